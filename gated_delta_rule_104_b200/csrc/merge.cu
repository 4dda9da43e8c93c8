// Merge of the bounded log into the dense base (DeltaLog page, Technical
// Summary, "Merge Phase": every M steps the accumulated logical state -- base
// plus replayed log entries -- is materialised back into the base), and the
// same merge fused with one step's read.
//
// Log-decay form. For log entries 0..n-1 (decays a_i, keys k_i, values v_i,
// strengths beta_i) write D(i, j) = prod_{m=j+1..i} a_m (= exp(Lambda_i -
// Lambda_j) with the page's log-decay metadata Lambda), gamma = D(n-1, -1).
// Every row s of the base evolves independently: with
//   G_i = s . Khat_i,  Khat_i = gamma_i o k_i          (a thin contraction)
//   C(i, j) = k_j . (D(i, j) o k_i), j < i
//   delta_i = beta_i (v_i[r] - G_i - sum_{j<i} C(i, j) delta_j)
// the merged row is s o gamma + sum_j delta_j F_j with F_j = k_j o D(n-1, j).
// The triangular solve is the same for every row: delta = X (v_r - G) with
// X = (I + Diag(beta) C)^{-1} Diag(beta), which the log keeps (each append
// adds its row), so the merge is two thin products
//   G = S Khat^T                 [rows x d_k] x [d_k x n]
//   S <- S o gamma + (V - G) W,  W = X^T F     [rows x n] x [n x d_k]
// with W formed once per head. That is 4 n d_k d_v FLOP against 2 d_k d_v
// state elements moved: a small dense contraction. For a block of entries
// [b, b + 16) of a longer log, X's diagonal block is the block's own X.
//
// Both products run on the tensor cores (mma.sync m16n8k8, TF32 in fp32
// accumulators). Plain TF32 keeps 10 mantissa bits, too few for the fp32
// state, so every operand is split as x = hi + lo (two TF32 values) and each
// product is formed as hi*hi + hi*lo + lo*hi, which recovers ~fp32 accuracy.
//
// RWKV6 (no delta correction) is the case X = I and no G: delta = V.
//
// Kernel: one block per (head, tile of up to 128 rows); warp w owns rows
// 16w..16w+15 of the tile. The entries are merged in blocks of NB = 8 or 16
// (a longer log is a chain of sub-merges; short blocks are padded with
// neutral entries k = 0, a = 1, beta = 0, v = 0). Per block:
//  1. stage the block's keys, decays, beta, X rows and the tile's values in
//     shared memory (all global loads issued before any shared store);
//  2. per key channel, running decay products give Khat, F and gamma; the
//     fused read's current entry (the block's last) has C(n, j) = k_n . F_j,
//     from which its X row follows;
//  3. W = X^T F;
//  4. per warp: G by tensor-core tiles, E = V - G moved from accumulator to
//     operand layout with quad shuffles, S o gamma + E W by tensor-core
//     tiles, the merged rows written back (and o = s_new . q for the fused
//     read) straight from the accumulator layout.
#include "launch.h"

namespace dl {

// ------------------------------------------------------------------ tensor-core helpers

__device__ __forceinline__ uint32_t tf32_of(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}
// x = hi + lo, both TF32 (x - hi is exact in fp32).
__device__ __forceinline__ void split_tf32(float x, uint32_t &hi, uint32_t &lo) {
    hi = tf32_of(x);
    lo = tf32_of(x - __uint_as_float(hi));
}
__device__ __forceinline__ void mma_tf32(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// d += a b with a = ah + al, b = bh + bl (the al bl term is below fp32 resolution).
__device__ __forceinline__ void mma3(float (&d)[4], const uint32_t (&ah)[4], const uint32_t (&al)[4], float b0,
                                     float b1) {
    uint32_t b0h, b0l, b1h, b1l;
    split_tf32(b0, b0h, b0l);
    split_tf32(b1, b1h, b1l);
    mma_tf32(d, al, b0h, b1h);
    mma_tf32(d, ah, b0l, b1l);
    mma_tf32(d, ah, b0h, b1h);
}

__device__ __forceinline__ float ld_state(const float *p) { return *p; }
__device__ __forceinline__ float ld_state(const bf16 *p) { return to_f(*p); }
__device__ __forceinline__ void st_state2(float *p, float x, float y) {
    __stcs(reinterpret_cast<float2 *>(p), make_float2(x, y));
}
__device__ __forceinline__ void st_state2(bf16 *p, float x, float y) {
    __stcs(reinterpret_cast<unsigned int *>(p), pack_bf2(x, y));
}

// ------------------------------------------------------------------ layout

__host__ __device__ constexpr size_t round4(size_t x) { return (x + 3) & ~(size_t)3; }

template <int DK, int NB>
struct MergeShape {
    static constexpr int ROWS = 64;     // base rows per block: 4 warps of 16
    static constexpr int KH = DK + 4;   // Khat row stride (conflict-free B-fragment reads)
    static constexpr int WS = DK + 8;   // F row stride (conflict-free B-fragment reads)
    static constexpr int XS = NB + 4;   // X row stride (conflict-free B-fragment reads)
    static constexpr int VS = ROWS + 4; // value row stride (conflict-free accumulator-layout reads)
    static constexpr int CW = DK / 32;  // key channels per lane (warp-wide dots)
};

// The block's base rows in shared memory: ROWS x DK elements of the state
// type, row-major with the 16-byte chunks of row r XOR-swizzled by
// f(r) = 2 (r mod 4) + (r / 4 mod 2), a permutation of 0..7. Over the 8 rows
// of a fragment f takes every value, so an 8-row x 4-column operand read hits
// 32 distinct banks; over each 4-row half it takes distinct pairs f / 2, so
// the accumulator-layout accesses (4 rows x 8 consecutive fp32 per half warp)
// do too. No padding.
template <class ST, int DK>
struct BaseTile {
    static constexpr int CE = 16 / (int)sizeof(ST);  // elements per 16-byte chunk
    static_assert(DK / CE >= 8, "swizzle spans 8 chunks");
    __device__ static __forceinline__ int off(int r, int c) {
        const int f = ((r & 3) << 1) | ((r >> 2) & 1);
        return r * DK + (((c / CE) ^ f) * CE) + (c % CE);
    }
};

// Shared memory (bytes) of one block for NB-entry sub-merges:
//   tile [ROWS][DK] of the tile type (swizzled base rows: float for an int8
//   base, else the state type), then floats:
//   kh [NB][KH] keys, turned into Khat in place
//   ff [NB][WS] F (channel decay: holds the decays until F replaces them)
//   fa [NB] head decays (padded to 4)   gn [DK] gamma   sq [DK] q
//   sx [NB][XS] X   sb [NB] beta   sv [NB][VS] the tile's values
//   sxw [4][XS] each warp's copy of the fused entry's X row
//   int8 base only: raw [ROWS][DK] codes, scl [ROWS] row scales, wsc [4][16]
//   the new row scales of each warp's rows
template <class ST, int DK, int NB>
__host__ __device__ constexpr size_t merge_smem_bytes() {
    using C = MergeShape<DK, NB>;
    constexpr bool Q8 = std::is_same<ST, int8_t>::value;
    using TT = typename std::conditional<Q8, float, ST>::type;
    const size_t floats = (size_t)NB * C::KH + (size_t)NB * C::WS + round4(NB) + DK + DK +
                          (size_t)NB * C::XS + round4(NB) + (size_t)NB * C::VS + 4 * (size_t)C::XS;
    const size_t q8 = Q8 ? (size_t)C::ROWS * DK + (size_t)C::ROWS * 4 + 64 * 4 : 0;
    return (size_t)C::ROWS * DK * sizeof(TT) + floats * sizeof(float) + q8;
}

__device__ __forceinline__ float2 ld_tile2(const float *p) { return *reinterpret_cast<const float2 *>(p); }
__device__ __forceinline__ float2 ld_tile2(const bf16 *p) {
    const uint32_t w = *reinterpret_cast<const uint32_t *>(p);
    return make_float2(bf_lo(w), bf_hi(w));
}
__device__ __forceinline__ void st_tile2(float *p, float x, float y) {
    *reinterpret_cast<float2 *>(p) = make_float2(x, y);
}
__device__ __forceinline__ void st_tile2(bf16 *p, float x, float y) {
    *reinterpret_cast<uint32_t *>(p) = pack_bf2(x, y);
}

// Accumulator layout (rows g, g + 8; columns 8i + 2t, 8i + 2t + 1) to A-operand
// layout (columns 8i + t, 8i + t + 4) of a 16 x 8NT tile, split into TF32 hi + lo.
template <int NT>
__device__ __forceinline__ void acc_to_operand(const float (&x)[NT][4], uint32_t (&hi)[NT][4],
                                               uint32_t (&lo)[NT][4], int lane) {
    const int t = lane & 3;
    const int s0 = (lane & ~3) | (t >> 1), s1 = s0 + 2;  // quad lanes holding columns t, t + 4
    const bool odd = t & 1;
#pragma unroll
    for (int i = 0; i < NT; ++i) {
        const float x00 = __shfl_sync(0xffffffffu, x[i][0], s0), x01 = __shfl_sync(0xffffffffu, x[i][1], s0);
        const float x10 = __shfl_sync(0xffffffffu, x[i][2], s0), x11 = __shfl_sync(0xffffffffu, x[i][3], s0);
        const float y00 = __shfl_sync(0xffffffffu, x[i][0], s1), y01 = __shfl_sync(0xffffffffu, x[i][1], s1);
        const float y10 = __shfl_sync(0xffffffffu, x[i][2], s1), y11 = __shfl_sync(0xffffffffu, x[i][3], s1);
        split_tf32(odd ? x01 : x00, hi[i][0], lo[i][0]);  // [g][8i + t]
        split_tf32(odd ? x11 : x10, hi[i][1], lo[i][1]);  // [g + 8][8i + t]
        split_tf32(odd ? y01 : y00, hi[i][2], lo[i][2]);  // [g][8i + t + 4]
        split_tf32(odd ? y11 : y10, hi[i][3], lo[i][3]);  // [g + 8][8i + t + 4]
    }
}

// ------------------------------------------------------------------ kernel

template <class ST, int DK, int KIND, bool WITH_CUR, int NB>
__global__ void __launch_bounds__(128, 4)
merge_kernel(ST *__restrict__ S, const void *__restrict__ log_k, const void *__restrict__ log_v,
             const void *__restrict__ log_b, const void *__restrict__ log_a, const float *__restrict__ log_x,
             int L, int n_log, const void *__restrict__ q, const void *__restrict__ k, const void *__restrict__ v,
             const void *__restrict__ beta, const void *__restrict__ a, float *__restrict__ o, int DV, bool bf,
             PoolIdx pool, int part, float *__restrict__ i8_scales) {
    using C = MergeShape<DK, NB>;
    // An int8 base (row scales in i8_scales) is widened into a float tile, merged
    // as a float base, and its rows rounded back to int8 when they are stored.
    constexpr bool Q8 = std::is_same<ST, int8_t>::value;
    using TT = typename std::conditional<Q8, float, ST>::type;
    using TL = BaseTile<TT, DK>;
    constexpr bool CHAN = Rule<KIND>::CHAN, DELTA = Rule<KIND>::DELTA;
    constexpr int KS = DK / 8;   // k-steps of the first product / column tiles of the second
    constexpr int NT = NB / 8;   // entry tiles
    constexpr int ROWS = C::ROWS;
    constexpr int nthr = 2 * ROWS;  // 4 warps, 16 rows each

    extern __shared__ float4 smem_raw[];
    TT *tile = reinterpret_cast<TT *>(smem_raw);
    float *kh = reinterpret_cast<float *>(tile + ROWS * DK);
    float *ff = kh + NB * C::KH;
    float *fa = ff + NB * C::WS;
    float *gn = fa + round4(NB);
    float *sq = gn + DK;
    float *sx = sq + DK;
    float *sb = sx + NB * C::XS;
    float *sv = sb + round4(NB);
    float *sxw = sv + NB * C::VS;
    int8_t *raw = reinterpret_cast<int8_t *>(sxw + 4 * C::XS);  // int8 base only
    float *scl = reinterpret_cast<float *>(raw + ROWS * DK);
    float *wsc = scl + ROWS;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, t = lane & 3;  // fragment coordinates
    const int tiles = DV / ROWS;
    const long long head = blockIdx.x / tiles;  // batch head (this step's inputs, o)
    const int row0 = (blockIdx.x % tiles) * ROWS;
    long long shead;                            // state / log head
    pdl_launch_dependents();  // a pool step's append part (other slots) may start beside this grid
    if (!pool_head(pool, part, head, shead, n_log)) return;  // the whole block: no barrier passed yet
    const int NTOT = n_log + (WITH_CUR ? 1 : 0);
    const long long lrow = shead * L;
    ST *Sw = S + (shead * DV + row0 + 16 * warp) * DK;  // this warp's 16 rows
    const int tr = 16 * warp;                           // and their first row in the tile

    // The block's base rows, fetched by cp.async right after the first entry
    // block's loads are issued (those come first, so that they do not queue
    // behind the tile); the tile lands while the key side is worked out.
    auto fetch_tile = [&]() {
        if constexpr (Q8) {  // the codes (unswizzled) and the row scales
            constexpr int CPR = DK / 16;
            const int8_t *src = S + (shead * DV + row0) * DK;
#pragma unroll 4
            for (int u = tid; u < ROWS * CPR; u += nthr) {
                const int r = u / CPR, ch = u % CPR;
                cp_async16(raw + r * DK + ch * 16, src + (long long)r * DK + ch * 16);
            }
            if (tid < ROWS / 4) cp_async16(scl + 4 * tid, i8_scales + shead * DV + row0 + 4 * tid);
        } else {
            constexpr int CPR = DK / TL::CE;  // chunks per row
            const ST *src = S + (shead * DV + row0) * DK;
#pragma unroll 4
            for (int u = tid; u < ROWS * CPR; u += nthr) {
                const int r = u / CPR, ch = u % CPR;
                cp_async16(tile + TL::off(r, ch * TL::CE), src + (long long)r * DK + ch * TL::CE);
            }
        }
        cp_async_commit();
    };

    float oacc[2] = {0.f, 0.f};  // o for rows g and g + 8 (fused read), partial over this lane's columns
    for (int b0 = 0; b0 < NTOT; b0 += NB) {
        const int nb = NTOT - b0 < NB ? NTOT - b0 : NB;
        const int nl = (n_log - b0 < nb ? n_log - b0 : nb);  // of which from the log (the rest: this step)
        const bool cur_here = WITH_CUR && nl < nb;
        const bool last = b0 + NB >= NTOT;

        // 1. entries b0 .. b0+nb-1 (log entries, then the fused read's own); all
        // global loads are issued before the first shared store.
        auto stage = [&](auto tag) {
            using IT = decltype(tag);
            constexpr int E = 16 / (int)sizeof(IT);
            constexpr int KC = DK / E;
            constexpr int KN = (NB * KC + 127) / 128;       // >= 128 threads per block
            constexpr int VN = (NB * 128 / E + 127) / 128;  // rows <= 128
            const int VC = ROWS / E;
            float kx[KN][E], ax[KN][E], vx[VN][E], qx[E];
            (void)ax;
            (void)qx;
            const bool qload = WITH_CUR && b0 == 0 && tid < KC;  // this step's q, with the first block
            if (qload) load_vec<E>(static_cast<const IT *>(q) + head * DK + tid * E, qx);
            auto key_src = [&](const void *logp, const void *cur, int r) -> const IT * {
                return r < nl ? static_cast<const IT *>(logp) + (lrow + b0 + r) * DK
                              : static_cast<const IT *>(cur) + head * DK;
            };
#pragma unroll
            for (int u = 0; u < KN; ++u) {
                const int c = tid + u * nthr, r = c / KC, col = (c % KC) * E;
                if (c < NB * KC && r < nb) {
                    load_vec<E>(key_src(log_k, k, r) + col, kx[u]);
                    if constexpr (CHAN) load_vec<E>(key_src(log_a, a, r) + col, ax[u]);
                }
            }
#pragma unroll
            for (int u = 0; u < VN; ++u) {
                const int c = tid + u * nthr, r = c / VC, col = (c % VC) * E;
                if (c < NB * VC && r < nb) {
                    const IT *src = r < nl ? static_cast<const IT *>(log_v) + (lrow + b0 + r) * DV
                                           : static_cast<const IT *>(v) + head * DV;
                    load_vec<E>(src + row0 + col, vx[u]);
                }
            }
            float bsc = 0.f, asc = 1.f;
            (void)asc;
            if (tid < nb) {
                if constexpr (DELTA)
                    bsc = tid < nl ? to_f(static_cast<const IT *>(log_b)[lrow + b0 + tid])
                                   : to_f(static_cast<const IT *>(beta)[head]);
                if constexpr (!CHAN)
                    asc = tid < nl ? to_f(static_cast<const IT *>(log_a)[lrow + b0 + tid])
                                   : to_f(static_cast<const IT *>(a)[head]);
            }
            // X(i, j), j <= i, of the logged entries (the block's diagonal block; the
            // current entry's row is formed below; padded entries are zero)
            constexpr int CN = (NB * NB + 127) / 128;
            float cval[CN];
#pragma unroll
            for (int u = 0; u < CN; ++u) {
                const int idx = tid + u * nthr, ci = idx / NB, cj = idx % NB;
                cval[u] = (DELTA && idx < NB * NB && cj <= ci && ci < nl) ? log_x[(lrow + b0 + ci) * L + b0 + cj]
                                                                            : 0.f;
            }
            if (b0 == 0) fetch_tile();
            auto put = [](float *dst, const float *x, bool real, float pad) {
#pragma unroll
                for (int e = 0; e < E; e += 4)
                    *reinterpret_cast<float4 *>(dst + e) =
                        real ? make_float4(x[e], x[e + 1], x[e + 2], x[e + 3]) : make_float4(pad, pad, pad, pad);
            };
#pragma unroll
            for (int u = 0; u < KN; ++u) {
                const int c = tid + u * nthr, r = c / KC, col = (c % KC) * E;
                if (c < NB * KC) {  // padded entries: k = 0, a = 1
                    put(kh + r * C::KH + col, kx[u], r < nb, 0.f);
                    if constexpr (CHAN) put(ff + r * C::WS + col, ax[u], r < nb, 1.f);
                }
            }
#pragma unroll
            for (int u = 0; u < VN; ++u) {
                const int c = tid + u * nthr, r = c / VC, col = (c % VC) * E;
                if (c < NB * VC) put(sv + r * C::VS + col, vx[u], r < nb, 0.f);
            }
            if (tid < NB) {
                sb[tid] = bsc;  // 0 for padded entries
                if constexpr (!CHAN) fa[tid] = asc;
            }
            if (qload) put(sq + tid * E, qx, true, 0.f);
#pragma unroll
            for (int u = 0; u < CN; ++u) {
                const int idx = tid + u * nthr, ci = idx / NB, cj = idx % NB;
                if (idx < NB * NB && !(cur_here && ci == nl)) sx[ci * C::XS + cj] = cval[u];
            }
        };
        if (bf) stage(bf16{});
        else stage(float{});
        __syncthreads();

        // 2. per key channel, in place: Khat_i = gamma_i o k_i, gamma,
        // F_j = k_j o D(NB-1, j) (padded entries have a = 1, so D(NB-1, j) = D(nb-1, j)).
        for (int c = tid; c < DK; c += nthr) {
            float ac[NB], kc[NB];
#pragma unroll
            for (int i = 0; i < NB; ++i) {
                ac[i] = CHAN ? ff[i * C::WS + c] : fa[i];
                kc[i] = kh[i * C::KH + c];
            }
            float gm = 1.f;
#pragma unroll
            for (int i = 0; i < NB; ++i) {
                gm *= ac[i];
                kh[i * C::KH + c] = gm * kc[i];
            }
            gn[c] = gm;
            float f = 1.f;
#pragma unroll
            for (int j = NB - 1; j >= 0; --j) {
                ff[j * C::WS + c] = kc[j] * f;
                f *= ac[j];
            }
        }
        cp_async_wait_all();  // this thread's share of the base tile has landed
        __syncthreads();
        if constexpr (Q8) {
            if (b0 == 0) {  // codes * scale into the float tile, 4 at a time
                for (int u = tid; u < ROWS * DK / 4; u += nthr) {
                    const int r = u / (DK / 4), c4 = (u % (DK / 4)) * 4;
                    const uint32_t w = *reinterpret_cast<const uint32_t *>(raw + r * DK + c4);
                    const float sc = scl[r];
                    *reinterpret_cast<float4 *>(tile + TL::off(r, c4)) =
                        make_float4((float)(int8_t)w * sc, (float)(int8_t)(w >> 8) * sc,
                                    (float)(int8_t)(w >> 16) * sc, (float)(int8_t)(w >> 24) * sc);
                }
                __syncthreads();
            }
        }
        // The fused read's current entry is the block's last real one: F_nl = k_nl
        // exactly (every later factor is a padded 1) and D(nl, j) is F_j's suffix
        // product, so C(nl, j) = F_nl . F_j. Every warp forms that C row and the
        // entry's X row itself, with no block barrier: lane-partial dots over its
        // key channels, one transposing butterfly (lane l ends with C(nl, l >> SH)),
        // then on lane j: X(nl, j) = -beta sum_{m=j..nl-1} C(nl, m) X(m, j),
        // X(nl, nl) = beta, kept in the warp's own row sxw.
        if (DELTA && cur_here) {
            constexpr int SH = NB == 16 ? 1 : 2;
            float fn[C::CW], pc[NB];
#pragma unroll
            for (int e = 0; e < C::CW; ++e) fn[e] = ff[nl * C::WS + e * 32 + lane];
#pragma unroll
            for (int j = 0; j < NB; ++j) {
                pc[j] = 0.f;
#pragma unroll
                for (int e = 0; e < C::CW; ++e) pc[j] = fmaf(fn[e], ff[j * C::WS + e * 32 + lane], pc[j]);
            }
            multi_sum<NB>(pc, lane);
            float acc = 0.f;
#pragma unroll
            for (int m = 0; m < NB; ++m) {
                const float cnm = __shfl_sync(0xffffffffu, pc[0], m << SH);
                if (lane <= m && m < nl) acc = fmaf(cnm, sx[m * C::XS + lane], acc);
            }
            const float bn = sb[nl];
            if (lane < NB) sxw[warp * C::XS + lane] = lane < nl ? -bn * acc : (lane == nl ? bn : 0.f);
            __syncwarp();
        }

        // 3. this warp's 16 rows: delta in the A-operand layout (split hi + lo).
        __syncwarp();  // a previous block's rows, written by this warp, are visible
        const int rg = 16 * warp + g;
        uint32_t xh[NT][4], xl[NT][4];
        if constexpr (!DELTA) {
            // delta = V, read straight into the operand layout (entries 8nt + t, + 4).
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const int i0 = 8 * nt + t;
                split_tf32(sv[i0 * C::VS + rg], xh[nt][0], xl[nt][0]);
                split_tf32(sv[i0 * C::VS + rg + 8], xh[nt][1], xl[nt][1]);
                split_tf32(sv[(i0 + 4) * C::VS + rg], xh[nt][2], xl[nt][2]);
                split_tf32(sv[(i0 + 4) * C::VS + rg + 8], xh[nt][3], xl[nt][3]);
            }
        } else {
            // G = S Khat^T, the A fragments from the base tile: a0 = S[g][8s + t],
            // a1 = S[g + 8][8s + t], a2 = S[g][8s + t + 4], a3 = S[g + 8][8s + t + 4].
            // (two accumulator sets, even and odd k-steps, halve the dependent chains)
            float acc1[NT][4], acc2[NT][4];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int x = 0; x < 4; ++x) acc1[nt][x] = acc2[nt][x] = 0.f;
#pragma unroll
            for (int s = 0; s < KS; ++s) {
                uint32_t ah[4], al[4];
                split_tf32(ld_state(tile + TL::off(tr + g, 8 * s + t)), ah[0], al[0]);
                split_tf32(ld_state(tile + TL::off(tr + g + 8, 8 * s + t)), ah[1], al[1]);
                split_tf32(ld_state(tile + TL::off(tr + g, 8 * s + t + 4)), ah[2], al[2]);
                split_tf32(ld_state(tile + TL::off(tr + g + 8, 8 * s + t + 4)), ah[3], al[3]);
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    const float *kp = kh + (8 * nt + g) * C::KH + 8 * s + t;
                    mma3((s & 1) ? acc2[nt] : acc1[nt], ah, al, kp[0], kp[4]);
                }
            }
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int x = 0; x < 4; ++x) acc1[nt][x] += acc2[nt][x];
            // E = V - G in the accumulator layout (rows g, g + 8; entries 8nt + 2t, +1).
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const int i0 = 8 * nt + 2 * t;
                acc1[nt][0] = sv[i0 * C::VS + rg] - acc1[nt][0];
                acc1[nt][1] = sv[(i0 + 1) * C::VS + rg] - acc1[nt][1];
                acc1[nt][2] = sv[i0 * C::VS + rg + 8] - acc1[nt][2];
                acc1[nt][3] = sv[(i0 + 1) * C::VS + rg + 8] - acc1[nt][3];
            }
            // delta = E X^T (the triangular solve, one small product per warp; X is
            // lower triangular, so tiles above the diagonal are skipped).
            acc_to_operand<NT>(acc1, xh, xl, lane);
            float dl[NT][4];
#pragma unroll
            for (int mt = 0; mt < NT; ++mt) {
#pragma unroll
                for (int x = 0; x < 4; ++x) dl[mt][x] = 0.f;
                const int xr = 8 * mt + g;  // the fused entry's row is the warp's own copy
                const float *xrow = (cur_here && xr == nl) ? sxw + warp * C::XS : sx + xr * C::XS;
#pragma unroll
                for (int kt = 0; kt <= mt; ++kt) {
                    const float *xp = xrow + 8 * kt + t;
                    mma3(dl[mt], xh[kt], xl[kt], xp[0], xp[4]);
                }
            }
            acc_to_operand<NT>(dl, xh, xl, lane);
        }
        // S <- S o gamma + delta F, one 16 x 8 column tile at a time (rows g, g + 8;
        // columns 8c + 2t, 8c + 2t + 1 of the accumulator layout): from the tile,
        // back to the tile for a following sub-merge (or, for an int8 base, for the
        // rounding below), else straight to HBM.
        float rmax0 = 0.f, rmax1 = 0.f;  // int8 base: |value| maxima of rows g, g + 8 (this lane's columns)
#pragma unroll 4
        for (int cb = 0; cb < KS; ++cb) {
            float dn[NT][4];  // one accumulator per entry tile: independent chains
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
                for (int x = 0; x < 4; ++x) dn[nt][x] = 0.f;
                const float *fp = ff + (8 * nt + t) * C::WS + 8 * cb + g;
                mma3(dn[nt], xh[nt], xl[nt], fp[0], fp[4 * C::WS]);
            }
            float d[4];
#pragma unroll
            for (int x = 0; x < 4; ++x) {
                d[x] = dn[0][x];
#pragma unroll
                for (int nt = 1; nt < NT; ++nt) d[x] += dn[nt][x];
            }
            const int col = 8 * cb + 2 * t;
            TT *p0 = tile + TL::off(tr + g, col), *p1 = tile + TL::off(tr + g + 8, col);
            const float2 r0 = ld_tile2(p0), r1 = ld_tile2(p1);
            float s00 = r0.x, s01 = r0.y, s10 = r1.x, s11 = r1.y;
            const float2 gv = *reinterpret_cast<const float2 *>(gn + col);
            s00 = fmaf(s00, gv.x, d[0]);
            s01 = fmaf(s01, gv.y, d[1]);
            s10 = fmaf(s10, gv.x, d[2]);
            s11 = fmaf(s11, gv.y, d[3]);
            if (WITH_CUR && last) {
                const float2 qv = *reinterpret_cast<const float2 *>(sq + col);
                oacc[0] = fmaf(s00, qv.x, fmaf(s01, qv.y, oacc[0]));
                oacc[1] = fmaf(s10, qv.x, fmaf(s11, qv.y, oacc[1]));
            }
            if constexpr (Q8) {
                st_tile2(p0, s00, s01);
                st_tile2(p1, s10, s11);
                rmax0 = fmaxf(rmax0, fmaxf(fabsf(s00), fabsf(s01)));
                rmax1 = fmaxf(rmax1, fmaxf(fabsf(s10), fabsf(s11)));
            } else if (last) {
                st_state2(Sw + g * DK + col, s00, s01);
                st_state2(Sw + (g + 8) * DK + col, s10, s11);
            } else {
                st_tile2(p0, s00, s01);
                st_tile2(p1, s10, s11);
            }
        }
        if constexpr (Q8) {
            if (last) {  // round the warp's 16 rows to int8 (one scale per row) and store them
#pragma unroll
                for (int off = 1; off <= 2; off <<= 1) {  // the quad holds a row's columns
                    rmax0 = fmaxf(rmax0, __shfl_xor_sync(0xffffffffu, rmax0, off));
                    rmax1 = fmaxf(rmax1, __shfl_xor_sync(0xffffffffu, rmax1, off));
                }
                if (t == 0) {
                    wsc[warp * 16 + g] = i8_scale(rmax0);
                    wsc[warp * 16 + g + 8] = i8_scale(rmax1);
                }
                __syncwarp();
                constexpr int CPR = DK / 16;  // 16-code chunks per row
                for (int i = lane; i < 16 * CPR; i += 32) {
                    const int rl = i / CPR, c0 = (i % CPR) * 16;
                    const float sc = wsc[warp * 16 + rl];
                    uint32_t wd[4];
#pragma unroll
                    for (int qd = 0; qd < 4; ++qd) {
                        const float4 x = *reinterpret_cast<const float4 *>(tile + TL::off(tr + rl, c0 + 4 * qd));
                        wd[qd] = (uint32_t)(i8_code(x.x, sc) & 0xff) | ((uint32_t)(i8_code(x.y, sc) & 0xff) << 8) |
                                 ((uint32_t)(i8_code(x.z, sc) & 0xff) << 16) |
                                 ((uint32_t)(i8_code(x.w, sc) & 0xff) << 24);
                    }
                    st_stream(Sw + rl * DK + c0, make_uint4(wd[0], wd[1], wd[2], wd[3]));
                }
                if (lane < 16) i8_scales[shead * DV + row0 + tr + lane] = wsc[warp * 16 + lane];
            }
        }
        __syncthreads();  // the next entry block reuses the shared buffers
    }

    if constexpr (WITH_CUR) {
        oacc[0] = group_sum<4>(oacc[0]);
        oacc[1] = group_sum<4>(oacc[1]);
        if (t == 0) {
            o[head * DV + row0 + 16 * warp + g] = oacc[0];
            o[head * DV + row0 + 16 * warp + g + 8] = oacc[1];
        }
    }
}

// ------------------------------------------------------------------ launch

template <class ST, int DK, int KD, bool WC, int NB>
static cudaError_t launch_merge_t(const StepParams &p, const LogParams &lg, int n_log, cudaStream_t st,
                                  const PoolIdx &pool, int part) {
    using C = MergeShape<DK, NB>;
    auto kern = merge_kernel<ST, DK, KD, WC, NB>;
    constexpr int rows = C::ROWS;
    const size_t smem = merge_smem_bytes<ST, DK, NB>();
    cudaError_t e = allow_smem(reinterpret_cast<const void *>(kern), smem);
    if (e != cudaSuccess) return e;
    const long long blocks = (long long)p.B * p.H * (p.dv / rows);
    // an int8 base's row scales follow its codes (all the state's heads: the pool's, or B*H)
    const long long state_heads = pool.slot ? (long long)pool.P * pool.H : (long long)p.B * p.H;
    float *i8_scales = std::is_same<ST, int8_t>::value
                           ? reinterpret_cast<float *>(static_cast<int8_t *>(p.S) + state_heads * p.dv * DK)
                           : nullptr;
    kern<<<(unsigned)blocks, rows * 2, smem, st>>>(static_cast<ST *>(p.S), lg.k, lg.v, lg.beta, lg.a, lg.x, lg.L,
                                                   n_log, p.q, p.k, p.v, p.beta, p.a, p.o, p.dv,
                                                   p.in_dt == DL_BF16, pool, part, i8_scales);
    return cudaGetLastError();
}

// Entry-block size: 8 when all entries fit, else 16 (a longer log runs as a
// chain of 16-entry sub-merges, the last one padded). A pool launch sizes it
// for the largest count a slot can hold.
template <class ST, int DK, int KD, bool WC>
static cudaError_t launch_merge_nb(const StepParams &p, const LogParams &lg, int n_log, cudaStream_t st,
                                   const PoolIdx &pool, int part) {
    const int nt = (pool.slot ? lg.L - 1 : n_log) + (WC ? 1 : 0);
    if (nt <= 8) return launch_merge_t<ST, DK, KD, WC, 8>(p, lg, n_log, st, pool, part);
    return launch_merge_t<ST, DK, KD, WC, 16>(p, lg, n_log, st, pool, part);
}

cudaError_t launch_merge(const StepParams &p, const LogParams &lg, int n_log, bool with_cur, cudaStream_t st,
                         const PoolIdx &pool, int part) {
    // The input dtype and d_v are run-time arguments of the merge kernel (they
    // only change staging and the grid), which keeps instantiations few.
    auto go = [&](auto st_t, auto dk_c) -> cudaError_t {
        using ST = decltype(st_t);
        constexpr int DK = decltype(dk_c)::value;
        auto with_kind = [&](auto kd_c) -> cudaError_t {
            constexpr int KD = decltype(kd_c)::value;
            if (with_cur) return launch_merge_nb<ST, DK, KD, true>(p, lg, n_log, st, pool, part);
            return launch_merge_nb<ST, DK, KD, false>(p, lg, n_log, st, pool, part);
        };
        if (p.kind == DL_RWKV6) return with_kind(std::integral_constant<int, DL_RWKV6>{});
        if (p.kind == DL_DECAY_CHANNEL) return with_kind(std::integral_constant<int, DL_DECAY_CHANNEL>{});
        return with_kind(std::integral_constant<int, DL_DECAY_HEAD>{});
    };
    auto with_dk = [&](auto st_t) -> cudaError_t {
        if (p.dk == 64) return go(st_t, std::integral_constant<int, 64>{});
        return go(st_t, std::integral_constant<int, 128>{});
    };
    if (p.s_dt == DL_BF16) return with_dk(bf16{});
    if (p.s_dt == DL_I8) return with_dk(int8_t{});
    return with_dk(float{});
}

// ------------------------------------------------------------------ pool counts

// After a pool step every listed slot holds one more entry, or none if this
// step was its L-th (merged); after a flush it holds none.
__global__ void pool_counts_kernel(const int *__restrict__ slot, int *__restrict__ counts, int B, int P, int L,
                                   bool advance) {
    const int b = blockIdx.x * blockDim.x + threadIdx.x;
    if (b >= B) return;
    const int s = slot[b];
    if (s < 0 || s >= P) return;  // flagged by the step's kernels
    const int c = counts[s];
    if (c < 0 || c >= L) return;
    counts[s] = (advance && c < L - 1) ? c + 1 : 0;
}

cudaError_t launch_pool_counts(const PoolIdx &pool, int B, bool advance, cudaStream_t st) {
    pool_counts_kernel<<<(B + 127) / 128, 128, 0, st>>>(pool.slot, pool.counts, B, pool.P, pool.L, advance);
    return cudaGetLastError();
}

}  // namespace dl
