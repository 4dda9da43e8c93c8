// Merge of the bounded log into the dense base (DeltaLog page, "Core
// Mechanism: Base + Log", the merge phase: at intervals the base absorbs every
// update the log holds and the log starts empty again), and the same merge
// fused with one step's read.
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
// adds its row), so per block of rows the merge is
//   G = S Khat^T                 [rows x d_k] x [d_k x n]
//   delta = (V - G) X^T          [rows x n] x [n x n], X lower triangular
//   S <- S o gamma + delta F     [rows x n] x [n x d_k]
// That is about 4 n d_k d_v FLOP against 2 d_k d_v state elements moved: a
// small dense contraction. For a block of entries [b, b + 16) of a longer log,
// X's diagonal block is the block's own X.
//
// All three products run on the tensor cores (mma.sync m16n8k8, TF32 in fp32
// accumulators). Plain TF32 keeps 10 mantissa bits, too few for the fp32
// state, so every operand is split as x = hi + lo (two TF32 values) and each
// product is formed as hi*hi + hi*lo + lo*hi, which recovers ~fp32 accuracy.
//
// RWKV6 (no delta correction) is the case X = I and no G: delta = V.
//
// Kernel: one 4-warp block per unit (head, tile of 64 rows); warp w owns rows
// 16w..16w+15 of the tile. The entries are merged in blocks of NB = 8 or 16
// (a longer log is a chain of sub-merges; short blocks are padded with
// neutral entries k = 0, a = 1, beta = 0, v = 0). Per entry block:
//  1. stage the block's keys, decays, beta, X rows and the tile's values in
//     shared memory (all global loads issued before any shared store; the
//     first block also starts the base tile's cp.async);
//  2. per key channel, running decay products give Khat, F and gamma; the
//     fused read's current entry (the block's last) has C(n, j) = F_n . F_j,
//     from which each warp forms its X row;
//  3. per warp: G by tensor-core tiles, E = V - G moved from accumulator to
//     operand layout with quad shuffles, delta = E X^T (lower tiles only),
//     then S o gamma + delta F by tensor-core tiles, the merged rows written
//     back (and o = s_new . q for the fused read) straight from the
//     accumulator layout.
// A pool step's merge part runs the same body over a compact grid (below).
#include "launch.h"
#include "guard.cuh"
#include "merge_layout.h"

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

// Four consecutive state elements (16 bytes of fp32, 8 of bf16), widened to fp32.
__device__ __forceinline__ float4 ld_tile4(const float *p) { return *reinterpret_cast<const float4 *>(p); }
__device__ __forceinline__ float4 ld_tile4(const bf16 *p) {
    const uint2 w = *reinterpret_cast<const uint2 *>(p);
    return make_float4(bf_lo(w.x), bf_hi(w.x), bf_lo(w.y), bf_hi(w.y));
}
__device__ __forceinline__ void st_tile4(float *p, float4 x) { *reinterpret_cast<float4 *>(p) = x; }
__device__ __forceinline__ void st_tile4(bf16 *p, float4 x) {
    *reinterpret_cast<uint2 *>(p) = make_uint2(pack_bf2(x.x, x.y), pack_bf2(x.z, x.w));
}
__device__ __forceinline__ void st_state4(float *p, float4 x) { __stcs(reinterpret_cast<float4 *>(p), x); }
__device__ __forceinline__ void st_state4(bf16 *p, float4 x) {
    __stcs(reinterpret_cast<uint2 *>(p), make_uint2(pack_bf2(x.x, x.y), pack_bf2(x.z, x.w)));
}

// Column order of the two products. Both are sums over, or maps of, the key
// columns, so any order that the state, Khat and F share gives the same
// result. Within each group of 16 columns [16j, 16j + 16):
//  - G's k-steps 2j + h (h = 0, 1) take fragment positions t and t + 4 to
//    columns 16j + 4t + 2h and 16j + 4t + 2h + 1;
//  - the update's column tiles 2j + h take accumulator column n to
//    16j + 4 (n / 2) + 2h + n mod 2.
// Either way lane (g, t) holds columns 16j + 4t .. 16j + 4t + 3 of its rows, so
// the base tile, Khat, gamma, q and the merged rows move 16 bytes per access.
// F is stored in the order the update's B fragments read it (f_pos, in
// merge_layout.h, with the block's shared-memory layout).

template <class ST, int DK, int NB>
__host__ __device__ constexpr size_t merge_smem_bytes() {
    return MergeRegions<(int)sizeof(ST), std::is_same<ST, int8_t>::value, DK, NB>::bytes;
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
             PoolIdx pool, int part, float *__restrict__ i8_scales, long long units) {
    using C = MergeShape<DK, NB>;
    // An int8 base (row scales in i8_scales) is widened into a float tile, merged
    // as a float base, and its rows rounded back to int8 when they are stored.
    constexpr bool Q8 = std::is_same<ST, int8_t>::value;
    using TT = typename std::conditional<Q8, float, ST>::type;
    using TL = BaseTile<(int)sizeof(TT), DK>;
    constexpr bool CHAN = Rule<KIND>::CHAN, DELTA = Rule<KIND>::DELTA;
    constexpr int NT = NB / 8;   // entry tiles
    constexpr int ROWS = C::ROWS;
    constexpr int nthr = 2 * ROWS;  // 4 warps, 16 rows each

    using RG = MergeRegions<(int)sizeof(ST), Q8, DK, NB>;
    extern __shared__ float4 smem_raw[];
    TT *tile = reinterpret_cast<TT *>(smem_raw);
    float *fl = reinterpret_cast<float *>(reinterpret_cast<uint8_t *>(smem_raw) + RG::tile_bytes);
    float *kh = fl + RG::kh;
    float *ff = fl + RG::ff;
    float *fa = fl + RG::fa;
    float *gn = fl + RG::gn;
    float *sq = fl + RG::sq;
    float *sx = fl + RG::sx;
    float *sb = fl + RG::sb;
    float *sv = fl + RG::sv;
    float *sxw = fl + RG::sxw;
    // int8 base only: the codes at the end of the (float) tile, the scales after sxw
    int8_t *raw = reinterpret_cast<int8_t *>(smem_raw) + RG::raw_bytes_off;
    float *scl = fl + RG::scl;
    float *wsc = fl + RG::wsc;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, t = lane & 3;  // fragment coordinates
    const int tiles = DV / ROWS;
    pdl_launch_dependents();  // a pool step's append part (other slots) may start beside this grid

    // A unit is (batch head, tile of ROWS rows); one unit per block, except in a
    // compact grid (a pool step's merge part, where only the slots on their L-th
    // entry merge). There block b owns units b, b + G, b + 2G, ... (G = gridDim.x):
    // it checks them 128 at a time, one per thread, keeps each warp's ballot of
    // those that merge in shared memory (xw[0..3], the batch in xw[4]), and merges
    // them one after another. The walk's state lives in shared memory, so that
    // nothing of it stays in registers across a merge.
    const bool compact = units != (long long)gridDim.x;
    uint32_t *xw = reinterpret_cast<uint32_t *>(fl + RG::xw);
    if (compact) {
        if (tid < 4) {
            DL_GUARD(xw + tid, 4) xw[tid] = 0u;
        }
        if (tid == 0) {
            DL_GUARD(xw + 4, 4) xw[4] = 0xffffffffu;  // batch -1: none checked yet
        }
        __syncthreads();
    }
    for (;;) {
        long long unit = blockIdx.x;
        if (compact) {
            int batch = (int)xw[4];
            uint32_t m[4] = {xw[0], xw[1], xw[2], xw[3]};
            bool done = false;
            while ((m[0] | m[1] | m[2] | m[3]) == 0u) {  // the next batch with a unit to merge
                ++batch;
                const long long u0 = (long long)blockIdx.x + (long long)batch * nthr * gridDim.x;
                if (u0 >= units) {
                    done = true;
                    break;
                }
                const long long u = u0 + (long long)tid * gridDim.x;
                bool mine = false;
                if (u < units) {
                    long long sh;
                    int nn = n_log;
                    mine = pool_head(pool, part, u / tiles, sh, nn);
                }
                const uint32_t bal = __ballot_sync(0xffffffffu, mine);
                __syncthreads();  // every thread has read the previous words
                if (lane == 0) {
                    DL_GUARD(xw + warp, 4) xw[warp] = bal;
                }
                __syncthreads();
#pragma unroll
                for (int w = 0; w < 4; ++w) m[w] = xw[w];
            }
            if (done) break;
            const int w = m[0] ? 0 : m[1] ? 1 : m[2] ? 2 : 3;
            const int bit = __ffs(m[w]) - 1;
            unit = (long long)blockIdx.x + ((long long)batch * nthr + 32 * w + bit) * gridDim.x;
            __syncthreads();  // every thread has read the words before they change
            if (tid == 0) {
                DL_GUARD(xw + w, 4) xw[w] = m[w] & (m[w] - 1u);
                DL_GUARD(xw + 4, 4) xw[4] = (uint32_t)batch;
            }
        }
        const long long head = unit / tiles;  // batch head (this step's inputs, o)
        const int row0 = (int)(unit % tiles) * ROWS;
        long long shead;                      // state / log head
        int n_log_u = n_log;                  // this unit's log count (a pool slot's own)
        // a unit that is not this launch's to merge (a pool slot at another count)
        // is left by the whole block before any barrier
        if (pool_head(pool, part, head, shead, n_log_u)) {
            const int n_log = n_log_u;
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
                        DL_GUARD(raw + r * DK + ch * 16, 16) cp_async16(raw + r * DK + ch * 16, src + (long long)r * DK + ch * 16);
                    }
                    if (tid < ROWS / 4) {
                        DL_GUARD(scl + 4 * tid, 16) cp_async16(scl + 4 * tid, i8_scales + shead * DV + row0 + 4 * tid);
                    }
                } else {
                    constexpr int CPR = DK / TL::CE;  // chunks per row
                    const ST *src = S + (shead * DV + row0) * DK;
#pragma unroll 4
                    for (int u = tid; u < ROWS * CPR; u += nthr) {
                        const int r = u / CPR, ch = u % CPR;
                        DL_GUARD(tile + TL::off(r, ch * TL::CE), 16)
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
                        cval[u] = (DELTA && idx < NB * NB && cj <= ci && ci < nl)
                                      ? log_x[(lrow + b0 + ci) * L + b0 + cj]
                                                                                    : 0.f;
                    }
                    if (b0 == 0) fetch_tile();
                    auto put = [](float *dst, const float *x, bool real, float pad) {
#pragma unroll
                        for (int e = 0; e < E; e += 4)
                            DL_GUARD(dst + e, 16) *reinterpret_cast<float4 *>(dst + e) =
                                real ? make_float4(x[e], x[e + 1], x[e + 2], x[e + 3])
                                     : make_float4(pad, pad, pad, pad);
                    };
#pragma unroll
                    for (int u = 0; u < KN; ++u) {
                        const int c = tid + u * nthr, r = c / KC, col = (c % KC) * E;
                        if (c < NB * KC) {  // padded entries: k = 0, a = 1
                            put(kh + C::kof(r, col), kx[u], r < nb, 0.f);
                            if constexpr (CHAN) put(ff + r * C::WS + col, ax[u], r < nb, 1.f);
                        }
                    }
#pragma unroll
                    for (int u = 0; u < VN; ++u) {
                        const int c = tid + u * nthr, r = c / VC, col = (c % VC) * E;
                        if (c < NB * VC) put(sv + r * C::VS + col, vx[u], r < nb, 0.f);
                    }
                    if (tid < NB) {
                        DL_GUARD(sb + tid, 4) sb[tid] = bsc;  // 0 for padded entries
                        if constexpr (!CHAN) {
                            DL_GUARD(fa + tid, 4) fa[tid] = asc;
                        }
                    }
                    if (qload) put(sq + tid * E, qx, true, 0.f);
#pragma unroll
                    for (int u = 0; u < CN; ++u) {
                        const int idx = tid + u * nthr, ci = idx / NB, cj = idx % NB;
                        if (idx < NB * NB && !(cur_here && ci == nl)) {
                            DL_GUARD(sx + ci * C::XS + cj, 4) sx[ci * C::XS + cj] = cval[u];
                        }
                    }
                };
                if (bf) stage(bf16{});
                else stage(float{});
                __syncthreads();

                // 2. per key channel, in place: Khat_i = gamma_i o k_i, gamma,
                // F_j = k_j o D(NB-1, j) (padded entries have a = 1, so D(NB-1, j) = D(nb-1, j)),
                // stored at f_pos(c): a column of the same warp (f_pos keeps c's group of 16).
                static_assert(DK <= nthr, "one key channel per thread");
                for (int c = tid; c < DK; c += nthr) {
                    float ac[NB], kc[NB];
#pragma unroll
                    for (int i = 0; i < NB; ++i) {
                        ac[i] = CHAN ? ff[i * C::WS + c] : fa[i];
                        kc[i] = kh[C::kof(i, c)];
                    }
                    float gm = 1.f;
#pragma unroll
                    for (int i = 0; i < NB; ++i) {
                        gm *= ac[i];
                        DL_GUARD(kh + C::kof(i, c), 4) kh[C::kof(i, c)] = gm * kc[i];
                    }
                    DL_GUARD(gn + c, 4) gn[c] = gm;
                    __syncwarp();  // the warp's lanes have read their decays before F lands over them
                    const int fc = f_pos(c);
                    float f = 1.f;
#pragma unroll
                    for (int j = NB - 1; j >= 0; --j) {
                        DL_GUARD(ff + j * C::WS + fc, 4) ff[j * C::WS + fc] = kc[j] * f;
                        f *= ac[j];
                    }
                }
                cp_async_wait_all();  // this thread's share of the base tile has landed
                __syncthreads();
                if constexpr (Q8) {
                    if (b0 == 0) {  // codes * scale into the float tile, 4 at a time
                        constexpr int WPT = ROWS * DK / 4 / nthr;  // code words per thread
                        static_assert(WPT * 4 * nthr == ROWS * DK, "whole words per thread");
                        uint32_t wv[WPT];
#pragma unroll
                        // word u holds the codes of row u / (DK/4), from column 4 (u % (DK/4))
                        for (int i = 0; i < WPT; ++i)
                            wv[i] = *reinterpret_cast<const uint32_t *>(raw + 4 * (tid + i * nthr));
                        __syncthreads();  // every code is in registers before the tile is written over them
#pragma unroll
                        for (int i = 0; i < WPT; ++i) {
                            const int u = tid + i * nthr, r = u / (DK / 4), c4 = (u % (DK / 4)) * 4;
                            const uint32_t w = wv[i];
                            const float sc = scl[r];
                            DL_GUARD(tile + TL::off(r, c4), 16) *reinterpret_cast<float4 *>(tile + TL::off(r, c4)) =
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
                    if (lane < NB) {
                        DL_GUARD(sxw + warp * C::XS + lane, 4)
                        sxw[warp * C::XS + lane] = lane < nl ? -bn * acc : (lane == nl ? bn : 0.f);
                    }
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
                    // G = S Khat^T in the column order above: k-step 2j + h has the A
                    // fragment a0 = S[g][c], a1 = S[g + 8][c], a2 = S[g][c + 1], a3 = S[g + 8][c + 1]
                    // with c = 16j + 4t + 2h, and B fragment Khat[8nt + g][c], Khat[8nt + g][c + 1].
                    // (two accumulator sets, even and odd k-steps, halve the dependent chains)
                    float acc1[NT][4], acc2[NT][4];
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                        for (int x = 0; x < 4; ++x) acc1[nt][x] = acc2[nt][x] = 0.f;
#pragma unroll
                    for (int j = 0; j < DK / 16; ++j) {
                        const float4 x0 = ld_tile4(tile + TL::off(tr + g, 16 * j + 4 * t));
                        const float4 x1 = ld_tile4(tile + TL::off(tr + g + 8, 16 * j + 4 * t));
                        uint32_t ah0[4], al0[4], ah1[4], al1[4];
                        split_tf32(x0.x, ah0[0], al0[0]);
                        split_tf32(x1.x, ah0[1], al0[1]);
                        split_tf32(x0.y, ah0[2], al0[2]);
                        split_tf32(x1.y, ah0[3], al0[3]);
                        split_tf32(x0.z, ah1[0], al1[0]);
                        split_tf32(x1.z, ah1[1], al1[1]);
                        split_tf32(x0.w, ah1[2], al1[2]);
                        split_tf32(x1.w, ah1[3], al1[3]);
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt) {
                            const float4 kv =
                                *reinterpret_cast<const float4 *>(kh + C::kof(8 * nt + g, 16 * j + 4 * t));
                            mma3(acc1[nt], ah0, al0, kv.x, kv.y);
                            mma3(acc2[nt], ah1, al1, kv.z, kv.w);
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
                // S <- S o gamma + delta F, two 16 x 8 column tiles at a time: tiles 2j and
                // 2j + 1 give lane (g, t) columns 16j + 4t .. + 3 of rows g and g + 8 (the
                // column order above); from the tile, back to the tile for a following
                // sub-merge (or, for an int8 base, for the rounding below), else straight
                // to HBM.
                float rmax0 = 0.f, rmax1 = 0.f;  // int8 base: |value| maxima of rows g, g + 8 (this lane's columns)
#pragma unroll 2
                for (int j = 0; j < DK / 16; ++j) {
                    float d[2][4];  // tile 2j + h: rows g, g + 8 at columns 16j + 4t + 2h, + 1
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        float dn[NT][4];  // one accumulator per entry tile: independent chains
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
                            for (int x = 0; x < 4; ++x) dn[nt][x] = 0.f;
                            const float *fp = ff + (8 * nt + t) * C::WS + 16 * j + 8 * h + g;
                            mma3(dn[nt], xh[nt], xl[nt], fp[0], fp[4 * C::WS]);
                        }
#pragma unroll
                        for (int x = 0; x < 4; ++x) {
                            d[h][x] = dn[0][x];
#pragma unroll
                            for (int nt = 1; nt < NT; ++nt) d[h][x] += dn[nt][x];
                        }
                    }
                    const int col = 16 * j + 4 * t;
                    TT *p0 = tile + TL::off(tr + g, col), *p1 = tile + TL::off(tr + g + 8, col);
                    const float4 r0 = ld_tile4(p0), r1 = ld_tile4(p1);
                    const float4 gv = *reinterpret_cast<const float4 *>(gn + col);
                    const float4 s0 = make_float4(fmaf(r0.x, gv.x, d[0][0]), fmaf(r0.y, gv.y, d[0][1]),
                                                  fmaf(r0.z, gv.z, d[1][0]), fmaf(r0.w, gv.w, d[1][1]));
                    const float4 s1 = make_float4(fmaf(r1.x, gv.x, d[0][2]), fmaf(r1.y, gv.y, d[0][3]),
                                                  fmaf(r1.z, gv.z, d[1][2]), fmaf(r1.w, gv.w, d[1][3]));
                    if (WITH_CUR && last) {
                        const float4 qv = *reinterpret_cast<const float4 *>(sq + col);
                        oacc[0] = fmaf(s0.x, qv.x, fmaf(s0.y, qv.y, fmaf(s0.z, qv.z, fmaf(s0.w, qv.w, oacc[0]))));
                        oacc[1] = fmaf(s1.x, qv.x, fmaf(s1.y, qv.y, fmaf(s1.z, qv.z, fmaf(s1.w, qv.w, oacc[1]))));
                    }
                    if constexpr (Q8) {
                        DL_GUARD(p0, 4 * sizeof(TT)) st_tile4(p0, s0);
                        DL_GUARD(p1, 4 * sizeof(TT)) st_tile4(p1, s1);
                        rmax0 = fmaxf(rmax0, fmaxf(fmaxf(fabsf(s0.x), fabsf(s0.y)), fmaxf(fabsf(s0.z), fabsf(s0.w))));
                        rmax1 = fmaxf(rmax1, fmaxf(fmaxf(fabsf(s1.x), fabsf(s1.y)), fmaxf(fabsf(s1.z), fabsf(s1.w))));
                    } else if (last) {
                        st_state4(Sw + g * DK + col, s0);
                        st_state4(Sw + (g + 8) * DK + col, s1);
                    } else {
                        DL_GUARD(p0, 4 * sizeof(TT)) st_tile4(p0, s0);
                        DL_GUARD(p1, 4 * sizeof(TT)) st_tile4(p1, s1);
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
                            DL_GUARD(wsc + warp * 16 + g, 4) wsc[warp * 16 + g] = i8_scale(rmax0);
                            DL_GUARD(wsc + warp * 16 + g + 8, 4) wsc[warp * 16 + g + 8] = i8_scale(rmax1);
                        }
                        __syncwarp();
                        constexpr int CPR = DK / 16;  // 16-code chunks per row
                        for (int i = lane; i < 16 * CPR; i += 32) {
                            const int rl = i / CPR, c0 = (i % CPR) * 16;
                            const float sc = wsc[warp * 16 + rl], inv = i8_inv(sc);
                            const bool fast = i8_fast(sc);
                            uint32_t wd[4];
#pragma unroll
                            for (int qd = 0; qd < 4; ++qd) {
                                const float4 x =
                                    *reinterpret_cast<const float4 *>(tile + TL::off(tr + rl, c0 + 4 * qd));
                                wd[qd] = fast ? i8_pack4<true>(x.x, x.y, x.z, x.w, sc, inv)
                                              : i8_pack4<false>(x.x, x.y, x.z, x.w, sc, inv);
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
        if (!compact) break;
        __syncthreads();  // thread 0's update of the walk is visible to all
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
    const long long units = (long long)p.B * p.H * (p.dv / rows);
    long long blocks = units;
    if (pool.slot && part == POOL_MERGE_FULL) {
        // only the slots on their L-th entry merge: a compact grid of as many blocks
        // as can be resident (4 per SM) walks all units and merges those
        int dev = 0, sms = 0;
        e = cudaGetDevice(&dev);
        if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return e;
        blocks = std::min<long long>(units, 4LL * sms);
    }
    // an int8 base's row scales follow its codes (all the state's heads: the pool's, or B*H)
    const long long state_heads = pool.slot ? (long long)pool.P * pool.H : (long long)p.B * p.H;
    float *i8_scales = std::is_same<ST, int8_t>::value
                           ? reinterpret_cast<float *>(static_cast<int8_t *>(p.S) + state_heads * p.dv * DK)
                           : nullptr;
    kern<<<(unsigned)blocks, rows * 2, smem, st>>>(static_cast<ST *>(p.S), lg.k, lg.v, lg.beta, lg.a, lg.x, lg.L,
                                                   n_log, p.q, p.k, p.v, p.beta, p.a, p.o, p.dv,
                                                   p.in_dt == DL_BF16, pool, part, i8_scales, units);
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
    // An fp32 or int8 base with d_k = 128 and at most 16 entries to merge goes
    // to the tcgen05 kernel (merge_tc.cu); every other case runs here.
    if (merge_tc_supported(p, n_log, with_cur, pool)) return launch_merge_tc(p, lg, n_log, with_cur, st);
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

// The guard word of this file's kernels (index-guard build; 0 otherwise).
cudaError_t read_guard_merge(unsigned int *flags, unsigned int *line, bool clear) {
    return read_guard_word(flags, line, clear);
}

}  // namespace dl
