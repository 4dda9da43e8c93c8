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
__device__ __forceinline__ void ld_state2(const float *p, float &x, float &y) {
    const float2 v = *reinterpret_cast<const float2 *>(p);
    x = v.x;
    y = v.y;
}
__device__ __forceinline__ void ld_state2(const bf16 *p, float &x, float &y) {
    const uint32_t w = *reinterpret_cast<const uint32_t *>(p);
    x = bf_lo(w);
    y = bf_hi(w);
}
__device__ __forceinline__ void st_state2(float *p, float x, float y) {
    __stcs(reinterpret_cast<float2 *>(p), make_float2(x, y));
}
__device__ __forceinline__ void st_state2(bf16 *p, float x, float y) {
    __stcs(reinterpret_cast<unsigned int *>(p), pack_bf2(x, y));
}

// ------------------------------------------------------------------ layout

__host__ __device__ constexpr size_t round4(size_t x) { return (x + 3) & ~(size_t)3; }

template <int DK>
struct MergeShape {
    static constexpr int KH = DK + 4;   // Khat row stride (conflict-free B-fragment reads)
    static constexpr int WS = DK + 8;   // W row stride (conflict-free B-fragment reads)
    static constexpr int CW = DK / 32;  // key channels per lane (warp-wide dots)
    __host__ __device__ static constexpr int rows(int dv) { return 64; }  // 4 warps per block
};

// Shared memory for one block of NB entries (all float):
//   fk [NB][DK] keys   fa: channel decay [NB][DK] or head decay [NB] (padded to 4)
//   ff [NB][DK] F      kh [NB][KH] Khat   sw [NB][WS] W
//   gn [DK] gamma      sq [DK] q          cm [NB] C row   sx [NB][NB] X   sb [NB] beta
//   sv [NB][rows] the tile's values
template <int DK, bool CHAN, int NB>
__host__ __device__ constexpr size_t merge_smem_bytes(int rows) {
    using C = MergeShape<DK>;
    const size_t floats = (size_t)NB * DK + (CHAN ? (size_t)NB * DK : round4(NB)) + (size_t)NB * DK +
                          (size_t)NB * C::KH + (size_t)NB * C::WS + DK + DK + round4(NB) + (size_t)NB * NB + round4(NB) +
                          (size_t)NB * rows;
    return floats * sizeof(float);
}

// ------------------------------------------------------------------ kernel

template <class ST, int DK, bool CHAN, bool WITH_CUR, int NB>
__global__ void __launch_bounds__(256, 2)
merge_kernel(ST *__restrict__ S, const void *__restrict__ log_k, const void *__restrict__ log_v,
             const void *__restrict__ log_b, const void *__restrict__ log_a, const float *__restrict__ log_x,
             int L, int n_log, const void *__restrict__ q, const void *__restrict__ k, const void *__restrict__ v,
             const void *__restrict__ beta, const void *__restrict__ a, float *__restrict__ o, int DV, bool bf) {
    using C = MergeShape<DK>;
    constexpr int KS = DK / 8;   // k-steps of the first product / column tiles of the second
    constexpr int NT = NB / 8;   // entry tiles
    const int ROWS = blockDim.x / 2;  // 16 rows per warp
    const int nthr = blockDim.x;
    const int NTOT = n_log + (WITH_CUR ? 1 : 0);

    extern __shared__ float4 smem_raw[];
    float *fk = reinterpret_cast<float *>(smem_raw);
    float *fa = fk + NB * DK;
    float *ff = fa + (CHAN ? NB * DK : (int)round4(NB));
    float *kh = ff + NB * DK;
    float *sw = kh + NB * C::KH;
    float *gn = sw + NB * C::WS;
    float *sq = gn + DK;
    float *cm = sq + DK;
    float *sx = cm + round4(NB);
    float *sb = sx + NB * NB;
    float *sv = sb + round4(NB);

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, t = lane & 3;  // fragment coordinates
    const int tiles = DV / ROWS;
    const long long head = blockIdx.x / tiles;
    const int row0 = (blockIdx.x % tiles) * ROWS;
    const long long lrow = head * L;
    ST *Sw = S + (head * DV + row0 + 16 * warp) * DK;  // this warp's 16 rows

    // First-product operand fragments of the warp's rows, fetched before anything
    // else (they land while the key side is prepared): a0 = S[g][8s + t],
    // a1 = S[g + 8][8s + t], a2 = S[g][8s + t + 4], a3 = S[g + 8][8s + t + 4].
    float afr[KS][4];
    auto load_afr = [&]() {
#pragma unroll
        for (int s = 0; s < KS; ++s) {
            afr[s][0] = ld_state(Sw + g * DK + 8 * s + t);
            afr[s][1] = ld_state(Sw + (g + 8) * DK + 8 * s + t);
            afr[s][2] = ld_state(Sw + g * DK + 8 * s + t + 4);
            afr[s][3] = ld_state(Sw + (g + 8) * DK + 8 * s + t + 4);
        }
    };
    if constexpr (WITH_CUR) {
        if (bf) stage_block(sq, DK, static_cast<const bf16 *>(q) + head * DK, DK, 1, DK, tid, nthr);
        else stage_block(sq, DK, static_cast<const float *>(q) + head * DK, DK, 1, DK, tid, nthr);
    }

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
            float kx[KN][E], ax[KN][E], vx[VN][E];
            (void)ax;
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
                cval[u] = (idx < NB * NB && cj <= ci && ci < nl) ? log_x[(lrow + b0 + ci) * L + b0 + cj] : 0.f;
            }
#pragma unroll
            for (int u = 0; u < KN; ++u) {
                const int c = tid + u * nthr, r = c / KC, col = (c % KC) * E;
                if (c < NB * KC) {
                    const bool real = r < nb;  // padded entries: k = 0, a = 1
#pragma unroll
                    for (int e = 0; e < E; ++e) {
                        fk[r * DK + col + e] = real ? kx[u][e] : 0.f;
                        if constexpr (CHAN) fa[r * DK + col + e] = real ? ax[u][e] : 1.f;
                    }
                }
            }
#pragma unroll
            for (int u = 0; u < VN; ++u) {
                const int c = tid + u * nthr, r = c / VC, col = (c % VC) * E;
                if (c < NB * VC) {
#pragma unroll
                    for (int e = 0; e < E; ++e) sv[r * ROWS + col + e] = r < nb ? vx[u][e] : 0.f;
                }
            }
            if (tid < NB) {
                sb[tid] = bsc;  // 0 for padded entries
                if constexpr (!CHAN) fa[tid] = asc;
            }
#pragma unroll
            for (int u = 0; u < CN; ++u) {
                const int idx = tid + u * nthr, ci = idx / NB;
                if (idx < NB * NB && !(cur_here && ci == nl)) sx[idx] = cval[u];
            }
        };
        if (bf) stage(bf16{});
        else stage(float{});
        __syncthreads();

        // 2. per key channel: Khat_i = gamma_i o k_i, gamma, F_j = k_j o D(nb-1, j).
        for (int c = tid; c < DK; c += nthr) {
            float ac[NB];
#pragma unroll
            for (int i = 0; i < NB; ++i) ac[i] = CHAN ? fa[i * DK + c] : fa[i];
            float gm = 1.f;
#pragma unroll
            for (int i = 0; i < NB; ++i) {
                gm *= ac[i];
                kh[i * C::KH + c] = gm * fk[i * DK + c];
            }
            gn[c] = gm;
            float f = 1.f;
#pragma unroll
            for (int j = NB - 1; j >= 0; --j) {
                ff[j * DK + c] = fk[j * DK + c] * f;
                f *= ac[j];
            }
        }
        __syncthreads();
        // The fused read's current entry is the block's last real one, so
        // D(nl, j) is F_j's suffix product: C(nl, j) = k_nl . F_j.
        if (cur_here) {
            for (int j = warp; j < nl; j += nthr / 32) {
                float pj = 0.f;
#pragma unroll
                for (int e = 0; e < C::CW; ++e) {
                    const int c = e * 32 + lane;
                    pj = fmaf(fk[nl * DK + c], ff[j * DK + c], pj);
                }
                pj = group_sum<32>(pj);
                if (lane == 0) cm[j] = pj;
            }
            __syncthreads();
            // its X row: X(nl, nl) = beta, X(nl, j) = -beta sum_{m=j..nl-1} C(nl, m) X(m, j)
            if (tid < NB) {
                const int j = tid;
                float acc = 0.f;
                for (int m = j; m < nl; ++m) acc = fmaf(cm[m], sx[m * NB + j], acc);
                sx[nl * NB + j] = j < nl ? -sb[nl] * acc : (j == nl ? sb[nl] : 0.f);
            }
            __syncthreads();
        }

        // 3. W = X^T F: W[j][c] = sum_{i>=j} X(i, j) F[i][c].
        for (int u = tid; u < NB * DK; u += nthr) {
            const int j = u / DK, c = u % DK;
            float acc = 0.f;
#pragma unroll
            for (int i = 0; i < NB; ++i) acc = fmaf(sx[i * NB + j], ff[i * DK + c], acc);
            sw[j * C::WS + c] = acc;
        }
        __syncthreads();

        // 4. this warp's 16 rows. G = S Khat^T.
        __syncwarp();  // a previous block's rows, written by this warp, are visible
        load_afr();
        float acc1[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int x = 0; x < 4; ++x) acc1[nt][x] = 0.f;
#pragma unroll
        for (int s = 0; s < KS; ++s) {
            uint32_t ah[4], al[4];
#pragma unroll
            for (int x = 0; x < 4; ++x) split_tf32(afr[s][x], ah[x], al[x]);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const float *kp = kh + (8 * nt + g) * C::KH + 8 * s + t;
                mma3(acc1[nt], ah, al, kp[0], kp[4]);
            }
        }
        // E = V - G (accumulator layout: rows g, g + 8; entries 8nt + 2t, 8nt + 2t + 1),
        // then moved to operand layout (entries 8nt + t, 8nt + t + 4) within each quad.
        const int rg = 16 * warp + g;
        uint32_t eh[NT][4], el[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int i0 = 8 * nt + 2 * t;
            const float e0 = sv[i0 * ROWS + rg] - acc1[nt][0];
            const float e1 = sv[(i0 + 1) * ROWS + rg] - acc1[nt][1];
            const float e2 = sv[i0 * ROWS + rg + 8] - acc1[nt][2];
            const float e3 = sv[(i0 + 1) * ROWS + rg + 8] - acc1[nt][3];
            const int s0 = (lane & ~3) | (t >> 1), s1 = s0 + 2;  // quad lanes holding entries t, t + 4
            const float x00 = __shfl_sync(0xffffffffu, e0, s0), x01 = __shfl_sync(0xffffffffu, e1, s0);
            const float x10 = __shfl_sync(0xffffffffu, e2, s0), x11 = __shfl_sync(0xffffffffu, e3, s0);
            const float y00 = __shfl_sync(0xffffffffu, e0, s1), y01 = __shfl_sync(0xffffffffu, e1, s1);
            const float y10 = __shfl_sync(0xffffffffu, e2, s1), y11 = __shfl_sync(0xffffffffu, e3, s1);
            const bool odd = t & 1;
            split_tf32(odd ? x01 : x00, eh[nt][0], el[nt][0]);  // E[g][8nt + t]
            split_tf32(odd ? x11 : x10, eh[nt][1], el[nt][1]);  // E[g + 8][8nt + t]
            split_tf32(odd ? y01 : y00, eh[nt][2], el[nt][2]);  // E[g][8nt + t + 4]
            split_tf32(odd ? y11 : y10, eh[nt][3], el[nt][3]);  // E[g + 8][8nt + t + 4]
        }
        // S <- S o gamma + E W, one 16 x 8 column tile at a time, written straight
        // from the accumulator layout (rows g, g + 8; columns 8c + 2t, 8c + 2t + 1).
#pragma unroll 4
        for (int cb = 0; cb < KS; ++cb) {
            float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const float *wp = sw + (8 * nt + t) * C::WS + 8 * cb + g;
                mma3(d, eh[nt], el[nt], wp[0], wp[4 * C::WS]);
            }
            const int col = 8 * cb + 2 * t;
            float s00, s01, s10, s11;
            ld_state2(Sw + g * DK + col, s00, s01);
            ld_state2(Sw + (g + 8) * DK + col, s10, s11);
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
            st_state2(Sw + g * DK + col, s00, s01);
            st_state2(Sw + (g + 8) * DK + col, s10, s11);
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

template <class ST, int DK, bool CHAN, bool WC, int NB>
static cudaError_t launch_merge_t(const StepParams &p, const LogParams &lg, int n_log, cudaStream_t st) {
    using C = MergeShape<DK>;
    auto kern = merge_kernel<ST, DK, CHAN, WC, NB>;
    const int rows = C::rows(p.dv);
    const size_t smem = merge_smem_bytes<DK, CHAN, NB>(rows);
    static bool configured = false;
    if (!configured) {
        const size_t want = merge_smem_bytes<DK, CHAN, NB>(rows);
        if (want > 48 * 1024) {
            cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)want);
            if (e != cudaSuccess) return e;
        }
        configured = true;
    }
    const long long blocks = (long long)p.B * p.H * (p.dv / rows);
    kern<<<(unsigned)blocks, rows * 2, smem, st>>>(static_cast<ST *>(p.S), lg.k, lg.v, lg.beta, lg.a, lg.x, lg.L,
                                                   n_log, p.q, p.k, p.v, p.beta, p.a, p.o, p.dv,
                                                   p.in_dt == DL_BF16);
    return cudaGetLastError();
}

// Entry-block size: 8 when all entries fit, else 16 (a longer log runs as a
// chain of 16-entry sub-merges, the last one padded).
template <class ST, int DK, bool CHAN, bool WC>
static cudaError_t launch_merge_nb(const StepParams &p, const LogParams &lg, int n_log, cudaStream_t st) {
    const int nt = n_log + (WC ? 1 : 0);
    if (nt <= 8) return launch_merge_t<ST, DK, CHAN, WC, 8>(p, lg, n_log, st);
    return launch_merge_t<ST, DK, CHAN, WC, 16>(p, lg, n_log, st);
}

cudaError_t launch_merge(const StepParams &p, const LogParams &lg, int n_log, bool with_cur, cudaStream_t st) {
    // The input dtype and d_v are run-time arguments of the merge kernel (they
    // only change staging and the grid), which keeps instantiations few.
    auto go = [&](auto st_t, auto dk_c) -> cudaError_t {
        using ST = decltype(st_t);
        constexpr int DK = decltype(dk_c)::value;
        if (p.chan) {
            if (with_cur) return launch_merge_nb<ST, DK, true, true>(p, lg, n_log, st);
            return launch_merge_nb<ST, DK, true, false>(p, lg, n_log, st);
        }
        if (with_cur) return launch_merge_nb<ST, DK, false, true>(p, lg, n_log, st);
        return launch_merge_nb<ST, DK, false, false>(p, lg, n_log, st);
    };
    auto with_dk = [&](auto st_t) -> cudaError_t {
        if (p.dk == 64) return go(st_t, std::integral_constant<int, 64>{});
        return go(st_t, std::integral_constant<int, 128>{});
    };
    if (p.s_dt == DL_BF16) return with_dk(bf16{});
    return with_dk(float{});
}

}  // namespace dl
