// Merge of the bounded log into the dense base (DeltaLog page, Technical
// Summary, "Merge Phase": every M steps the accumulated logical state -- base
// plus replayed log entries -- is materialised back into the base), and the
// same merge fused with one step's read.
//
// Log-decay form. For log entries 1..n (decays a_i, keys k_i, values v_i,
// strengths beta_i) write D(i, j) = prod_{m=j+1..i} a_m (= exp(Lambda_i -
// Lambda_j) with the page's log-decay metadata Lambda), gamma_i = D(i, 0).
// Every row s_bar of the base evolves independently:
//   s_i = s_bar o gamma_i + sum_{j<=i} delta_j (k_j o D(i, j)),
//   delta_i = beta_i (v_i[r] - G_i - sum_{j<i} C(i, j) delta_j),
//   G_i = s_bar . (gamma_i o k_i),   C(i, j) = sum_c k_i[c] D(i, j)[c] k_j[c],
// and the merged row is s_n = s_bar o gamma_n + sum_j delta_j F_j with
// F_j = k_j o D(n, j). Per head this is two thin contractions of the base
// (G = S_bar Khat^T, then delta F) around an n x n triangular solve per row:
// 4 n d_k d_v FLOP against 2 d_k d_v state elements moved, about 4 FMA per
// state byte at n = 16 -- close to the B200's CUDA-core/HBM balance.
//
// Kernel: one 256-thread block per (head, 64-row value tile); four adjacent
// lanes share a row, each holding every fourth 16-byte chunk of it in
// registers, so the base is read and written with coalesced 64-byte runs and
// never staged in shared memory. The n entries are merged in blocks of at
// most 16 -- merging n entries is the same as merging the first 16 and then
// the next 16 into the result -- with the row kept in fp32 registers between
// blocks and rounded to the state dtype once, at the end.
//  1. The block issues its base loads first (they land during 2-3).
//  2. Per entry block, the key side is staged into shared memory: k, a,
//     beta, the tile's values.
//  3. One thread per key channel forms Khat_i = gamma_i o k_i, F_j and
//     gamma_n from running decay products. C(i, j) comes from the log
//     metadata (the append that logged entry i computed it); the fused read's
//     current entry is the block's last, so its row is just k_n . F_j.
//  4. Each thread contracts its columns of the row against Khat (the four
//     lanes of a row read four adjacent chunks: one broadcast wavefront),
//     the row's partial G are summed over its four lanes, delta is solved
//     in registers and the row updated. After the last block the row is
//     streamed out; the fused read also forms o = s_new . q.
#include "launch.h"

namespace dl {

template <class ST, int DK>
struct MergeShape {
    static constexpr int VEC = StateVec<ST>::N;              // elements per 16-byte chunk
    static constexpr int CPR = DK * (int)sizeof(ST) / 16;     // chunks per row
    static constexpr int TPR = 4;                             // threads per row
    static constexpr int CPT = CPR / TPR;                     // chunks per thread
    static constexpr int ROWS = 64;                           // rows per block
    static constexpr int THREADS = ROWS * TPR;
    static constexpr int WARPS = THREADS / 32;
    static constexpr int CW = DK / 32;                        // key channels per lane (C matrix)
    // base tile rows in shared memory, padded by 64 bytes so that the eight
    // lanes of a quarter-warp (two rows x four chunks) hit distinct banks
    static constexpr int TSTRIDE = CPR * 16 + 64;
    static constexpr int TILE_BYTES = ROWS * TSTRIDE;
    static_assert(CPT >= 1 && CPT * TPR == CPR, "row split");
};

// One input element (fp32 or bf16, chosen at run time) widened to float.
__device__ __forceinline__ float ld_in(const void *p, long long i, bool bf) {
    return bf ? to_f(static_cast<const bf16 *>(p)[i]) : static_cast<const float *>(p)[i];
}

__host__ __device__ constexpr size_t round4(size_t x) { return (x + 3) & ~(size_t)3; }

// Shared-memory layout after the base tile, for one block of NB entries
// (all float):
//   fk [nb][DK]  keys                                 (16-byte aligned)
//   fa           channel decay: [nb][DK]; head decay: nb scalars (padded to 4)
//   kh [nb][DK]  Khat_i = gamma_i o k_i
//   ff [nb][DK]  F_j = k_j o D(nb, j)
//   gn [DK], sq [DK]                                  (vector reads)
//   cm [nb][nb], sb [nb], sv [nb][ROWS]               (scalar reads)
template <class ST, int DK, bool CHAN, int NB>
__host__ __device__ constexpr size_t merge_smem_bytes() {
    using C = MergeShape<ST, DK>;
    constexpr int nb = NB, rows = C::ROWS;
    const size_t floats = (size_t)nb * DK + (CHAN ? (size_t)nb * DK : round4(nb)) + 2 * (size_t)nb * DK + DK +
                          DK + (size_t)nb * nb + nb + (size_t)nb * rows;
    return (size_t)C::TILE_BYTES + floats * sizeof(float);
}

template <class ST, int DK, bool CHAN, bool WITH_CUR, int NB>
__global__ void __launch_bounds__(256, 2)
merge_kernel(ST *__restrict__ S, const void *__restrict__ log_k, const void *__restrict__ log_v,
             const void *__restrict__ log_b, const void *__restrict__ log_a, const float *__restrict__ log_c,
             int L, int n_log,
             const void *__restrict__ q, const void *__restrict__ k, const void *__restrict__ v,
             const void *__restrict__ beta, const void *__restrict__ a, float *__restrict__ o, int DV,
             bool bf) {
    using C = MergeShape<ST, DK>;
    constexpr int VEC = C::VEC, ROWS = C::ROWS, EPT = C::CPT * VEC;
    const int NT = n_log + (WITH_CUR ? 1 : 0);  // entries merged

    extern __shared__ float4 smem_raw[];
    unsigned char *tile = reinterpret_cast<unsigned char *>(smem_raw);         // the base tile
    float *fk = reinterpret_cast<float *>(tile + C::TILE_BYTES);  // keys
    float *fa = fk + (size_t)NB * DK;                             // decays
    float *kh = fa + (CHAN ? (size_t)NB * DK : round4(NB));       // Khat
    float *ff = kh + (size_t)NB * DK;                             // F
    float *gn = ff + (size_t)NB * DK;
    float *sq = gn + DK;
    float *cm = sq + DK;
    float *sb = cm + (size_t)NB * NB;
    float *sv = sb + NB;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int tiles = DV / ROWS;
    const long long head = blockIdx.x / tiles;
    const int row0 = (blockIdx.x % tiles) * ROWS;
    const int rl = tid / C::TPR, part = tid % C::TPR;  // row in tile, which quarter of the chunks
    ST *grow = S + (head * DV + row0 + rl) * DK;
    const long long lrow = head * L;

    // 1. the base tile -> padded shared rows, asynchronously (no registers held);
    // issued right after the first entry block's key-side loads, so the small
    // operands are not queued behind the 32-64 KB of state.
    auto issue_tile = [&]() {
        const unsigned char *gt = reinterpret_cast<const unsigned char *>(S + (head * DV + row0) * DK);
#pragma unroll
        for (int u = 0; u < C::CPT; ++u) {
            const int g = tid + u * C::THREADS, r = g / C::CPR, c = g % C::CPR;
            cp_async16(tile + r * C::TSTRIDE + c * 16, gt + (size_t)r * (C::CPR * 16) + c * 16);
        }
        cp_async_commit();
    };
    if constexpr (WITH_CUR) {
        if (bf) stage_block(sq, DK, static_cast<const bf16 *>(q) + head * DK, DK, 1, DK, tid, C::THREADS);
        else stage_block(sq, DK, static_cast<const float *>(q) + head * DK, DK, 1, DK, tid, C::THREADS);
    }

    float srow[EPT];  // this thread's columns of the row, fp32, across entry blocks
    for (int b0 = 0; b0 < NT; b0 += NB) {
        const int nb = NT - b0 < NB ? NT - b0 : NB;
        const int nl = (n_log - b0 < nb ? n_log - b0 : nb);  // of which from the log (the rest: this step)

        // 2. entries b0 .. b0+nb-1: log entries, then (fused read) this step's.
        // Every global load of the block is issued before the first shared store.
        auto stage = [&](auto tag) {
            using IT = decltype(tag);
            constexpr int E = 16 / (int)sizeof(IT);      // elements per 16-byte chunk
            constexpr int KC = DK / E, VC = ROWS / E;     // chunks per key row / per value slice
            constexpr int KN = (NB * KC + C::THREADS - 1) / C::THREADS;
            constexpr int VN = (NB * VC + C::THREADS - 1) / C::THREADS;
            float kx[KN][E], ax[KN][E], vx[VN][E];
            (void)ax;
            auto key_src = [&](const void *logp, const void *cur, int r) -> const IT * {
                return r < nl ? static_cast<const IT *>(logp) + (lrow + b0 + r) * DK
                              : static_cast<const IT *>(cur) + head * DK;
            };
#pragma unroll
            for (int u = 0; u < KN; ++u) {
                const int c = tid + u * C::THREADS, r = c / KC, col = (c % KC) * E;
                if (r < nb) {
                    load_vec<E>(key_src(log_k, k, r) + col, kx[u]);
                    if constexpr (CHAN) load_vec<E>(key_src(log_a, a, r) + col, ax[u]);
                }
            }
#pragma unroll
            for (int u = 0; u < VN; ++u) {
                const int c = tid + u * C::THREADS, r = c / VC, col = (c % VC) * E;
                if (r < nb) {
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
            // C(i, j) for the logged entries of the block (the current entry's row,
            // if any, is formed below); zero elsewhere.
            float cval = 0.f;
            const int ci = tid / NB, cj = tid % NB;
            if (tid < NB * NB && cj < ci && ci < nl) cval = log_c[(lrow + b0 + ci) * L + b0 + cj];
            if (b0 == 0) issue_tile();
#pragma unroll
            for (int u = 0; u < KN; ++u) {
                const int c = tid + u * C::THREADS, r = c / KC, col = (c % KC) * E;
                if (r < nb) {
#pragma unroll
                    for (int e = 0; e < E; ++e) {
                        fk[r * DK + col + e] = kx[u][e];
                        if constexpr (CHAN) fa[r * DK + col + e] = ax[u][e];
                    }
                }
            }
#pragma unroll
            for (int u = 0; u < VN; ++u) {
                const int c = tid + u * C::THREADS, r = c / VC, col = (c % VC) * E;
                if (r < nb) {
#pragma unroll
                    for (int e = 0; e < E; ++e) sv[r * ROWS + col + e] = vx[u][e];
                }
            }
            if (tid < nb) {
                sb[tid] = bsc;
                if constexpr (!CHAN) fa[tid] = asc;
            }
            if (tid < NB * NB && !(WITH_CUR && nl < nb && ci == nl && cj < nl)) cm[tid] = cval;
        };
        if (bf) stage(bf16{});
        else stage(float{});
        // Entries nb..NB-1 of a short block are neutral: k = 0, a = 1, beta = 0,
        // v = 0 leave gamma, F and every delta unchanged, so all loops below run
        // over the full compile-time NB without bound checks.
        for (int i = nb * DK + tid; i < NB * DK; i += C::THREADS) {
            fk[i] = 0.f;
            if constexpr (CHAN) fa[i] = 1.f;
        }
        for (int i = nb + tid; i < NB; i += C::THREADS) {
            if constexpr (!CHAN) fa[i] = 1.f;
            sb[i] = 0.f;
        }
        for (int i = nb * ROWS + tid; i < NB * ROWS; i += C::THREADS) sv[i] = 0.f;
        __syncthreads();

        // 3. Per key channel: Khat_i = gamma_i o k_i, gamma_nb and F_j = k_j o D(nb, j)
        // (running decay products; padded entries have a = 1).
        for (int c = tid; c < DK; c += C::THREADS) {
            float ac[NB];
#pragma unroll
            for (int i = 0; i < NB; ++i) ac[i] = CHAN ? fa[i * DK + c] : fa[i];
            float g = 1.f;
#pragma unroll
            for (int i = 0; i < NB; ++i) {
                g *= ac[i];
                kh[i * DK + c] = g * fk[i * DK + c];
            }
            gn[c] = g;
            float f = 1.f;
#pragma unroll
            for (int j = NB - 1; j >= 0; --j) {
                ff[j * DK + c] = fk[j * DK + c] * f;
                f *= ac[j];
            }
        }
        __syncthreads();
        // C(i, j) = sum_c k_i[c] k_j[c] prod_{m=j+1..i} a_m[c] for j < i came with the
        // staging (logged entries carry their rows). The fused read's current
        // entry is the block's last real entry nl, so D(nl, j) is the suffix
        // product of F_j and its row is a plain dot: C(nl, j) = k_nl . F_j.
        const bool cur_here = WITH_CUR && nl < nb;
        if (cur_here) {
            for (int j = warp; j < nl; j += C::WARPS) {
                float pj = 0.f;
#pragma unroll
                for (int e = 0; e < C::CW; ++e) {
                    const int c = e * 32 + lane;
                    pj = fmaf(fk[nl * DK + c], ff[j * DK + c], pj);
                }
                pj = group_sum<32>(pj);
                if (lane == 0) cm[nl * NB + j] = pj;
            }
        }

        if (b0 == 0) {  // this thread's chunks of its row: chunk part + 4 m
            cp_async_wait_all();
            __syncthreads();
#pragma unroll
            for (int m = 0; m < C::CPT; ++m) {
                float x[VEC];
                StateVec<ST>::unpack(
                    *reinterpret_cast<const uint4 *>(tile + rl * C::TSTRIDE + (part + C::TPR * m) * 16), x);
#pragma unroll
                for (int e = 0; e < VEC; ++e) srow[m * VEC + e] = x[e];
            }
        }

        // 4. G_i = s . Khat_i over this thread's columns, then over the row's 4 lanes.
        // Entry-outer loops: one uniform bound check per entry, and every shared
        // load a compile-time offset from one per-thread base.
        const float *khp = kh + part * VEC, *fkp = ff + part * VEC;
        float acc[NB];
#pragma unroll
        for (int i = 0; i < NB; ++i) {
            float p0 = 0.f, p1 = 0.f;  // two partial chains per entry
#pragma unroll
            for (int m = 0; m < C::CPT; ++m) {
                float kv[VEC];
                load_vec<VEC>(khp + i * DK + m * C::TPR * VEC, kv);
#pragma unroll
                for (int e = 0; e < VEC; ++e) {
                    if ((m + e) & 1) p1 = fmaf(srow[m * VEC + e], kv[e], p1);
                    else p0 = fmaf(srow[m * VEC + e], kv[e], p0);
                }
            }
            acc[i] = group_sum<C::TPR>(p0 + p1);
        }
        if (cur_here) __syncthreads();  // the current entry's C row is complete
        // forward substitution (each of the 4 lanes redundantly): acc <- delta
#pragma unroll
        for (int i = 0; i < NB; ++i) {
            float t = sv[i * ROWS + rl] - acc[i];
#pragma unroll
            for (int j = 0; j < i; ++j) t = fmaf(-cm[i * NB + j], acc[j], t);
            acc[i] = sb[i] * t;
        }
        // s <- s o gamma_nb + sum_j delta_j F_j
#pragma unroll
        for (int m = 0; m < C::CPT; ++m) {
            float gv[VEC];
            load_vec<VEC>(gn + part * VEC + m * C::TPR * VEC, gv);
#pragma unroll
            for (int e = 0; e < VEC; ++e) srow[m * VEC + e] *= gv[e];
        }
#pragma unroll
        for (int j = 0; j < NB; ++j) {
            const float dj = acc[j];
#pragma unroll
            for (int m = 0; m < C::CPT; ++m) {
                float fv[VEC];
                load_vec<VEC>(fkp + j * DK + m * C::TPR * VEC, fv);
#pragma unroll
                for (int e = 0; e < VEC; ++e) srow[m * VEC + e] = fmaf(dj, fv[e], srow[m * VEC + e]);
            }
        }
        __syncthreads();  // the next entry block reuses the shared buffers
    }

    // 5. the merged row, streamed back (rounded once for a bf16 state); o = s_new . q (fused read).
    float oacc = 0.f;
#pragma unroll
    for (int m = 0; m < C::CPT; ++m) {
        const int c0 = (part + C::TPR * m) * VEC;
        float x[VEC];
#pragma unroll
        for (int e = 0; e < VEC; ++e) x[e] = srow[m * VEC + e];
        if constexpr (WITH_CUR) {
            float qv[VEC];
            load_vec<VEC>(sq + c0, qv);
#pragma unroll
            for (int e = 0; e < VEC; ++e) oacc = fmaf(x[e], qv[e], oacc);
        }
        st_stream(grow + c0, StateVec<ST>::pack(x));
    }
    if constexpr (WITH_CUR) {
        oacc = group_sum<C::TPR>(oacc);
        if (part == 0) o[head * DV + row0 + rl] = oacc;
    }
}

template <class ST, int DK, bool CHAN, bool WC, int NB>
static cudaError_t launch_merge_t(const StepParams &p, const LogParams &lg, int n_log, cudaStream_t st) {
    using C = MergeShape<ST, DK>;
    auto kern = merge_kernel<ST, DK, CHAN, WC, NB>;
    const size_t smem = merge_smem_bytes<ST, DK, CHAN, NB>();
    static bool configured = false;
    if (!configured && smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        configured = true;
    }
    const long long blocks = (long long)p.B * p.H * (p.dv / C::ROWS);
    kern<<<(unsigned)blocks, C::THREADS, smem, st>>>(static_cast<ST *>(p.S), lg.k, lg.v, lg.beta, lg.a, lg.c,
                                                    lg.L, n_log, p.q, p.k, p.v, p.beta, p.a, p.o, p.dv,
                                                    p.in_dt == DL_BF16);
    return cudaGetLastError();
}

// Entry-block size: the smallest of 4, 8, 16 that holds all entries (16 for
// longer logs, whose last block is padded).
template <class ST, int DK, bool CHAN, bool WC>
static cudaError_t launch_merge_nb(const StepParams &p, const LogParams &lg, int n_log, cudaStream_t st) {
    const int nt = n_log + (WC ? 1 : 0);
    if (nt <= 4) return launch_merge_t<ST, DK, CHAN, WC, 4>(p, lg, n_log, st);
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
