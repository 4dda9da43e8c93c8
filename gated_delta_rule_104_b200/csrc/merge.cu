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
// (G = S_bar Khat^T, then delta F) around an n x n triangular solve per row,
// 4 n d_k d_v FLOP against 2 d_k d_v state elements moved.
//
// Kernel: one block per (head, value tile), one thread per state row.
//  1. The tile (up to 64 KB) is copied into padded shared-memory rows with
//     16-byte cp.async (no registers held), overlapping steps 2-3.
//  2. The key side is staged once per block: k, a, beta, the tile's values.
//  3. C(i, j) by warps (lanes over key channels, shuffle reductions); then,
//     one thread per key channel, the running decay products turn the staged
//     keys in place into Khat_i = gamma_i o k_i and F_j, plus gamma_n.
//  4. Each thread contracts its own row against Khat (broadcast shared
//     reads), solves for delta in registers, forms the new row in place and,
//     for the fused read, o = s_new . q.
//  5. The tile is written back with coalesced 16-byte streaming stores.
#include "launch.h"

namespace dl {

template <class ST, int DK>
struct MergeShape {
    static constexpr int VEC = StateVec<ST>::N;
    static constexpr int ROW_BYTES = DK * (int)sizeof(ST);
    static constexpr int CH = ROW_BYTES / 16;                  // 16-byte chunks per row
    static constexpr int CAP = 65536 / ROW_BYTES < 256 ? 65536 / ROW_BYTES : 256;
    static constexpr int RSTRIDE = ROW_BYTES + 16;             // padded row stride (bytes)
    static constexpr int CW = DK / 32;                         // key channels per lane
    // rows (= threads) per block for a given d_v: a whole head when it fits
    // in 64 KB (and 256 threads), else equal value tiles of CAP rows.
    __host__ __device__ static constexpr int rows(int dv) { return dv < CAP ? dv : CAP; }
};

// One input element (fp32 or bf16, chosen at run time) widened to float.
__device__ __forceinline__ float ld_in(const void *p, long long i, bool bf) {
    return bf ? to_f(static_cast<const bf16 *>(p)[i]) : static_cast<const float *>(p)[i];
}

// Shared-memory layout for nt merged entries (floats after the padded rows):
//   fk [nt][DK]  keys, turned into F in place        (16-byte aligned)
//   fa           channel decay: [nt][DK], turned into Khat in place;
//                head decay: nt scalars (padded to 4)
//   kh [nt][DK]  Khat (head decay only; aliases fa otherwise)
//   gn [DK], sq [DK]                                 (vector reads)
//   cm [nt][nt], sb [nt], sv [nt][ROWS]              (scalar reads)
__host__ __device__ constexpr size_t round4(size_t x) { return (x + 3) & ~(size_t)3; }

template <class ST, int DK, bool CHAN>
__host__ __device__ constexpr size_t merge_smem_bytes(int nt, int rows) {
    using C = MergeShape<ST, DK>;
    const size_t floats = (size_t)nt * DK
                        + (CHAN ? (size_t)nt * DK : round4(nt))
                        + (CHAN ? 0 : (size_t)nt * DK)
                        + DK + DK
                        + (size_t)nt * nt + nt + (size_t)nt * rows;
    return (size_t)rows * C::RSTRIDE + floats * sizeof(float);
}

template <class ST, int DK, bool CHAN, int NMAX, bool WITH_CUR>
__global__ void __launch_bounds__(256)
merge_kernel(ST *__restrict__ S, const void *__restrict__ log_k, const void *__restrict__ log_v,
             const void *__restrict__ log_b, const void *__restrict__ log_a, int L, int n_log,
             const void *__restrict__ q, const void *__restrict__ k, const void *__restrict__ v,
             const void *__restrict__ beta, const void *__restrict__ a, float *__restrict__ o,
             int DV, bool bf) {
    using C = MergeShape<ST, DK>;
    constexpr int VEC = C::VEC;
    const int ROWS = blockDim.x;                 // = MergeShape::rows(DV)
    const int TILES = DV / ROWS;
    const int WARPS = ROWS / 32;
    const int NT = n_log + (WITH_CUR ? 1 : 0);   // entries merged, 1..NMAX

    extern __shared__ float4 smem_raw[];
    unsigned char *rows = reinterpret_cast<unsigned char *>(smem_raw);
    float *fk = reinterpret_cast<float *>(rows + (size_t)ROWS * C::RSTRIDE);  // k, then F
    float *fa = fk + (size_t)NT * DK;                         // a (channel: then Khat)
    float *kh = CHAN ? fa : fa + round4(NT);                  // Khat
    float *gn = kh + (size_t)NT * DK;
    float *sq = gn + DK;
    float *cm = sq + DK;
    float *sb = cm + (size_t)NT * NT;
    float *sv = sb + NT;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const long long head = blockIdx.x / TILES;
    const int tile = blockIdx.x % TILES;
    const int row0 = tile * ROWS;
    unsigned char *gtile = reinterpret_cast<unsigned char *>(S + (head * DV + row0) * DK);

    // 1. base tile -> padded shared rows, asynchronously.
    for (int g = tid; g < ROWS * C::CH; g += ROWS) {
        const int r = g / C::CH, c = g % C::CH;
        cp_async16(rows + (size_t)r * C::RSTRIDE + c * 16, gtile + (size_t)r * C::ROW_BYTES + c * 16);
    }
    cp_async_commit();

    // 2. key side and values (log entries 0..n_log-1, then this step's): flat,
    // vectorised loads with several in flight per thread.
    const long long lrow = head * L;
    auto stage = [&](auto tag) {
        using IT = decltype(tag);
        stage_block(fk, DK, static_cast<const IT *>(log_k) + lrow * DK, DK, n_log, DK, tid, ROWS);
        if constexpr (CHAN) stage_block(fa, DK, static_cast<const IT *>(log_a) + lrow * DK, DK, n_log, DK, tid, ROWS);
        stage_block(sv, ROWS, static_cast<const IT *>(log_v) + lrow * DV + row0, DV, n_log, ROWS, tid, ROWS);
        if constexpr (WITH_CUR) {
            stage_block(fk + (size_t)n_log * DK, DK, static_cast<const IT *>(k) + head * DK, DK, 1, DK, tid, ROWS);
            if constexpr (CHAN)
                stage_block(fa + (size_t)n_log * DK, DK, static_cast<const IT *>(a) + head * DK, DK, 1, DK, tid, ROWS);
            stage_block(sq, DK, static_cast<const IT *>(q) + head * DK, DK, 1, DK, tid, ROWS);
            stage_block(sv + (size_t)n_log * ROWS, ROWS, static_cast<const IT *>(v) + head * DV + row0, DV, 1, ROWS,
                        tid, ROWS);
        }
    };
    if (bf) stage(bf16{});
    else stage(float{});
    for (int i = tid; i < n_log; i += ROWS) {
        if constexpr (!CHAN) fa[i] = ld_in(log_a, lrow + i, bf);
        sb[i] = ld_in(log_b, lrow + i, bf);
    }
    if (WITH_CUR && tid == 0) {
        if constexpr (!CHAN) fa[n_log] = ld_in(a, head, bf);
        sb[n_log] = ld_in(beta, head, bf);
    }
    __syncthreads();

    // 3a. C(i, j) = sum_c k_i[c] k_j[c] prod_{m=j+1..i} a_m[c], for j < i.
    for (int j = warp; j < NT - 1; j += WARPS) {
        float y[C::CW];
#pragma unroll
        for (int e = 0; e < C::CW; ++e) y[e] = fk[(size_t)j * DK + e * 32 + lane];
#pragma unroll 4
        for (int i = j + 1; i < NT; ++i) {
            float p = 0.f;
#pragma unroll
            for (int e = 0; e < C::CW; ++e) {
                const int c = e * 32 + lane;
                y[e] *= CHAN ? fa[(size_t)i * DK + c] : fa[i];
                p = fmaf(fk[(size_t)i * DK + c], y[e], p);
            }
            p = group_sum<32>(p);
            if (lane == 0) cm[i * NT + j] = p;
        }
    }
    __syncthreads();

    // 3b. per key channel: Khat_i = gamma_i o k_i, gamma_n, F_j = k_j o D(n, j).
    for (int c = tid; c < DK; c += ROWS) {
        float ac[NMAX];
#pragma unroll
        for (int i = 0; i < NMAX; ++i)
            if (i < NT) ac[i] = CHAN ? fa[(size_t)i * DK + c] : fa[i];
        float g = 1.f;
#pragma unroll
        for (int i = 0; i < NMAX; ++i)
            if (i < NT) {
                g *= ac[i];
                kh[(size_t)i * DK + c] = g * fk[(size_t)i * DK + c];
            }
        gn[c] = g;
        float f = 1.f;
#pragma unroll
        for (int j = NMAX - 1; j >= 0; --j)
            if (j < NT) {
                fk[(size_t)j * DK + c] *= f;
                f *= ac[j];
            }
    }
    cp_async_wait_all();
    __syncthreads();

    // 4. one thread per row.
    const int r = tid;
    unsigned char *my = rows + (size_t)r * C::RSTRIDE;
    float acc[NMAX];
#pragma unroll
    for (int i = 0; i < NMAX; ++i) acc[i] = 0.f;
    for (int c = 0; c < C::CH; ++c) {               // G_i = s_bar . Khat_i
        float s[VEC];
        StateVec<ST>::unpack(*reinterpret_cast<const uint4 *>(my + c * 16), s);
#pragma unroll
        for (int i = 0; i < NMAX; ++i) {
            if (i >= NT) break;
            float kv[VEC];
            load_vec<VEC>(kh + (size_t)i * DK + c * VEC, kv);
#pragma unroll
            for (int e = 0; e < VEC; ++e) acc[i] = fmaf(s[e], kv[e], acc[i]);
        }
    }
#pragma unroll
    for (int i = 0; i < NMAX; ++i) {                // forward substitution: acc <- delta
        if (i >= NT) break;
        float t = sv[(size_t)i * ROWS + r] - acc[i];
#pragma unroll
        for (int j = 0; j < i; ++j) t = fmaf(-cm[i * NT + j], acc[j], t);
        acc[i] = sb[i] * t;
    }
    float oacc = 0.f;
    for (int c = 0; c < C::CH; ++c) {               // s_new = s_bar o gamma_n + sum_j delta_j F_j
        float s[VEC], gv[VEC];
        StateVec<ST>::unpack(*reinterpret_cast<const uint4 *>(my + c * 16), s);
        load_vec<VEC>(gn + c * VEC, gv);
#pragma unroll
        for (int e = 0; e < VEC; ++e) s[e] *= gv[e];
#pragma unroll
        for (int j = 0; j < NMAX; ++j) {
            if (j >= NT) break;
            float fv[VEC];
            load_vec<VEC>(fk + (size_t)j * DK + c * VEC, fv);
#pragma unroll
            for (int e = 0; e < VEC; ++e) s[e] = fmaf(acc[j], fv[e], s[e]);
        }
        if constexpr (WITH_CUR) {
            float qv[VEC];
            load_vec<VEC>(sq + c * VEC, qv);
#pragma unroll
            for (int e = 0; e < VEC; ++e) oacc = fmaf(s[e], qv[e], oacc);
        }
        *reinterpret_cast<uint4 *>(my + c * 16) = StateVec<ST>::pack(s);
    }
    if constexpr (WITH_CUR) o[head * DV + row0 + r] = oacc;
    __syncthreads();

    // 5. write the tile back, coalesced.
    for (int g = tid; g < ROWS * C::CH; g += ROWS) {
        const int rr = g / C::CH, c = g % C::CH;
        st_stream(gtile + (size_t)rr * C::ROW_BYTES + c * 16,
                  *reinterpret_cast<const uint4 *>(rows + (size_t)rr * C::RSTRIDE + c * 16));
    }
}

template <class ST, int DK, bool CHAN, int NMAX, bool WC>
static cudaError_t launch_merge_t(const StepParams &p, const LogParams &lg, int n_log, cudaStream_t st) {
    using C = MergeShape<ST, DK>;
    auto kern = merge_kernel<ST, DK, CHAN, NMAX, WC>;
    const int rows = C::rows(p.dv);
    const int nt = n_log + (WC ? 1 : 0);
    const size_t smem = merge_smem_bytes<ST, DK, CHAN>(nt, rows);
    static size_t configured = 48 * 1024;
    if (smem > configured) {
        const size_t want = merge_smem_bytes<ST, DK, CHAN>(NMAX, C::CAP);
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)want);
        if (e != cudaSuccess) return e;
        configured = want;
    }
    const long long blocks = (long long)p.B * p.H * (p.dv / rows);
    kern<<<(unsigned)blocks, rows, smem, st>>>(static_cast<ST *>(p.S), lg.k, lg.v, lg.beta, lg.a, lg.L, n_log,
                                               p.q, p.k, p.v, p.beta, p.a, p.o, p.dv, p.in_dt == DL_BF16);
    return cudaGetLastError();
}

template <class ST, int DK, bool CH>
static cudaError_t launch_merge_n(const StepParams &p, const LogParams &lg, int n_log, bool with_cur,
                                  cudaStream_t st) {
    const int nt = n_log + (with_cur ? 1 : 0);
    if (with_cur) {
        if (nt <= 16) return launch_merge_t<ST, DK, CH, 16, true>(p, lg, n_log, st);
        if (nt <= 32) return launch_merge_t<ST, DK, CH, 32, true>(p, lg, n_log, st);
        return launch_merge_t<ST, DK, CH, 64, true>(p, lg, n_log, st);
    }
    if (nt <= 16) return launch_merge_t<ST, DK, CH, 16, false>(p, lg, n_log, st);
    if (nt <= 32) return launch_merge_t<ST, DK, CH, 32, false>(p, lg, n_log, st);
    return launch_merge_t<ST, DK, CH, 64, false>(p, lg, n_log, st);
}

cudaError_t launch_merge(const StepParams &p, const LogParams &lg, int n_log, bool with_cur, cudaStream_t st) {
    // The input dtype and d_v are run-time arguments of the merge kernel (they
    // only change staging and the block size), which keeps instantiations few.
    auto go = [&](auto st_t, auto dk_c) -> cudaError_t {
        using ST = decltype(st_t);
        constexpr int DK = decltype(dk_c)::value;
        if (p.chan) return launch_merge_n<ST, DK, true>(p, lg, n_log, with_cur, st);
        return launch_merge_n<ST, DK, false>(p, lg, n_log, with_cur, st);
    };
    auto with_dk = [&](auto st_t) -> cudaError_t {
        if (p.dk == 64) return go(st_t, std::integral_constant<int, 64>{});
        return go(st_t, std::integral_constant<int, 128>{});
    };
    if (p.s_dt == DL_BF16) return with_dk(bf16{});
    return with_dk(float{});
}

}  // namespace dl
