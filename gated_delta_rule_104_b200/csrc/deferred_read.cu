// Deferred step: append this step's factors to the log and read
// o = S_n q from the unwritten base plus the log (DeltaLog page, Technical
// Summary, "Append Phase", and "Kernel Implementation": value-tile
// parallelism, key-side metadata computed once and shared by the value
// tiles, a "ReplayPrep" stage then "AppendDecode" stages).
//
// With A_i = Diag(a_i)(I - beta_i k_i k_i^T), the logical state after log
// entries 1..n is S_n = S_bar A_1...A_n + sum_i beta_i v_i k_i^T A_{i+1}...A_n,
// so o = S_n q needs only
//   key side (once per head):   x_n = q; for i = n..1:
//        c_i = k_i . x_i,  s_i = beta_i c_i,  x_{i-1} = a_i o (x_i - s_i k_i)
//   value side (per row r):     o_r = S_bar[r] . x_0 + sum_i s_i v_i[r].
// The base is read once and never written.
//
// One 256-thread block per (head, value tile); a tile holds up to 64 KB of
// the base. The block first issues all of its base loads into registers
// (16 x 16 bytes per thread at most), then stages the log entries it needs
// into shared memory, writes the new entry (tile 0 only), runs the key-side
// recursion in warp 0 while the base loads are in flight, and finally every
// warp finishes its rows with group shuffle reductions.
#include "launch.h"

namespace dl {

template <class ST, int DK, int DV>
struct ReadShape {
    static constexpr int VEC = StateVec<ST>::N;
    static constexpr int G = DK / VEC;                 // lanes per row
    static constexpr int RPW = 32 / G;                 // rows per warp-wide load
    static constexpr int ROW_BYTES = DK * (int)sizeof(ST);
    static constexpr int ROWS = DV < 65536 / ROW_BYTES ? DV : 65536 / ROW_BYTES;  // rows per block
    static constexpr int TILES = DV / ROWS;
    static constexpr int WARPS = 8;
    static constexpr int THREADS = WARPS * 32;
    static constexpr int NV = ROWS / (WARPS * RPW);    // 16-byte base loads per thread
    static constexpr int CW = DK / 32;                 // key columns per lane in the recursion
    static constexpr int SVS = ROWS + 1;               // padded stride of staged values
    static_assert(NV >= 1 && NV * WARPS * RPW == ROWS, "tile shape");
};

// Shared-memory floats needed for a log holding n entries before this step.
template <class ST, int DK, int DV, bool CHAN>
__host__ __device__ constexpr size_t read_smem_floats(int n) {
    using C = ReadShape<ST, DK, DV>;
    return (size_t)(n + 1) * DK                    // k
         + (size_t)(n + 1) * (CHAN ? DK : 1)       // a
         + (size_t)(n + 1)                         // beta
         + (size_t)(n + 1) * C::SVS                // v (this tile's rows)
         + (size_t)(n + 1)                         // s
         + DK;                                     // x_0
}

template <class IT>
__device__ __forceinline__ void stage_contig(float *dst, const IT *src, int count, int tid, int nthreads) {
    constexpr int E = 16 / (int)sizeof(IT);  // elements per 16-byte chunk
    const int chunks = count / E;
    for (int c = tid; c < chunks; c += nthreads) {
        float x[E];
        load_vec<E>(src + c * E, x);
#pragma unroll
        for (int e = 0; e < E; ++e) dst[c * E + e] = x[e];
    }
    for (int i = chunks * E + tid; i < count; i += nthreads) dst[i] = to_f(src[i]);
}

template <class IT>
__device__ __forceinline__ void copy_contig(IT *dst, const IT *src, int count, int tid, int nthreads) {
    constexpr int E = 16 / (int)sizeof(IT);
    const int chunks = count / E;
    for (int c = tid; c < chunks; c += nthreads)
        *reinterpret_cast<uint4 *>(dst + c * E) = *reinterpret_cast<const uint4 *>(src + c * E);
    for (int i = chunks * E + tid; i < count; i += nthreads) dst[i] = src[i];
}

template <class ST, class IT, int DK, int DV, bool CHAN>
__global__ void __launch_bounds__(256, 2)
append_read_kernel(const ST *__restrict__ Sbar, const IT *__restrict__ q, const IT *__restrict__ k,
                   const IT *__restrict__ v, const IT *__restrict__ beta, const IT *__restrict__ a,
                   float *__restrict__ o, IT *__restrict__ log_k, IT *__restrict__ log_v,
                   IT *__restrict__ log_b, IT *__restrict__ log_a, int L, int n) {
    using C = ReadShape<ST, DK, DV>;
    constexpr int VEC = C::VEC;
    extern __shared__ float4 smem_raw[];
    float *sk = reinterpret_cast<float *>(smem_raw);
    float *sa = sk + (size_t)(n + 1) * DK;
    float *sb = sa + (size_t)(n + 1) * (CHAN ? DK : 1);
    float *sv = sb + (n + 1);
    float *ss = sv + (size_t)(n + 1) * C::SVS;
    float *sx = ss + (n + 1);

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const long long head = blockIdx.x / C::TILES;
    const int tile = blockIdx.x % C::TILES;
    const int row0 = tile * C::ROWS;                 // first row of the tile within the head
    const int sub = lane / C::G;
    const int col = (lane % C::G) * VEC;

    // D3 operands first: this thread's slice of the base (NV rows x 16 bytes).
    const ST *bsrc = Sbar + (head * DV + row0 + (long long)warp * C::NV * C::RPW + sub) * DK + col;
    uint4 raw[C::NV];
#pragma unroll
    for (int j = 0; j < C::NV; ++j) raw[j] = ld_ro_stream(bsrc + (long long)j * C::RPW * DK);

    // Stage log entries 0..n-1 and this step's factors as entry n.
    const long long lrow = head * L;                 // first log slot of this head
    stage_contig(sk, log_k + lrow * DK, n * DK, tid, C::THREADS);
    stage_contig(sk + (size_t)n * DK, k + head * DK, DK, tid, C::THREADS);
    if constexpr (CHAN) {
        stage_contig(sa, log_a + lrow * DK, n * DK, tid, C::THREADS);
        stage_contig(sa + (size_t)n * DK, a + head * DK, DK, tid, C::THREADS);
    } else {
        for (int i = tid; i < n; i += C::THREADS) sa[i] = to_f(log_a[lrow + i]);
        if (tid == 0) sa[n] = to_f(a[head]);
    }
    for (int i = tid; i < n; i += C::THREADS) sb[i] = to_f(log_b[lrow + i]);
    if (tid == 0) sb[n] = to_f(beta[head]);
    for (int i = 0; i < n; ++i)
        stage_contig(sv + (size_t)i * C::SVS, log_v + (lrow + i) * DV + row0, C::ROWS, tid, C::THREADS);
    stage_contig(sv + (size_t)n * C::SVS, v + head * DV + row0, C::ROWS, tid, C::THREADS);

    // D1: append (k, v, beta, a) as entry n, unchanged. One tile per head writes it.
    if (tile == 0) {
        copy_contig(log_k + (lrow + n) * DK, k + head * DK, DK, tid, C::THREADS);
        copy_contig(log_v + (lrow + n) * DV, v + head * DV, DV, tid, C::THREADS);
        if constexpr (CHAN) copy_contig(log_a + (lrow + n) * DK, a + head * DK, DK, tid, C::THREADS);
        else if (tid == 0) log_a[lrow + n] = a[head];
        if (tid == 0) log_b[lrow + n] = beta[head];
    }
    __syncthreads();

    // D2: key-side recursion (ReplayPrep), warp 0, lanes own CW key columns.
    if (warp == 0) {
        const int c0 = lane * C::CW;
        float x[C::CW];
        load_vec<C::CW>(q + head * DK + c0, x);
        for (int i = n; i >= 0; --i) {
            float kk[C::CW], ai[C::CW];
            load_vec<C::CW>(sk + (size_t)i * DK + c0, kk);
            if constexpr (CHAN) {
                load_vec<C::CW>(sa + (size_t)i * DK + c0, ai);
            } else {
#pragma unroll
                for (int e = 0; e < C::CW; ++e) ai[e] = sa[i];
            }
            float c = 0.f;
#pragma unroll
            for (int e = 0; e < C::CW; ++e) c = fmaf(kk[e], x[e], c);
            c = group_sum<32>(c);
            const float si = sb[i] * c;
#pragma unroll
            for (int e = 0; e < C::CW; ++e) x[e] = ai[e] * fmaf(-si, kk[e], x[e]);
            if (lane == 0) ss[i] = si;
        }
#pragma unroll
        for (int e = 0; e < C::CW; ++e) sx[c0 + e] = x[e];
    }
    __syncthreads();

    // D3: o_r = S_bar[r] . x_0 + sum_i s_i v_i[r]  (AppendDecode).
    float xv[VEC];
#pragma unroll
    for (int e = 0; e < VEC; ++e) xv[e] = sx[col + e];
    const int gl = lane % C::G;
#pragma unroll
    for (int j = 0; j < C::NV; ++j) {
        const int rl = (warp * C::NV + j) * C::RPW + sub;   // row within the tile
        float s[VEC];
        StateVec<ST>::unpack(raw[j], s);
        float acc = 0.f;
#pragma unroll
        for (int e = 0; e < VEC; ++e) acc = fmaf(s[e], xv[e], acc);
        for (int i = gl; i <= n; i += C::G) acc = fmaf(ss[i], sv[(size_t)i * C::SVS + rl], acc);
        acc = group_sum<C::G>(acc);
        if (gl == 0) o[head * DV + row0 + rl] = acc;
    }
}

cudaError_t launch_append_read(const StepParams &p, const LogParams &lg, int n, cudaStream_t st) {
    return dispatch(p, [&](auto st_t, auto it_t, auto dk_c, auto dv_c, auto ch_c) -> cudaError_t {
        using ST = decltype(st_t);
        using IT = decltype(it_t);
        constexpr int DK = decltype(dk_c)::value;
        constexpr int DV = decltype(dv_c)::value;
        constexpr bool CH = decltype(ch_c)::value;
        using C = ReadShape<ST, DK, DV>;
        auto kern = append_read_kernel<ST, IT, DK, DV, CH>;
        const size_t smem = read_smem_floats<ST, DK, DV, CH>(n) * sizeof(float);
        static size_t configured = 48 * 1024;  // per instantiation
        if (smem > configured) {
            const size_t want = read_smem_floats<ST, DK, DV, CH>(DL_MAX_LOG - 1) * sizeof(float);
            cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)want);
            if (e != cudaSuccess) return e;
            configured = want;
        }
        const long long blocks = (long long)p.B * p.H * C::TILES;
        kern<<<(unsigned)blocks, C::THREADS, smem, st>>>(
            static_cast<const ST *>(p.S), static_cast<const IT *>(p.q), static_cast<const IT *>(p.k),
            static_cast<const IT *>(p.v), static_cast<const IT *>(p.beta), static_cast<const IT *>(p.a),
            p.o, static_cast<IT *>(lg.k), static_cast<IT *>(lg.v), static_cast<IT *>(lg.beta),
            static_cast<IT *>(lg.a), lg.L, n);
        return cudaGetLastError();
    });
}

}  // namespace dl
