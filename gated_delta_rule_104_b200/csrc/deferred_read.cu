// Deferred step: append this step's factors to the log and read
// o = S_n q from the unwritten base plus the log (DeltaLog page, Technical
// Summary, "Append Phase", and "Kernel Implementation": key-side metadata
// computed once per slot-head in a "ReplayPrep" stage and shared by the value
// tiles, which then run in parallel "AppendDecode" stages).
//
// With A_i = Diag(a_i)(I - beta_i k_i k_i^T), the logical state after log
// entries 1..n is S_n = S_bar A_1...A_n + sum_i beta_i v_i k_i^T A_{i+1}...A_n,
// so o = S_n q needs only
//   key side (once per head):   x_n = q; for i = n..1:
//        c_i = k_i . x_i,  s_i = beta_i c_i,  x_{i-1} = a_i o (x_i - s_i k_i)
//        and w = sum_i s_i v_i            (a d_v vector)
//   value side (per row r):     o_r = S_bar[r] . x_0 + w_r.
// The base is read once and never written.
//
// Two kernels, chained with programmatic dependent launch:
//   replay_prep   one warp per head: appends the entry, runs the serial
//                 recursion (lanes own d_k/32 key columns, one shuffle
//                 reduction per entry) and w, and stores (x_0, w) in the
//                 caller's workspace [B*H][d_k + d_v] fp32.
//   append_decode a pure streaming pass over the base, laid out like the
//                 eager kernel (a row spread over 16-byte lane slices, 8 loads
//                 in flight per thread, no shared memory, no block barrier).
//                 It may start while replay_prep still runs: it issues its
//                 base loads first and waits for the prep grid only before
//                 reading the workspace.
#include <mutex>

#include "launch.h"

namespace dl {

// ------------------------------------------------------------------ prep

template <class IT, int DK, int DV, bool CHAN>
__global__ void __launch_bounds__(256)
replay_prep_kernel(const IT *__restrict__ q, const IT *__restrict__ k, const IT *__restrict__ v,
                   const IT *__restrict__ beta, const IT *__restrict__ a, IT *__restrict__ log_k,
                   IT *__restrict__ log_v, IT *__restrict__ log_b, IT *__restrict__ log_a, int L, int n,
                   float *__restrict__ work, long long heads) {
    pdl_launch_dependents();
    constexpr int CW = DK / 32;   // key columns per lane
    constexpr int RV = DV / 32;   // value rows per lane
    constexpr int CHUNK = 4;      // log entries fetched together
    const int lane = threadIdx.x & 31;
    const long long head = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (head >= heads) return;
    const long long lrow = head * L;
    const int c0 = lane * CW, r0 = lane * RV;

    // This step's entry (index n), from the inputs.
    float kc[CW], ac[CW], vc[RV], x[CW];
    load_vec<CW>(k + head * DK + c0, kc);
    load_vec<RV>(v + head * DV + r0, vc);
    load_vec<CW>(q + head * DK + c0, x);
    if constexpr (CHAN) {
        load_vec<CW>(a + head * DK + c0, ac);
    } else {
        const float as = to_f(a[head]);
#pragma unroll
        for (int e = 0; e < CW; ++e) ac[e] = as;
    }
    const float bc = to_f(beta[head]);

    // D1: the entry is appended unchanged (raw input elements).
#pragma unroll
    for (int e = 0; e < CW; ++e) log_k[(lrow + n) * DK + c0 + e] = k[head * DK + c0 + e];
#pragma unroll
    for (int e = 0; e < RV; ++e) log_v[(lrow + n) * DV + r0 + e] = v[head * DV + r0 + e];
    if constexpr (CHAN) {
#pragma unroll
        for (int e = 0; e < CW; ++e) log_a[(lrow + n) * DK + c0 + e] = a[head * DK + c0 + e];
    } else if (lane == 0) {
        log_a[lrow + n] = a[head];
    }
    if (lane == 0) log_b[lrow + n] = beta[head];

    // D2: the recursion, newest entry first.
    float w[RV];
#pragma unroll
    for (int e = 0; e < RV; ++e) w[e] = 0.f;
    auto step = [&](const float (&kk)[CW], const float (&aa)[CW], float bb, const float (&vv)[RV]) {
        float c = 0.f;
#pragma unroll
        for (int e = 0; e < CW; ++e) c = fmaf(kk[e], x[e], c);
        c = group_sum<32>(c);
        const float s = bb * c;
#pragma unroll
        for (int e = 0; e < CW; ++e) x[e] = aa[e] * fmaf(-s, kk[e], x[e]);
#pragma unroll
        for (int e = 0; e < RV; ++e) w[e] = fmaf(s, vv[e], w[e]);
    };
    step(kc, ac, bc, vc);
    for (int top = n - 1; top >= 0; top -= CHUNK) {
        float kk[CHUNK][CW], aa[CHUNK][CW], vv[CHUNK][RV], bb[CHUNK];
#pragma unroll
        for (int j = 0; j < CHUNK; ++j) {
            const int i = top - j;
            if (i < 0) break;
            load_vec<CW>(log_k + (lrow + i) * DK + c0, kk[j]);
            load_vec<RV>(log_v + (lrow + i) * DV + r0, vv[j]);
            if constexpr (CHAN) {
                load_vec<CW>(log_a + (lrow + i) * DK + c0, aa[j]);
            } else {
                const float as = to_f(log_a[lrow + i]);
#pragma unroll
                for (int e = 0; e < CW; ++e) aa[j][e] = as;
            }
            bb[j] = to_f(log_b[lrow + i]);
        }
#pragma unroll
        for (int j = 0; j < CHUNK; ++j) {
            if (top - j < 0) break;
            step(kk[j], aa[j], bb[j], vv[j]);
        }
    }

    // (x_0, w) -> workspace.
    float *wk = work + head * (DK + DV);
#pragma unroll
    for (int e = 0; e < CW; ++e) wk[c0 + e] = x[e];
#pragma unroll
    for (int e = 0; e < RV; ++e) wk[DK + r0 + e] = w[e];
}

// ------------------------------------------------------------------ decode

template <class ST, int DK>
struct DecodeShape {
    static constexpr int VEC = StateVec<ST>::N;
    static constexpr int G = DK / VEC;       // lanes per row
    static constexpr int RPW = 32 / G;       // rows per warp-wide load
    static constexpr int R = 8;              // loads in flight per thread
    static constexpr int UNIT = R * RPW;     // rows per warp
    static constexpr int WARPS = 8;
};

template <class ST, int DK, int DV>
__global__ void __launch_bounds__(256)
append_decode_kernel(const ST *__restrict__ Sbar, const float *__restrict__ work, float *__restrict__ o,
                     long long num_units) {
    using C = DecodeShape<ST, DK>;
    constexpr int VEC = C::VEC;
    static_assert(DV % C::UNIT == 0, "unit divides d_v");
    const int lane = threadIdx.x & 31;
    const long long unit = (long long)blockIdx.x * C::WARPS + (threadIdx.x >> 5);
    const bool active = unit < num_units;
    const long long row0 = unit * C::UNIT;
    const long long head = row0 / DV;
    const int rin0 = (int)(row0 - head * DV);
    const int sub = lane / C::G;
    const int col = (lane % C::G) * VEC;

    // D3 operands: the base rows first (read only, streamed).
    uint4 raw[C::R];
    if (active) {
        const ST *src = Sbar + (row0 + sub) * DK + col;
#pragma unroll
        for (int r = 0; r < C::R; ++r) raw[r] = ld_ro_stream(src + (long long)r * C::RPW * DK);
    }
    pdl_wait();  // replay_prep's (x_0, w) are complete and visible from here on
    if (!active) return;
    const float *wk = work + head * (DK + DV);
    float xv[VEC];
    load_vec<VEC>(wk + col, xv);
#pragma unroll
    for (int r = 0; r < C::R; ++r) {
        float s[VEC];
        StateVec<ST>::unpack(raw[r], s);
        float acc = 0.f;
#pragma unroll
        for (int e = 0; e < VEC; ++e) acc = fmaf(s[e], xv[e], acc);
        acc = group_sum<C::G>(acc);
        const int rr = rin0 + r * C::RPW + sub;
        if ((lane % C::G) == 0) o[head * DV + rr] = acc + wk[DK + rr];
    }
}

size_t read_work_bytes(int B, int H, int dk, int dv) { return (size_t)B * H * (dk + dv) * sizeof(float); }

template <class ST, int DK, int DV>
static cudaError_t launch_decode(const StepParams &p, const float *work, cudaStream_t st) {
    using C = DecodeShape<ST, DK>;
    const long long units = (long long)p.B * p.H * DV / C::UNIT;
    const long long blocks = (units + C::WARPS - 1) / C::WARPS;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)blocks);
    cfg.blockDim = dim3(C::WARPS * 32);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, append_decode_kernel<ST, DK, DV>, static_cast<const ST *>(p.S), work, p.o,
                              units);
}

cudaError_t launch_append_read(const StepParams &p, const LogParams &lg, int n, float *work, cudaStream_t st) {
    return dispatch(p, [&](auto st_t, auto it_t, auto dk_c, auto dv_c, auto ch_c) -> cudaError_t {
        using ST = decltype(st_t);
        using IT = decltype(it_t);
        constexpr int DK = decltype(dk_c)::value;
        constexpr int DV = decltype(dv_c)::value;
        constexpr bool CH = decltype(ch_c)::value;
        const long long heads = (long long)p.B * p.H;
        replay_prep_kernel<IT, DK, DV, CH><<<(unsigned)((heads + 7) / 8), 256, 0, st>>>(
            static_cast<const IT *>(p.q), static_cast<const IT *>(p.k), static_cast<const IT *>(p.v),
            static_cast<const IT *>(p.beta), static_cast<const IT *>(p.a), static_cast<IT *>(lg.k),
            static_cast<IT *>(lg.v), static_cast<IT *>(lg.beta), static_cast<IT *>(lg.a), lg.L, n, work, heads);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        e = launch_decode<ST, DK, DV>(p, work, st);
        if (e != cudaSuccess) return e;
        return cudaGetLastError();
    });
}

// ------------------------------------------------------------------ no-allocation variant
//
// dl_log_append_read_noalloc runs the same two kernels with their scratch in
// this fixed module-level array instead of a caller-provided workspace, for
// callers that cannot allocate device memory. The array belongs to the CUDA
// module of this file, so every device that loads the library holds it until
// the process exits. All calls share it: calls whose kernels overlap on the
// GPU (different streams, or different host threads) race on it and must be
// serialised by the caller. Nothing in it needs clearing between calls:
// replay_prep writes every (x_0, w) value the decode kernel then reads.
static __device__ __align__(256) float g_noalloc_work[DL_NOALLOC_WORK_BYTES / sizeof(float)];

// Device address of g_noalloc_work on the current device. Host code may not
// hand the symbol itself to a kernel (on the host it names a host-side
// stand-in), so the address is looked up with cudaGetSymbolAddress once per
// device, with that device current, and cached.
static cudaError_t noalloc_work_address(float **out) {
    constexpr int kMaxDevices = 64;
    static std::mutex mu;
    static float *addr[kMaxDevices] = {};
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (addr[dev] == nullptr) {
        float *ptr = nullptr;
        e = cudaGetSymbolAddress((void **)&ptr, g_noalloc_work);
        if (e != cudaSuccess) return e;
        addr[dev] = ptr;
    }
    *out = addr[dev];
    return cudaSuccess;
}

cudaError_t launch_append_read_noalloc(const StepParams &p, const LogParams &lg, int n, cudaStream_t st) {
    float *work = nullptr;
    cudaError_t e = noalloc_work_address(&work);
    if (e != cudaSuccess) return e;
    return launch_append_read(p, lg, n, work, st);
}

}  // namespace dl
