// Deferred step: append this step's factors to the log and read
// o = S_n q from the unwritten base plus the log (DeltaLog page, Technical
// Summary, "Append Phase", and "Kernel Implementation": the key-side work is
// done once per (sequence, head) in a "ReplayPrep" stage, and its results serve
// every value tile, each an "AppendDecode" stage running in parallel).
//
// With A_e = Diag(a_e)(I - beta_e k_e k_e^T), entries e = 0..n (n is this
// step's, the newest), the logical state is S_bar A_0 ... A_n-style replayed
// and o = S_n q needs only, per head, the vector x_0 and the scalars s_e of
// the key-side recursion (x <- q; for e = n..0: s_e = beta_e k_e . x,
// x <- a_e o (x - s_e k_e)), then per row r: o_r = S_bar[r] . x_0 + w_r with
// w = sum_e s_e v_e. The base is read once and never written.
//
// ReplayPrep evaluates that recursion in parallel form. With the decay
// products D(j, e) = prod_{m=e+1..j} a_m (the page's log-decay metadata as
// products) and the decayed key inner products C(j, e) = k_e . (D(j, e) o k_j)
// for e < j:
//   d_e = k_e . (D(n, e) o q)                    (independent dots)
//   s_e = beta_e (d_e - sum_{j>e} C(j, e) s_j), i.e. s = X^T d with
//   X = (I + Diag(beta) C)^{-1} Diag(beta)       (lower triangular)
//   x_0 = gamma_n o q - sum_e s_e (gamma_e o k_e),  gamma_e = prod_{m<=e} a_m.
// X only ever gains a row when an entry is appended,
//   X(n, n) = beta_n,  X(n, j) = -beta_n sum_{m=j..n-1} C(n, m) X(m, j),
// so it is kept with the log (log.x): each append forms the new entry's C
// row (the same kind of dots as d_e), extends X by one row and stores it. A
// read is then two parallel dot passes with no serial solve, and the merge
// uses the same X.
// RWKV6 (no delta correction: A_e = Diag(a_e), value added raw) is the case
// X = I: s_e = d_e and x_0 = gamma_n o q.
//
// Two kernels, chained with programmatic dependent launch:
//   replay_prep   one warp per head: stages the head's log keys and decays
//                 in shared memory (cp.async), appends the entry, forms all
//                 d_e and C(n, e) with one transposing butterfly per 32
//                 entries, back-substitutes s, and stores (x_0, w) in the
//                 caller's workspace [B*H][d_k + d_v] fp32.
//   append_decode a pure streaming pass over the base (a row spread over
//                 16-byte lane slices, 8 loads in flight per thread, no
//                 shared memory, no block barrier). It may start while
//                 replay_prep still runs: it issues its base loads first and
//                 waits for the prep grid only before reading the workspace.
#include "launch.h"
#include "guard.cuh"
#include "prep.cuh"
#include "fused_layout.h"
#include "tc.cuh"

namespace dl {

// ------------------------------------------------------------------ prep

template <class IT, int DK, int DV, int KIND, int EMAX>
__global__ void __launch_bounds__(128)
replay_prep_kernel(const IT *__restrict__ q, const IT *__restrict__ k, const IT *__restrict__ v,
                   const IT *__restrict__ beta, const IT *__restrict__ a, IT *__restrict__ log_k,
                   IT *__restrict__ log_v, IT *__restrict__ log_b, IT *__restrict__ log_a,
                   float *__restrict__ log_x, int L, int n, float *__restrict__ work, long long heads,
                   PoolIdx pool) {
    pdl_launch_dependents();
    using P = PrepSmem<(int)sizeof(IT), DK, EMAX, Rule<KIND>::CHAN>;
    extern __shared__ float4 smem_raw[];
    const int warp = threadIdx.x >> 5;
    unsigned char *base = reinterpret_cast<unsigned char *>(smem_raw) + (size_t)warp * P::BYTES;
    // A pool step launches this kernel as a programmatic dependent of its merge
    // part (which works on other slots), so the two overlap; every warp waits
    // for that grid before it exits, so that this grid's completion implies the
    // merge's for the kernels after it. (A no-op for an ordinary launch.)
    const long long head = (long long)blockIdx.x * (blockDim.x / 32) + warp;  // batch head (inputs, work)
    long long shead;  // state / log head (a pool slot's, or the batch head itself)
    if (head >= heads || !pool_head(pool, POOL_APPEND, head, shead, n)) {
        pdl_wait();
        return;
    }
    prep_head<IT, DK, DV, KIND, EMAX, false>(q, k, v, beta, a, log_k, log_v, log_b, log_a, log_x, L, n, head, shead,
                                             base, work + head * (DK + DV));
    pdl_wait();
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
                     long long num_units, PoolIdx pool, const float *__restrict__ row_scale) {
    using C = DecodeShape<ST, DK>;
    constexpr int VEC = C::VEC;
    static_assert(DV % C::UNIT == 0, "unit divides d_v");
    const int lane = threadIdx.x & 31;
    const long long unit = (long long)blockIdx.x * C::WARPS + (threadIdx.x >> 5);
    const long long row0 = unit * C::UNIT;
    const long long head = row0 / DV;  // batch head (work, o)
    const int rin0 = (int)(row0 - head * DV);
    const int sub = lane / C::G;
    const int col = (lane % C::G) * VEC;
    long long shead = head;  // state head
    int n_unused = 0;
    const bool active = unit < num_units && pool_head(pool, POOL_APPEND, head, shead, n_unused);

    // D3 operands: the base rows first (read only, streamed); an int8 base's
    // row scales with them.
    constexpr bool Q8 = std::is_same<ST, int8_t>::value;
    uint4 raw[C::R];
    float rsc[Q8 ? C::R : 1];
    if (active) {
        const uint64_t stream = l2_policy_stream();
        const ST *src = Sbar + (shead * DV + rin0 + sub) * DK + col;
#pragma unroll
        for (int r = 0; r < C::R; ++r) raw[r] = ld_ro_hint(src + (long long)r * C::RPW * DK, stream);
        if constexpr (Q8) {
#pragma unroll
            for (int r = 0; r < C::R; ++r) rsc[r] = row_scale[shead * DV + rin0 + r * C::RPW + sub];
        }
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
        if constexpr (Q8) acc *= rsc[r];
        const int rr = rin0 + r * C::RPW + sub;
        if ((lane % C::G) == 0) o[head * DV + rr] = acc + wk[DK + rr];
    }
}

// ------------------------------------------------------------------ fused append-read
//
// The same step in one persistent kernel (one block per SM; layout and roles
// in fused_layout.h), so that ReplayPrep runs under the base stream instead
// of ahead of it: prep warps work through the block's heads a few heads ahead
// of the decode warps and hand each head's (x_0, w) over in shared memory;
// decode warps keep NBUF bulk copies of the base in flight per warp and form
// o exactly as append_decode does (the same products and sums in the same
// order, so the two paths agree bit for bit). Used for logs of up to 16
// entries on an fp32 or bf16 base without a slot pool; no workspace.
// Every mbarrier wait is bounded (about two seconds); a wait that runs out
// sets bit 0 of g_read_faults and the block leaves its loops, waits for the
// copies it has in flight, and returns.

__device__ unsigned int g_read_faults = 0;

namespace {

__device__ __forceinline__ uint64_t read_globaltimer() {
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}
// Wait for the phase of `bar` with parity `par`; false once about two seconds
// have passed (setting *abort and the fault bit) or another warp gave up.
__device__ __forceinline__ bool fused_wait(uint64_t *bar, uint32_t par, volatile int *abort) {
    if (tc::mbar_try_wait(bar, par)) return true;
    const uint64_t t0 = read_globaltimer();
    for (uint32_t i = 0;; ++i) {
        if (tc::mbar_try_wait(bar, par)) return true;
        if ((i & 63u) == 63u) {
            if (*abort) return false;
            if (read_globaltimer() - t0 > 2000000000ull) {
                *abort = 1;
                atomicOr(&g_read_faults, 1u);
                return false;
            }
        }
    }
}
// The same without the abort check: for draining a warp's own copies.
__device__ __forceinline__ void fused_drain(uint64_t *bar, uint32_t par) {
    const uint64_t t0 = read_globaltimer();
    while (!tc::mbar_try_wait(bar, par)) {
        if (read_globaltimer() - t0 > 2000000000ull) {
            atomicOr(&g_read_faults, 1u);
            return;
        }
    }
}

}  // namespace

template <class IT, class ST, int DK, int DV, int KIND>
__global__ void __launch_bounds__(fused::Layout<(int)sizeof(IT), (int)sizeof(ST), DK, DV, Rule<KIND>::CHAN>::WARPS * 32, 1)
append_read_fused_kernel(const ST *__restrict__ Sbar, const IT *__restrict__ q, const IT *__restrict__ k,
                         const IT *__restrict__ v, const IT *__restrict__ beta, const IT *__restrict__ a,
                         IT *__restrict__ log_k, IT *__restrict__ log_v, IT *__restrict__ log_b,
                         IT *__restrict__ log_a, float *__restrict__ log_x, int L, int n, float *__restrict__ o,
                         long long heads) {
    using LY = fused::Layout<(int)sizeof(IT), (int)sizeof(ST), DK, DV, Rule<KIND>::CHAN>;
    using C = DecodeShape<ST, DK>;
    constexpr int VEC = C::VEC, NP = LY::NP, ND = fused::ND, NBUF = fused::NBUF, NSLOT = LY::NSLOT,
                  UPH = LY::UPH;
    static_assert(C::UNIT == LY::UNIT_ROWS, "a bulk copy holds one decode unit");
    static_assert(DV % LY::UNIT_ROWS == 0, "units tile a head");
    extern __shared__ float4 smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
    uint64_t *full = reinterpret_cast<uint64_t *>(sm + LY::BAR_FULL);
    uint64_t *freeb = reinterpret_cast<uint64_t *>(sm + LY::BAR_FREE);
    uint64_t *ringb = reinterpret_cast<uint64_t *>(sm + LY::BAR_RING);
    volatile int *abort = reinterpret_cast<volatile int *>(sm + LY::ABORT_OFF);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nh = heads > (long long)blockIdx.x ? (int)((heads - 1 - blockIdx.x) / gridDim.x) + 1 : 0;

    // Launched as a programmatic dependent of the kernel before it: the block
    // sets up its barriers while that kernel drains, and touches no global
    // memory before the wait (the base, the log and the inputs may all be
    // that kernel's output). The kernel after it may likewise start early.
    pdl_launch_dependents();
    if (threadIdx.x == 0) {
        for (int s = 0; s < NSLOT; ++s) {
            tc::mbar_init(&full[s], 32);     // the prep warp's 32 lanes
            tc::mbar_init(&freeb[s], UPH);   // one arrival per decode unit of the head
        }
        for (int u = 0; u < ND * NBUF; ++u) tc::mbar_init(&ringb[u], 1);
        *abort = 0;
        tc::mbar_init_fence();
    }
    __syncthreads();
    pdl_wait();

    if (warp < NP) {
        // ------------------------------------------------ ReplayPrep, heads warp, warp + NP, ...
        unsigned char *base = sm + LY::prep(warp);
        for (int i = warp; i < nh; i += NP) {
            const int s = i % NSLOT;
            if (i >= NSLOT && !fused_wait(&freeb[s], (uint32_t)((i / NSLOT - 1) & 1), abort)) break;
            const long long head = (long long)blockIdx.x + (long long)i * gridDim.x;
            prep_head<IT, DK, DV, KIND, fused::EMAX, true>(q, k, v, beta, a, log_k, log_v, log_b, log_a, log_x, L,
                                                             n, head, head, base,
                                                             reinterpret_cast<float *>(sm + LY::slot(s)));
            tc::mbar_arrive(&full[s]);  // each lane after its own stores of x_0 and w
        }
    } else {
        // ------------------------------------------------ AppendDecode, units d, d + ND, ... of the block's heads
        const int d = warp - NP;
        const int nf = nh * UPH;
        const int sub = lane / C::G, col = (lane % C::G) * VEC;
        // (a buffer is refilled only after every lane's reads of it have
        // returned their values, which the unit's sums consumed)
        auto issue = [&](int f, int b) {
            if (lane == 0) {
                const long long head = (long long)blockIdx.x + (long long)(f / UPH) * gridDim.x;
                uint64_t *bar = &ringb[d * NBUF + b];
                tc::mbar_arrive_expect_tx(bar, fused::UNIT_BYTES);
                tc::bulk_load(sm + LY::ring(d, b), Sbar + (head * DV + (long long)(f % UPH) * LY::UNIT_ROWS) * DK,
                              fused::UNIT_BYTES, bar);
            }
        };
        int issued = 0;
        for (int b = 0; b < NBUF && d + b * ND < nf; ++b, ++issued) issue(d + b * ND, b);
        int t = 0;
        for (;; ++t) {
            const int f = d + t * ND;
            if (f >= nf) break;
            const int b = t % NBUF, i = f / UPH, j = f % UPH, s = i % NSLOT;
            if (!fused_wait(&ringb[d * NBUF + b], (uint32_t)((t / NBUF) & 1), abort)) break;
            if (!fused_wait(&full[s], (uint32_t)((i / NSLOT) & 1), abort)) break;
            const long long head = (long long)blockIdx.x + (long long)i * gridDim.x;
            const ST *tile = reinterpret_cast<const ST *>(sm + LY::ring(d, b));
            const float *sl = reinterpret_cast<const float *>(sm + LY::slot(s));
            float xv[VEC], res[C::R];
#pragma unroll
            for (int e = 0; e < VEC; ++e) xv[e] = sl[col + e];
            const bool writer = (lane % C::G) == 0;
#pragma unroll
            for (int r = 0; r < C::R; ++r) {
                const int ru = r * C::RPW + sub;  // row within the unit
                float sv[VEC];
                StateVec<ST>::unpack(*reinterpret_cast<const uint4 *>(tile + ru * DK + col), sv);
                float acc = 0.f;
#pragma unroll
                for (int e = 0; e < VEC; ++e) acc = fmaf(sv[e], xv[e], acc);
                acc = group_sum<C::G>(acc);
                res[r] = writer ? acc + sl[DK + j * LY::UNIT_ROWS + ru] : 0.f;
            }
            // the unit reads nothing more of slot s or of buffer b: hand the
            // slot back and refill the buffer before the unit's stores, so that
            // neither waits behind them
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&freeb[s]);
            if (f + NBUF * ND < nf) {
                issue(f + NBUF * ND, b);
                ++issued;
            }
#pragma unroll
            for (int r = 0; r < C::R; ++r)
                if (writer) o[head * DV + j * LY::UNIT_ROWS + r * C::RPW + sub] = res[r];
        }
        // after a wait gave up: the copies this warp still has in flight land
        // before the block exits
        if (lane == 0)
            for (int u = t; u < issued; ++u) fused_drain(&ringb[d * NBUF + u % NBUF], (uint32_t)((u / NBUF) & 1));
        __syncwarp();
    }
}

template <class IT, class ST, int DK, int DV, int KD>
static cudaError_t launch_fused(const StepParams &p, const LogParams &lg, int n, cudaStream_t st) {
    using LY = fused::Layout<(int)sizeof(IT), (int)sizeof(ST), DK, DV, Rule<KD>::CHAN>;
    static_assert(LY::REQUEST <= fused::SMEM_LIMIT, "layout fits the shared memory a block may request");
    static_assert(LY::NP >= 1, "at least one prep warp");
    auto kern = append_read_fused_kernel<IT, ST, DK, DV, KD>;
    cudaError_t e = allow_smem(reinterpret_cast<const void *>(kern), LY::REQUEST);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 0;
    e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    const long long heads = (long long)p.B * p.H;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)std::min<long long>(heads, sms));
    cfg.blockDim = dim3(LY::WARPS * 32);
    cfg.dynamicSmemBytes = LY::REQUEST;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kern, static_cast<const ST *>(p.S), static_cast<const IT *>(p.q),
                           static_cast<const IT *>(p.k), static_cast<const IT *>(p.v),
                           static_cast<const IT *>(p.beta), static_cast<const IT *>(p.a), static_cast<IT *>(lg.k),
                           static_cast<IT *>(lg.v), static_cast<IT *>(lg.beta), static_cast<IT *>(lg.a), lg.x, lg.L,
                           n, p.o, heads);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

size_t read_work_bytes(int B, int H, int dk, int dv) { return (size_t)B * H * (dk + dv) * sizeof(float); }

template <class ST, int DK, int DV>
static cudaError_t launch_decode(const StepParams &p, const float *work, cudaStream_t st, const PoolIdx &pool) {
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
    // an int8 base's row scales follow its codes (all the state's heads: the pool's, or B*H)
    const long long state_heads = pool.slot ? (long long)pool.P * pool.H : (long long)p.B * p.H;
    const float *row_scale = std::is_same<ST, int8_t>::value
                                 ? reinterpret_cast<const float *>(static_cast<const int8_t *>(p.S) +
                                                                   state_heads * DV * DK)
                                 : nullptr;
    return cudaLaunchKernelEx(&cfg, append_decode_kernel<ST, DK, DV>, static_cast<const ST *>(p.S), work, p.o,
                              units, pool, row_scale);
}

template <class IT, int DK, int DV, int KD, int EMAX>
static cudaError_t launch_prep(const StepParams &p, const LogParams &lg, int n, float *work, cudaStream_t st,
                               const PoolIdx &pool) {
    using P = PrepSmem<(int)sizeof(IT), DK, EMAX, Rule<KD>::CHAN>;
    constexpr int WARPS = prep_warps(EMAX);
    auto kern = replay_prep_kernel<IT, DK, DV, KD, EMAX>;
    const size_t smem = (size_t)WARPS * P::BYTES;
    cudaError_t e = allow_smem(reinterpret_cast<const void *>(kern), smem);
    if (e != cudaSuccess) return e;
    const long long heads = (long long)p.B * p.H;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((heads + WARPS - 1) / WARPS));
    cfg.blockDim = dim3(WARPS * 32);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pool.slot ? 1 : 0;  // a pool step overlaps it with its merge part
    return cudaLaunchKernelEx(&cfg, kern, static_cast<const IT *>(p.q), static_cast<const IT *>(p.k),
                              static_cast<const IT *>(p.v), static_cast<const IT *>(p.beta),
                              static_cast<const IT *>(p.a), static_cast<IT *>(lg.k), static_cast<IT *>(lg.v),
                              static_cast<IT *>(lg.beta), static_cast<IT *>(lg.a), lg.x, lg.L, n, work, heads, pool);
}

// The two-kernel form (replay_prep, then append_decode with the workspace).
static cudaError_t launch_append_read_split(const StepParams &p, const LogParams &lg, int n, float *work,
                                           cudaStream_t st, const PoolIdx &pool) {
    return dispatch(p, [&](auto st_t, auto it_t, auto dk_c, auto dv_c, auto ch_c) -> cudaError_t {
        using ST = decltype(st_t);
        using IT = decltype(it_t);
        constexpr int DK = decltype(dk_c)::value;
        constexpr int DV = decltype(dv_c)::value;
        constexpr int KD = decltype(ch_c)::value;
        cudaError_t e;
        const int emax = prep_emax(lg.L);
        if (emax == 16) e = launch_prep<IT, DK, DV, KD, 16>(p, lg, n, work, st, pool);
        else if (emax == 32) e = launch_prep<IT, DK, DV, KD, 32>(p, lg, n, work, st, pool);
        else e = launch_prep<IT, DK, DV, KD, 64>(p, lg, n, work, st, pool);
        if (e != cudaSuccess) return e;
        if (p.s_dt == DL_I8) e = launch_decode<int8_t, DK, DV>(p, work, st, pool);
        else e = launch_decode<ST, DK, DV>(p, work, st, pool);
        if (e != cudaSuccess) return e;
        return cudaGetLastError();
    });
}

// The one-kernel form pays where each block has many heads to pipeline: its
// first head's ReplayPrep is exposed once per launch, and with a few heads per
// SM (or 256-row heads, whose ReplayPrep is twice as long) the two-kernel form,
// whose prep grid covers every head at once, measured faster.
bool fused_read_supported(const StepParams &p, int L, const PoolIdx &pool) {
    if (pool.slot != nullptr || !(p.s_dt == DL_F32 || p.s_dt == DL_BF16) || prep_emax(L) != fused::EMAX ||
        p.dv > 128)
        return false;
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return false;
    return (long long)p.B * p.H >= (long long)fused::MIN_HEADS_PER_SM * sms;
}

cudaError_t launch_append_read(const StepParams &p, const LogParams &lg, int n, float *work, cudaStream_t st,
                               const PoolIdx &pool) {
    if (!fused_read_supported(p, lg.L, pool)) return launch_append_read_split(p, lg, n, work, st, pool);
    return dispatch(p, [&](auto st_t, auto it_t, auto dk_c, auto dv_c, auto ch_c) -> cudaError_t {
        using ST = decltype(st_t);
        using IT = decltype(it_t);
        constexpr int DV = decltype(dv_c)::value;
        if constexpr (DV <= 128)
            return launch_fused<IT, ST, decltype(dk_c)::value, DV, decltype(ch_c)::value>(p, lg, n, st);
        else
            return launch_append_read_split(p, lg, n, work, st, pool);
    });
}

// ------------------------------------------------------------------ no-allocation variant
//
// dl_log_append_read_noalloc runs the two-kernel form of the step
// (replay_prep, then append_decode) for every shape, with its scratch in
// this fixed module-level array instead of a caller-provided workspace, for
// callers that cannot allocate device memory. The array belongs to the CUDA
// module of this file, so every device that loads the library holds it until
// the process exits. All calls share it: calls whose kernels overlap on the
// GPU (different streams, or different host threads) race on it and must be
// serialised by the caller. Nothing in it needs clearing between calls:
// replay_prep writes every (x_0, w) value the decode kernel then reads.
static __device__ __align__(256) float g_noalloc_work[DL_NOALLOC_WORK_BYTES / sizeof(float)];

// Device address of g_noalloc_work in the current context. Host code may not
// hand the symbol itself to a kernel (on the host it names a host-side
// stand-in), so the address is looked up with cudaGetSymbolAddress, with the
// caller's device current. The lookup is made on every call rather than
// cached: the array belongs to the module loaded in one context, and after a
// device or primary-context reset (or under a context the caller made itself)
// a cached address would point at memory the array no longer occupies. Once
// the module is loaded in a context the lookup is a host-side table read; the
// first call in a context may load the module.
static cudaError_t noalloc_work_address(float **out) {
    float *ptr = nullptr;
    const cudaError_t e = cudaGetSymbolAddress((void **)&ptr, g_noalloc_work);
    if (e != cudaSuccess) return e;
    *out = ptr;
    return cudaSuccess;
}

cudaError_t launch_append_read_noalloc(const StepParams &p, const LogParams &lg, int n, cudaStream_t st) {
    float *work = nullptr;
    cudaError_t e = noalloc_work_address(&work);
    if (e != cudaSuccess) return e;
    return launch_append_read_split(p, lg, n, work, st, PoolIdx{});
}

cudaError_t read_read_faults(unsigned int *out, bool clear) {
    cudaError_t e = cudaMemcpyFromSymbol(out, g_read_faults, sizeof(unsigned int));
    if (e == cudaSuccess && clear) {
        const unsigned int zero = 0;
        e = cudaMemcpyToSymbol(g_read_faults, &zero, sizeof(unsigned int));
    }
    return e;
}

// The guard word of this file's kernels (index-guard build; 0 otherwise).
cudaError_t read_guard_read(unsigned int *flags, unsigned int *line, bool clear) {
    return read_guard_word(flags, line, clear);
}

}  // namespace dl
