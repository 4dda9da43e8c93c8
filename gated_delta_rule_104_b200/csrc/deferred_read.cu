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
#include "prep_layout.h"

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
    constexpr bool CHAN = Rule<KIND>::CHAN, DELTA = Rule<KIND>::DELTA;
    using P = PrepSmem<(int)sizeof(IT), DK, EMAX, CHAN>;
    constexpr int CW = DK / 32;            // key columns per lane (contiguous)
    constexpr int RV = DV / 32;            // value rows per lane
    constexpr int CH = EMAX < 32 ? EMAX : 32;  // entries per butterfly
    constexpr int E = 16 / (int)sizeof(IT);    // elements per 16-byte chunk
    extern __shared__ float4 smem_raw[];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    unsigned char *base = reinterpret_cast<unsigned char *>(smem_raw) + (size_t)warp * P::BYTES;
    IT *sk = reinterpret_cast<IT *>(base + P::K_OFF);
    IT *sa = reinterpret_cast<IT *>(base + P::A_OFF);
    float *fl = reinterpret_cast<float *>(base + P::F_OFF);
    float *fas = fl + P::AS, *fbeta = fl + P::BETA, *fd = fl + P::D, *fcn = fl + P::CN, *fs = fl + P::S,
          *xrow = fl + P::XROW;

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
    const long long lrow = shead * L;
    const int c0 = lane * CW, r0 = lane * RV;
    // The log stays L2-resident between steps: its loads and stores carry an
    // evict-last policy (the base streams through with evict-first); the
    // cp.async staging copies carry none.
    const uint64_t keep = l2_policy_keep();

    // Stage keys and decays of entries 0..n-1 (log) and n (this step), raw.
    for (int u = lane; u < (n + 1) * (DK / E); u += 32) {
        const int e = u / (DK / E), col = (u % (DK / E)) * E;
        if (e < n) {
            DL_GUARD(sk + e * DK + col, 16) cp_async16(sk + e * DK + col, log_k + (lrow + e) * DK + col);
            if constexpr (CHAN) {
                DL_GUARD(sa + e * DK + col, 16) cp_async16(sa + e * DK + col, log_a + (lrow + e) * DK + col);
            }
        } else {
            DL_GUARD(sk + e * DK + col, 16) cp_async16(sk + e * DK + col, k + head * DK + col);
            if constexpr (CHAN) {
                DL_GUARD(sa + e * DK + col, 16) cp_async16(sa + e * DK + col, a + head * DK + col);
            }
        }
    }
    cp_async_commit();
    // Everything else the head needs is loaded next, all loads before the first
    // store that consumes one (a warp issues in order: a store waiting on its
    // load would hold back every load behind it).
    constexpr int SB = (EMAX + 31) / 32;
    RawCopy<1, IT> bx[SB], ax[SB];  // beta and a head-wise decay of entries lane, lane + 32 (<= n), raw
#pragma unroll
    for (int i = 0; i < SB; ++i) {
        const int e = lane + 32 * i;
        if (e <= n) {
            if constexpr (DELTA) {
                if (e < n) bx[i].load_hint(log_b + lrow + e, keep);
                else bx[i].load(beta + head);
            }
            if constexpr (!CHAN) {
                if (e < n) ax[i].load_hint(log_a + lrow + e, keep);
                else ax[i].load(a + head);
            }
        }
    }
    // X rows of the logged entries (rows j < n, columns e <= j), XB per lane a batch.
    constexpr int XB = 8;
    float xx[XB];
    auto x_load = [&](int base) {
#pragma unroll
        for (int i = 0; i < XB; ++i) {
            const int u = base + i * 32 + lane, j = u / EMAX, e = u % EMAX;
            xx[i] = 0.f;
            if (DELTA && u < n * EMAX && e <= j) {
                float t1[1];
                load_vec_hint<1>(log_x + (lrow + j) * L + e, t1, keep);
                xx[i] = t1[0];
            }
        }
    };
    auto x_store = [&](int base) {
#pragma unroll
        for (int i = 0; i < XB; ++i) {
            const int u = base + i * 32 + lane, j = u / EMAX, e = u % EMAX;
            if (DELTA && u < n * EMAX && e <= j) {
                DL_GUARD(xrow + j * EMAX + e, 4) xrow[j * EMAX + e] = xx[i];
            }
        }
    };
    x_load(0);
    // D1: the entry is appended unchanged (raw input elements).
    RawCopy<CW, IT> ck, ca;
    RawCopy<RV, IT> cv;
    ck.load(k + head * DK + c0);
    cv.load(v + head * DV + r0);
    if constexpr (CHAN) ca.load(a + head * DK + c0);
    float qv[CW];
    load_vec<CW>(q + head * DK + c0, qv);
    // the stores
#pragma unroll
    for (int i = 0; i < SB; ++i) {
        const int e = lane + 32 * i;
        if (e <= n) {
            float t1[1];
            if constexpr (DELTA) {
                bx[i].widen(t1);
                DL_GUARD(fbeta + e, 4) fbeta[e] = t1[0];
            }
            if constexpr (!CHAN) {
                ax[i].widen(t1);
                DL_GUARD(fas + e, 4) fas[e] = t1[0];
            }
        }
    }
    x_store(0);
    for (int base = 32 * XB; DELTA && base < n * EMAX; base += 32 * XB) {  // longer logs only
        x_load(base);
        x_store(base);
    }
    ck.store(log_k + (lrow + n) * DK + c0, keep);
    cv.store(log_v + (lrow + n) * DV + r0, keep);
    if constexpr (CHAN) {
        ca.store(log_a + (lrow + n) * DK + c0, keep);
    } else if (lane == 0) {
        copy_hint<1>(log_a + lrow + n, a + head, keep);
    }
    if (DELTA && lane == 0) copy_hint<1>(log_b + lrow + n, beta + head, keep);
    cp_async_wait_all();
    __syncwarp();

    auto decay = [&](int e, float (&ae)[CW]) {
        if constexpr (CHAN) {
            load_vec<CW>(sa + e * DK + c0, ae);
        } else {
#pragma unroll
            for (int c = 0; c < CW; ++c) ae[c] = fas[e];
        }
    };

    // d_e = k_e . (D(n, e) o q) and C(n, e) = k_e . (D(n, e) o k_n), newest first.
    float z[CW], y[CW];
#pragma unroll
    for (int c = 0; c < CW; ++c) z[c] = qv[c];
    load_vec<CW>(sk + n * DK + c0, y);
    for (int top = n; top >= 0; top -= CH) {
        float pd[CH], pc[CH];
#pragma unroll
        for (int jj = 0; jj < CH; ++jj) {
            pd[jj] = 0.f;
            pc[jj] = 0.f;
            const int e = top - jj;
            if (e >= 0) {
                float ke[CW], ae[CW];
                load_vec<CW>(sk + e * DK + c0, ke);
                decay(e, ae);
#pragma unroll
                for (int c = 0; c < CW; ++c) {
                    pd[jj] = fmaf(ke[c], z[c], pd[jj]);
                    z[c] *= ae[c];
                    if constexpr (DELTA) {
                        pc[jj] = fmaf(ke[c], y[c], pc[jj]);
                        y[c] *= ae[c];
                    }
                }
            }
        }
        multi_sum<CH>(pd, lane);
        if constexpr (DELTA) multi_sum<CH>(pc, lane);
        constexpr int shift = CH == 32 ? 0 : CH == 16 ? 1 : CH == 8 ? 2 : 3;
        const int e = top - (lane >> shift);
        if ((lane & ((1 << shift) - 1)) == 0 && e >= 0) {
            DL_GUARD(fd + e, 4) fd[e] = pd[0];
            DL_GUARD(fcn + e, 4) fcn[e] = pc[0];  // (C(n, n) is not used)
        }
    }
    __syncwarp();
    // X row n: X(n, n) = beta_n, X(n, j) = -beta_n sum_{m=j..n-1} C(n, m) X(m, j).
    const float bn = DELTA ? fbeta[n] : 0.f;
    for (int j = lane; DELTA && j <= n; j += 32) {
        float acc = 0.f;
#pragma unroll 4
        for (int m = j; m < n; ++m) acc = fmaf(fcn[m], xrow[m * EMAX + j], acc);
        const float xnj = j == n ? bn : -bn * acc;
        DL_GUARD(xrow + n * EMAX + j, 4) xrow[n * EMAX + j] = xnj;
        st_hint(log_x + (lrow + n) * L + j, __float_as_uint(xnj), keep);
    }
    __syncwarp();
    // s_e = sum_{i=e..n} X(i, e) d_i (the back-substitution, as one dot per entry).
    for (int e = lane; e <= n; e += 32) {
        float acc = 0.f;
        if constexpr (DELTA) {
#pragma unroll 4
            for (int i = e; i <= n; ++i) acc = fmaf(xrow[i * EMAX + e], fd[i], acc);
        } else {
            acc = fd[e];
        }
        DL_GUARD(fs + e, 4) fs[e] = acc;
    }
    __syncwarp();

    // x_0 = gamma_n o q - sum_e s_e (gamma_e o k_e);  w = sum_e s_e v_e.
    float g[CW], xs[CW];
#pragma unroll
    for (int c = 0; c < CW; ++c) {
        g[c] = 1.f;
        xs[c] = 0.f;
    }
#pragma unroll 4
    for (int e = 0; e <= n; ++e) {
        float ke[CW], ae[CW];
        load_vec<CW>(sk + e * DK + c0, ke);
        decay(e, ae);
        const float se = fs[e];
#pragma unroll
        for (int c = 0; c < CW; ++c) {
            g[c] *= ae[c];
            if constexpr (DELTA) xs[c] = fmaf(se * g[c], ke[c], xs[c]);
        }
    }
    float w[RV];
#pragma unroll
    for (int r = 0; r < RV; ++r) w[r] = 0.f;
    // Entries in batches of VB: a batch's raw words are all loaded before any is
    // widened (a widening right after its load would stall the loads behind it).
    constexpr int VB = 8;
    using VC = RawCopy<RV, IT>;
    for (int e0 = 0; e0 <= n; e0 += VB) {
        VC raw[VB];
#pragma unroll
        for (int i = 0; i < VB; ++i) {
            const int e = e0 + i;
            if (e < n) raw[i].load_hint(log_v + (lrow + e) * DV + r0, keep);
            else if (e == n) raw[i].load(v + head * DV + r0);
        }
#pragma unroll
        for (int i = 0; i < VB; ++i) {
            const int e = e0 + i;
            if (e <= n) {
                const float se = fs[e];
                float ve[RV];
                raw[i].widen(ve);
#pragma unroll
                for (int r = 0; r < RV; ++r) w[r] = fmaf(se, ve[r], w[r]);
            }
        }
    }

    float *wk = work + head * (DK + DV);
#pragma unroll
    for (int c = 0; c < CW; ++c) wk[c0 + c] = fmaf(g[c], qv[c], -xs[c]);
#pragma unroll
    for (int r = 0; r < RV; ++r) wk[DK + r0 + r] = w[r];
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

cudaError_t launch_append_read(const StepParams &p, const LogParams &lg, int n, float *work, cudaStream_t st,
                               const PoolIdx &pool) {
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
    return launch_append_read(p, lg, n, work, st);
}

// The guard word of this file's kernels (index-guard build; 0 otherwise).
cudaError_t read_guard_read(unsigned int *flags, unsigned int *line, bool clear) {
    return read_guard_word(flags, line, clear);
}

}  // namespace dl
