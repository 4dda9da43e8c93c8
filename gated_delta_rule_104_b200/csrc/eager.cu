// Eager decode step (DeltaLog page, Technical Summary, "Problem: The
// State-Update Tax": the eager schedule reads and writes the whole
// [B, H, d_v, d_k] state every token).
//
// Per (b, h), with S' = S Diag(a):
//   u = S' k,  p = S' q,  S <- S' + beta (v - u) k^T,  o = p + beta (v - u) (k . q)
// which is S_t = S_{t-1} Diag(a)(I - beta k k^T) + beta v k^T and o = S_t q.
// RWKV6 (raw-value update, no delta correction) takes d = v in place of
// beta (v - u): S <- S' + v k^T, o = p + v (k . q).
//
// HBM-bound streaming kernel (about 1 FLOP per state byte). Layout: one state
// row (d_k contiguous elements, 128-512 bytes) is spread over a group of G
// lanes, 16 bytes (4 fp32 or 8 bf16) per lane, so each warp-wide 16-byte load
// covers 32/G whole rows: fully coalesced 512-byte transactions. A warp owns
// R such loads (a "unit" of R*32/G consecutive rows of one head) and issues
// all of them before any arithmetic, so each thread keeps R*16 bytes in
// flight; with 8 warps per block and full occupancy an SM holds ~128 KB of
// outstanding loads. The row dots S'k and S'q are group shuffle reductions.
// No shared memory, no block barriers: each warp is independent.
#include "launch.h"

namespace dl {

template <class ST, int DK>
struct EagerShape {
    static constexpr int VEC = StateVec<ST>::N;   // elements per lane
    static constexpr int G = DK / VEC;            // lanes per row
    static constexpr int RPW = 32 / G;            // rows per warp-wide load
    static constexpr int R = 4;                   // loads per warp unit
    static constexpr int UNIT = R * RPW;          // rows per warp unit
    static constexpr int WARPS = 8;
    static_assert(G >= 1 && G <= 32 && 32 % G == 0, "row group");
};

template <class ST, class IT, int DK, int DV, int KIND>
__global__ void __launch_bounds__(256)
eager_step_kernel(ST *__restrict__ S, const IT *__restrict__ q, const IT *__restrict__ k,
                  const IT *__restrict__ v, const IT *__restrict__ beta, const IT *__restrict__ a,
                  float *__restrict__ o, long long num_units) {
    using C = EagerShape<ST, DK>;
    constexpr int VEC = C::VEC;
    constexpr bool CHAN = Rule<KIND>::CHAN, DELTA = Rule<KIND>::DELTA;
    const int lane = threadIdx.x & 31;
    const long long unit = (long long)blockIdx.x * C::WARPS + (threadIdx.x >> 5);
    if (unit >= num_units) return;  // whole warps leave together

    const long long row0 = unit * C::UNIT;       // first row (over B*H*d_v)
    const long long head = row0 / DV;
    const int rin0 = (int)(row0 - head * DV);    // row within the head
    const int sub = lane / C::G;                 // row within one warp-wide load
    const int col = (lane % C::G) * VEC;         // first key column of this lane

    // E1: state loads first (R independent 16-byte loads per thread).
    ST *srow = S + (row0 + sub) * DK + col;
    uint4 raw[C::R];
#pragma unroll
    for (int r = 0; r < C::R; ++r) raw[r] = ld_stream(srow + (long long)r * C::RPW * DK);

    // This step's operands for the head (shared by all rows of the head).
    float kk[VEC], qq[VEC], aa[VEC];
    load_vec<VEC>(k + head * DK + col, kk);
    load_vec<VEC>(q + head * DK + col, qq);
    if constexpr (CHAN) {
        load_vec<VEC>(a + head * DK + col, aa);
    } else {
        const float as = to_f(a[head]);
#pragma unroll
        for (int e = 0; e < VEC; ++e) aa[e] = as;
    }
    const float b = DELTA ? to_f(beta[head]) : 1.f;
    float vr[C::R];
#pragma unroll
    for (int r = 0; r < C::R; ++r) vr[r] = to_f(v[head * DV + rin0 + r * C::RPW + sub]);

    float kq = 0.f;
#pragma unroll
    for (int e = 0; e < VEC; ++e) kq = fmaf(kk[e], qq[e], kq);
    kq = group_sum<C::G>(kq);

#pragma unroll
    for (int r = 0; r < C::R; ++r) {
        float s[VEC];
        StateVec<ST>::unpack(raw[r], s);
        float u = 0.f, pq = 0.f;
#pragma unroll
        for (int e = 0; e < VEC; ++e) {
            s[e] *= aa[e];                           // E2: decay
            if constexpr (DELTA) u = fmaf(s[e], kk[e], u);  // E3: S'k
            pq = fmaf(s[e], qq[e], pq);              //     S'q
        }
        if constexpr (DELTA) u = group_sum<C::G>(u);
        pq = group_sum<C::G>(pq);
        const float d = DELTA ? b * (vr[r] - u) : vr[r];  // E4: beta (v - S'k), or v
#pragma unroll
        for (int e = 0; e < VEC; ++e) s[e] = fmaf(d, kk[e], s[e]);
        st_stream(srow + (long long)r * C::RPW * DK, StateVec<ST>::pack(s));
        if ((lane % C::G) == 0)            // E5: o = S_t q
            o[head * DV + rin0 + r * C::RPW + sub] = fmaf(d, kq, pq);
    }
}

cudaError_t launch_eager(const StepParams &p, cudaStream_t st) {
    return dispatch(p, [&](auto st_t, auto it_t, auto dk_c, auto dv_c, auto ch_c) -> cudaError_t {
        using ST = decltype(st_t);
        using IT = decltype(it_t);
        constexpr int DK = decltype(dk_c)::value;
        constexpr int DV = decltype(dv_c)::value;
        constexpr int KD = decltype(ch_c)::value;
        using C = EagerShape<ST, DK>;
        static_assert(DV % C::UNIT == 0, "unit divides d_v");
        const long long rows = (long long)p.B * p.H * DV;
        const long long units = rows / C::UNIT;
        const long long blocks = (units + C::WARPS - 1) / C::WARPS;
        eager_step_kernel<ST, IT, DK, DV, KD><<<(unsigned)blocks, C::WARPS * 32, 0, st>>>(
            static_cast<ST *>(p.S), static_cast<const IT *>(p.q), static_cast<const IT *>(p.k),
            static_cast<const IT *>(p.v), static_cast<const IT *>(p.beta), static_cast<const IT *>(p.a),
            p.o, units);
        return cudaGetLastError();
    });
}

}  // namespace dl
