// Shared device helpers for the decode-step kernels: element types, widening
// vector loads, bf16 packing and group reductions. sm_100a only.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace dl {

using bf16 = __nv_bfloat16;

// ---------------------------------------------------------------- scalars

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(bf16 x) { return __bfloat162float(x); }

// bf16 bit pattern (low / high half of a 32-bit word) widened exactly.
__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Two floats rounded to nearest-even bf16, packed (first in the low half).
__device__ __forceinline__ uint32_t pack_bf2(float lo, float hi) {
    __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&p);
}

// ---------------------------------------------------------------- loads

// N consecutive elements of T at p (aligned to N * sizeof(T) bytes, at most
// 16) widened to float. Plain cached loads (small, reused operands).
template <int N>
__device__ __forceinline__ void load_vec(const float *p, float (&x)[N]) {
    static_assert(N % 2 == 0, "even");
    if constexpr (N % 4 == 0) {
#pragma unroll
        for (int i = 0; i < N; i += 4) {
            float4 v = *reinterpret_cast<const float4 *>(p + i);
            x[i] = v.x; x[i + 1] = v.y; x[i + 2] = v.z; x[i + 3] = v.w;
        }
    } else {
#pragma unroll
        for (int i = 0; i < N; i += 2) {
            float2 v = *reinterpret_cast<const float2 *>(p + i);
            x[i] = v.x; x[i + 1] = v.y;
        }
    }
}

template <int N>
__device__ __forceinline__ void load_vec(const bf16 *p, float (&x)[N]) {
    static_assert(N % 2 == 0, "even");
    if constexpr (N % 8 == 0) {
#pragma unroll
        for (int i = 0; i < N; i += 8) {
            uint4 v = *reinterpret_cast<const uint4 *>(p + i);
            x[i] = bf_lo(v.x); x[i + 1] = bf_hi(v.x);
            x[i + 2] = bf_lo(v.y); x[i + 3] = bf_hi(v.y);
            x[i + 4] = bf_lo(v.z); x[i + 5] = bf_hi(v.z);
            x[i + 6] = bf_lo(v.w); x[i + 7] = bf_hi(v.w);
        }
    } else if constexpr (N % 4 == 0) {
#pragma unroll
        for (int i = 0; i < N; i += 4) {
            uint2 v = *reinterpret_cast<const uint2 *>(p + i);
            x[i] = bf_lo(v.x); x[i + 1] = bf_hi(v.x);
            x[i + 2] = bf_lo(v.y); x[i + 3] = bf_hi(v.y);
        }
    } else {
#pragma unroll
        for (int i = 0; i < N; i += 2) {
            uint32_t v = *reinterpret_cast<const uint32_t *>(p + i);
            x[i] = bf_lo(v); x[i + 1] = bf_hi(v);
        }
    }
}

// 16-byte state vectors: 4 floats or 8 bf16 held in a uint4.
template <class ST> struct StateVec;
template <> struct StateVec<float> {
    static constexpr int N = 4;
    __device__ __forceinline__ static void unpack(const uint4 &r, float (&x)[4]) {
        x[0] = __uint_as_float(r.x); x[1] = __uint_as_float(r.y);
        x[2] = __uint_as_float(r.z); x[3] = __uint_as_float(r.w);
    }
    __device__ __forceinline__ static uint4 pack(const float (&x)[4]) {
        return make_uint4(__float_as_uint(x[0]), __float_as_uint(x[1]),
                          __float_as_uint(x[2]), __float_as_uint(x[3]));
    }
};
template <> struct StateVec<bf16> {
    static constexpr int N = 8;
    __device__ __forceinline__ static void unpack(const uint4 &r, float (&x)[8]) {
        x[0] = bf_lo(r.x); x[1] = bf_hi(r.x); x[2] = bf_lo(r.y); x[3] = bf_hi(r.y);
        x[4] = bf_lo(r.z); x[5] = bf_hi(r.z); x[6] = bf_lo(r.w); x[7] = bf_hi(r.w);
    }
    __device__ __forceinline__ static uint4 pack(const float (&x)[8]) {
        return make_uint4(pack_bf2(x[0], x[1]), pack_bf2(x[2], x[3]),
                          pack_bf2(x[4], x[5]), pack_bf2(x[6], x[7]));
    }
};

// int8 state codes (a deferred base of type DL_I8): 16 per 16-byte slice,
// widened here; the row scale is applied by the caller.
template <> struct StateVec<int8_t> {
    static constexpr int N = 16;
    __device__ __forceinline__ static void unpack(const uint4 &r, float (&x)[16]) {
        const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) x[4 * i + j] = (float)(int8_t)(w[i] >> (8 * j));
    }
};

// The int8 state's row rounding: scale = max|value| / 127, code = the nearest
// integer to value / scale (ties to even) in [-127, 127]; an all-zero row has
// scale 0 and every code 0.
//
// The quotient value / scale is formed without a division per element, from
// the row's reciprocal inv = 1 / scale (one correctly rounded division per
// row): q0 = value * inv, then one fused correction q0 + (value - q0 scale) inv,
// which is the correctly rounded quotient (Markstein's one-step correction of
// a quotient from a correctly rounded reciprocal; the residual is exact in
// one FMA). Checked against fp32 division on 3.2e8 quotients, near half-
// integers included, for scales from 1e-32 to 1e28; rows whose scale lies
// outside [2^-100, 2^90] (inside that range) divide instead (a choice made
// once per row), and the GPU conversion test compares the codes with the
// oracle's fp32 division bit for bit.
__device__ __forceinline__ float i8_scale(float row_max) { return row_max / 127.f; }
// Whether a row takes the reciprocal form (its scale is 0 or in [2^-100, 2^90]),
// and the reciprocal it uses (0 for a zero row, whose codes then come out 0).
__device__ __forceinline__ bool i8_fast(float scale) {
    return scale == 0.f || (scale >= 0x1p-100f && scale <= 0x1p90f);
}
__device__ __forceinline__ float i8_inv(float scale) { return scale == 0.f ? 0.f : 1.f / scale; }
__device__ __forceinline__ int i8_clamp(int c) { return c > 127 ? 127 : (c < -127 ? -127 : c); }
// the code of x in a row with i8_fast(scale), without a branch
__device__ __forceinline__ int i8_code(float x, float scale, float inv) {
    const float q0 = __fmul_rn(x, inv);
    return i8_clamp(__float2int_rn(fmaf(fmaf(-q0, scale, x), inv, q0)));
}
// the code of x in any row, by division
__device__ __forceinline__ int i8_code_div(float x, float scale) {
    return scale == 0.f ? 0 : i8_clamp(__float2int_rn(x / scale));
}
// four codes packed into a word, low byte first (FAST: the row takes the
// reciprocal form)
template <bool FAST>
__device__ __forceinline__ uint32_t i8_pack4(float a, float b, float c, float d, float scale, float inv) {
    int k0, k1, k2, k3;
    if constexpr (FAST) {
        k0 = i8_code(a, scale, inv), k1 = i8_code(b, scale, inv), k2 = i8_code(c, scale, inv),
        k3 = i8_code(d, scale, inv);
    } else {
        k0 = i8_code_div(a, scale), k1 = i8_code_div(b, scale), k2 = i8_code_div(c, scale),
        k3 = i8_code_div(d, scale);
    }
    return (uint32_t)(k0 & 0xff) | ((uint32_t)(k1 & 0xff) << 8) | ((uint32_t)(k2 & 0xff) << 16) |
           ((uint32_t)(k3 & 0xff) << 24);
}
__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, off));
    return x;
}

// Streaming 16-byte state accesses: the state is touched once per step, so
// it is read and written with the evict-first (".cs") cache hint and kept out
// of L1, leaving L2 to the small per-step operands.
__device__ __forceinline__ uint4 ld_stream(const void *p) {
    return __ldcs(reinterpret_cast<const uint4 *>(p));
}
__device__ __forceinline__ void st_stream(void *p, const uint4 &v) {
    __stcs(reinterpret_cast<uint4 *>(p), v);
}
// Read-only state (the deferred base between merges): non-coherent path,
// no L1 allocation.
__device__ __forceinline__ uint4 ld_ro_stream(const void *p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

// L2 residency policies (createpolicy). The deferred path keeps its log --
// a few hundred bytes per head per entry -- in L2 across steps (evict_last),
// while the base state streams through once per step (evict_first).
__device__ __forceinline__ uint64_t l2_policy_keep() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ uint64_t l2_policy_stream() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}
// Read-only 16-byte stream load under an L2 policy, no L1 allocation.
__device__ __forceinline__ uint4 ld_ro_hint(const void *p, uint64_t pol) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0, %1, %2, %3}, [%4], %5;"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p), "l"(pol));
    return r;
}
// Loads / stores of small operands under an L2 policy (bytes: 2, 4, 8, 16).
template <int BYTES> struct HintWord;
template <> struct HintWord<2> { using T = unsigned short; };
template <> struct HintWord<4> { using T = uint32_t; };
template <> struct HintWord<8> { using T = uint2; };
template <> struct HintWord<16> { using T = uint4; };

__device__ __forceinline__ void st_hint(void *p, unsigned short v, uint64_t pol) {
    asm volatile("st.global.L2::cache_hint.b16 [%0], %1, %2;" ::"l"(p), "h"(v), "l"(pol) : "memory");
}
__device__ __forceinline__ void st_hint(void *p, uint32_t v, uint64_t pol) {
    asm volatile("st.global.L2::cache_hint.b32 [%0], %1, %2;" ::"l"(p), "r"(v), "l"(pol) : "memory");
}
__device__ __forceinline__ void st_hint(void *p, uint2 v, uint64_t pol) {
    asm volatile("st.global.L2::cache_hint.v2.b32 [%0], {%1, %2}, %3;" ::"l"(p), "r"(v.x), "r"(v.y), "l"(pol)
                 : "memory");
}
__device__ __forceinline__ void st_hint(void *p, uint4 v, uint64_t pol) {
    asm volatile("st.global.L2::cache_hint.v4.b32 [%0], {%1, %2, %3, %4}, %5;" ::"l"(p), "r"(v.x), "r"(v.y),
                 "r"(v.z), "r"(v.w), "l"(pol)
                 : "memory");
}
__device__ __forceinline__ void ld_hint(const void *p, unsigned short &v, uint64_t pol) {
    asm volatile("ld.global.L2::cache_hint.b16 %0, [%1], %2;" : "=h"(v) : "l"(p), "l"(pol));
}
__device__ __forceinline__ void ld_hint(const void *p, uint32_t &v, uint64_t pol) {
    asm volatile("ld.global.L2::cache_hint.b32 %0, [%1], %2;" : "=r"(v) : "l"(p), "l"(pol));
}
__device__ __forceinline__ void ld_hint(const void *p, uint2 &v, uint64_t pol) {
    asm volatile("ld.global.L2::cache_hint.v2.b32 {%0, %1}, [%2], %3;" : "=r"(v.x), "=r"(v.y) : "l"(p), "l"(pol));
}
__device__ __forceinline__ void ld_hint(const void *p, uint4 &v, uint64_t pol) {
    asm volatile("ld.global.L2::cache_hint.v4.b32 {%0, %1, %2, %3}, [%4], %5;"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p), "l"(pol));
}
// Copy N elements of T (N * sizeof(T) a power of two >= 2 bytes, aligned to
// min(16, that)) from src to dst, writing under an L2 policy.
template <int N, class T>
__device__ __forceinline__ void copy_hint(T *dst, const T *src, uint64_t pol) {
    constexpr int BYTES = N * (int)sizeof(T), W = BYTES < 16 ? BYTES : 16, K = BYTES / W;
    using Word = typename HintWord<W>::T;
#pragma unroll
    for (int i = 0; i < K; ++i)
        st_hint(reinterpret_cast<unsigned char *>(dst) + i * W,
                *reinterpret_cast<const Word *>(reinterpret_cast<const unsigned char *>(src) + i * W), pol);
}
// The same copy split in two, so that several copies' loads can be in flight
// before the first store: load() reads the words, store() writes them.
template <int N, class T>
struct RawCopy {
    static constexpr int BYTES = N * (int)sizeof(T), W = BYTES < 16 ? BYTES : 16, K = BYTES / W;
    using Word = typename HintWord<W>::T;
    Word w[K];
    __device__ __forceinline__ void load(const T *src) {
#pragma unroll
        for (int i = 0; i < K; ++i)
            w[i] = *reinterpret_cast<const Word *>(reinterpret_cast<const unsigned char *>(src) + i * W);
    }
    __device__ __forceinline__ void load_hint(const T *src, uint64_t pol) {
#pragma unroll
        for (int i = 0; i < K; ++i) ld_hint(reinterpret_cast<const unsigned char *>(src) + i * W, w[i], pol);
    }
    __device__ __forceinline__ void store(T *dst, uint64_t pol) const {
#pragma unroll
        for (int i = 0; i < K; ++i) st_hint(reinterpret_cast<unsigned char *>(dst) + i * W, w[i], pol);
    }
    // the N elements widened to float
    __device__ __forceinline__ void widen(float (&x)[N]) const {
        const T *e = reinterpret_cast<const T *>(w);
#pragma unroll
        for (int i = 0; i < N; ++i) x[i] = to_f(e[i]);
    }
};
// N elements of T (as load_vec) read under an L2 policy, widened to float.
template <int N, class T>
__device__ __forceinline__ void load_vec_hint(const T *p, float (&x)[N], uint64_t pol) {
    constexpr int BYTES = N * (int)sizeof(T), W = BYTES < 16 ? BYTES : 16, K = BYTES / W, PER = W / (int)sizeof(T);
    using Word = typename HintWord<W>::T;
#pragma unroll
    for (int i = 0; i < K; ++i) {
        Word w;
        ld_hint(reinterpret_cast<const unsigned char *>(p) + i * W, w, pol);
        const T *e = reinterpret_cast<const T *>(&w);
#pragma unroll
        for (int j = 0; j < PER; ++j) x[i * PER + j] = to_f(e[j]);
    }
}

// ---------------------------------------------------------------- reductions

// Sum over aligned groups of G consecutive lanes (G a power of two <= 32);
// every lane of the group receives the group's sum.
template <int G>
__device__ __forceinline__ float group_sum(float x) {
#pragma unroll
    for (int off = G / 2; off > 0; off >>= 1)
        x += __shfl_xor_sync(0xffffffffu, x, off);
    return x;
}

// Sum each of N values (N a power of two, 2..32) over all 32 lanes of the
// warp at once with a transposing butterfly: every exchange step halves the
// values a lane keeps, so the whole reduction costs N - 1 + (5 - log2 N)
// shuffles instead of 5 N. Afterwards v[0] of lane l holds the warp-wide sum
// of entry l >> (5 - log2 N).
template <int N>
__device__ __forceinline__ void multi_sum(float (&v)[N], int lane) {
    static_assert(N >= 2 && N <= 32 && (N & (N - 1)) == 0, "power of two");
#pragma unroll
    for (int half = N / 2, off = 16; half >= 1; half >>= 1, off >>= 1) {
        const bool upper = (lane & off) != 0;
#pragma unroll
        for (int i = 0; i < half; ++i) {
            const float keep = upper ? v[i + half] : v[i];
            const float send = upper ? v[i] : v[i + half];
            v[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
        }
    }
    constexpr int steps = (N == 2 ? 1 : N == 4 ? 2 : N == 8 ? 3 : N == 16 ? 4 : 5);
#pragma unroll
    for (int off = 16 >> steps; off > 0; off >>= 1) v[0] += __shfl_xor_sync(0xffffffffu, v[0], off);
}

// ---------------------------------------------------------------- staging

// Copy a rows x cols block of IT (each row contiguous in global memory, row
// r at src + r * src_stride; cols a multiple of 16 / sizeof(IT)) into shared
// memory as float with row stride dst_stride. All threads of the block take
// part; the flat chunk loop is unrolled so several 16-byte loads are in
// flight per thread before the first shared store.
template <class IT>
__device__ __forceinline__ void stage_block(float *dst, int dst_stride, const IT *src, long long src_stride,
                                            int rows, int cols, int tid, int nthreads) {
    constexpr int E = 16 / (int)sizeof(IT);
    const int cpr = cols / E;  // chunks per row
    const int total = rows * cpr;
#pragma unroll 4
    for (int c = tid; c < total; c += nthreads) {
        const int r = c / cpr, j = (c - r * cpr) * E;
        float x[E];
        load_vec<E>(src + r * src_stride + j, x);
#pragma unroll
        for (int e = 0; e < E; ++e) dst[r * dst_stride + j + e] = x[e];
    }
}

// ---------------------------------------------------------------- PDL

// Programmatic dependent launch: a producer lets the next kernel in the
// stream start early; the consumer waits for the producer's completion (and
// memory) only where it first reads the producer's results. Both are no-ops
// when the launch did not opt in.
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// ---------------------------------------------------------------- async copy

__device__ __forceinline__ void cp_async16(void *smem_dst, const void *gmem_src) {
    uint32_t s = static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst));
    asm volatile("cp.async.cg.shared.global.L2::128B [%0], [%1], 16;" ::"r"(s), "l"(gmem_src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

}  // namespace dl
