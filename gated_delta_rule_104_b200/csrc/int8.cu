// Conversions between a float32 / bfloat16 state and the int8 layout of a
// deferred base (DL_I8: int8 codes row-major, then one float scale per row;
// value = code * scale). One warp per state row of d_k elements.
#include "launch.h"

namespace dl {

template <class ST>
__global__ void __launch_bounds__(256)
to_i8_kernel(const ST *__restrict__ S, int8_t *__restrict__ codes, float *__restrict__ scales, long long rows,
             int dk) {
    const long long r = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (r >= rows) return;
    const ST *row = S + r * dk;
    float m = 0.f;
    for (int c = lane; c < dk; c += 32) m = fmaxf(m, fabsf(to_f(row[c])));
    const float sc = i8_scale(warp_max(m)), inv = i8_inv(sc);
    if (i8_fast(sc))
        for (int c = lane; c < dk; c += 32) codes[r * dk + c] = (int8_t)i8_code(to_f(row[c]), sc, inv);
    else
        for (int c = lane; c < dk; c += 32) codes[r * dk + c] = (int8_t)i8_code_div(to_f(row[c]), sc);
    if (lane == 0) scales[r] = sc;
}

__device__ __forceinline__ void store_elem(float *p, float x) { *p = x; }
__device__ __forceinline__ void store_elem(bf16 *p, float x) { *p = __float2bfloat16_rn(x); }

template <class ST>
__global__ void __launch_bounds__(256)
from_i8_kernel(const int8_t *__restrict__ codes, const float *__restrict__ scales, ST *__restrict__ S,
               long long rows, int dk) {
    const long long r = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (r >= rows) return;
    const float sc = scales[r];
    for (int c = lane; c < dk; c += 32) store_elem(S + r * dk + c, (float)codes[r * dk + c] * sc);
}

cudaError_t launch_to_i8(const void *S, dl_dtype s_dt, void *S_i8, long long rows, int dk, cudaStream_t st) {
    int8_t *codes = static_cast<int8_t *>(S_i8);
    float *scales = reinterpret_cast<float *>(codes + rows * dk);
    const unsigned blocks = (unsigned)((rows + 7) / 8);
    if (s_dt == DL_BF16)
        to_i8_kernel<bf16><<<blocks, 256, 0, st>>>(static_cast<const bf16 *>(S), codes, scales, rows, dk);
    else
        to_i8_kernel<float><<<blocks, 256, 0, st>>>(static_cast<const float *>(S), codes, scales, rows, dk);
    return cudaGetLastError();
}

cudaError_t launch_from_i8(const void *S_i8, void *S, dl_dtype s_dt, long long rows, int dk, cudaStream_t st) {
    const int8_t *codes = static_cast<const int8_t *>(S_i8);
    const float *scales = reinterpret_cast<const float *>(codes + rows * dk);
    const unsigned blocks = (unsigned)((rows + 7) / 8);
    if (s_dt == DL_BF16)
        from_i8_kernel<bf16><<<blocks, 256, 0, st>>>(codes, scales, static_cast<bf16 *>(S), rows, dk);
    else
        from_i8_kernel<float><<<blocks, 256, 0, st>>>(codes, scales, static_cast<float *>(S), rows, dk);
    return cudaGetLastError();
}

}  // namespace dl
