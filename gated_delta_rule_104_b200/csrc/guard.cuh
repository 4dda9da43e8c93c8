// Index guard of the debug build. Compiled with DL_INDEX_GUARD, every
// shared-memory write of the kernels (plain stores and the destinations of
// cp.async copies) first checks that its bytes lie inside the block's dynamic
// shared memory and that its address is aligned for its width; a write that
// fails the check is skipped and recorded in the translation unit's guard
// word (bit 1; the source line of the first such write is kept beside it).
// The ordinary build compiles every check away.
//
//   DL_GUARD(ptr, bytes) statement;
//
// prefixes the statement that writes `bytes` at `ptr`; the statement runs only
// when the check passes. Use it on a statement of its own (inside braces when
// it is the body of an if).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#ifdef DL_INDEX_GUARD

namespace dl {

extern __shared__ float4 dl_guard_dyn_smem[];  // the base of the block's dynamic shared memory

namespace {

__device__ unsigned int g_guard[2];             // [0]: bit 1 = a write was out of bounds; [1]: its source line

__device__ __forceinline__ bool guard_ok(const void *p, unsigned bytes, int line) {
    const uint32_t a = (uint32_t)__cvta_generic_to_shared(p);
    const uint32_t base = (uint32_t)__cvta_generic_to_shared(dl_guard_dyn_smem);
    uint32_t size;
    asm volatile("mov.u32 %0, %%dynamic_smem_size;" : "=r"(size));
    const unsigned al = bytes >= 16 ? 16u : bytes;
    if (a >= base && a - base + bytes <= size && a % al == 0) return true;
    atomicOr(&g_guard[0], 2u);
    atomicCAS(&g_guard[1], 0u, (unsigned)line);
    return false;
}

// The unit's guard word and line (and zero both when clear).
inline cudaError_t read_guard_word(unsigned int *flags, unsigned int *line, bool clear) {
    unsigned int w[2] = {0u, 0u};
    cudaError_t e = cudaMemcpyFromSymbol(w, g_guard, sizeof(w));
    if (e == cudaSuccess && clear) {
        const unsigned int z[2] = {0u, 0u};
        e = cudaMemcpyToSymbol(g_guard, z, sizeof(z));
    }
    *flags = w[0];
    *line = w[1];
    return e;
}

}  // namespace
}  // namespace dl

#define DL_GUARD(p, n) \
    if (!::dl::guard_ok((p), (unsigned)(n), __LINE__)) { \
    } else

#else

namespace dl {
namespace {
inline cudaError_t read_guard_word(unsigned int *flags, unsigned int *line, bool) {
    *flags = 0u;
    *line = 0u;
    return cudaSuccess;
}
}  // namespace
}  // namespace dl

#define DL_GUARD(p, n)

#endif
