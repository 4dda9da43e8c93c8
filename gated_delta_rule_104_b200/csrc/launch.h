// Internal launcher interface between the C-ABI layer (api.cu) and the
// kernels. Arguments are already validated when these are called.
#pragma once

#include <algorithm>
#include <mutex>
#include <set>
#include <type_traits>
#include <utility>

#include "../../include/deltalog.h"
#include "common.cuh"

namespace dl {

struct StepParams {
    void *S;             // [B, H, d_v, d_k] state or deferred base
    const void *q, *k, *v, *beta, *a;  // this step's inputs (may be null for a plain merge)
    float *o;            // [B, H, d_v] output (may be null for a plain merge)
    int B, H, dk, dv;
    int kind;            // dl_decay: GDN (head decay), KDA (channel decay), RWKV6 (channel decay, no delta)
    dl_dtype s_dt, in_dt;
    bool chan() const { return kind != DL_DECAY_HEAD; }
};

// Compile-time rule of a kernel instantiation (the dl_decay value).
template <int KIND>
struct Rule {
    static constexpr bool CHAN = KIND != DL_DECAY_HEAD;  // a decay value per key channel
    static constexpr bool DELTA = KIND != DL_RWKV6;      // delta-rule correction (beta, S'k)
};

struct LogParams {
    void *k, *v, *beta, *a;  // [B, H, L, *]
    float *x;                // [B, H, L, L] rows of X = (I + Diag(beta) C)^{-1} Diag(beta), e <= j
    int L;
};

// Slot indirection of the pool entry points. With slot == nullptr (the plain
// entry points) batch head i is state/log head i and the log count is the
// launch's scalar n. Otherwise batch row b works on state and log slot
// slot[b] with counts[slot[b]] entries; a launch only takes the rows its part
// of the step owns (PoolPart), and rows whose slot or count is out of range
// are skipped (and flagged in *status, when given).
enum PoolPart { POOL_APPEND = 0, POOL_MERGE_FULL = 1, POOL_FLUSH = 2 };
struct PoolIdx {
    const int *slot = nullptr;  // [B] slot of each batch row
    int *counts = nullptr;        // [P] log entries held per slot
    int *status = nullptr;        // optional error word (bit 0: a slot or count out of range)
    int P = 0, H = 1, L = 0;
};

// Batch head -> (state head, count) for one part of a pool step; false if the
// head is not this launch's to process.
__device__ __forceinline__ bool pool_head(const PoolIdx &pi, int part, long long head, long long &shead, int &n) {
    if (pi.slot == nullptr) {
        shead = head;
        return true;
    }
    const long long b = head / pi.H;
    const int h = (int)(head - b * pi.H);
    const int s = pi.slot[b];
    const int c = (s >= 0 && s < pi.P) ? pi.counts[s] : -1;
    if (c < 0 || c >= pi.L) {
        if (pi.status && h == 0) atomicOr(pi.status, 1);
        return false;
    }
    shead = (long long)s * pi.H + h;
    n = c;
    if (part == POOL_APPEND) return c < pi.L - 1;
    if (part == POOL_MERGE_FULL) return c == pi.L - 1;
    return c > 0;  // POOL_FLUSH
}

// Lets `kern` use `bytes` (> 48 KB) of dynamic shared memory on the current
// device: set once per (kernel, device), thread-safe; a no-op for 48 KB or less.
inline cudaError_t allow_smem(const void *kern, size_t bytes) {
    if (bytes <= 48 * 1024) return cudaSuccess;
    static std::mutex mu;
    static std::set<std::pair<const void *, int>> done;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(mu);
    if (done.count({kern, dev})) return cudaSuccess;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e == cudaSuccess) done.insert({kern, dev});
    return e;
}

cudaError_t launch_eager(const StepParams &p, cudaStream_t st);
// Deferred read. The fused one-kernel form (fused_read_supported: an fp32 or
// bf16 base, logs of up to 16 entries, no slot pool) needs no workspace; the
// two-kernel form takes read_work_bytes() of fp32 workspace (x_0 and w per head).
bool fused_read_supported(const StepParams &p, int L, const PoolIdx &pool);
cudaError_t launch_append_read(const StepParams &p, const LogParams &lg, int n, float *work, cudaStream_t st,
                               const PoolIdx &pool = PoolIdx{});
size_t read_work_bytes(int B, int H, int dk, int dv);
// The same with the scratch in a fixed module array (DL_NOALLOC_WORK_BYTES).
cudaError_t launch_append_read_noalloc(const StepParams &p, const LogParams &lg, int n, cudaStream_t st);
// Merge n_log log entries (plus, if with_cur, this step's inputs as one more
// entry, and then o = S_new q) into the base.
cudaError_t launch_merge(const StepParams &p, const LogParams &lg, int n_log, bool with_cur,
                         cudaStream_t st, const PoolIdx &pool = PoolIdx{}, int part = POOL_MERGE_FULL);
// The same merge on the tcgen05 tensor cores (merge_tc.cu), for the cases
// merge_tc_supported() accepts: an fp32 or int8 base, d_k = 128, d_v a
// multiple of 128, 1..16 entries in all, no slot pool.
bool merge_tc_supported(const StepParams &p, int n_log, bool with_cur, const PoolIdx &pool);
cudaError_t launch_merge_tc(const StepParams &p, const LogParams &lg, int n_log, bool with_cur, cudaStream_t st);
// The tensor-core kernels' fault word (bit 0: a bounded wait ran out), read
// synchronously; cleared afterwards when `clear`.
cudaError_t read_tc_faults(unsigned int *out, bool clear);
// The same for the fused append-read kernel (deferred_read.cu).
cudaError_t read_read_faults(unsigned int *out, bool clear);
// index-guard words of the kernels' files (bit 1: a shared-memory write out of
// bounds was skipped; line: the source line of the first); 0 in the ordinary build
cudaError_t read_guard_merge(unsigned int *flags, unsigned int *line, bool clear);
cudaError_t read_guard_read(unsigned int *flags, unsigned int *line, bool clear);
cudaError_t read_guard_merge_tc(unsigned int *flags, unsigned int *line, bool clear);
// State conversions to / from the int8 layout (rows = B*H*d_v rows of d_k).
cudaError_t launch_to_i8(const void *S, dl_dtype s_dt, void *S_i8, long long rows, int dk, cudaStream_t st);
cudaError_t launch_from_i8(const void *S_i8, void *S, dl_dtype s_dt, long long rows, int dk, cudaStream_t st);

// Pool bookkeeping after a step (advance = true: count + 1, or 0 after the L-th
// entry merged) or a flush (advance = false: count = 0), for each batch row's slot.
cudaError_t launch_pool_counts(const PoolIdx &pool, int B, bool advance, cudaStream_t st);

// Calls f(ST{}, IT{}, DK_constant, DV_constant, KIND_constant) with the
// compile-time types/sizes matching the runtime description.
template <class F>
cudaError_t dispatch(const StepParams &p, F &&f) {
    auto with_chan = [&](auto st, auto it, auto dk, auto dv) -> cudaError_t {
        switch (p.kind) {
            case DL_DECAY_HEAD: return f(st, it, dk, dv, std::integral_constant<int, DL_DECAY_HEAD>{});
            case DL_DECAY_CHANNEL: return f(st, it, dk, dv, std::integral_constant<int, DL_DECAY_CHANNEL>{});
            case DL_RWKV6: return f(st, it, dk, dv, std::integral_constant<int, DL_RWKV6>{});
        }
        return cudaErrorInvalidValue;
    };
    auto with_dv = [&](auto st, auto it, auto dk) -> cudaError_t {
        switch (p.dv) {
            case 64: return with_chan(st, it, dk, std::integral_constant<int, 64>{});
            case 128: return with_chan(st, it, dk, std::integral_constant<int, 128>{});
            case 256: return with_chan(st, it, dk, std::integral_constant<int, 256>{});
        }
        return cudaErrorInvalidValue;
    };
    auto with_dk = [&](auto st, auto it) -> cudaError_t {
        switch (p.dk) {
            case 64: return with_dv(st, it, std::integral_constant<int, 64>{});
            case 128: return with_dv(st, it, std::integral_constant<int, 128>{});
        }
        return cudaErrorInvalidValue;
    };
    auto with_it = [&](auto st) -> cudaError_t {
        if (p.in_dt == DL_BF16) return with_dk(st, bf16{});
        return with_dk(st, float{});
    };
    if (p.s_dt == DL_BF16) return with_it(bf16{});
    return with_it(float{});
}

}  // namespace dl
