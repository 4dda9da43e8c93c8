// Internal launcher interface between the C-ABI layer (api.cu) and the
// kernels. Arguments are already validated when these are called.
#pragma once

#include <type_traits>

#include "../../include/deltalog.h"
#include "common.cuh"

namespace dl {

struct StepParams {
    void *S;             // [B, H, d_v, d_k] state or deferred base
    const void *q, *k, *v, *beta, *a;  // this step's inputs (may be null for a plain merge)
    float *o;            // [B, H, d_v] output (may be null for a plain merge)
    int B, H, dk, dv;
    bool chan;           // channel-wise decay (KDA) vs head-wise (GDN)
    dl_dtype s_dt, in_dt;
};

struct LogParams {
    void *k, *v, *beta, *a;  // [B, H, L, *]
    float *x;                // [B, H, L, L] rows of X = (I + Diag(beta) C)^{-1} Diag(beta), e <= j
    int L;
};

cudaError_t launch_eager(const StepParams &p, cudaStream_t st);
// Deferred read: needs read_work_bytes() of fp32 workspace (x_0 and w per head).
cudaError_t launch_append_read(const StepParams &p, const LogParams &lg, int n, float *work, cudaStream_t st);
size_t read_work_bytes(int B, int H, int dk, int dv);
// The same with the scratch in a fixed module array (DL_NOALLOC_WORK_BYTES).
cudaError_t launch_append_read_noalloc(const StepParams &p, const LogParams &lg, int n, cudaStream_t st);
// Merge n_log log entries (plus, if with_cur, this step's inputs as one more
// entry, and then o = S_new q) into the base.
cudaError_t launch_merge(const StepParams &p, const LogParams &lg, int n_log, bool with_cur,
                         cudaStream_t st);

// Calls f(ST{}, IT{}, DK_constant, DV_constant, CHAN_constant) with the
// compile-time types/sizes matching the runtime description.
template <class F>
cudaError_t dispatch(const StepParams &p, F &&f) {
    auto with_chan = [&](auto st, auto it, auto dk, auto dv) -> cudaError_t {
        if (p.chan) return f(st, it, dk, dv, std::true_type{});
        return f(st, it, dk, dv, std::false_type{});
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
