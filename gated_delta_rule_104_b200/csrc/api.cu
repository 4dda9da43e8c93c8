// C-ABI layer of libdeltalog: host-side argument checks (before any CUDA
// call), then dispatch to the kernels. Declarations and the contract of each
// entry point are in include/deltalog.h.
#include <stdarg.h>
#include <stdint.h>
#include <stdio.h>

#include "launch.h"

namespace {

thread_local char g_err[512] = "";

dl_status fail(dl_status s, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof(g_err), fmt, ap);
    va_end(ap);
    return s;
}

dl_status ok() {
    g_err[0] = '\0';
    return DL_OK;
}

size_t elem_size(dl_dtype t) { return t == DL_BF16 ? 2 : 4; }
bool valid_dtype(int t) { return t == DL_F32 || t == DL_BF16; }
bool valid_state_dtype(int t) { return t == DL_F32 || t == DL_BF16 || t == DL_I8; }
// Bytes of BH heads of d_v x d_k state (DL_I8: codes, then a float scale per row).
size_t state_bytes(dl_dtype t, size_t bh, int dk, int dv) {
    if (t == DL_I8) return bh * dv * dk + bh * dv * sizeof(float);
    return bh * dv * dk * elem_size(t);
}
bool valid_decay(int t) { return t == DL_DECAY_HEAD || t == DL_DECAY_CHANNEL || t == DL_RWKV6; }

struct Buf {
    const char *name;
    const void *p;
    size_t bytes;
    size_t align;
    bool unused = false;  // not read by this kind (may be null)
};

bool overlaps(const Buf &a, const Buf &b) {
    if (a.unused || b.unused || !a.p || !b.p || !a.bytes || !b.bytes) return false;
    const uintptr_t a0 = (uintptr_t)a.p, b0 = (uintptr_t)b.p;
    return a0 < b0 + b.bytes && b0 < a0 + a.bytes;
}

dl_status check_bufs(const Buf *bufs, int nb) {
    for (int i = 0; i < nb; ++i) {
        if (bufs[i].unused) continue;
        if (!bufs[i].p) return fail(DL_ERR_INVALID_ARG, "%s is a null pointer", bufs[i].name);
        if ((uintptr_t)bufs[i].p % bufs[i].align)
            return fail(DL_ERR_INVALID_ARG, "%s is not %zu-byte aligned", bufs[i].name, bufs[i].align);
    }
    return DL_OK;
}

// Writers must not overlap anything else in the call.
dl_status check_overlap(const Buf *writers, int nw, const Buf *all, int na) {
    for (int i = 0; i < nw; ++i)
        for (int j = 0; j < na; ++j) {
            if (writers[i].p == all[j].p && writers[i].name == all[j].name) continue;
            if (overlaps(writers[i], all[j]))
                return fail(DL_ERR_INVALID_ARG, "%s overlaps %s", writers[i].name, all[j].name);
        }
    return DL_OK;
}

dl_status check_dims(int B, int H, int dk, int dv, int s_dt, int in_dt) {
    if (B < 1 || H < 1) return fail(DL_ERR_INVALID_ARG, "B and H must be >= 1 (got B=%d, H=%d)", B, H);
    if ((long long)B * H > (1LL << 26)) return fail(DL_ERR_UNSUPPORTED, "B*H=%lld exceeds 2^26", (long long)B * H);
    if (!valid_state_dtype(s_dt)) return fail(DL_ERR_INVALID_ARG, "unknown state dtype %d", s_dt);
    if (!valid_dtype(in_dt)) return fail(DL_ERR_INVALID_ARG, "unknown input dtype %d", in_dt);
    if (dk != 64 && dk != 128) return fail(DL_ERR_UNSUPPORTED, "d_k=%d not in {64, 128}", dk);
    if (dv != 64 && dv != 128 && dv != 256) return fail(DL_ERR_UNSUPPORTED, "d_v=%d not in {64, 128, 256}", dv);
    return DL_OK;
}

// Step operands: S, q, k, v, beta, a, o (indices fixed for the callers).
int step_bufs(Buf *out, const void *S, const char *sname, dl_dtype s_dt, const void *q, const void *k,
              const void *v, const void *beta, const void *a, dl_dtype in_dt, const float *o, int B,
              int H, int dk, int dv, int kind) {
    const size_t bh = (size_t)B * H, is = elem_size(in_dt);
    const bool chan = kind != DL_DECAY_HEAD;
    out[0] = {sname, S, state_bytes(s_dt, bh, dk, dv), 16};
    out[1] = {"q", q, bh * dk * is, 16};
    out[2] = {"k", k, bh * dk * is, 16};
    out[3] = {"v", v, bh * dv * is, 16};
    out[4] = {"beta", beta, bh * is, is, kind == DL_RWKV6};
    out[5] = chan ? Buf{"a", a, bh * dk * is, 16} : Buf{"a", a, bh * is, is};
    out[6] = {"o", o, bh * dv * sizeof(float), 16};
    return 7;
}

dl_status check_log(const dl_log *log, Buf *out, dl_dtype in_dt, int B, int H, int dk, int dv, int kind) {
    const bool chan = kind != DL_DECAY_HEAD;
    if (!log) return fail(DL_ERR_INVALID_ARG, "log is a null pointer");
    if (!valid_dtype(log->dtype)) return fail(DL_ERR_INVALID_ARG, "unknown log dtype %d", (int)log->dtype);
    if (log->L < 1 || log->L > DL_MAX_LOG)
        return fail(DL_ERR_UNSUPPORTED, "log capacity L=%d not in 1..%d", log->L, DL_MAX_LOG);
    if (log->dtype != in_dt) return fail(DL_ERR_UNSUPPORTED, "log dtype differs from the input dtype");
    const size_t bhl = (size_t)B * H * log->L, is = elem_size(in_dt);
    out[0] = {"log.k", log->k, bhl * dk * is, 16};
    out[1] = {"log.v", log->v, bhl * dv * is, 16};
    out[2] = {"log.beta", log->beta, bhl * is, is, kind == DL_RWKV6};
    out[3] = chan ? Buf{"log.a", log->a, bhl * dk * is, 16} : Buf{"log.a", log->a, bhl * is, is};
    out[4] = {"log.x", log->x, bhl * log->L * sizeof(float), 16, kind == DL_RWKV6};
    return DL_OK;
}

dl_status cuda_status(cudaError_t e, const char *what) {
    if (e != cudaSuccess) return fail(DL_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
    return ok();
}

dl_status eager_step(void *S, dl_dtype s_dt, const void *q, const void *k, const void *v, const void *beta,
                     const void *a, dl_dtype in_dt, float *o, int B, int H, int dk, int dv,
                     cudaStream_t stream, int kind) {
    dl_status s = check_dims(B, H, dk, dv, s_dt, in_dt);
    if (s != DL_OK) return s;
    if (s_dt == DL_I8) return fail(DL_ERR_UNSUPPORTED, "the eager step takes a float32 or bfloat16 state");
    Buf b[7];
    int nb = step_bufs(b, S, "S", s_dt, q, k, v, beta, a, in_dt, o, B, H, dk, dv, kind);
    if ((s = check_bufs(b, nb)) != DL_OK) return s;
    const Buf writers[2] = {b[0], b[6]};  // S and o are written
    if ((s = check_overlap(writers, 2, b, nb)) != DL_OK) return s;
    dl::StepParams p{S, q, k, v, beta, a, o, B, H, dk, dv, kind, s_dt, in_dt};
    return cuda_status(dl::launch_eager(p, stream), "eager step launch");
}

}  // namespace

extern "C" {

dl_status dl_gdn_decode_step(void *S, dl_dtype s_dtype, const void *q, const void *k, const void *v,
                             const void *beta, const void *a, dl_dtype in_dtype, float *o, int B, int H,
                             int d_k, int d_v, cudaStream_t stream) {
    return eager_step(S, s_dtype, q, k, v, beta, a, in_dtype, o, B, H, d_k, d_v, stream, DL_DECAY_HEAD);
}

dl_status dl_kda_decode_step(void *S, dl_dtype s_dtype, const void *q, const void *k, const void *v,
                             const void *beta, const void *a, dl_dtype in_dtype, float *o, int B, int H,
                             int d_k, int d_v, cudaStream_t stream) {
    return eager_step(S, s_dtype, q, k, v, beta, a, in_dtype, o, B, H, d_k, d_v, stream, DL_DECAY_CHANNEL);
}

dl_status dl_rwkv6_decode_step(void *S, dl_dtype s_dtype, const void *q, const void *k, const void *v,
                               const void *a, dl_dtype in_dtype, float *o, int B, int H, int d_k, int d_v,
                               cudaStream_t stream) {
    return eager_step(S, s_dtype, q, k, v, nullptr, a, in_dtype, o, B, H, d_k, d_v, stream, DL_RWKV6);
}

dl_status dl_log_append_read(const void *S_base, dl_dtype s_dtype, dl_decay kind, const dl_log *log, int n,
                             const void *q, const void *k, const void *v, const void *beta, const void *a,
                             dl_dtype in_dtype, float *o, int B, int H, int d_k, int d_v,
                             cudaStream_t stream) {
    dl_status s = check_dims(B, H, d_k, d_v, s_dtype, in_dtype);
    if (s != DL_OK) return s;
    if (!valid_decay(kind)) return fail(DL_ERR_INVALID_ARG, "unknown decay kind %d", (int)kind);
    Buf b[13];
    int nb = step_bufs(b, S_base, "S_base", s_dtype, q, k, v, beta, a, in_dtype, o, B, H, d_k, d_v, kind);
    if ((s = check_log(log, b + nb, in_dtype, B, H, d_k, d_v, kind)) != DL_OK) return s;
    nb += 5;
    if ((s = check_bufs(b, nb)) != DL_OK) return s;
    if (n < 0) return fail(DL_ERR_INVALID_ARG, "n=%d is negative", n);
    if (n >= log->L) return fail(DL_ERR_LOG_FULL, "log holds n=%d of L=%d entries: merge first", n, log->L);
    const size_t need = dl::read_work_bytes(B, H, d_k, d_v);
    b[nb] = {"log.work", log->work, need, 16};
    if ((s = check_bufs(b + nb, 1)) != DL_OK) return s;
    if (log->work_bytes < need)
        return fail(DL_ERR_INVALID_ARG, "log.work holds %zu bytes, needs %zu", log->work_bytes, need);
    ++nb;
    // written: o, the log (slot n, metadata row n) and its workspace; the base is only read.
    const Buf writers[7] = {b[6], b[7], b[8], b[9], b[10], b[11], b[12]};
    if ((s = check_overlap(writers, 7, b, nb)) != DL_OK) return s;
    dl::StepParams p{const_cast<void *>(S_base), q, k, v, beta, a, o, B, H, d_k, d_v, kind, s_dtype, in_dtype};
    dl::LogParams lg{log->k, log->v, log->beta, log->a, log->x, log->L};
    return cuda_status(dl::launch_append_read(p, lg, n, static_cast<float *>(log->work), stream),
                       "append-read launch");
}

dl_status dl_log_merge(void *S_base, dl_dtype s_dtype, dl_decay kind, const dl_log *log, int n, int B, int H,
                       int d_k, int d_v, cudaStream_t stream) {
    dl_status s = check_dims(B, H, d_k, d_v, s_dtype, log ? (int)log->dtype : (int)DL_F32);
    if (s != DL_OK) return s;
    if (!valid_decay(kind)) return fail(DL_ERR_INVALID_ARG, "unknown decay kind %d", (int)kind);
    if (!log) return fail(DL_ERR_INVALID_ARG, "log is a null pointer");
    Buf b[6];
    b[0] = {"S_base", S_base, state_bytes(s_dtype, (size_t)B * H, d_k, d_v), 16};
    if ((s = check_log(log, b + 1, log->dtype, B, H, d_k, d_v, kind)) != DL_OK) return s;
    if ((s = check_bufs(b, 6)) != DL_OK) return s;
    if (n < 1 || n > log->L) return fail(DL_ERR_INVALID_ARG, "merge needs 1 <= n <= L (n=%d, L=%d)", n, log->L);
    const Buf writers[1] = {b[0]};
    if ((s = check_overlap(writers, 1, b, 6)) != DL_OK) return s;
    const Buf logw[5] = {b[1], b[2], b[3], b[4], b[5]};
    if ((s = check_overlap(logw, 5, b + 1, 5)) != DL_OK) return s;
    dl::StepParams p{S_base, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, B, H, d_k, d_v, kind,
                     s_dtype, log->dtype};
    dl::LogParams lg{log->k, log->v, log->beta, log->a, log->x, log->L};
    return cuda_status(dl::launch_merge(p, lg, n, false, stream), "merge launch");
}

dl_status dl_log_merge_read(void *S_base, dl_dtype s_dtype, dl_decay kind, const dl_log *log, int n,
                            const void *q, const void *k, const void *v, const void *beta, const void *a,
                            dl_dtype in_dtype, float *o, int B, int H, int d_k, int d_v,
                            cudaStream_t stream) {
    dl_status s = check_dims(B, H, d_k, d_v, s_dtype, in_dtype);
    if (s != DL_OK) return s;
    if (!valid_decay(kind)) return fail(DL_ERR_INVALID_ARG, "unknown decay kind %d", (int)kind);
    Buf b[12];
    int nb = step_bufs(b, S_base, "S_base", s_dtype, q, k, v, beta, a, in_dtype, o, B, H, d_k, d_v, kind);
    if ((s = check_log(log, b + nb, in_dtype, B, H, d_k, d_v, kind)) != DL_OK) return s;
    nb += 5;
    if ((s = check_bufs(b, nb)) != DL_OK) return s;
    if (n < 0) return fail(DL_ERR_INVALID_ARG, "n=%d is negative", n);
    if (n >= log->L) return fail(DL_ERR_LOG_FULL, "log holds n=%d of L=%d entries: merge first", n, log->L);
    const Buf writers[2] = {b[0], b[6]};  // the base and o
    if ((s = check_overlap(writers, 2, b, nb)) != DL_OK) return s;
    dl::StepParams p{S_base, q, k, v, beta, a, o, B, H, d_k, d_v, kind, s_dtype, in_dtype};
    dl::LogParams lg{log->k, log->v, log->beta, log->a, log->x, log->L};
    return cuda_status(dl::launch_merge(p, lg, n, true, stream), "merge-read launch");
}

dl_status dl_log_append_read_noalloc(const void *S_base, dl_dtype s_dtype, dl_decay kind, const dl_log *log,
                                     int n, const void *q, const void *k, const void *v, const void *beta,
                                     const void *a, dl_dtype in_dtype, float *o, int B, int H, int d_k, int d_v,
                                     cudaStream_t stream) {
    dl_status s = check_dims(B, H, d_k, d_v, s_dtype, in_dtype);
    if (s != DL_OK) return s;
    if (!valid_decay(kind)) return fail(DL_ERR_INVALID_ARG, "unknown decay kind %d", (int)kind);
    Buf b[12];
    int nb = step_bufs(b, S_base, "S_base", s_dtype, q, k, v, beta, a, in_dtype, o, B, H, d_k, d_v, kind);
    if ((s = check_log(log, b + nb, in_dtype, B, H, d_k, d_v, kind)) != DL_OK) return s;
    nb += 5;
    if ((s = check_bufs(b, nb)) != DL_OK) return s;
    if (n < 0) return fail(DL_ERR_INVALID_ARG, "n=%d is negative", n);
    if (n >= log->L) return fail(DL_ERR_LOG_FULL, "log holds n=%d of L=%d entries: merge first", n, log->L);
    const size_t need = dl::read_work_bytes(B, H, d_k, d_v);
    if (need > DL_NOALLOC_WORK_BYTES)
        return fail(DL_ERR_UNSUPPORTED,
                    "B*H*(d_k+d_v)*4 = %zu bytes of scratch exceeds the built-in %zu-byte array "
                    "(DL_NOALLOC_WORK_BYTES); use dl_log_append_read with a workspace",
                    need, (size_t)DL_NOALLOC_WORK_BYTES);
    const Buf writers[6] = {b[6], b[7], b[8], b[9], b[10], b[11]};  // o and the log
    if ((s = check_overlap(writers, 6, b, nb)) != DL_OK) return s;
    dl::StepParams p{const_cast<void *>(S_base), q, k, v, beta, a, o, B, H, d_k, d_v, kind, s_dtype, in_dtype};
    dl::LogParams lg{log->k, log->v, log->beta, log->a, log->x, log->L};
    return cuda_status(dl::launch_append_read_noalloc(p, lg, n, stream), "no-alloc append-read launch");
}

// ------------------------------------------------------------------ slot pool

static dl_status pool_checks(const dl_pool *pool, dl_decay kind, const int *slot, dl_dtype in_dt, int B, int H,
                             int d_k, int d_v, Buf *b, int &nb) {
    if (!pool) return fail(DL_ERR_INVALID_ARG, "pool is a null pointer");
    dl_status s = check_dims(B, H, d_k, d_v, pool->s_dtype, in_dt);
    if (s != DL_OK) return s;
    if (!valid_decay(kind)) return fail(DL_ERR_INVALID_ARG, "unknown decay kind %d", (int)kind);
    if (pool->P < 1) return fail(DL_ERR_INVALID_ARG, "pool.P=%d must be >= 1", pool->P);
    if (B > pool->P) return fail(DL_ERR_INVALID_ARG, "B=%d rows need distinct slots but P=%d", B, pool->P);
    if ((long long)pool->P * H > (1LL << 26)) return fail(DL_ERR_UNSUPPORTED, "P*H exceeds 2^26");
    if ((s = check_log(&pool->log, b + nb, in_dt, pool->P, H, d_k, d_v, kind)) != DL_OK) return s;
    nb += 5;
    b[nb++] = {"pool.n", pool->n, (size_t)pool->P * sizeof(int), 4};
    b[nb++] = {"slot", slot, (size_t)B * sizeof(int), 4};
    b[nb++] = {"pool.status", pool->status, sizeof(int), 4, pool->status == nullptr};
    return DL_OK;
}

dl_status dl_pool_step(const dl_pool *pool, dl_decay kind, const int *slot, const void *q, const void *k,
                       const void *v, const void *beta, const void *a, dl_dtype in_dtype, float *o, int B, int H,
                       int d_k, int d_v, cudaStream_t stream) {
    Buf b[17];
    int nb = 7;
    if (pool) step_bufs(b, pool->S, "pool.S", pool->s_dtype, q, k, v, beta, a, in_dtype, o, B, H, d_k, d_v, kind);
    dl_status s = pool_checks(pool, kind, slot, in_dtype, B, H, d_k, d_v, b, nb);
    if (s != DL_OK) return s;
    b[0].bytes = state_bytes(pool->s_dtype, (size_t)pool->P * H, d_k, d_v);  // the whole pool
    const size_t need = dl::read_work_bytes(B, H, d_k, d_v);
    b[nb++] = {"log.work", pool->log.work, need, 16};
    if ((s = check_bufs(b, nb)) != DL_OK) return s;
    if (pool->log.work_bytes < need)
        return fail(DL_ERR_INVALID_ARG, "log.work holds %zu bytes, needs %zu", pool->log.work_bytes, need);
    // written: the pool's bases (merging slots), o, the logs, counts, status, workspace
    const Buf writers[10] = {b[0], b[6], b[7], b[8], b[9], b[10], b[11], b[12], b[14], b[15]};
    if ((s = check_overlap(writers, 10, b, nb)) != DL_OK) return s;
    dl::StepParams p{pool->S, q, k, v, beta, a, o, B, H, d_k, d_v, kind, pool->s_dtype, in_dtype};
    const dl_log *lg0 = &pool->log;
    dl::LogParams lg{lg0->k, lg0->v, lg0->beta, lg0->a, lg0->x, lg0->L};
    dl::PoolIdx pi;
    pi.slot = slot;
    pi.counts = pool->n;
    pi.status = pool->status;
    pi.P = pool->P;
    pi.H = H;
    pi.L = lg0->L;
    // the merge part (rows on their L-th entry) first; the append part of the
    // other rows runs beside it (programmatic dependent launch), then the counts
    cudaError_t e = dl::launch_merge(p, lg, lg0->L - 1, true, stream, pi, dl::POOL_MERGE_FULL);
    if (e == cudaSuccess) e = dl::launch_append_read(p, lg, 0, static_cast<float *>(lg0->work), stream, pi);
    if (e == cudaSuccess) e = dl::launch_pool_counts(pi, B, true, stream);
    return cuda_status(e, "pool step launch");
}

dl_status dl_pool_flush(const dl_pool *pool, dl_decay kind, const int *slot, int B, int H, int d_k, int d_v,
                        cudaStream_t stream) {
    Buf b[10];
    int nb = 1;
    if (pool) b[0] = {"pool.S", pool->S, state_bytes(pool->s_dtype, (size_t)pool->P * H, d_k, d_v), 16};
    dl_status s = pool_checks(pool, kind, slot, pool ? pool->log.dtype : DL_F32, B, H, d_k, d_v, b, nb);
    if (s != DL_OK) return s;
    if ((s = check_bufs(b, nb)) != DL_OK) return s;
    const Buf writers[3] = {b[0], b[6], b[8]};  // bases, counts, status
    if ((s = check_overlap(writers, 3, b, nb)) != DL_OK) return s;
    dl::StepParams p{pool->S, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, B, H, d_k, d_v, kind,
                     pool->s_dtype, pool->log.dtype};
    const dl_log *lg0 = &pool->log;
    dl::LogParams lg{lg0->k, lg0->v, lg0->beta, lg0->a, lg0->x, lg0->L};
    dl::PoolIdx pi;
    pi.slot = slot;
    pi.counts = pool->n;
    pi.status = pool->status;
    pi.P = pool->P;
    pi.H = H;
    pi.L = lg0->L;
    cudaError_t e = dl::launch_merge(p, lg, lg0->L - 1, false, stream, pi, dl::POOL_FLUSH);
    if (e == cudaSuccess) e = dl::launch_pool_counts(pi, B, false, stream);
    return cuda_status(e, "pool flush launch");
}

size_t dl_state_bytes(dl_dtype s_dtype, int B, int H, int d_k, int d_v) {
    if (B < 1 || H < 1 || d_k < 1 || d_v < 1 || !valid_state_dtype(s_dtype)) return 0;
    return state_bytes(s_dtype, (size_t)B * H, d_k, d_v);
}

static dl_status convert_checks(const void *S, dl_dtype s_dtype, const void *S_i8, int B, int H, int d_k, int d_v) {
    dl_status s = check_dims(B, H, d_k, d_v, s_dtype, DL_F32);
    if (s != DL_OK) return s;
    if (s_dtype == DL_I8) return fail(DL_ERR_INVALID_ARG, "the other state must be float32 or bfloat16");
    const size_t bh = (size_t)B * H;
    Buf b[2] = {{"S", S, state_bytes(s_dtype, bh, d_k, d_v), 16}, {"S_i8", S_i8, state_bytes(DL_I8, bh, d_k, d_v), 16}};
    if ((s = check_bufs(b, 2)) != DL_OK) return s;
    return check_overlap(b, 2, b, 2);
}

dl_status dl_state_to_i8(const void *S, dl_dtype s_dtype, void *S_i8, int B, int H, int d_k, int d_v,
                         cudaStream_t stream) {
    dl_status s = convert_checks(S, s_dtype, S_i8, B, H, d_k, d_v);
    if (s != DL_OK) return s;
    return cuda_status(dl::launch_to_i8(S, s_dtype, S_i8, (long long)B * H * d_v, d_k, stream), "to-int8 launch");
}

dl_status dl_state_from_i8(const void *S_i8, void *S, dl_dtype s_dtype, int B, int H, int d_k, int d_v,
                           cudaStream_t stream) {
    dl_status s = convert_checks(S, s_dtype, S_i8, B, H, d_k, d_v);
    if (s != DL_OK) return s;
    return cuda_status(dl::launch_from_i8(S_i8, S, s_dtype, (long long)B * H * d_v, d_k, stream),
                       "from-int8 launch");
}

const char *dl_status_string(dl_status s) {
    switch (s) {
        case DL_OK: return "ok";
        case DL_ERR_INVALID_ARG: return "invalid argument";
        case DL_ERR_UNSUPPORTED: return "unsupported size or dtype";
        case DL_ERR_LOG_FULL: return "log full";
        case DL_ERR_CUDA: return "CUDA launch error";
    }
    return "unknown status";
}

const char *dl_last_error(void) { return g_err; }

size_t dl_log_work_bytes(int B, int H, int d_k, int d_v) {
    if (B < 1 || H < 1 || d_k < 1 || d_v < 1) return 0;
    return dl::read_work_bytes(B, H, d_k, d_v);
}

int dl_abi_version(void) { return DL_ABI_VERSION; }

dl_status dl_device_faults(unsigned int *flags, int clear) {
    if (!flags) return fail(DL_ERR_INVALID_ARG, "flags is a null pointer");
    *flags = 0;
    unsigned int w = 0;
    dl_status st = cuda_status(dl::read_tc_faults(&w, clear != 0), "fault word read");
    if (st != DL_OK) return st;
    *flags = w;
    st = cuda_status(dl::read_read_faults(&w, clear != 0), "fault word read");
    if (st != DL_OK) return st;
    *flags |= w;
    struct {
        const char *file;
        cudaError_t (*read)(unsigned int *, unsigned int *, bool);
    } const units[] = {{"merge.cu", dl::read_guard_merge},
                       {"deferred_read.cu", dl::read_guard_read},
                       {"merge_tc.cu", dl::read_guard_merge_tc}};
    for (const auto &u : units) {
        unsigned int g = 0, line = 0;
        st = cuda_status(u.read(&g, &line, clear != 0), "guard word read");
        if (st != DL_OK) return st;
        if (g) {
            *flags |= g;
            snprintf(g_err, sizeof g_err, "index guard: an out-of-bounds shared-memory write was skipped (%s:%u)",
                          u.file, line);
        }
    }
    return DL_OK;
}

int dl_index_guard_build(void) {
#ifdef DL_INDEX_GUARD
    return 1;
#else
    return 0;
#endif
}

}  // extern "C"
