/*
 * deltalog.h -- C ABI of the gated delta-rule decode-step library (sm_100a).
 *
 * The operation (DeltaLog: Deferred Materialization of Recurrent States for
 * Linear Attention Decoding, Technical Summary, "Problem" and "Kernel
 * Implementation"): for each sequence b < B and head h < H, a recurrent state
 * S in R^{d_v x d_k} is advanced by one decode step with q, k in R^{d_k},
 * v in R^{d_v}, a scalar beta and a decay a,
 *
 *     S_t = S_{t-1} Diag(a_t) (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,
 *     o_t = S_t q_t,
 *
 * where the decay is one scalar per head for Gated DeltaNet (GDN) and one
 * value per key channel for Kimi Delta Attention (KDA). The third model of
 * the page's operator list, RWKV6 (per-key decay, raw-value update with no
 * delta-rule correction, "Kernel Implementation"), is
 *
 *     S_t = S_{t-1} Diag(a_t) + v_t k_t^T,    o_t = S_t q_t
 *
 * (beta is not used; RWKV6's per-channel "bonus" on the current token is not
 * defined on the page and is not computed).
 *
 * Two schedules:
 *   eager     -- dl_gdn_decode_step / dl_kda_decode_step read S, apply the
 *                step and write S back every token (section "Problem: The
 *                State-Update Tax").
 *   deferred  -- the DeltaLog schedule (section "Methodology", "Core
 *                Mechanism: Base + Log" and "Traffic Model"): a dense base
 *                S_bar is left unwritten while each step appends its factors
 *                (k, v, beta, a) to a bounded per-head log and reads o from
 *                base + log (dl_log_append_read); once the log is full the
 *                caller merges it into the base (dl_log_merge), or fuses the
 *                merge with that step's read (dl_log_merge_read).
 *
 * Conventions for every entry point
 *   Pointers   device pointers (cudaMalloc'd or equivalent), row-major and
 *              contiguous with the layouts given per argument. S, q, k, v, o,
 *              a channel-wise decay and the log's k, v and channel-wise a must
 *              be 16-byte aligned; beta and a head-wise decay need only their
 *              element alignment. Misaligned -> DL_ERR_INVALID_ARG.
 *   Element    dl_dtype of S (s_dtype) and of q, k, v, beta, a and the log
 *   types      (in_dtype; the log's dtype must equal in_dtype). o is float.
 *   Shapes     B, H >= 1; d_k in {64, 128}; d_v in {64, 128, 256}; log
 *              capacity L in 1..64. Other sizes -> DL_ERR_UNSUPPORTED.
 *   Ownership  the caller owns every buffer. The library allocates no device
 *              memory, keeps no state between calls and never synchronises:
 *              the work is enqueued on `stream` (0 = legacy default stream).
 *   Aliasing   o must not overlap any input or S; the log must not overlap S.
 *              Overlap -> DL_ERR_INVALID_ARG.
 *   Errors     arguments are checked on the host before anything is enqueued;
 *              a failed check enqueues nothing and returns its status. A
 *              launch failure returns DL_ERR_CUDA. Faults during execution
 *              surface at the caller's next synchronisation. After any
 *              non-OK return, dl_last_error() describes the cause (per thread).
 */
#ifndef DELTALOG_H
#define DELTALOG_H

#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

#define DL_ABI_VERSION 9
#define DL_MAX_LOG 64

typedef enum {
    DL_OK = 0,
    DL_ERR_INVALID_ARG = 1, /* null / misaligned / overlapping pointer, bad enum, B or H < 1, bad n */
    DL_ERR_UNSUPPORTED = 2, /* d_k, d_v or L outside the supported set; log dtype != in_dtype */
    DL_ERR_LOG_FULL = 3,    /* append with n >= L (merge first) */
    DL_ERR_CUDA = 4         /* the kernel launch failed (cudaGetLastError) */
} dl_status;

/* Element types. DL_I8 is a state type only, and only for a deferred base
 * (dl_log_append_read, dl_log_merge, dl_log_merge_read, the no-alloc read and
 * the pool): the base is held as int8 codes with one fp32 scale per state row
 * (a value channel), packed in one buffer -- B*H*d_v*d_k int8 codes, row-major
 * as for the other types, then B*H*d_v fp32 scales (dl_state_bytes) -- and an
 * element's value is code * scale. Every merge re-rounds the rows it writes:
 * scale = max|row| / 127, code = the nearest integer to value / scale, ties to
 * even, clamped to [-127, 127] (an all-zero row stays zero), each step one
 * correctly rounded fp32 operation on the row's fp32 values. (The low-precision base of the DAMP
 * abstract, "Decay-Aware Mixed-Precision Recurrent-State Quantization": with
 * the deferred schedule the base is rounded once per merge, not every step.)
 * The eager steps take DL_F32 or DL_BF16 only (DL_I8 -> DL_ERR_UNSUPPORTED). */
typedef enum { DL_F32 = 0, DL_BF16 = 1, DL_I8 = 2 } dl_dtype;

/* The model's update rule: its decay shape and whether the delta-rule
 * correction applies. */
typedef enum {
    DL_DECAY_HEAD = 0,    /* a is one scalar per (b, h, step): GDN */
    DL_DECAY_CHANNEL = 1, /* a is one value per key channel: KDA  */
    DL_RWKV6 = 2          /* a per key channel, raw-value update, no beta: RWKV6 */
} dl_decay;

/* Caller-owned bounded log of a deferred state: per (b, h) up to L entries of
 * the raw step factors, stored unchanged in `dtype` (lossless), their
 * log-decay metadata, and a small fp32 workspace the deferred read uses to
 * hand its per-head key-side results to the value tiles.
 * (The page's log holds each step's small update factors with log-decay
 * metadata, Technical Summary, "Core Mechanism: Base + Log"; here the decay products
 * are recomputed from the stored decays where they are needed, and the
 * triangular solve they lead to is kept as x below.)
 *   k     [B, H, L, d_k]
 *   v     [B, H, L, d_v]
 *   beta  [B, H, L]
 *   a     [B, H, L] (DL_DECAY_HEAD) or [B, H, L, d_k] (DL_DECAY_CHANNEL, DL_RWKV6)
 *   x     [B, H, L, L] float: the log's metadata, row j holding X(j, e) for
 *         e <= j, where X = (I + Diag(beta) C)^{-1} Diag(beta) and
 *         C(j, e) = sum_c k_e[c] k_j[c] prod_{m=e+1..j} a_m[c] for e < j (the
 *         decayed key inner products: the page's "log-decay metadata",
 *         Technical Summary, "Core Mechanism: Base + Log", kept as products
 *         rather than logarithms). X is lower triangular and gains one row per
 *         append, so dl_log_append_read writes row n for the entry it appends;
 *         the deferred read and the merge read it. Log entries must therefore
 *         be written by dl_log_append_read. 16-byte aligned.
 *         DL_RWKV6 has no correction (X is the identity): beta and x are not
 *         used and may be null.
 *   work  at least dl_log_work_bytes(B, H, d_k, d_v) bytes, 16-byte aligned,
 *         contents irrelevant between calls (only dl_log_append_read uses it)
 * The number of valid entries n (the same for every head) is tracked by the
 * caller and passed to each call; entries 0..n-1 are valid. */
typedef struct {
    void *k;
    void *v;
    void *beta;
    void *a;
    float *x;
    dl_dtype dtype;
    int L;
    void *work;
    size_t work_bytes;
} dl_log;

/* Eager GDN step (head-wise decay), in place.
 *   S     [B, H, d_v, d_k] s_dtype, read and overwritten with S_t
 *   q, k  [B, H, d_k] in_dtype      v [B, H, d_v] in_dtype
 *   beta  [B, H] in_dtype           a [B, H] in_dtype (one decay per head)
 *   o     [B, H, d_v] float, written with S_t q
 * A bf16 S is updated in fp32 and rounded to nearest-even when stored. */
dl_status dl_gdn_decode_step(void *S, dl_dtype s_dtype,
                             const void *q, const void *k, const void *v,
                             const void *beta, const void *a, dl_dtype in_dtype,
                             float *o, int B, int H, int d_k, int d_v,
                             cudaStream_t stream);

/* Eager KDA step (channel-wise decay): as dl_gdn_decode_step, except
 *   a     [B, H, d_k] in_dtype (one decay per key channel). */
dl_status dl_kda_decode_step(void *S, dl_dtype s_dtype,
                             const void *q, const void *k, const void *v,
                             const void *beta, const void *a, dl_dtype in_dtype,
                             float *o, int B, int H, int d_k, int d_v,
                             cudaStream_t stream);

/* Eager RWKV6 step (channel-wise decay, raw-value update), in place:
 *   S_t = S_{t-1} Diag(a) + v k^T,  o = S_t q.
 * Arguments as dl_kda_decode_step without beta. */
dl_status dl_rwkv6_decode_step(void *S, dl_dtype s_dtype,
                               const void *q, const void *k, const void *v,
                               const void *a, dl_dtype in_dtype,
                               float *o, int B, int H, int d_k, int d_v,
                               cudaStream_t stream);

/* Bytes of log workspace (dl_log.work) the deferred read needs:
 * B * H * (d_k + d_v) * 4. */
size_t dl_log_work_bytes(int B, int H, int d_k, int d_v);

/* Deferred step: append this step's (k, v, beta, a) to the log as entry n and
 * write o = S_n q, where S_n is the base with log entries 0..n replayed, read
 * without materialising it (Technical Summary, "Append Phase" and
 * "Kernel Implementation": key-side coefficients computed once per head, then
 * value tiles read the base). S_base is only read.
 *   S_base [B, H, d_v, d_k] s_dtype (read only)
 *   log    entries 0..n-1 read, entry n written; log->work is overwritten
 *          (missing or smaller than dl_log_work_bytes -> DL_ERR_INVALID_ARG)
 *   n      entries already in the log, 0 <= n < L; n >= L -> DL_ERR_LOG_FULL
 *   q, k, v, beta, a, o: as the eager step of the same kind (DL_RWKV6: beta
 *          is not used and may be null).
 * With an fp32 or bf16 base and L <= 16 the step runs as one persistent
 * kernel (the key-side work of each head done in shared memory a few heads
 * ahead of the base stream) and log->work is checked but not used; otherwise
 * (an int8 base, L > 16) as two kernels that hand the key-side results over
 * in log->work. Both forms give the same results, bit for bit. */
dl_status dl_log_append_read(const void *S_base, dl_dtype s_dtype, dl_decay kind,
                             const dl_log *log, int n,
                             const void *q, const void *k, const void *v,
                             const void *beta, const void *a, dl_dtype in_dtype,
                             float *o, int B, int H, int d_k, int d_v,
                             cudaStream_t stream);

/* Merge log entries 0..n-1 into the base in place: S_base <- S_n (Technical
 * Summary, "Merge Phase"). Afterwards the caller treats the log as empty.
 *   n      1 <= n <= L, else DL_ERR_INVALID_ARG
 * A bf16 base is merged in fp32 and rounded once when stored. */
dl_status dl_log_merge(void *S_base, dl_dtype s_dtype, dl_decay kind,
                       const dl_log *log, int n,
                       int B, int H, int d_k, int d_v, cudaStream_t stream);

/* The merge fused with a step's read: S_base <- the base with log entries
 * 0..n-1 and then this step's (k, v, beta, a) replayed, and o = (new S_base) q.
 * Equivalent to dl_log_append_read(n) followed by dl_log_merge(n + 1), with one
 * pass over the base instead of two; the log slot n is not written.
 *   n      entries already in the log, 0 <= n < L; n >= L -> DL_ERR_LOG_FULL */
dl_status dl_log_merge_read(void *S_base, dl_dtype s_dtype, dl_decay kind,
                            const dl_log *log, int n,
                            const void *q, const void *k, const void *v,
                            const void *beta, const void *a, dl_dtype in_dtype,
                            float *o, int B, int H, int d_k, int d_v,
                            cudaStream_t stream);

/* Deferred step that allocates nothing and needs no workspace from the caller.
 *
 * The paper has no counterpart to this entry point; it exists for callers
 * that cannot allocate device memory, such as a serving engine whose caching
 * allocator has already reserved the device's memory for its state pool, a
 * plugin host that hands a kernel only its input and output buffers, or a
 * latency-critical decode loop where a cudaMalloc would synchronise the
 * device. It computes exactly what dl_log_append_read computes, with the same
 * arguments and checks, always in the two-kernel form of that step, except
 * that log->work is ignored (it may be null):
 * the per-head scratch lives in a fixed array of DL_NOALLOC_WORK_BYTES inside
 * the library, which every device that loads the library keeps until the
 * process exits.
 *   Limit      B * H * (d_k + d_v) * 4 <= DL_NOALLOC_WORK_BYTES (16 MiB, e.g.
 *              B * H = 16384 heads at d_k = d_v = 128); larger -> DL_ERR_UNSUPPORTED.
 *   Set-up     every call looks up the array's device address in the current
 *              context (cudaGetSymbolAddress, with the caller's device
 *              current), so the address stays right after a device reset or
 *              under a context the caller made. The first call in a context
 *              may load the library's module there; make that first call
 *              before any stream capture.
 *   Sharing    every call uses the same array and leaves its contents behind;
 *              calls whose work overlaps on the GPU (other streams or host
 *              threads) race on it, so the caller must serialise them. No
 *              part of the array needs clearing between calls.
 * It calls no cudaMalloc, cudaFree or other allocating routine. */
#define DL_NOALLOC_WORK_BYTES (16u << 20)
dl_status dl_log_append_read_noalloc(const void *S_base, dl_dtype s_dtype, dl_decay kind,
                                     const dl_log *log, int n,
                                     const void *q, const void *k, const void *v,
                                     const void *beta, const void *a, dl_dtype in_dtype,
                                     float *o, int B, int H, int d_k, int d_v,
                                     cudaStream_t stream);

/* A pool of per-sequence deferred states for continuous batching: the
 * sequences of a decode batch own slots of a preallocated pool, and each slot
 * keeps its own log fill (the page's per-"slot-head" state, Technical
 * Summary, "Kernel Implementation"; its vLLM-based serving stack, "System
 * Implementation and Evaluation").
 *   S       [P, H, d_v, d_k] s_dtype: the base of every slot
 *   P       slots, >= 1
 *   n       [P] int32, device: the log entries each slot holds, 0 <= n[s] < L.
 *           dl_pool_step and dl_pool_flush update it. When a new sequence
 *           takes slot s, the caller writes its initial state into S[s] and
 *           sets n[s] = 0.
 *   status  optional (may be null) int32, device: a step or flush ORs in 1
 *           when a batch row's slot is outside [0, P) or that slot's count
 *           outside [0, L); such a row is skipped (o not written).
 *   log     the slots' logs: k [P, H, L, d_k], v [P, H, L, d_v], beta [P, H, L],
 *           a [P, H, L] or [P, H, L, d_k], x [P, H, L, L] (as dl_log with B = P);
 *           log.work must hold dl_log_work_bytes(B, H, d_k, d_v) for the batch.
 * Alignment and aliasing rules as for the other entry points; n, status and
 * slot need 4-byte alignment. */
typedef struct {
    void *S;
    dl_dtype s_dtype;
    int P;
    int *n;
    int *status;
    dl_log log;
} dl_pool;

/* One decode step of B sequences of a pool. Batch row b works on slot slot[b]
 * (int32 [B], device; the slots of one call must be distinct). With
 * c = n[slot[b]] before the call:
 *   c < L - 1   append this step's factors as the slot's entry c and read
 *               o = S_c q from base + log (dl_log_append_read); n <- c + 1
 *   c = L - 1   merge the slot's c entries and this step into its base and
 *               read o from the new base (dl_log_merge_read); n <- 0
 * so every sequence follows its own deferred schedule whatever the fills of
 * the others. q, k, v, beta, a and o are batch tensors [B, H, ...] as for
 * dl_log_append_read; B <= P. */
dl_status dl_pool_step(const dl_pool *pool, dl_decay kind, const int *slot,
                       const void *q, const void *k, const void *v,
                       const void *beta, const void *a, dl_dtype in_dtype,
                       float *o, int B, int H, int d_k, int d_v,
                       cudaStream_t stream);

/* Merge the log of every listed slot into its base (slots holding n[s] > 0
 * entries) and set n[s] = 0: afterwards S[slot[b]] is the dense state of
 * that sequence (for a sequence that ends, or a state handed elsewhere). */
dl_status dl_pool_flush(const dl_pool *pool, dl_decay kind, const int *slot,
                        int B, int H, int d_k, int d_v, cudaStream_t stream);

/* Bytes of a [B, H, d_v, d_k] state of element type s_dtype (for DL_I8 the
 * codes and the row scales); 0 for a bad argument. */
size_t dl_state_bytes(dl_dtype s_dtype, int B, int H, int d_k, int d_v);

/* Round a state into the int8 layout of DL_I8 (scale per row, ties to even):
 *   S     [B, H, d_v, d_k] s_dtype (DL_F32 or DL_BF16), read
 *   S_i8  dl_state_bytes(DL_I8, ...) bytes, written; 16-byte aligned, no overlap */
dl_status dl_state_to_i8(const void *S, dl_dtype s_dtype, void *S_i8,
                         int B, int H, int d_k, int d_v, cudaStream_t stream);

/* The values of an int8 state (code * scale) into S of type s_dtype (DL_F32 or
 * DL_BF16, rounded to nearest-even for DL_BF16). */
dl_status dl_state_from_i8(const void *S_i8, void *S, dl_dtype s_dtype,
                           int B, int H, int d_k, int d_v, cudaStream_t stream);

/* Static text for a status code. */
const char *dl_status_string(dl_status s);

/* Description of the most recent non-OK return on the calling thread ("" if
 * none). The pointer stays valid until the thread's next dl_* call. */
const char *dl_last_error(void);

/* DL_ABI_VERSION of the built library. */
int dl_abi_version(void);

/* Fault word of the library's kernels on the current device. The kernels that
 * wait on on-chip barriers (the tcgen05 merge of dl_log_merge and
 * dl_log_merge_read, and the one-kernel form of dl_log_append_read) bound
 * every such wait; a wait that runs out (about two
 * seconds; it means a bug, not a slow GPU) sets bit 0 here, abandons its work
 * (the state it was merging is then unspecified) and returns, so the device
 * stays usable. In the index-guard build (dl_index_guard_build() == 1), bit 1
 * means that a kernel skipped a shared-memory write that lay outside its
 * block's shared memory or was misaligned (a bug; that call's results are
 * wrong); dl_last_error() then names the source file and line of the first
 * one. *flags receives the word; clear != 0 resets it to 0.
 * Synchronous: it waits for the device's pending work (cudaMemcpyFromSymbol).
 * No counterpart on the pages: it is a health check of this library. */
dl_status dl_device_faults(unsigned int *flags, int clear);

/* 1 in the index-guard debug build (libdeltalog_guard.so, compiled with
 * DL_INDEX_GUARD: every shared-memory write of the kernels checks its bounds
 * and alignment first, and a write that fails is skipped and reported through
 * dl_device_faults), else 0. The guard build computes the same results as the
 * ordinary one, more slowly. No counterpart on the pages. */
int dl_index_guard_build(void);

#ifdef __cplusplus
}
#endif

#endif /* DELTALOG_H */
