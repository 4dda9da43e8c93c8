// ReplayPrep for one (sequence, head), done by one warp (DeltaLog page,
// Technical Summary, "Append Phase" and "Kernel Implementation": the
// key-side work of a read is done once per head and serves every value
// tile). Used by replay_prep_kernel (deferred_read.cu), which writes the
// result to a global workspace, and by the fused append-read kernel
// (append_read_fused.cu), which keeps it in shared memory.
//
// Appends entry n = (k, v, beta, a) of this step to the log unchanged and its
// row of X, then evaluates the key-side recursion in parallel form:
//   d_e = k_e . (D(n, e) o q), C(n, e) = k_e . (D(n, e) o k_n),
//   X(n, n) = beta_n, X(n, j) = -beta_n sum_{m=j..n-1} C(n, m) X(m, j),
//   s = X^T d,
//   x_0 = gamma_n o q - sum_e s_e (gamma_e o k_e),  w = sum_e s_e v_e,
// and stores out[0 .. DK) = x_0 and out[DK .. DK + DV) = w. `base` is the
// warp's staging area of PrepSmem<sizeof(IT), DK, EMAX, CHAN>::BYTES in shared
// memory; `head` indexes this step's inputs, `shead` the log. OUT_SMEM says
// that `out` is in shared memory (its stores are then index-guarded in the
// debug build).
#pragma once

#include "launch.h"
#include "guard.cuh"
#include "prep_layout.h"

namespace dl {

template <class IT, int DK, int DV, int KIND, int EMAX, bool OUT_SMEM>
__device__ __forceinline__ void prep_head(const IT *__restrict__ q, const IT *__restrict__ k,
                                          const IT *__restrict__ v, const IT *__restrict__ beta,
                                          const IT *__restrict__ a, IT *__restrict__ log_k, IT *__restrict__ log_v,
                                          IT *__restrict__ log_b, IT *__restrict__ log_a, float *__restrict__ log_x,
                                          int L, int n, long long head, long long shead, unsigned char *base,
                                          float *out) {
    constexpr bool CHAN = Rule<KIND>::CHAN, DELTA = Rule<KIND>::DELTA;
    using P = PrepSmem<(int)sizeof(IT), DK, EMAX, CHAN>;
    constexpr int CW = DK / 32;            // key columns per lane (contiguous)
    constexpr int RV = DV / 32;            // value rows per lane
    constexpr int CH = EMAX < 32 ? EMAX : 32;  // entries per butterfly
    constexpr int E = 16 / (int)sizeof(IT);    // elements per 16-byte chunk
    const int lane = threadIdx.x & 31;
    IT *sk = reinterpret_cast<IT *>(base + P::K_OFF);
    IT *sa = reinterpret_cast<IT *>(base + P::A_OFF);
    float *fl = reinterpret_cast<float *>(base + P::F_OFF);
    float *fas = fl + P::AS, *fbeta = fl + P::BETA, *fd = fl + P::D, *fcn = fl + P::CN, *fs = fl + P::S,
          *xrow = fl + P::XROW;

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

#pragma unroll
    for (int c = 0; c < CW; ++c) {
        const float x0 = fmaf(g[c], qv[c], -xs[c]);
        if constexpr (OUT_SMEM) {
            DL_GUARD(out + c0 + c, 4) out[c0 + c] = x0;
        } else {
            out[c0 + c] = x0;
        }
    }
#pragma unroll
    for (int r = 0; r < RV; ++r) {
        if constexpr (OUT_SMEM) {
            DL_GUARD(out + DK + r0 + r, 4) out[DK + r0 + r] = w[r];
        } else {
            out[DK + r0 + r] = w[r];
        }
    }
}

}  // namespace dl
