// Merge of the bounded log into an fp32 or int8 base on the 5th-generation
// tensor cores (DeltaLog page, "Core Mechanism: Base + Log", the merge phase:
// the base absorbs every update the log holds and the log starts empty
// again), alone or fused with one step's read.
//
// An int8 base (codes with one fp32 scale per row; the low-precision base of
// the DAMP abstract) takes the same path: the loader brings the unit's codes
// by one TMA box into the tile's last column chunk and its row scales by a
// bulk copy; each thread widens its row (code * scale, fp32) into the fp32
// tile as it makes its pass over the row, the tensor cores reading each half
// of the tile once the group has written it; the merged row is rounded back
// (scale = max|row| / 127, codes to nearest, ties to even) and stored from
// registers.
//
// The arithmetic is the log-decay form of merge.cu (same symbols): for a
// block of n <= 16 entries with decays a_i, keys k_i, values v_i, strengths
// beta_i, per 128-row tile S of one head
//   G     = S Khat^T,          Khat_i = gamma_i o k_i, gamma_i = prod_{m<=i} a_m
//   delta = X (V - G)          X = (I + Diag(beta) C)^{-1} Diag(beta), kept with the log
//   S    <- S o gamma_{n-1} + delta F,   F_j = k_j o prod_{m=j+1..n-1} a_m
// (RWKV6: delta = V, no G). The fused read's own entry is the block's last,
// and its X row is formed here from C(n, j) = F_n . F_j.
//
// Both products run as tcgen05.mma kind::tf32 with fp32 accumulators in
// tensor memory. A TF32 operand read keeps the top 19 bits of each fp32 word
// (the rest are ignored), so every operand x is split as hi + lo with
// hi = x with its low 13 mantissa bits cleared and lo = x - hi (exact), and
// each product is formed from the three terms hi*hi + hi*lo + lo*hi (lo*lo
// is below fp32 resolution; G also takes it, at no cost). The state tile,
// as the TMA load leaves it in shared memory, is already its own hi part.
//   G:        D_G[:, 0:16]  = S_hi Khat_hi^T + S_lo Khat_hi^T
//             D_G[:, 16:32] = S_hi Khat_lo^T + S_lo Khat_lo^T    (N = 32)
//             A = the state tile (shared memory) or S_lo (tensor memory),
//             B = [Khat_hi; Khat_lo] (shared memory), 16 + 16 MMAs of K = 8
//   write-back: D = delta_hi F_hi + delta_hi F_lo + delta_lo F_hi    (N = 128)
//             A = [delta_hi | delta_lo] (tensor memory), B = [F_hi | F_lo]
//             (shared memory), 6 MMAs of K = 8
//
// CTA: one per SM, persistent over units (unit = (head, 128-row tile)), in
// these roles:
//   warp 0    loads: the unit's state tile by TMA (four 32-column boxes,
//             128-byte swizzle) and its raw log entries and X block
//             (cp.async; the few scalars by plain loads issued first) into one
//             of two stages; after the unit is merged, stores the tile back by
//             TMA and refills the stage with the unit two ahead;
//   warp 1, 2 issue the products of compute group 0, 1 (one thread each);
//             warp 1 also allocates tensor memory;
//   groups    NWG (two when their operand tiles fit the shared memory beside
//             the stages, else one) groups of 4 warps; group w merges units
//             w, w + NWG, ... with its own operand tiles and its own 256
//             columns of tensor memory, so one group works while the other's
//             products run. Thread t of a group owns state row
//             r = 32 (warp % 4) + lane (its tensor-memory lane) and key
//             channel c = r. Per unit: Khat, F and gamma from the raw entries
//             (and the fused entry's X row), S_lo into tensor memory, then
//             delta from G, then the write-back S o gamma + D into the tile
//             (and o = S_new q for the fused read).
// Every wait on an mbarrier is bounded; a wait that runs out sets a bit of
// the module's fault word and the CTA drains and returns.
#include "launch.h"
#include "guard.cuh"
#include "merge_tc_layout.h"
#include "tc.cuh"

namespace dl {

// Fault word of the tensor-core kernels (bit 0: a bounded wait ran out).
__device__ unsigned int g_tc_faults = 0;

namespace {

using namespace mtc;

// ---------------------------------------------------------------- bounded waits

__device__ __forceinline__ uint64_t globaltimer() {
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}
// Wait for the phase of `bar` with parity `par`; gives up after about two
// seconds, or at once once another role has given up (*abort set).
__device__ __forceinline__ bool wait_bar(uint64_t *bar, uint32_t par, volatile int *abort) {
    if (tc::mbar_try_wait(bar, par)) return true;
    const uint64_t t0 = globaltimer();
    for (uint32_t i = 0;; ++i) {
        if (tc::mbar_try_wait(bar, par)) return true;
        if ((i & 63u) == 63u) {
            if (*abort) return false;
            if (globaltimer() - t0 > 2000000000ull) {
                *abort = 1;
                atomicOr(&g_tc_faults, 1u);
                return false;
            }
        }
    }
}

__device__ __forceinline__ void cp_async_bar_arrive(uint64_t *bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(tc::smem_u32(bar)) : "memory");
}

// Unit index -> (batch head, first row of the tile).
struct Unit {
    long long head;
    int row0;
};
__device__ __forceinline__ Unit unit_of(long long u, int tiles) { return {u / tiles, (int)(u % tiles) * ROWS}; }

template <class IT>
__device__ __forceinline__ float ld_in(const IT *p) {
    return to_f(*p);
}

// ---------------------------------------------------------------- kernel

// cp.async of 4 bytes (the X block's floats: rows of the log's [L, L] matrix
// are only 4-byte aligned).
__device__ __forceinline__ void cp_async4(void *smem_dst, const void *gmem_src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(tc::smem_u32(smem_dst)), "l"(gmem_src) : "memory");
}

template <class IT, int KIND, bool WITH_CUR, int NWG, bool Q8>
__global__ void __launch_bounds__(threads_for(NWG), 1)
merge_tc_kernel(const __grid_constant__ CUtensorMap map_s, const __grid_constant__ CUtensorMap map_st,
                const IT *__restrict__ log_k, const IT *__restrict__ log_v, const IT *__restrict__ log_b,
                const IT *__restrict__ log_a, const float *__restrict__ log_x, int L, int n_log,
                const IT *__restrict__ q, const IT *__restrict__ k, const IT *__restrict__ v,
                const IT *__restrict__ beta, const IT *__restrict__ a, float *__restrict__ o, int DV,
                long long units, int8_t *__restrict__ codes, float *__restrict__ i8_scales) {
    constexpr bool CHAN = Rule<KIND>::CHAN, DELTA = Rule<KIND>::DELTA;
    constexpr Layout LY{sizeof(IT), CHAN, NWG, Q8};
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + LY.off_bar());
    uint32_t *tslot = reinterpret_cast<uint32_t *>(sm + LY.off_tslot());
    volatile int *abort = reinterpret_cast<volatile int *>(sm + LY.off_abort());
    auto B_FULL = [&](int s) { return &bars[s]; };
    auto B_FREE = [&](int s) { return &bars[NS + s]; };
    auto B_KH = [&](int w) { return &bars[2 * NS + 6 * w + 0]; };
    auto B_LO = [&](int w) { return &bars[2 * NS + 6 * w + 1]; };      // completes twice per unit
    auto B_LOFREE = [&](int w) { return &bars[2 * NS + 6 * w + 2]; };
    auto B_G = [&](int w) { return &bars[2 * NS + 6 * w + 3]; };
    auto B_DELTA = [&](int w) { return &bars[2 * NS + 6 * w + 4]; };
    auto B_D = [&](int w) { return &bars[2 * NS + 6 * w + 5]; };

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int tiles = DV / ROWS;
    const int nb = n_log + (WITH_CUR ? 1 : 0);  // entries merged (<= NB)
    const int n_mine = units > blockIdx.x ? (int)((units - 1 - blockIdx.x) / gridDim.x) + 1 : 0;

    if (tid == 0) {
        for (int s = 0; s < NS; ++s) {
            tc::mbar_init(B_FULL(s), 1 + 32);  // the loader's byte count + its lanes' cp.async arrivals
            tc::mbar_init(B_FREE(s), 1);
        }
        for (int w = 0; w < NWG; ++w)
            for (int b = 0; b < 6; ++b) tc::mbar_init(&bars[2 * NS + 6 * w + b], 1);
        *abort = 0;
        tc::mbar_init_fence();
    }
    if (warp == 1) {
        tc::tmem_alloc(tslot, tmem_cols_for(NWG));
        tc::tmem_relinquish();
    }
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tbase = *tslot;

    if (warp == 0) {
        // ------------------------------------------------ loads
        if (lane == 0) {
            tc::tma_prefetch_desc(&map_s);
            tc::tma_prefetch_desc(&map_st);
        }
        constexpr uint32_t KB = DK * sizeof(IT), VB = ROWS * sizeof(IT);  // one entry's key / value-tile bytes
        // the unit's base: the fp32 tile, or the int8 codes (ROWS x DK bytes) and row scales
        constexpr uint32_t BASE_TX = Q8 ? (uint32_t)(ROWS * DK + ROWS * 4) : (uint32_t)LY.tile();
        const uint32_t tx = BASE_TX + (uint32_t)nb * (KB * (CHAN ? 2 : 1) + VB) + (WITH_CUR ? KB : 0);
        for (int i = 0; i < n_mine; ++i) {
            const int s = i % NS;
            if (i >= NS && !wait_bar(B_FREE(s), (uint32_t)((i / NS - 1) & 1), abort)) break;
            uint8_t *st = sm + LY.stage(s);
            const Unit un = unit_of((long long)blockIdx.x + (long long)i * gridDim.x, tiles);
            const long long lrow = un.head * L;
            uint64_t *full = B_FULL(s);
            // the state tile by TMA; the raw entries by bulk copies spread over
            // the lanes: logged ones from the log (contiguous per head), the
            // fused read's own from this step's inputs
            if (lane == 0) tc::mbar_arrive_expect_tx(full, tx);
            __syncwarp();
            uint8_t *rk = st + LY.off_raw_k(), *ra = st + LY.off_raw_a(), *rv = st + LY.off_raw_v();
            if constexpr (Q8) {
                if (lane == 0) tc::tma_load_2d(st + LY.off_codes(), &map_s, 0, (int)(un.head * DV + un.row0), full);
                if (lane == 1) tc::bulk_load(st + LY.off_scl(), i8_scales + un.head * DV + un.row0, ROWS * 4, full);
            } else if (lane < NCHUNK) {
                tc::tma_load_2d(st + LY.off_tile() + lane * (ROWS * 128), &map_s, lane * CHUNK,
                                (int)(un.head * DV + un.row0), full);
            }
            if (lane == NCHUNK && n_log > 0) tc::bulk_load(rk, log_k + lrow * DK, (uint32_t)n_log * KB, full);
            if (CHAN && lane == NCHUNK + 1 && n_log > 0)
                tc::bulk_load(ra, log_a + lrow * DK, (uint32_t)n_log * KB, full);
            if (WITH_CUR && lane == NCHUNK + 2) {
                tc::bulk_load(rk + raw_k_off(n_log, 0, sizeof(IT)), k + un.head * DK, KB, full);
                if constexpr (CHAN) tc::bulk_load(ra + raw_k_off(n_log, 0, sizeof(IT)), a + un.head * DK, KB, full);
                tc::bulk_load(st + LY.off_raw_q(), q + un.head * DK, KB, full);
            }
            if (lane >= 16 && lane - 16 < nb) {  // value tiles: lane 16 + e copies entry e's
                const int e = lane - 16;
                const IT *src = e < n_log ? log_v + (lrow + e) * DV + un.row0 : v + un.head * DV + un.row0;
                tc::bulk_load(rv + raw_v_off(e, 0, sizeof(IT)), src, VB, full);
            }
            if constexpr (DELTA) {  // the X block: X(j, e), e <= j < n_log
                uint8_t *sc = st + LY.off_sc();
                for (int u = lane; u < NB * NB; u += 32) {
                    const int j = u / NB, e = u % NB;
                    if (j < n_log && e <= j) cp_async4(sc + sc_x(j, e), log_x + (lrow + j) * L + e);
                }
            }
            cp_async_bar_arrive(full);
        }
        cp_async_wait_all();
    } else if (warp >= 1 && warp <= NWG) {
        // ------------------------------------------------ products of group w (one thread)
        const int w = warp - 1;
        if (lane == 0) {
            constexpr uint32_t ID_G = tc::instr_desc(tc::FMT_TF32, false, false, ROWS, 2 * NB);
            constexpr uint32_t ID_W = tc::instr_desc(tc::FMT_TF32, false, false, ROWS, DK);
            const uint32_t kh = tc::smem_u32(sm + LY.group(w) + LY.g_kh());
            const uint32_t ff = tc::smem_u32(sm + LY.group(w) + LY.g_ff());
            const uint32_t tw = tbase + (uint32_t)w * TMEM_COLS_PER_GROUP;
            for (int j = 0, i = w; i < n_mine; ++j, i += NWG) {
                const int s = i % NS;
                const uint32_t par = (uint32_t)(j & 1);
                if constexpr (DELTA) {
                    // G: the tile part as soon as Khat is in place, then the S_lo
                    // part in two halves of the key columns as the group writes them
                    if (!wait_bar(B_KH(w), par, abort)) break;
                    tc::tc_fence_after();
                    const uint32_t tile = tc::smem_u32(sm + LY.stage(s) + LY.off_tile());
                    if constexpr (!Q8) {  // the TMA tile is in place already
#pragma unroll
                        for (int kk = 0; kk < DK / 8; ++kk) {
                            const uint64_t ad = tc::smem_desc(tile + g_a_start(kk), 16, 1024, tc::SWZ_128);
                            const uint64_t bd = tc::smem_desc(kh + g_b_start(kk), 16, 1024, tc::SWZ_128);
                            tc::mma_ss_tf32(tw + COL_G, ad, bd, ID_G, kk > 0);
                        }
                    }
                    bool ok = true;
#pragma unroll
                    for (int h = 0; h < 2 && ok; ++h) {
                        if (!wait_bar(B_LO(w), (uint32_t)h, abort)) {
                            ok = false;
                            break;
                        }
                        tc::tc_fence_after();
                        if constexpr (Q8) {  // the half of the fp32 tile the group has just written
#pragma unroll
                            for (int kq = 0; kq < DK / 16; ++kq) {
                                const int kk = h * (DK / 16) + kq;
                                const uint64_t ad = tc::smem_desc(tile + g_a_start(kk), 16, 1024, tc::SWZ_128);
                                const uint64_t bd = tc::smem_desc(kh + g_b_start(kk), 16, 1024, tc::SWZ_128);
                                tc::mma_ss_tf32(tw + COL_G, ad, bd, ID_G, kk > 0);
                            }
                        }
#pragma unroll
                        for (int kq = 0; kq < DK / 16; ++kq) {
                            const int kk = h * (DK / 16) + kq;
                            const uint64_t bd = tc::smem_desc(kh + g_b_start(kk), 16, 1024, tc::SWZ_128);
                            tc::mma_ts_tf32(tw + COL_G, tw + COL_LO + 8 * kq, bd, ID_G, true);
                        }
                        tc::mma_commit(h == 0 ? B_LOFREE(w) : B_G(w));
                    }
                    if (!ok) break;
                }
                if (!wait_bar(B_DELTA(w), par, abort)) break;
                tc::tc_fence_after();
#pragma unroll
                for (int m = 0; m < 6; ++m) {  // onto S o gamma
                    const uint64_t bd = tc::smem_desc(ff + wb_b_start(m), 16, 1024, tc::SWZ_128);
                    tc::mma_ts_tf32(tw + COL_SG, tw + COL_DL + wb_a_col(m), bd, ID_W, true);
                }
                tc::mma_commit(B_D(w));
            }
        }
        __syncwarp();
    } else if (warp >= CTRL_WARPS) {
        // ------------------------------------------------ compute group w (128 threads)
        const int w = (warp - CTRL_WARPS) / 4;
        const int ct = tid - 32 * CTRL_WARPS - 128 * w;  // 0..127
        const int quad = warp & 3;                       // tensor-memory lane quadrant
        const int r = 32 * quad + lane;                  // state row of this thread (and its key channel)
        const int c = r;
        const uint32_t trow = tbase + (uint32_t)w * TMEM_COLS_PER_GROUP + ((uint32_t)(32 * quad) << 16);
        uint8_t *gp = sm + LY.group(w);
        float *gam = reinterpret_cast<float *>(gp + LY.g_gam());
        float *qf = reinterpret_cast<float *>(gp + LY.g_qf());
        float *cn = reinterpret_cast<float *>(gp + LY.g_cn());
        float *red = reinterpret_cast<float *>(gp + LY.g_red());
        uint8_t *kh = gp + LY.g_kh();
        uint8_t *ff = gp + LY.g_ff();
        const int bar_id = 1 + w;
        // the unit's scalars from global memory (head-wise decays of every
        // entry, which each thread needs all of, and the fused entry's beta),
        // fetched one unit of the group ahead: behind the stages' bulk loads a
        // plain load takes about as long as a unit
        float adec_n[NB], bcur_n = 0.f;
        auto fetch = [&](int i) {
            const long long head = ((long long)blockIdx.x + (long long)i * gridDim.x) / tiles;
#pragma unroll
            for (int e = 0; e < NB; ++e) {
                adec_n[e] = 1.f;
                if (!CHAN && e < nb && i < n_mine)
                    adec_n[e] = e < n_log ? ld_in(log_a + head * L + e) : ld_in(a + head);
            }
            if (DELTA && WITH_CUR && i < n_mine) bcur_n = ld_in(beta + head);
        };
        fetch(w);
        for (int j = 0, i = w; i < n_mine; ++j, i += NWG) {
            const int s = i % NS;
            const uint32_t par = (uint32_t)(j & 1);
            uint8_t *st = sm + LY.stage(s);
            uint8_t *tile = st + LY.off_tile();
            const IT *rk = reinterpret_cast<const IT *>(st + LY.off_raw_k());
            const IT *ra = reinterpret_cast<const IT *>(st + LY.off_raw_a());
            const IT *rv = reinterpret_cast<const IT *>(st + LY.off_raw_v());
            const IT *rq = reinterpret_cast<const IT *>(st + LY.off_raw_q());
            uint8_t *sc = st + LY.off_sc();
            auto scf = [&](size_t off) { return *reinterpret_cast<const float *>(sc + off); };
            const Unit un = unit_of((long long)blockIdx.x + (long long)i * gridDim.x, tiles);
            float adec[NB];
#pragma unroll
            for (int e = 0; e < NB; ++e) adec[e] = adec_n[e];
            const float bcur = bcur_n;
            fetch(i + NWG);
            if (!wait_bar(B_FULL(s), (uint32_t)((i / NS) & 1), abort)) break;
            if (j > 0) tc::named_sync(bar_id, 128);  // every warp's last stores have read its quarter of Khat

            // 1. key side for channel c: Khat (hi and lo parts), F, gamma, q
            float kc[NB], ac[NB];
#pragma unroll
            for (int e = 0; e < NB; ++e) {
                const bool real = e < nb;
                kc[e] = real ? to_f(rk[raw_k_off(e, c, 1)]) : 0.f;
                ac[e] = real ? (CHAN ? to_f(ra[raw_k_off(e, c, 1)]) : adec[e]) : 1.f;
            }
            {
                float g = 1.f;
#pragma unroll
                for (int e = 0; e < NB; ++e) {
                    g *= ac[e];
                    if constexpr (DELTA) {
                        const float x = g * kc[e], hi = tc::tf32_trunc(x);
                        DL_GUARD(kh + kh_off(e, c), 4) *reinterpret_cast<float *>(kh + kh_off(e, c)) = hi;
                        DL_GUARD(kh + kh_off(NB + e, c), 4) *reinterpret_cast<float *>(kh + kh_off(NB + e, c)) = x - hi;
                    }
                }
                DL_GUARD(gam + c, 4) gam[c] = g;
                if constexpr (WITH_CUR) {
                    DL_GUARD(qf + c, 4) qf[c] = to_f(rq[raw_q_off(c, 1)]);
                }
            }
            float fv[NB];  // F_e[c], into row c of F (this warp's quarter of F, which its last stores have read)
            {
                float f = 1.f;
#pragma unroll
                for (int e = NB - 1; e >= 0; --e) {
                    fv[e] = kc[e] * f;
                    f *= ac[e];
                }
                if (lane == 0) tc::bulk_wait_read<0>();
                __syncwarp();
#pragma unroll
                for (int u = 0; u < 8; ++u) {  // 16-byte pieces: hi of entries 4u.. (u < 4), lo (u >= 4)
                    float4 wv;
                    float *wp = reinterpret_cast<float *>(&wv);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float x = fv[(4 * u + e) % NB], hi = tc::tf32_trunc(x);
                        wp[e] = u < 4 ? hi : x - hi;
                    }
                    DL_GUARD(ff + ff_off(c, 4 * u), 16) *reinterpret_cast<float4 *>(ff + ff_off(c, 4 * u)) = wv;
                }
            }
            tc::fence_async_smem();       // Khat and F are read by the tensor cores
            tc::named_sync(bar_id, 128);  // Khat, gamma and q of every channel are in place
            if (DELTA && ct == 0) tc::mbar_arrive(B_KH(w));

            // 2. one pass over the tile row: S o gamma into [COL_SG, +128), and
            //    S_lo = S - hi(S) into [COL_LO, +64) one half of the columns at a
            //    time (the second half once G has read the first); for the fused
            //    read also (S o gamma) . q
            float oacc = 0.f;
            // an int8 base: this row's scale; chunk ch's 32 codes are pieces 2ch and
            // 2ch + 1 of the row in the code box, read before the chunk's fp32
            // columns are written (chunk 3's columns overwrite the row's codes)
            const float rs = Q8 ? *reinterpret_cast<const float *>(st + LY.off_scl() + 4 * r) : 0.f;
            auto row_chunk = [&](int ch, uint32_t (&lo)[32]) {
                uint32_t y[32];
                uint4 cw[2];
                if constexpr (Q8) {
                    cw[0] = *reinterpret_cast<const uint4 *>(st + LY.off_codes() + code_off(r, 2 * ch));
                    cw[1] = *reinterpret_cast<const uint4 *>(st + LY.off_codes() + code_off(r, 2 * ch + 1));
                }
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int col = ch * CHUNK + 4 * u;
                    float4 x;
                    if constexpr (Q8) {  // codes 4u .. 4u + 3 of the chunk, widened and scaled
                        const uint4 &c4 = cw[u / 4];
                        const uint32_t wd = (u % 4) == 0 ? c4.x : (u % 4) == 1 ? c4.y : (u % 4) == 2 ? c4.z : c4.w;
                        x = make_float4((float)(int8_t)(wd & 0xff) * rs, (float)(int8_t)((wd >> 8) & 0xff) * rs,
                                        (float)(int8_t)((wd >> 16) & 0xff) * rs, (float)(int8_t)(wd >> 24) * rs);
                        if constexpr (DELTA) {  // the fp32 tile is the A operand of G's tile part
                            DL_GUARD(tile + tile_off(r, col), 16) *reinterpret_cast<float4 *>(tile + tile_off(r, col)) = x;
                        }
                    } else {
                        x = *reinterpret_cast<const float4 *>(tile + tile_off(r, col));
                    }
                    const float4 gv = *reinterpret_cast<const float4 *>(gam + col);
                    const float4 sg = make_float4(x.x * gv.x, x.y * gv.y, x.z * gv.z, x.w * gv.w);
                    y[4 * u + 0] = __float_as_uint(sg.x);
                    y[4 * u + 1] = __float_as_uint(sg.y);
                    y[4 * u + 2] = __float_as_uint(sg.z);
                    y[4 * u + 3] = __float_as_uint(sg.w);
                    if constexpr (DELTA) {
                        lo[4 * u + 0] = __float_as_uint(x.x - tc::tf32_trunc(x.x));
                        lo[4 * u + 1] = __float_as_uint(x.y - tc::tf32_trunc(x.y));
                        lo[4 * u + 2] = __float_as_uint(x.z - tc::tf32_trunc(x.z));
                        lo[4 * u + 3] = __float_as_uint(x.w - tc::tf32_trunc(x.w));
                    }
                    if constexpr (WITH_CUR) {
                        const float4 qv = *reinterpret_cast<const float4 *>(qf + col);
                        oacc = fmaf(sg.x, qv.x, fmaf(sg.y, qv.y, fmaf(sg.z, qv.z, fmaf(sg.w, qv.w, oacc))));
                    }
                }
                tc::tmem_st32(trow + COL_SG + ch * CHUNK, y);
            };
            {
                uint32_t lo[32];
                row_chunk(0, lo);
                if constexpr (DELTA) tc::tmem_st32(trow + COL_LO, lo);
                row_chunk(1, lo);
                if constexpr (DELTA) {
                    tc::tmem_st32(trow + COL_LO + CHUNK, lo);
                    tc::tmem_wait_st();
                    tc::tc_fence_before();
                    if constexpr (Q8) tc::fence_async_smem();  // the tile's first half is read by the tensor cores
                    tc::named_sync(bar_id, 128);
                    if (ct == 0) tc::mbar_arrive(B_LO(w));  // first half
                }
                row_chunk(2, lo);
                if constexpr (DELTA) {
                    if (!wait_bar(B_LOFREE(w), par, abort)) break;  // G has read the first half
                    tc::tc_fence_after();
                    tc::tmem_st32(trow + COL_LO, lo);
                }
                row_chunk(3, lo);
                if constexpr (DELTA) {
                    tc::tmem_st32(trow + COL_LO + CHUNK, lo);
                    tc::tmem_wait_st();
                    tc::tc_fence_before();
                    if constexpr (Q8) tc::fence_async_smem();  // and its second half
                    tc::named_sync(bar_id, 128);
                    if (ct == 0) tc::mbar_arrive(B_LO(w));  // second half
                }
            }
            // 3. while G runs, for the fused read: the sums over key channels that
            //    its entry's X row and its output need, C(nb-1, e) = F_{nb-1} . F_e
            //    (every factor after the entry is a padded 1, so F_{nb-1} = k_{nb-1})
            //    and (F q)_e; then the entry's X row
            if constexpr (WITH_CUR) {
                const int nl = nb - 1;
                const float fn = to_f(rk[raw_k_off(nl, c, 1)]);
                const float qc = qf[c];
                float p[2 * NB];
#pragma unroll
                for (int e = 0; e < NB; ++e) {
                    p[e] = (DELTA && e < nl) ? fn * fv[e] : 0.f;
                    p[NB + e] = fv[e] * qc;
                }
                multi_sum<2 * NB>(p, lane);  // lane l: this warp's sum of item l
                DL_GUARD(red + quad * 2 * NB + lane, 4) red[quad * 2 * NB + lane] = p[0];
                tc::named_sync(bar_id, 128);
                if (ct < 2 * NB) {
                    DL_GUARD(cn + ct, 4) cn[ct] = red[ct] + red[2 * NB + ct] + red[4 * NB + ct] + red[6 * NB + ct];
                }
                tc::named_sync(bar_id, 128);
                if (DELTA && ct <= nl) {
                    // X(nl, ct) = -beta_nl sum_{m = ct..nl-1} C(nl, m) X(m, ct); X(nl, nl) = beta_nl
                    float acc = 0.f;
#pragma unroll
                    for (int m = 0; m < NB; ++m)
                        if (m >= ct && m < nl) acc = fmaf(cn[m], scf(sc_x(m, ct)), acc);
                    DL_GUARD(sc + sc_x(nl, ct), 4) *reinterpret_cast<float *>(sc + sc_x(nl, ct)) = ct == nl ? bcur : -bcur * acc;
                }
                if constexpr (DELTA) tc::named_sync(bar_id, 128);
            }
            float vr[NB];
#pragma unroll
            for (int e = 0; e < NB; ++e) vr[e] = e < nb ? to_f(rv[raw_v_off(e, r, 1)]) : 0.f;

            // 4. delta = X (V - G) for row r (RWKV6: delta = V) into [COL_DL, +32)
            float dl[NB];
            if constexpr (DELTA) {
                if (!wait_bar(B_G(w), par, abort)) break;
                tc::tc_fence_after();
                uint32_t gr[32];
                tc::tmem_ld32(trow + COL_G, gr);
                tc::tmem_wait_ld();
                float ev[NB];
#pragma unroll
                for (int e = 0; e < NB; ++e) ev[e] = vr[e] - (__uint_as_float(gr[e]) + __uint_as_float(gr[NB + e]));
#pragma unroll
                for (int e = 0; e < NB; ++e) {
                    float xr[NB];  // row e of X (entries past the diagonal are not read)
#pragma unroll
                    for (int m4 = 0; m4 <= e / 4; ++m4) {
                        const float4 x4 = *reinterpret_cast<const float4 *>(sc + sc_x(e, 4 * m4));
                        xr[4 * m4 + 0] = x4.x;
                        xr[4 * m4 + 1] = x4.y;
                        xr[4 * m4 + 2] = x4.z;
                        xr[4 * m4 + 3] = x4.w;
                    }
                    float acc = 0.f;
#pragma unroll
                    for (int m = 0; m <= e; ++m) acc = fmaf(xr[m], ev[m], acc);
                    dl[e] = e < nb ? acc : 0.f;
                }
            } else {
#pragma unroll
                for (int e = 0; e < NB; ++e) dl[e] = vr[e];
            }
            {
                uint32_t wd[32];
#pragma unroll
                for (int e = 0; e < NB; ++e) {
                    const float hi = tc::tf32_trunc(dl[e]);
                    wd[e] = __float_as_uint(hi);
                    wd[NB + e] = __float_as_uint(dl[e] - hi);
                }
                tc::tmem_st32(trow + COL_DL, wd);
            }
            tc::tmem_wait_st();
            tc::tc_fence_before();
            tc::named_sync(bar_id, 128);
            if (ct == 0) {
                tc::mbar_arrive(B_DELTA(w));
                tc::mbar_arrive(B_FREE(s));  // the unit reads nothing more of its stage
            }
            if constexpr (WITH_CUR) {  // o = (S o gamma) . q + delta . (F q)
#pragma unroll
                for (int e = 0; e < NB; ++e) oacc = fmaf(dl[e], cn[NB + e], oacc);
                o[un.head * DV + un.row0 + r] = oacc;
            }

            // 5. S_new = [COL_SG, +128) after the write-back: each warp's 32 rows
            //    to HBM by TMA, 32 columns at a time, through two staging tiles
            //    used in turn: the warp's quarters of Khat (which G has finished
            //    reading) and of F (which the write-back has). Before a tile is
            //    rewritten, the store that last used it has read it: stores
            //    complete their reads in order, so waiting until at most one is
            //    still reading suffices, at the next chunk and at the unit's end.
            if (!wait_bar(B_D(w), par, abort)) break;
            tc::tc_fence_after();
            if constexpr (Q8) {
                // an int8 base: the row's max over two reads of its 128 columns, then
                // its codes (16-byte stores of the row's own 128 bytes) and its scale
                float mx = 0.f;
#pragma unroll 1
                for (int ch = 0; ch < NCHUNK; ++ch) {
                    uint32_t d[32];
                    tc::tmem_ld32(trow + COL_SG + ch * CHUNK, d);
                    tc::tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) mx = fmaxf(mx, fabsf(__uint_as_float(d[i])));
                }
                const float sc = i8_scale(mx), inv = i8_inv(sc);
                int8_t *crow = codes + (un.head * DV + un.row0 + r) * (long long)DK;
                auto store_codes = [&](auto fast_c) {
                    constexpr bool FAST = decltype(fast_c)::value;
#pragma unroll 1
                    for (int ch = 0; ch < NCHUNK; ++ch) {
                        uint32_t d[32];
                        tc::tmem_ld32(trow + COL_SG + ch * CHUNK, d);
                        tc::tmem_wait_ld();
                        uint32_t wd[8];
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            wd[i] = i8_pack4<FAST>(__uint_as_float(d[4 * i + 0]), __uint_as_float(d[4 * i + 1]),
                                                   __uint_as_float(d[4 * i + 2]), __uint_as_float(d[4 * i + 3]), sc,
                                                   inv);
                        st_stream(crow + ch * CHUNK, make_uint4(wd[0], wd[1], wd[2], wd[3]));
                        st_stream(crow + ch * CHUNK + 16, make_uint4(wd[4], wd[5], wd[6], wd[7]));
                    }
                };
                if (i8_fast(sc))
                    store_codes(std::true_type{});
                else
                    store_codes(std::false_type{});
                i8_scales[un.head * DV + un.row0 + r] = sc;
            } else {
#pragma unroll 1
                for (int ch = 0; ch < NCHUNK; ++ch) {
                    uint32_t d[32];
                    tc::tmem_ld32(trow + COL_SG + ch * CHUNK, d);
                    uint8_t *buf = sm + LY.group(w) + LY.out_buf(quad, ch & 1);
                    if (ch >= 1 && lane == 0) tc::bulk_wait_read<1>();
                    __syncwarp();
                    tc::tmem_wait_ld();
#pragma unroll
                    for (int u = 0; u < 8; ++u)
                        DL_GUARD(buf + tile_off(lane, 4 * u), 16) *reinterpret_cast<uint4 *>(buf + tile_off(lane, 4 * u)) =
                            make_uint4(d[4 * u + 0], d[4 * u + 1], d[4 * u + 2], d[4 * u + 3]);
                    tc::fence_async_smem();  // the staging tile is read by the TMA store
                    __syncwarp();
                    if (lane == 0) {
                        tc::tma_store_2d(&map_st, ch * CHUNK, (int)(un.head * DV + un.row0 + 32 * quad), buf);
                        tc::bulk_commit();
                    }
                }
                // the warp's quarter of Khat, rewritten by the next unit's key side,
                // is free once the third store has read it; the fourth may still be
                // reading the warp's quarter of F, which the next F write waits for
                if (lane == 0) tc::bulk_wait_read<1>();
                __syncwarp();
            }
            tc::tc_fence_before();  // [COL_SG, +128) is rewritten by the group's next unit
        }
        if (lane == 0) tc::bulk_wait_all();  // the warp's last stores have landed
    }
    // drain: every role has left its loop; products in flight have completed
    // (the compute warps waited for the last one, or the CTA gave up)
    __syncthreads();
    if (warp == 1) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tbase, tmem_cols_for(NWG));
    }
}

// ---------------------------------------------------------------- host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link
// against the driver library); looked up once.
EncodeTiledFn encoder() {
    static EncodeTiledFn fn = []() -> EncodeTiledFn {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        return reinterpret_cast<EncodeTiledFn>(p);
    }();
    return fn;
}

// The fp32 state [rows, 128] as a tensor map of box_cols x box_rows boxes
// (box_cols x 4 bytes = the swizzle span: 32 columns with 128-byte swizzle,
// 16 with 64-byte).
cudaError_t state_map(CUtensorMap *m, void *S, unsigned long long rows, unsigned box_cols, unsigned box_rows) {
    EncodeTiledFn fn = encoder();
    if (!fn) return cudaErrorNotSupported;
    const cuuint64_t dims[2] = {(cuuint64_t)DK, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)DK * 4};
    const cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
    const cuuint32_t es[2] = {1, 1};
    const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, S, dims, strides, box, es,
                          CU_TENSOR_MAP_INTERLEAVE_NONE,
                          box_cols == 32 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// The int8 codes [rows, 128] as a tensor map of 128 x 128 boxes (one unit's
// codes; 128-byte rows under 128-byte swizzle).
cudaError_t code_map(CUtensorMap *m, void *codes, unsigned long long rows) {
    EncodeTiledFn fn = encoder();
    if (!fn) return cudaErrorNotSupported;
    const cuuint64_t dims[2] = {(cuuint64_t)DK, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)DK};
    const cuuint32_t box[2] = {(cuuint32_t)DK, (cuuint32_t)ROWS};
    const cuuint32_t es[2] = {1, 1};
    const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, codes, dims, strides, box, es,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

template <class IT, int KD, bool WC, bool Q8>
cudaError_t launch_tc_t(const StepParams &p, const LogParams &lg, int n_log, cudaStream_t st) {
    constexpr int NWG = groups_for(sizeof(IT), Rule<KD>::CHAN, Q8);
    constexpr Layout LY{sizeof(IT), Rule<KD>::CHAN, NWG, Q8};
    static_assert(LY.request() <= SMEM_LIMIT, "layout fits the shared memory a block may request");
    auto kern = merge_tc_kernel<IT, KD, WC, NWG, Q8>;
    cudaError_t e = allow_smem(reinterpret_cast<const void *>(kern), LY.request());
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 0;
    e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    const long long heads = (long long)p.B * p.H;
    CUtensorMap map, map_st;  // loads: 32 x 128 boxes; each warp's stores: 32 x 32 boxes
    int8_t *codes = nullptr;
    float *scales = nullptr;
    if constexpr (Q8) {  // codes [heads * d_v, 128], then one fp32 scale per row
        codes = static_cast<int8_t *>(p.S);
        scales = reinterpret_cast<float *>(codes + heads * p.dv * DK);
        e = code_map(&map, p.S, (unsigned long long)heads * p.dv);
        map_st = map;  // not used: the rows are stored from registers
    } else {
        e = state_map(&map, p.S, (unsigned long long)heads * p.dv, CHUNK, ROWS);
        if (e == cudaSuccess) e = state_map(&map_st, p.S, (unsigned long long)heads * p.dv, CHUNK, 32);
    }
    if (e != cudaSuccess) return e;
    const long long units = heads * (p.dv / ROWS);
    const unsigned grid = (unsigned)std::min<long long>(units, sms);
    kern<<<grid, threads_for(NWG), LY.request(), st>>>(
        map, map_st, static_cast<const IT *>(lg.k), static_cast<const IT *>(lg.v), static_cast<const IT *>(lg.beta),
        static_cast<const IT *>(lg.a), lg.x, lg.L, n_log, static_cast<const IT *>(p.q), static_cast<const IT *>(p.k),
        static_cast<const IT *>(p.v), static_cast<const IT *>(p.beta), static_cast<const IT *>(p.a), p.o, p.dv,
        units, codes, scales);
    return cudaGetLastError();
}

}  // namespace

bool merge_tc_supported(const StepParams &p, int n_log, bool with_cur, const PoolIdx &pool) {
    const long long rows = (long long)p.B * p.H * p.dv;
    return pool.slot == nullptr && (p.s_dt == DL_F32 || p.s_dt == DL_I8) && p.dk == DK && p.dv % ROWS == 0 &&
           n_log + (with_cur ? 1 : 0) <= NB && n_log + (with_cur ? 1 : 0) >= 1 && rows < (1LL << 31) &&
           encoder() != nullptr;
}

cudaError_t launch_merge_tc(const StepParams &p, const LogParams &lg, int n_log, bool with_cur, cudaStream_t st) {
    auto with_kind = [&](auto it_t, auto kd_c) -> cudaError_t {
        using IT = decltype(it_t);
        constexpr int KD = decltype(kd_c)::value;
        if (p.s_dt == DL_I8) {
            if (with_cur) return launch_tc_t<IT, KD, true, true>(p, lg, n_log, st);
            return launch_tc_t<IT, KD, false, true>(p, lg, n_log, st);
        }
        if (with_cur) return launch_tc_t<IT, KD, true, false>(p, lg, n_log, st);
        return launch_tc_t<IT, KD, false, false>(p, lg, n_log, st);
    };
    auto with_it = [&](auto it_t) -> cudaError_t {
        if (p.kind == DL_RWKV6) return with_kind(it_t, std::integral_constant<int, DL_RWKV6>{});
        if (p.kind == DL_DECAY_CHANNEL) return with_kind(it_t, std::integral_constant<int, DL_DECAY_CHANNEL>{});
        return with_kind(it_t, std::integral_constant<int, DL_DECAY_HEAD>{});
    };
    if (p.in_dt == DL_BF16) return with_it(bf16{});
    return with_it(float{});
}

cudaError_t read_tc_faults(unsigned int *out, bool clear) {
    cudaError_t e = cudaMemcpyFromSymbol(out, g_tc_faults, sizeof(unsigned int));
    if (e == cudaSuccess && clear) {
        const unsigned int zero = 0;
        e = cudaMemcpyToSymbol(g_tc_faults, &zero, sizeof(unsigned int));
    }
    return e;
}

// The guard word of this file's kernels (index-guard build; 0 otherwise).
cudaError_t read_guard_merge_tc(unsigned int *flags, unsigned int *line, bool clear) {
    return read_guard_word(flags, line, clear);
}

}  // namespace dl
