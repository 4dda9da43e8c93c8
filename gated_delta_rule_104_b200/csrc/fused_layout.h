// Shared-memory layout of the fused append-read kernel (deferred_read.cu,
// append_read_fused_kernel), in host- and device-callable form, so that a
// host program can replay the addresses the kernel forms and check them
// against the regions below. The kernel serves d_v <= 128 (d_v = 256 layouts
// are laid out and replayed too, but the read takes its two-kernel form there).
//
// One persistent block per SM, in two roles that work on the block's heads
// (batch heads blockIdx.x, blockIdx.x + gridDim.x, ...) in order:
//   NP prep warps     warp p runs ReplayPrep for the block's heads p, p + NP,
//                     ... in its own staging area (PrepSmem), and leaves the
//                     head's (x_0, w) in slot i mod NSLOT of a ring;
//   ND decode warps   stream the base by bulk copies of UNIT_BYTES (a unit:
//                     UNIT_ROWS consecutive rows of one head) into a ring of
//                     NBUF buffers per warp, and form o = S_bar x_0 + w for
//                     the units d, d + ND, ... of the block's heads.
// Regions (byte offsets from the 128-aligned base of dynamic shared memory):
//   prep   [NP][PrepSmem::BYTES]
//   slots  [NSLOT][DK + DV] fp32
//   ring   [ND][NBUF][UNIT_BYTES]
//   bars   full[NSLOT], free[NSLOT], ring[ND][NBUF] (8-byte mbarriers), then
//          one int: the abort flag
#pragma once

#include <stddef.h>

#include "prep_layout.h"

#ifndef DL_HD
#if defined(__CUDACC__)
#define DL_HD __host__ __device__
#else
#define DL_HD
#endif
#endif

namespace dl {

namespace fused {

constexpr int EMAX = 16;                  // log entries the fused kernel stages (L <= 16)
constexpr int ND = 8;                     // decode warps
constexpr int NBUF = 3;                   // base buffers in flight per decode warp
constexpr int UNIT_BYTES = 4096;          // one bulk copy: 32 lanes x 8 rows' 16-byte slices
constexpr int MIN_HEADS_PER_SM = 32;      // the one-kernel read is used from this many heads per SM
// prep warps at most: 12, or 8 where ReplayPrep holds more per lane (fp32
// inputs), so that the block's registers (65536 over its threads) leave no
// prep warp spilling
DL_HD constexpr int np_max(int IB, int DV) { return (IB == 4 || DV > 128) ? 8 : 12; }
constexpr int SMEM_LIMIT = 227 * 1024;    // dynamic shared memory a block may request
constexpr int ALIGN_SLACK = 128;          // the kernel aligns its base up to 128 bytes

DL_HD constexpr int align_up(int x, int a) { return (x + a - 1) / a * a; }

// IB: bytes of an input element; SB: bytes of a base element.
template <int IB, int SB, int DK, int DV, bool CHAN>
struct Layout {
    using P = PrepSmem<IB, DK, EMAX, CHAN>;
    static constexpr int UNIT_ROWS = UNIT_BYTES / (DK * SB);
    static constexpr int UPH = DV / UNIT_ROWS;  // units per head
    static constexpr int SLOT_BYTES = (DK + DV) * 4;
    static constexpr int RING_BYTES = ND * NBUF * UNIT_BYTES;
    // a prep warp costs its staging area and two slots of the ring
    static constexpr int PER_PREP = P::BYTES + 2 * SLOT_BYTES;
    static constexpr int FIXED = RING_BYTES + ALIGN_SLACK + 256 + 8 * ND * NBUF + 16;
    static constexpr int NP_CAP = np_max(IB, DV);
    static constexpr int NP_FIT = (SMEM_LIMIT - FIXED - 16 * NP_CAP * 2) / PER_PREP;
    static constexpr int NP = NP_FIT < NP_CAP ? NP_FIT : NP_CAP;
    static constexpr int NSLOT = 2 * NP;
    static constexpr int WARPS = NP + ND;

    static constexpr int PREP_OFF = 0;
    static constexpr int SLOT_OFF = align_up(PREP_OFF + NP * P::BYTES, 128);
    static constexpr int RING_OFF = align_up(SLOT_OFF + NSLOT * SLOT_BYTES, 128);
    static constexpr int BAR_OFF = RING_OFF + RING_BYTES;
    static constexpr int BAR_FULL = BAR_OFF;
    static constexpr int BAR_FREE = BAR_FULL + 8 * NSLOT;
    static constexpr int BAR_RING = BAR_FREE + 8 * NSLOT;
    static constexpr int ABORT_OFF = BAR_RING + 8 * ND * NBUF;
    static constexpr int BYTES = ABORT_OFF + 16;
    static constexpr int REQUEST = BYTES + ALIGN_SLACK;

    DL_HD static constexpr int prep(int p) { return PREP_OFF + p * P::BYTES; }
    DL_HD static constexpr int slot(int s) { return SLOT_OFF + s * SLOT_BYTES; }
    DL_HD static constexpr int ring(int d, int b) { return RING_OFF + (d * NBUF + b) * UNIT_BYTES; }
};

}  // namespace fused

}  // namespace dl
