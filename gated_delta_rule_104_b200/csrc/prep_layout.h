// Shared-memory layout of the replay-prep kernel (deferred_read.cu), in host-
// and device-callable form, so that a host program can replay the addresses
// the kernel forms and check them against the regions below.
//
// One warp per head; each warp of the block owns one staging area of BYTES:
//   sk [EMAX][DK] the log keys and this step's key (raw input elements)
//   sa [EMAX][DK] the same for channel decays (channel decay only)
//   floats: as [EMAX] head-wise decays, beta [EMAX], d [EMAX], cn [EMAX],
//           s [EMAX], xrow [EMAX][EMAX] the X rows of the log and the new entry
#pragma once

#include <stddef.h>

#ifndef DL_HD
#if defined(__CUDACC__)
#define DL_HD __host__ __device__
#else
#define DL_HD
#endif
#endif

namespace dl {

template <int IB, int DK, int EMAX, bool CHAN>
struct PrepSmem {
    static constexpr int ROWB = DK * IB;                          // bytes of one key row
    static constexpr int K_OFF = 0;
    static constexpr int A_OFF = K_OFF + EMAX * ROWB;              // channel decays (raw)
    static constexpr int F_OFF = A_OFF + (CHAN ? EMAX * ROWB : 0);
    // float offsets from F_OFF
    static constexpr int AS = 0, BETA = AS + EMAX, D = BETA + EMAX, CN = D + EMAX, S = CN + EMAX,
                         XROW = S + EMAX;
    static constexpr int FLOATS = XROW + EMAX * EMAX;
    static constexpr int BYTES = F_OFF + FLOATS * 4;
};

// log capacity -> staging capacity (entries) and warps (heads) per block
DL_HD constexpr int prep_emax(int L) { return L <= 16 ? 16 : L <= 32 ? 32 : 64; }
DL_HD constexpr int prep_warps(int emax) { return emax <= 32 ? 4 : 2; }

}  // namespace dl
