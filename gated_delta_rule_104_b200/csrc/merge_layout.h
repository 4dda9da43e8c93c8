// Shared-memory layout of the warp-MMA merge kernel (merge.cu), in host- and
// device-callable form, so that a host program can replay the addresses the
// kernel forms and check them against the regions below.
//
// One block merges ROWS = 64 base rows of one head (4 warps of 16 rows). Its
// dynamic shared memory, in order:
//   tile [ROWS][DK] of the tile type (swizzled base rows: float for an int8
//        base, else the state type), then floats:
//   kh [NB][KH] keys, turned into Khat in place
//   ff [NB][WS] F (channel decay: holds the decays until F replaces them)
//   fa [NB] head decays (padded to 4)   gn [DK] gamma   sq [DK] q
//   sx [NB][XS] X   sb [NB] beta   sv [NB][VS] the tile's values
//   sxw [4][XS] each warp's copy of the fused entry's X row
//   int8 base only: scl [ROWS] row scales, wsc [4][16] the new row scales of
//        each warp's rows (the codes [ROWS][DK] land in the last ROWS * DK
//        bytes of the float tile and are read out into registers before it is
//        widened over them)
//   xw [5] a compact grid's walk: four ballots and the batch index, in
//        XW_BYTES (16-byte granules)
#pragma once

#include <stddef.h>
#include <stdint.h>

#ifndef DL_HD
#if defined(__CUDACC__)
#define DL_HD __host__ __device__
#else
#define DL_HD
#endif
#endif

namespace dl {

DL_HD constexpr size_t round4(size_t x) { return (x + 3) & ~(size_t)3; }

// Column order of the two products (merge.cu): F is stored in the order the
// update's B fragments read it, column c at position f_pos(c) = 16j + 8h + n
// of its group of 16.
DL_HD inline int f_pos(int c) { return (c & ~15) | (((c >> 1) & 1) << 3) | (((c >> 2) & 3) << 1) | (c & 1); }

template <int DK, int NB>
struct MergeShape {
    static constexpr int ROWS = 64;     // base rows per block: 4 warps of 16
    static constexpr int KH = DK;       // Khat row stride (no padding: the rows are swizzled, kof)
    static constexpr int WS = DK + 8;   // F row stride (conflict-free B-fragment reads)
    static constexpr int XS = NB + 4;   // X row stride (conflict-free B-fragment reads)
    static constexpr int VS = ROWS + 4; // value row stride (conflict-free accumulator-layout reads)
    static constexpr int CW = DK / 32;  // key channels per lane (warp-wide dots)
    // Khat element (i, c): the 16-byte chunks of row i XOR-swizzled by 4 (i mod 2),
    // so that a 16-byte B-fragment read (rows 2m and 2m + 1 in one 8-lane phase)
    // hits every bank; a pair of chunks 2u, 2u + 1 stays adjacent.
    DL_HD static inline int kof(int i, int c) { return i * KH + ((((c >> 2) ^ ((i & 1) << 2)) << 2) | (c & 3)); }
};

// The block's base rows: ROWS x DK elements of TB bytes, row-major, with the
// 16-byte chunks of row r XOR-swizzled by f(r). Every access is lane (g, t)
// moving columns 16j + 4t .. + 3 of row g (or g + 8):
//  - fp32: one 128-byte phase is 8 lanes, rows r, r + 1 with 4 chunks each;
//    f(r) = 4 (r mod 2) puts the two rows in opposite halves of the banks;
//  - bf16: one phase is 16 lanes of 8 bytes, rows r .. r + 3 with a chunk pair
//    each; f(r) = 2 (r mod 4) puts the four pairs on distinct banks.
// No padding.
template <int TB, int DK>
struct BaseTile {
    static constexpr int CE = 16 / TB;  // elements per 16-byte chunk
    static_assert(DK / CE >= 8, "swizzle spans 8 chunks");
    DL_HD static inline int off(int r, int c) {
        const int f = CE == 4 ? (r & 1) << 2 : (r & 3) << 1;
        return r * DK + (((c / CE) ^ f) * CE) + (c % CE);
    }
};

constexpr size_t XW_BYTES = 32;  // the compact walk's five words, padded to 16-byte granules

// Offsets of the regions: the tile in bytes from the base, the rest in floats
// from the end of the tile (xw: in floats too, a uint32 array). SB is the
// state element's size; Q8 an int8 base (then the tile holds floats).
template <int SB, bool Q8, int DK, int NB>
struct MergeRegions {
    using C = MergeShape<DK, NB>;
    static constexpr int TB = Q8 ? 4 : SB;  // tile element bytes
    static constexpr size_t tile_bytes = (size_t)C::ROWS * DK * TB;
    static constexpr size_t kh = 0;
    static constexpr size_t ff = kh + (size_t)NB * C::KH;
    static constexpr size_t fa = ff + (size_t)NB * C::WS;
    static constexpr size_t gn = fa + round4(NB);
    static constexpr size_t sq = gn + DK;
    static constexpr size_t sx = sq + DK;
    static constexpr size_t sb = sx + (size_t)NB * C::XS;
    static constexpr size_t sv = sb + round4(NB);
    static constexpr size_t sxw = sv + (size_t)NB * C::VS;
    static constexpr size_t scl = sxw + 4 * (size_t)C::XS;  // int8 base only
    static constexpr size_t wsc = scl + C::ROWS;             // int8 base only
    static constexpr size_t xw = Q8 ? wsc + 64 : scl;
    // the int8 codes: bytes from the base (the last ROWS * DK bytes of the float tile)
    static constexpr size_t raw_bytes_off = (size_t)C::ROWS * DK * (TB - 1);
    static constexpr size_t floats = xw;  // float words before xw
    static constexpr size_t bytes = tile_bytes + floats * 4 + XW_BYTES;
};

}  // namespace dl
