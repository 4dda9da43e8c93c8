// Shared-memory and tensor-memory layout of the tensor-core merge kernel
// (merge_tc.cu), in host- and device-callable form, so that a host program
// can replay every address the kernel forms and check it against the
// regions below (bounds, alignment, no overlap of live regions).
//
// One unit = one 128-row tile of one head's d_v x 128 fp32 state. A CTA keeps
// two pipeline stages, each holding one unit's state tile (as the TMA load
// leaves it) and the raw log entries its merge needs; a stage is released as
// soon as its unit no longer reads it (before the write-back), not when the
// unit's result has been stored. NWG compute groups (1 or 2) each keep their
// own operand tiles (Khat and F, which double as staging tiles for the TMA
// stores of the result), a few vectors, and their own 256 columns of tensor
// memory; group w merges the units i = w, w + NWG, ... of the CTA.
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
namespace mtc {

constexpr int ROWS = 128;     // state rows per unit (the M of every product)
constexpr int DK = 128;       // key width
constexpr int NB = 16;        // log entries merged per unit (the K of the write-back product)
constexpr int NS = 2;         // pipeline stages
constexpr int CHUNK = 32;     // fp32 columns per 128-byte swizzle row
constexpr int NCHUNK = DK / CHUNK;
constexpr int CTRL_WARPS = 4; // warp 0 loads, warps 1 and 2 issue products (group 0, 1), warp 3 idle
constexpr uint32_t TMEM_COLS_PER_GROUP = 256;
// A group's tensor memory (columns from the group's base):
//   [0, 128)   S o gamma, written while the tile is read for S_lo; the
//              write-back accumulates delta F onto it, giving S_new
//   [128, 192) S_lo for one half of the key columns at a time (the A operand
//              of G's second half, two rounds of 8 K-steps)
//   [192, 224) G = S Khat^T (hi half of Khat, then lo half)
//   [224, 256) delta hi (16 columns) | delta lo (16 columns)
constexpr int COL_SG = 0;
constexpr int COL_LO = 128;
constexpr int COL_G = 192;
constexpr int COL_DL = 224;
constexpr size_t SMEM_LIMIT = 232448;  // dynamic shared memory a block may request (227 KiB)

DL_HD constexpr size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
DL_HD constexpr int threads_for(int nwg) { return 32 * CTRL_WARPS + 128 * nwg; }
DL_HD constexpr uint32_t tmem_cols_for(int nwg) { return nwg == 1 ? 256u : 512u; }

// Offsets (bytes) from the CTA's 1024-aligned shared-memory base.
struct Layout {
    size_t in_size;  // bytes of one input element (2: bf16, 4: fp32)
    bool chan;       // one decay per key channel (else per entry)
    int nwg;         // compute groups
    bool q8 = false; // an int8 base: the unit's codes land in the tile's last column chunk (box 3,
                     // rows of 128 codes under the same 128-byte swizzle) and its row scales in
                     // the stage's scale region; the compute group writes the widened fp32 tile

    // ---- one stage
    DL_HD constexpr size_t tile() const { return (size_t)ROWS * DK * 4; }  // 64 KiB, 4 column chunks of 16 KiB
    DL_HD constexpr size_t raw_k() const { return (size_t)NB * DK * in_size; }
    DL_HD constexpr size_t raw_a() const { return chan ? raw_k() : 0; }
    DL_HD constexpr size_t raw_v() const { return (size_t)NB * ROWS * in_size; }
    DL_HD constexpr size_t raw_q() const { return (size_t)DK * in_size; }
    DL_HD constexpr size_t sc_floats() const { return NB * NB; }  // the X block
    DL_HD constexpr size_t off_tile() const { return 0; }
    DL_HD constexpr size_t off_raw_k() const { return off_tile() + tile(); }
    DL_HD constexpr size_t off_raw_a() const { return off_raw_k() + raw_k(); }
    DL_HD constexpr size_t off_raw_v() const { return off_raw_a() + raw_a(); }
    DL_HD constexpr size_t off_raw_q() const { return off_raw_v() + raw_v(); }
    DL_HD constexpr size_t off_sc() const { return off_raw_q() + raw_q(); }
    DL_HD constexpr size_t off_scl() const { return off_sc() + sc_floats() * 4; }  // int8 row scales [128]
    DL_HD constexpr size_t scl_bytes() const { return q8 ? (size_t)ROWS * 4 : 0; }
    DL_HD constexpr size_t off_codes() const { return off_tile() + (size_t)(NCHUNK - 1) * ROWS * 128; }
    DL_HD constexpr size_t stage_bytes() const { return round_up(off_scl() + scl_bytes(), 1024); }
    DL_HD constexpr size_t stage(int s) const { return (size_t)s * stage_bytes(); }

    // ---- one compute group's regions (from the group's base)
    // Khat, the B operand of G: 32 rows (entries' hi parts 0..15, lo parts
    // 16..31) x 128 key channels, K-major, 128-byte swizzle; column chunk c =
    // channels 32c..32c+31 is a [32 x 128 B] block at 4 KiB c.
    DL_HD constexpr size_t g_kh() const { return 0; }
    DL_HD constexpr size_t kh_bytes() const { return (size_t)2 * NB * DK * 4; }
    // F, the B operand of the write-back: 128 rows (key channels) x 32
    // (entries' hi parts 0..15, lo parts 16..31), K-major, 128-byte swizzle;
    // rows 32q..32q+31 are the quarter q (4 KiB).
    DL_HD constexpr size_t g_ff() const { return g_kh() + kh_bytes(); }
    DL_HD constexpr size_t ff_bytes() const { return (size_t)DK * 2 * NB * 4; }
    // the staging tiles of the result's TMA stores, two per warp of the group
    // (used in turn): warp quad q (rows 32q..32q+31) stages one 32-column
    // chunk of its rows, [32 rows x 128 B] with 128-byte swizzle. Tile 0 is
    // the warp's quarter of Khat (free once G has read it), tile 1 its quarter
    // of F (free once the write-back has read it).
    DL_HD constexpr size_t out_buf(int quad, int b) const {
        return (b == 0 ? g_kh() : g_ff()) + (size_t)quad * 32 * 128;
    }
    DL_HD constexpr size_t g_gam() const { return g_ff() + ff_bytes(); }    // gamma [128] floats
    DL_HD constexpr size_t g_qf() const { return g_gam() + DK * 4; }        // q widened [128] floats
    // the fused read's sums over key channels: C(n, e) (16) then (F q)_e (16)
    DL_HD constexpr size_t g_cn() const { return g_qf() + DK * 4; }
    DL_HD constexpr size_t g_red() const { return g_cn() + 2 * NB * 4; }    // [4 warps][32] partial sums
    DL_HD constexpr size_t group_bytes() const { return round_up(g_red() + 4 * 2 * NB * 4, 1024); }
    DL_HD constexpr size_t group(int w) const { return stage(NS) + (size_t)w * group_bytes(); }

    // ---- barriers and words
    DL_HD constexpr size_t off_bar() const { return group(nwg); }
    // full[NS], free[NS], then per group: kh_ready, lo_ready (twice per unit),
    // lo_free, g_done, delta_ready, d_done
    DL_HD constexpr int nbar() const { return 2 * NS + 6 * nwg; }
    DL_HD constexpr size_t off_tslot() const { return off_bar() + (size_t)nbar() * 8; }
    DL_HD constexpr size_t off_abort() const { return off_tslot() + 4; }
    DL_HD constexpr size_t end() const { return off_abort() + 4; }
    // dynamic shared memory to request: the layout plus slack to align the base to 1024
    DL_HD constexpr size_t request() const { return end() + 1024; }
};

// Byte offsets inside one stage's raw buffers (in_size-byte elements): key or
// channel decay c of entry e, value row r of entry e, query element c; and
// X(j, e) of the unit's X block (floats).
DL_HD constexpr size_t raw_k_off(int e, int c, size_t in_size) { return ((size_t)e * DK + c) * in_size; }
DL_HD constexpr size_t raw_v_off(int e, int r, size_t in_size) { return ((size_t)e * ROWS + r) * in_size; }
DL_HD constexpr size_t raw_q_off(int c, size_t in_size) { return (size_t)c * in_size; }
DL_HD constexpr size_t sc_x(int j, int e) { return (size_t)(j * NB + e) * 4; }

// Shared-memory start addresses (byte offsets from the operand's base) of the
// descriptors of the K = 8 step kk of G: A = the state tile, B = Khat. Both
// K-major with 128-byte swizzle and 1024-byte stride between 8-row groups.
DL_HD constexpr uint32_t g_a_start(int kk) { return (uint32_t)((kk / 4) * (ROWS * 128) + (kk % 4) * 32); }
DL_HD constexpr uint32_t g_b_start(int kk) { return (uint32_t)((kk / 4) * (2 * NB * 128) + (kk % 4) * 32); }
// The write-back's six K = 8 steps m: A columns in tensor memory (from
// COL_DL) and the byte offset of B inside F: delta_hi F_hi (2 steps),
// delta_hi F_lo (2), delta_lo F_hi (2). G's second half takes its A operand
// (S_lo) from tensor-memory columns COL_B + 8 kk.
DL_HD constexpr int wb_a_col(int m) { return m < 4 ? (m % 2) * 8 : 16 + (m % 2) * 8; }
DL_HD constexpr uint32_t wb_b_start(int m) { return (uint32_t)((m < 4 ? m : m - 4) * 32); }

// Byte offset inside the state tile of fp32 element (row r, column c): column
// chunk c / 32 at 16 KiB each, rows 128 bytes apart inside it, the 16-byte
// pieces of a row permuted by the 128-byte swizzle (the layout a tensor-map
// load with 128-byte swizzling writes, and the tensor cores' canonical K-major
// layout).
DL_HD constexpr uint32_t swz128(uint32_t off) { return off ^ ((off & 0x380u) >> 3); }
DL_HD constexpr uint32_t tile_off(int r, int c) {
    return (uint32_t)((c / CHUNK) * (ROWS * 128)) + swz128((uint32_t)(r * 128 + (c % CHUNK) * 4));
}
// Khat element (row n in 0..31, channel c) inside Khat.
DL_HD constexpr uint32_t kh_off(int n, int c) {
    return (uint32_t)((c / CHUNK) * (2 * NB * 128)) + swz128((uint32_t)(n * 128 + (c % CHUNK) * 4));
}
// F element (channel c, column j in 0..31) inside F.
DL_HD constexpr uint32_t ff_off(int c, int j) { return swz128((uint32_t)(c * 128 + j * 4)); }
// Groups the launch can afford: two when their regions fit beside the
// two stages, else one.
DL_HD constexpr int groups_for(size_t in_size, bool chan, bool q8 = false) {
    return Layout{in_size, chan, 2, q8}.request() <= SMEM_LIMIT ? 2 : 1;
}
// Byte offset inside the int8 code box (box 3 of the tile) of the 16-code
// piece j (codes 16j..16j+15) of row r: rows 128 bytes apart, pieces permuted
// by the same 128-byte swizzle, so row r's codes stay inside row r's 128 bytes
// of the box (which its own fp32 columns 96..127 overwrite last).
DL_HD constexpr uint32_t code_off(int r, int j) { return swz128((uint32_t)(r * 128 + j * 16)); }

}  // namespace mtc
}  // namespace dl
