// Host replay of every shared-memory, tensor-memory and global address the
// tensor-core merge kernel (gated_delta_rule_104_b200/csrc/merge_tc.cu)
// forms, for every instantiation (input element size, channel or head decay,
// delta rule or RWKV6, fused read or not, fp32 or int8 base) and every entry
// count it accepts. With an int8 base it also checks that each thread reads
// its row's codes before its own fp32 columns overwrite them, and that no
// thread writes over another row's codes.
// It uses the same layout functions as the kernel (merge_tc_layout.h) and
// walks the kernel's loops with their bounds, checking that each access lies
// inside its region, is aligned for its width, that regions do not overlap,
// that the swizzled layouts are one-to-one, that the operand tiles the
// threads write are the ones the descriptors make the tensor cores read, and
// that the whole layout fits the requested dynamic shared memory.
//
// Usage: merge_tc_replay [shrink <region> <bytes>]
//   shrink: the bounds table believes <region> is <bytes> shorter than the
//   layout says (a planted overrun: the replay must then fail).
// Exit status 0: every check passed; 1: a check failed (printed).
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <map>
#include <set>
#include <string>
#include <vector>

#include "merge_tc_layout.h"

using namespace dl::mtc;

namespace {

int failures = 0;
std::map<std::string, long> shrink;

void fail(const char *what, const std::string &ctx) {
    if (failures < 20) std::printf("FAIL %s: %s\n", what, ctx.c_str());
    ++failures;
}

struct Region {
    std::string name;
    size_t off, bytes;
};

struct Replay {
    size_t in_size;
    bool chan, delta, with_cur, q8;
    Layout ly;
    std::vector<Region> regions;

    Replay(size_t in, bool ch, bool de, bool wc, bool q)
        : in_size(in), chan(ch), delta(de), with_cur(wc), q8(q), ly{in, ch, groups_for(in, ch, q), q} {
        for (int s = 0; s < NS; ++s) {
            const std::string p = "stage" + std::to_string(s) + ".";
            add(p + "tile", ly.stage(s) + ly.off_tile(), ly.tile());
            if (q8) add(p + "scl", ly.stage(s) + ly.off_scl(), ly.scl_bytes());
            add(p + "raw_k", ly.stage(s) + ly.off_raw_k(), ly.raw_k());
            if (chan) add(p + "raw_a", ly.stage(s) + ly.off_raw_a(), ly.raw_a());
            add(p + "raw_v", ly.stage(s) + ly.off_raw_v(), ly.raw_v());
            add(p + "raw_q", ly.stage(s) + ly.off_raw_q(), ly.raw_q());
            add(p + "sc", ly.stage(s) + ly.off_sc(), ly.sc_floats() * 4);
        }
        for (int w = 0; w < ly.nwg; ++w) {
            const std::string p = "group" + std::to_string(w) + ".";
            add(p + "kh", ly.group(w) + ly.g_kh(), ly.kh_bytes());
            add(p + "ff", ly.group(w) + ly.g_ff(), ly.ff_bytes());
            add(p + "gam", ly.group(w) + ly.g_gam(), DK * 4);
            add(p + "qf", ly.group(w) + ly.g_qf(), DK * 4);
            add(p + "cn", ly.group(w) + ly.g_cn(), 2 * NB * 4);        // C(n, e) then (F q)_e
            add(p + "red", ly.group(w) + ly.g_red(), 4 * 2 * NB * 4);  // [4 warps][32]
        }
        add("bar", ly.off_bar(), (size_t)ly.nbar() * 8);
        add("tslot", ly.off_tslot(), 4);
        add("abort", ly.off_abort(), 4);
    }
    std::string tag() const {
        char b[96];
        std::snprintf(b, sizeof b, "in%zu %s %s %s %s", in_size, chan ? "chan" : "head", delta ? "delta" : "rwkv6",
                      with_cur ? "fused" : "merge", q8 ? "int8 base" : "fp32 base");
        return b;
    }
    void add(const std::string &name, size_t off, size_t bytes) {
        // a planted shrink applies to every stage's region of that name
        for (auto &kv : shrink) {
            const std::string &n = kv.first;
            if (name == n || (name.size() > n.size() && name.compare(name.size() - n.size(), n.size(), n) == 0 &&
                              name[name.size() - n.size() - 1] == '.'))
                bytes = bytes > (size_t)kv.second ? bytes - kv.second : 0;
        }
        regions.push_back({name, off, bytes});
    }
    const Region &region(const std::string &name) const {
        for (auto &r : regions)
            if (r.name == name) return r;
        std::printf("no region %s\n", name.c_str());
        std::exit(2);
    }
    // an access of `bytes` at `off` (from the region's start) of width-aligned data
    void acc(const std::string &name, size_t off, size_t bytes, size_t align, const char *what) {
        const Region &r = region(name);
        if (off + bytes > r.bytes) fail("out of region", tag() + " " + name + " " + what + " off " + std::to_string(off));
        if ((r.off + off) % align) fail("misaligned", tag() + " " + name + " " + what);
    }

    void layout_checks() {
        if (ly.request() > SMEM_LIMIT) fail("request above 227 KiB", tag());
        if (ly.end() + 1023 > ly.request()) fail("no room for the 1024-byte base alignment", tag());
        if (ly.stage_bytes() % 1024) fail("stage not 1024-aligned", tag());
        for (int w = 0; w < ly.nwg; ++w)
            if ((ly.group(w) + ly.g_kh()) % 1024 || (ly.group(w) + ly.g_ff()) % 1024)
                fail("operand region not 1024-aligned", tag());
        if (ly.nwg < 1 || ly.nwg > 2 || (int)tmem_cols_for(ly.nwg) < ly.nwg * (int)TMEM_COLS_PER_GROUP)
            fail("tensor memory for the groups", tag());
        for (size_t i = 0; i < regions.size(); ++i) {
            if (regions[i].off + regions[i].bytes > ly.end()) fail("region beyond the layout", regions[i].name);
            for (size_t j = i + 1; j < regions.size(); ++j) {
                const Region &a = regions[i], &b = regions[j];
                if (a.bytes && b.bytes && a.off < b.off + b.bytes && b.off < a.off + a.bytes)
                    fail("overlapping regions", a.name + " / " + b.name);
            }
        }
        for (int s = 0; s < NS; ++s)
            for (int ch = 0; ch < NCHUNK; ++ch)
                if ((ly.stage(s) + ly.off_tile() + ch * ROWS * 128) % 1024) fail("TMA box not 1024-aligned", tag());
    }

    // warp 0: TMA boxes and bulk copies of the raw entries (lane 0), cp.async of the X block
    void producer(int n_log, int L) {
        const int nb = n_log + (with_cur ? 1 : 0);
        const size_t KB = DK * in_size, VB = ROWS * in_size;
        for (int s = 0; s < NS; ++s) {
            const std::string p = "stage" + std::to_string(s) + ".";
            size_t tx = 0;
            if (q8) {  // the codes' one TMA box into the tile's last column chunk, the scales by a bulk copy
                if (ly.off_codes() - ly.off_tile() != (size_t)(NCHUNK - 1) * ROWS * 128) fail("code box offset", tag());
                acc(p + "tile", ly.off_codes() - ly.off_tile(), ROWS * DK, 1024, "code TMA box");
                tx += ROWS * DK;
                acc(p + "scl", 0, ROWS * 4, 16, "row scales");
                tx += ROWS * 4;
            } else {
                for (int ch = 0; ch < NCHUNK; ++ch) {
                    acc(p + "tile", ch * ROWS * 128, ROWS * 128, 1024, "TMA box");
                    tx += ROWS * 128;
                }
            }
            // (lanes 16 + e copy entry e's value tile: every entry has a lane)
            if (nb > 16) fail("more entries than value-copy lanes", tag());
            auto bulk = [&](const std::string &reg, size_t off, size_t bytes, const char *what) {
                if (bytes % 16) fail("bulk copy size not a multiple of 16", tag() + " " + what);
                acc(reg, off, bytes, 16, what);
                tx += bytes;
            };
            if (n_log > 0) {
                bulk(p + "raw_k", raw_k_off(0, 0, in_size), n_log * KB, "log keys");
                if (chan) bulk(p + "raw_a", raw_k_off(0, 0, in_size), n_log * KB, "log decays");
            }
            for (int e = 0; e < n_log; ++e) bulk(p + "raw_v", raw_v_off(e, 0, in_size), VB, "log values");
            if (with_cur) {
                bulk(p + "raw_k", raw_k_off(n_log, 0, in_size), KB, "step key");
                if (chan) bulk(p + "raw_a", raw_k_off(n_log, 0, in_size), KB, "step decays");
                bulk(p + "raw_v", raw_v_off(n_log, 0, in_size), VB, "step values");
                bulk(p + "raw_q", raw_q_off(0, in_size), KB, "step query");
            }
            // the byte count the loader expects (merge_tc.cu: tx)
            const size_t base_tx = q8 ? (size_t)ROWS * DK + ROWS * 4 : ly.tile();
            const size_t expect = base_tx + (size_t)nb * (KB * (chan ? 2 : 1) + VB) + (with_cur ? KB : 0);
            if (tx != expect) fail("expected bytes differ from the bytes copied", tag());
            if (tx >= (1u << 20)) fail("transaction count beyond the mbarrier's range", tag());
            for (int lane = 0; lane < 32; ++lane)
                if (delta)
                    for (int u = lane; u < NB * NB; u += 32) {
                        const int j = u / NB, e = u % NB;
                        if (j < n_log && e <= j) {
                            acc(p + "sc", sc_x(j, e), 4, 4, "X block");
                            // the global element read: row j < n_log <= L of the head's [L, L] block
                            if (j >= L || e >= L) fail("X read outside the head's block", tag());
                        }
                    }
        }
    }

    // compute group w: key side, fused X row, S_lo, delta, write-back (128 threads)
    void compute(int n_log, int w) {
        const int nb = n_log + (with_cur ? 1 : 0);
        const std::string p = "stage" + std::to_string(w % NS) + ".";
        const std::string gp = "group" + std::to_string(w) + ".";
        std::set<uint32_t> khs, ffs, tiles;
        for (int ct = 0; ct < 128; ++ct) {
            const int warp = CTRL_WARPS + 4 * w + ct / 32, lane = ct % 32, quad = warp & 3, r = 32 * quad + lane,
                      c = r;
            if (warp >= threads_for(ly.nwg) / 32) fail("warp outside the block", tag());
            if (r < 0 || r >= ROWS) fail("row outside the tile", tag());
            for (int j = 0; j < NB; ++j) {
                if (j < nb) {
                    acc(p + "raw_k", raw_k_off(j, c, in_size), in_size, in_size, "k read");
                    if (chan) acc(p + "raw_a", raw_k_off(j, c, in_size), in_size, in_size, "a read");
                    acc(p + "raw_v", raw_v_off(j, r, in_size), in_size, in_size, "v read");
                }
                if (delta) {
                    acc(gp + "kh", kh_off(j, c), 4, 4, "Khat hi");
                    acc(gp + "kh", kh_off(NB + j, c), 4, 4, "Khat lo");
                    khs.insert(kh_off(j, c));
                    khs.insert(kh_off(NB + j, c));
                    for (int m4 = 0; m4 <= j / 4; ++m4) acc(p + "sc", sc_x(j, 4 * m4), 16, 16, "X row piece");
                }
            }
            acc(gp + "gam", c * 4, 4, 4, "gamma");
            if (with_cur) {
                acc(gp + "qf", c * 4, 4, 4, "q widened");
                acc(p + "raw_q", raw_q_off(c, in_size), in_size, in_size, "q raw read");
            }
            for (int u = 0; u < 8; ++u) {
                acc(gp + "ff", ff_off(c, 4 * u), 16, 16, "F piece");
                // F row c lies in the warp's own quarter of F (its staging tile 1)
                const size_t q1 = ly.out_buf(quad, 1) - ly.g_ff();
                if (ff_off(c, 4 * u) < q1 || ff_off(c, 4 * u) + 16 > q1 + 32 * 128)
                    fail("F piece outside the warp's own quarter", tag());
                for (int e = 0; e < 4; ++e) {
                    if (ff_off(c, 4 * u + e) != ff_off(c, 4 * u) + 4u * e) fail("F piece not contiguous", tag());
                    ffs.insert(ff_off(c, 4 * u + e));
                }
            }
            if (with_cur) {  // the fused read's sums over key channels and its entry's X row
                const int nl = nb - 1;
                acc(p + "raw_k", raw_k_off(nl, c, in_size), in_size, in_size, "fused key");
                acc(p + "raw_q", raw_q_off(c, in_size), in_size, in_size, "fused q");
                acc(gp + "red", (quad * 2 * NB + lane) * 4, 4, 4, "red write");
                if (ct < 2 * NB) {
                    for (int q4 = 0; q4 < 4; ++q4) acc(gp + "red", (q4 * 2 * NB + ct) * 4, 4, 4, "red read");
                    acc(gp + "cn", ct * 4, 4, 4, "cn write");
                }
                if (delta && ct <= nl) {
                    for (int m = ct; m < nl; ++m) {
                        acc(gp + "cn", m * 4, 4, 4, "cn read");
                        acc(p + "sc", sc_x(m, ct), 4, 4, "X read (fused row)");
                    }
                    acc(p + "sc", sc_x(nl, ct), 4, 4, "fused X row write");
                }
                for (int e = 0; e < NB; ++e) acc(gp + "cn", (NB + e) * 4, 4, 4, "F q read");
            }
            if (q8) {
                acc(p + "scl", r * 4, 4, 4, "row scale");
                // chunk ch reads pieces 2ch, 2ch + 1 of the row's codes, then writes its
                // fp32 columns; no chunk may write a code byte that a later chunk reads
                std::set<uint32_t> written;
                for (int ch = 0; ch < NCHUNK; ++ch) {
                    for (int j = 2 * ch; j < 2 * ch + 2; ++j) {
                        const uint32_t co = (uint32_t)(ly.off_codes() - ly.off_tile()) + code_off(r, j);
                        acc(p + "tile", co, 16, 16, "code piece");
                        for (uint32_t b = co; b < co + 16; ++b)
                            if (written.count(b)) fail("a code piece read after its bytes were overwritten", tag());
                        if (co < (uint32_t)(ly.off_codes() - ly.off_tile()) + r * 128u ||
                            co + 16 > (uint32_t)(ly.off_codes() - ly.off_tile()) + (r + 1) * 128u)
                            fail("a code piece outside its row's 128 bytes", tag());
                    }
                    if (delta)
                        for (int col = ch * CHUNK; col < (ch + 1) * CHUNK; col += 4)
                            for (uint32_t b = tile_off(r, col); b < tile_off(r, col) + 16; ++b) written.insert(b);
                }
                // what the tile's writes overwrite of other rows' codes: nothing
                for (uint32_t b : written) {
                    const uint32_t cb = (uint32_t)(ly.off_codes() - ly.off_tile());
                    if (b >= cb && (b - cb) / 128 != (uint32_t)r) fail("a tile write over another row's codes", tag());
                }
            }
            for (int col = 0; col < DK; col += 4) {
                acc(p + "tile", tile_off(r, col), 16, 16, "tile piece");
                if (col < CHUNK)  // the warp's two staging tiles: its 32 rows of one 32-column chunk
                    for (int b = 0; b < 2; ++b) {
                        const char *reg = b == 0 ? "kh" : "ff";
                        const size_t base = b == 0 ? ly.g_kh() : ly.g_ff();
                        const size_t o = ly.out_buf(quad, b) - base + tile_off(lane, col);
                        acc(gp + reg, o, 16, 16, "staging piece");
                        if (tile_off(lane, col) >= 32 * 128) fail("staging piece outside its tile", tag());
                        if ((ly.group(w) + ly.out_buf(quad, b)) % 1024) fail("staging tile not 1024-aligned", tag());
                    }
                acc(gp + "gam", col * 4, 16, 16, "gamma piece");
                if (with_cur) acc(gp + "qf", col * 4, 16, 16, "q piece");
                for (int e = 0; e < 4; ++e) {
                    if (tile_off(r, col + e) != tile_off(r, col) + 4u * e) fail("tile piece not contiguous", tag());
                    tiles.insert(tile_off(r, col + e));
                    (void)e;
                }
            }
            // tensor memory: S o gamma chunks, the two S_lo halves, G, delta, the write-back's 16-column reads
            for (int ch = 0; ch < NCHUNK; ++ch)
                if (COL_SG + ch * CHUNK + 32 > COL_LO) fail("S o gamma columns run into S_lo", tag());
            for (int h = 0; h < 2; ++h)
                if (COL_LO + h * CHUNK + 32 > COL_G) fail("S_lo columns run into G", tag());
            for (int c16 = 0; c16 < DK / 16; ++c16)
                if (COL_SG + 16 * c16 + 16 > COL_LO) fail("write-back read past S_new", tag());
        }
        if (delta && khs.size() != (size_t)2 * NB * DK) fail("Khat layout not one-to-one", tag());
        if (ffs.size() != (size_t)DK * 2 * NB) fail("F layout not one-to-one", tag());
        if (tiles.size() != (size_t)ROWS * DK) fail("tile layout not one-to-one", tag());
    }

    // what the descriptors make the tensor cores read: K-major, 128-byte
    // swizzle, 8-row groups 1024 bytes apart, 32 bytes of K per step. The
    // element (row, k) a step reads must be the one the threads wrote there.
    static uint32_t desc_elem(uint32_t start, int row, int k) {
        // start = group-aligned base + byte offset of the step within the 128-byte row
        const uint32_t base = start & ~127u, within = start & 127u;
        return base + (uint32_t)(row / 8) * 1024 + swz128((uint32_t)((row % 8) * 128) + within + 4u * k);
    }
    void descriptors() {
        // G, A = the state tile: step kk reads rows 0..127, channels 8kk..8kk+7
        for (int kk = 0; kk < DK / 8; ++kk)
            for (int row = 0; row < ROWS; ++row)
                for (int k = 0; k < 8; ++k) {
                    const uint32_t a = desc_elem(g_a_start(kk), row, k);
                    if (a != tile_off(row, 8 * kk + k)) fail("G's A operand is not the tile element", tag());
                    if (delta) {
                        if (row < 2 * NB) {
                            const uint32_t b = desc_elem(g_b_start(kk), row, k);
                            if (b != kh_off(row, 8 * kk + k)) fail("G's B operand is not the Khat element", tag());
                            if (b + 4 > ly.kh_bytes()) fail("G's B read outside Khat", tag());
                        }
                    }
                    if (a + 4 > ly.tile()) fail("G's A read outside the tile", tag());
                }
        // write-back, B = F: step m reads rows (channels) 0..127, entries of its 8-column slice
        for (int m = 0; m < 6; ++m) {
            const int jbase = (m < 4 ? m : m - 4) * 8;  // column of F in [hi 0..15 | lo 16..31]
            for (int row = 0; row < DK; ++row)
                for (int k = 0; k < 8; ++k) {
                    const uint32_t b = desc_elem(wb_b_start(m), row, k);
                    if (b != ff_off(row, jbase + k)) fail("write-back's B operand is not the F element", tag());
                    if (b + 4 > ly.ff_bytes()) fail("write-back's B read outside F", tag());
                }
            // A in tensor memory: delta columns of the same entries (hi for m < 4, lo after)
            const int acol = COL_DL + wb_a_col(m);
            const int entry0 = (m % 2) * 8, part = m < 4 ? 0 : 1;  // which half of [hi | lo]
            if (acol != COL_DL + part * NB + entry0) fail("write-back's A columns", tag());
            const bool b_lo = (m == 2 || m == 3);
            if ((b_lo ? NB : 0) + entry0 != jbase) fail("write-back pairs the wrong F half", tag());
            if (acol + 8 > (int)TMEM_COLS_PER_GROUP) fail("tensor-memory column out of range", tag());
        }
        // G's second product: A = S_lo, columns COL_LO + 8 kq for the 8 K-steps of each half
        for (int kq = 0; kq < DK / 16; ++kq)
            if (COL_LO + 8 * kq + 8 > COL_G) fail("S_lo A columns out of range", tag());
        // S o gamma [0, 128) | S_lo [128, 192) | G [192, 224) | delta [224, 256)
        if (COL_SG + DK > COL_LO || COL_LO + DK / 2 > COL_G || COL_G + 2 * NB > COL_DL ||
            COL_DL + 2 * NB > (int)TMEM_COLS_PER_GROUP)
            fail("tensor-memory regions overlap or overflow", tag());
    }
};

}  // namespace

int main(int argc, char **argv) {
    for (int i = 1; i < argc; ++i) {
        if (std::strcmp(argv[i], "shrink") == 0 && i + 2 < argc) {
            shrink[argv[i + 1]] = std::atol(argv[i + 2]);
            i += 2;
        }
    }
    int cases = 0;
    for (int q8 = 0; q8 < 2; ++q8)
    for (size_t in : {2, 4})
        for (int chan = 0; chan < 2; ++chan)
            for (int delta = 0; delta < 2; ++delta)
                for (int wc = 0; wc < 2; ++wc) {
                    if (!delta && !chan) continue;  // RWKV6 has channel decay
                    Replay rp(in, chan, delta, wc, q8);
                    rp.layout_checks();
                    rp.descriptors();
                    for (int n_log = wc ? 0 : 1; n_log + wc <= NB; ++n_log) {
                        // L: the log capacity; fused reads need n_log < L, merges n_log <= L
                        const int L = wc ? n_log + 1 : n_log;
                        rp.producer(n_log, L);
                        for (int w = 0; w < rp.ly.nwg; ++w) rp.compute(n_log, w);
                        ++cases;
                    }
                }
    std::printf("%d cases, %d failures\n", cases, failures);
    return failures ? 1 : 0;
}
