// Host replay of the shared-memory addresses (and the log's global rows)
// that the warp-MMA merge kernel (gated_delta_rule_104_b200/csrc/merge.cu,
// its compact pool walk included), the replay-prep kernel and the fused
// append-read kernel (gated_delta_rule_104_b200/csrc/deferred_read.cu, the
// latter's ReplayPrep from prep.cuh) form, for every instantiation and every
// log fill they accept. The region offsets and the swizzles come from the
// kernels' own layout headers (merge_layout.h, prep_layout.h,
// fused_layout.h); the loops are the kernels' loops with their bounds. Each
// access is checked to lie inside its region and to be aligned for its
// width; the regions must not overlap and must fit the dynamic shared memory
// the launch requests.
//
// Usage: merge_replay [merge | prep | fused] [shrink <region> <bytes>]...
//   merge, prep, fused: replay only that kernel.
//   shrink: the bounds table believes <region> is <bytes> shorter than the
//   layout says (a planted overrun: the replay must then fail; it stops at
//   the first failure).
// Exit status 0: every check passed; 1: a check failed (printed).
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <map>
#include <set>
#include <string>
#include <vector>

#include "merge_layout.h"
#include "prep_layout.h"
#include "fused_layout.h"

using namespace dl;

namespace {

int failures = 0;
std::map<std::string, long> shrink;
constexpr size_t SMEM_LIMIT = 232448;  // dynamic shared memory a block may request (227 KiB)

void fail(const char *what, const std::string &ctx) {
    if (failures < 20) std::printf("FAIL %s: %s\n", what, ctx.c_str());
    ++failures;
    if (!shrink.empty()) std::exit(1);  // a planted overrun: the first failure is the answer
}

struct Region {
    std::string name;
    size_t off, bytes;
    bool overlay;  // lies inside another region by design (int8 codes inside the float tile)
};

struct Table {
    std::string tag;
    std::vector<Region> regions;
    void add(const std::string &name, size_t off, size_t bytes, bool overlay = false) {
        auto it = shrink.find(name);
        if (it != shrink.end()) bytes = bytes > (size_t)it->second ? bytes - it->second : 0;
        regions.push_back({name, off, bytes, overlay});
    }
    const Region &region(const std::string &name) const {
        for (auto &r : regions)
            if (r.name == name) return r;
        std::printf("no region %s\n", name.c_str());
        std::exit(2);
    }
    // `bytes` at byte offset `off` from the region's start, `align`-aligned in shared memory
    void acc(const std::string &name, long off, size_t bytes, size_t align, const char *what) {
        const Region &r = region(name);
        if (off < 0 || (size_t)off + bytes > r.bytes)
            fail("out of region", tag + " " + name + " " + what + " off " + std::to_string(off));
        if ((r.off + (size_t)off) % align) fail("misaligned", tag + " " + name + " " + what);
    }
    void no_overlap(size_t end) {
        for (size_t i = 0; i < regions.size(); ++i) {
            if (regions[i].off + regions[i].bytes > end) fail("region beyond the layout", tag + " " + regions[i].name);
            for (size_t j = i + 1; j < regions.size(); ++j) {
                const Region &a = regions[i], &b = regions[j];
                if (a.overlay || b.overlay) continue;
                if (a.bytes && b.bytes && a.off < b.off + b.bytes && b.off < a.off + a.bytes)
                    fail("overlapping regions", tag + " " + a.name + " / " + b.name);
            }
        }
    }
};

// ---------------------------------------------------------------- merge.cu

template <int SB, bool Q8, int DK, int NB>
struct MergeReplay {
    using C = MergeShape<DK, NB>;
    using RG = MergeRegions<SB, Q8, DK, NB>;
    static constexpr int TB = RG::TB, ROWS = C::ROWS, nthr = 2 * ROWS, NT = NB / 8;
    using TL = BaseTile<TB, DK>;
    bool chan, delta;
    int in_bytes;
    Table t;

    MergeReplay(bool ch, bool de, int ib) : chan(ch), delta(de), in_bytes(ib) {
        char b[96];
        std::snprintf(b, sizeof b, "state%d%s dk%d nb%d %s %s in%d", SB, Q8 ? "(i8)" : "", DK, NB,
                      ch ? "chan" : "head", de ? "delta" : "rwkv6", ib);
        t.tag = b;
        const size_t F = RG::tile_bytes;  // floats start here
        t.add("tile", 0, RG::tile_bytes);
        if (Q8) t.add("raw", RG::raw_bytes_off, (size_t)ROWS * DK, true);
        t.add("kh", F + RG::kh * 4, (size_t)NB * C::KH * 4);
        t.add("ff", F + RG::ff * 4, (size_t)NB * C::WS * 4);
        t.add("fa", F + RG::fa * 4, round4(NB) * 4);
        t.add("gn", F + RG::gn * 4, (size_t)DK * 4);
        t.add("sq", F + RG::sq * 4, (size_t)DK * 4);
        t.add("sx", F + RG::sx * 4, (size_t)NB * C::XS * 4);
        t.add("sb", F + RG::sb * 4, round4(NB) * 4);
        t.add("sv", F + RG::sv * 4, (size_t)NB * C::VS * 4);
        t.add("sxw", F + RG::sxw * 4, (size_t)4 * C::XS * 4);
        if (Q8) {
            t.add("scl", F + RG::scl * 4, (size_t)ROWS * 4);
            t.add("wsc", F + RG::wsc * 4, (size_t)64 * 4);
        }
        t.add("xw", F + RG::xw * 4, XW_BYTES);
    }
    void f(const char *reg, long idx, int n, size_t align, const char *what) {  // float index
        t.acc(reg, idx * 4, (size_t)n * 4, align, what);
    }
    void tile(int r, int c, int n, const char *what) {  // n consecutive tile elements
        const int o = TL::off(r, c);
        for (int e = 0; e < n; ++e)
            if (TL::off(r, c + e) != o + e) fail("tile elements not contiguous", t.tag + " " + what);
        t.acc("tile", (long)o * TB, (size_t)n * TB, (size_t)n * TB, what);
    }

    void layout() {
        if (RG::bytes > SMEM_LIMIT) fail("request above 227 KiB", t.tag);
        t.no_overlap(RG::bytes);
        std::set<int> seen;  // the tile swizzle is one-to-one
        for (int r = 0; r < ROWS; ++r)
            for (int c = 0; c < DK; ++c) seen.insert(TL::off(r, c));
        if (seen.size() != (size_t)ROWS * DK || *seen.rbegin() >= ROWS * DK) fail("tile swizzle", t.tag);
        std::set<int> ks;
        for (int i = 0; i < NB; ++i)
            for (int c = 0; c < DK; ++c) ks.insert(C::kof(i, c));
        if (ks.size() != (size_t)NB * DK || *ks.rbegin() >= NB * C::KH) fail("Khat swizzle", t.tag);
        std::set<int> fs;
        for (int c = 0; c < DK; ++c) fs.insert(f_pos(c));
        if (fs.size() != (size_t)DK || *fs.rbegin() >= DK) fail("F column order", t.tag);
    }

    void run(int n_log, bool wc, int L) {
        const int E = 16 / in_bytes, KC = DK / E, VC = ROWS / E;
        const int KN = (NB * KC + nthr - 1) / nthr, VN = (NB * ROWS / E + nthr - 1) / nthr;
        // the tile fetch
        if (Q8) {
            for (int u = 0; u < ROWS * (DK / 16); ++u) {
                const int r = u / (DK / 16), ch = u % (DK / 16);
                t.acc("raw", (long)r * DK + ch * 16, 16, 16, "cp.async codes");
            }
            for (int tid = 0; tid < ROWS / 4; ++tid) f("scl", 4 * tid, 4, 16, "cp.async scales");
            const int WPT = ROWS * DK / 4 / nthr;
            for (int tid = 0; tid < nthr; ++tid)
                for (int i = 0; i < WPT; ++i) {
                    const int u = tid + i * nthr, r = u / (DK / 4), c4 = (u % (DK / 4)) * 4;
                    t.acc("raw", 4L * u, 4, 4, "code word");
                    tile(r, c4, 4, "widened codes");
                    f("scl", r, 1, 4, "scale");
                }
        } else {
            const int CE = TL::CE;
            for (int u = 0; u < ROWS * (DK / CE); ++u) {
                const int r = u / (DK / CE), ch = u % (DK / CE);
                tile(r, ch * CE, CE, "cp.async tile");
            }
        }
        // the pool walk's words
        for (int i = 0; i < 5; ++i) f("xw", i, 1, 4, "walk word");
        const int NTOT = n_log + (wc ? 1 : 0);
        for (int b0 = 0; b0 < NTOT; b0 += NB) {
            const int nb = NTOT - b0 < NB ? NTOT - b0 : NB;
            const int nl = n_log - b0 < nb ? n_log - b0 : nb;
            const bool cur = wc && nl < nb;
            for (int tid = 0; tid < nthr; ++tid) {
                // staging
                for (int u = 0; u < KN; ++u) {
                    const int c = tid + u * nthr, r = c / KC, col = (c % KC) * E;
                    if (c >= NB * KC) continue;
                    for (int e = 0; e < E; e += 4) {
                        for (int x = 0; x < 4; ++x)
                            if (C::kof(r, col + e + x) != C::kof(r, col + e) + x)
                                fail("Khat piece not contiguous", t.tag);
                        f("kh", C::kof(r, col + e), 4, 16, "put keys");
                        if (chan) f("ff", (long)r * C::WS + col + e, 4, 16, "put decays");
                    }
                }
                for (int u = 0; u < VN; ++u) {
                    const int c = tid + u * nthr, r = c / VC, col = (c % VC) * E;
                    if (c < NB * VC)
                        for (int e = 0; e < E; e += 4) f("sv", (long)r * C::VS + col + e, 4, 16, "put values");
                }
                if (tid < NB) {
                    f("sb", tid, 1, 4, "beta");
                    if (!chan) f("fa", tid, 1, 4, "head decay");
                }
                if (tid < KC) f("sq", (long)tid * E, E, 16, "put q");
                for (int u = 0; u < (NB * NB + nthr - 1) / nthr; ++u) {
                    const int idx = tid + u * nthr, ci = idx / NB, cj = idx % NB;
                    if (idx >= NB * NB) continue;
                    if (delta && cj <= ci && ci < nl && (b0 + ci >= L || b0 + cj >= L))
                        fail("X read outside the head's block", t.tag);
                    if (!(cur && ci == nl)) f("sx", (long)ci * C::XS + cj, 1, 4, "X");
                }
                // key side, one channel per thread
                for (int c = tid; c < DK; c += nthr)
                    for (int i = 0; i < NB; ++i) {
                        if (chan) f("ff", (long)i * C::WS + c, 1, 4, "decay read");
                        else f("fa", i, 1, 4, "head decay read");
                        f("kh", C::kof(i, c), 1, 4, "Khat");
                        f("ff", (long)i * C::WS + f_pos(c), 1, 4, "F");
                        f("gn", c, 1, 4, "gamma");
                    }
            }
            for (int warp = 0; warp < 4; ++warp) {
                const int tr = 16 * warp;
                for (int lane = 0; lane < 32; ++lane) {
                    const int g = lane >> 2, tq = lane & 3, rg = tr + g;
                    if (delta && cur) {  // the fused entry's C and X rows
                        for (int e = 0; e < C::CW; ++e) f("ff", (long)nl * C::WS + e * 32 + lane, 1, 4, "F_nl");
                        for (int j = 0; j < NB; ++j)
                            for (int e = 0; e < C::CW; ++e) f("ff", (long)j * C::WS + e * 32 + lane, 1, 4, "F_j");
                        for (int m = 0; m < NB; ++m)
                            if (lane <= m && m < nl) f("sx", (long)m * C::XS + lane, 1, 4, "X for the fused row");
                        f("sb", nl, 1, 4, "fused beta");
                        if (lane < NB) f("sxw", (long)warp * C::XS + lane, 1, 4, "fused X row");
                    }
                    if (delta)
                        for (int j = 0; j < DK / 16; ++j) {
                            const int c = 16 * j + 4 * tq;
                            tile(rg, c, 4, "G A");
                            tile(rg + 8, c, 4, "G A");
                            for (int nt = 0; nt < NT; ++nt) {
                                for (int x = 0; x < 4; ++x)
                                    if (C::kof(8 * nt + g, c + x) != C::kof(8 * nt + g, c) + x)
                                        fail("G's B piece not contiguous", t.tag);
                                f("kh", C::kof(8 * nt + g, c), 4, 16, "G B");
                            }
                        }
                    for (int nt = 0; nt < NT; ++nt) {
                        if (delta) {  // V - G in the accumulator layout
                            const int i0 = 8 * nt + 2 * tq;
                            for (int ii = i0; ii <= i0 + 1; ++ii) {
                                f("sv", (long)ii * C::VS + rg, 1, 4, "value");
                                f("sv", (long)ii * C::VS + rg + 8, 1, 4, "value");
                            }
                        } else {  // delta = V in the operand layout
                            const int i0 = 8 * nt + tq;
                            for (int ii : {i0, i0 + 4}) {
                                f("sv", (long)ii * C::VS + rg, 1, 4, "value (operand)");
                                f("sv", (long)ii * C::VS + rg + 8, 1, 4, "value (operand)");
                            }
                        }
                    }
                    if (delta)
                        for (int mt = 0; mt < NT; ++mt) {
                            const int xr = 8 * mt + g;
                            const bool own = cur && xr == nl;
                            for (int kt = 0; kt <= mt; ++kt)
                                for (int d = 0; d <= 4; d += 4) {
                                    if (own) f("sxw", (long)warp * C::XS + 8 * kt + tq + d, 1, 4, "X row (fused)");
                                    else f("sx", (long)xr * C::XS + 8 * kt + tq + d, 1, 4, "X row");
                                }
                        }
                    for (int j = 0; j < DK / 16; ++j) {
                        for (int h = 0; h < 2; ++h)
                            for (int nt = 0; nt < NT; ++nt) {
                                const long p = (long)(8 * nt + tq) * C::WS + 16 * j + 8 * h + g;
                                f("ff", p, 1, 4, "update B");
                                f("ff", p + 4 * C::WS, 1, 4, "update B");
                            }
                        const int col = 16 * j + 4 * tq;
                        tile(tr + g, col, 4, "write-back");
                        tile(tr + g + 8, col, 4, "write-back");
                        f("gn", col, 4, 16, "gamma piece");
                        f("sq", col, 4, 16, "q piece");
                    }
                    if (Q8) {
                        f("wsc", warp * 16 + g, 1, 4, "row scale");
                        f("wsc", warp * 16 + g + 8, 1, 4, "row scale");
                        const int CPR = DK / 16;
                        for (int i = lane; i < 16 * CPR; i += 32) {
                            const int rl = i / CPR, c0 = (i % CPR) * 16;
                            f("wsc", warp * 16 + rl, 1, 4, "pack scale");
                            for (int qd = 0; qd < 4; ++qd) tile(tr + rl, c0 + 4 * qd, 4, "pack");
                        }
                    }
                }
            }
        }
    }
};

template <int SB, bool Q8, int DK, int NB>
int merge_cases() {
    int cases = 0;
    for (int chan = 0; chan < 2; ++chan)
        for (int delta = 0; delta < 2; ++delta)
            for (int ib : {2, 4}) {
                if (!delta && !chan) continue;  // RWKV6 has channel decay
                MergeReplay<SB, Q8, DK, NB> rp(chan, delta, ib);
                rp.layout();
                for (int L : {1, 8, 16, 17, 64})  // one or several entry blocks, a ragged last block
                    for (int n_log = 0; n_log <= L; ++n_log)
                        for (int wc = 0; wc < 2; ++wc) {
                            // every fill up to 17; at 64 the block edges (1, 8 and 16 entries,
                            // the fused entry alone in or at the end of a block)
                            if (L == 64 && !(n_log <= 1 || n_log % 16 <= 1 || n_log % 16 == 15 || n_log >= 62))
                                continue;
                            if (wc && n_log == L) continue;  // a fused read needs a free slot
                            if (!wc && n_log == 0) continue;
                            rp.run(n_log, wc, L);
                            ++cases;
                        }
            }
    return cases;
}

// ---------------------------------------------------------------- prep (deferred_read.cu)

template <int IB, int DK, int DV, int EMAX, bool CHAN>
struct PrepReplay {
    using P = PrepSmem<IB, DK, EMAX, CHAN>;
    static constexpr int CW = DK / 32, E = 16 / IB, CH = EMAX < 32 ? EMAX : 32, SBN = (EMAX + 31) / 32, XB = 8;
    bool delta;
    int WARPS;  // staging areas laid out from offset 0: the prep kernel's warps, or the fused kernel's prep warps
    Table t;
    PrepReplay(bool de, int warps = prep_warps(EMAX), const char *kernel = "prep") : delta(de), WARPS(warps) {
        char b[96];
        std::snprintf(b, sizeof b, "%s in%d dk%d dv%d emax%d %s %s", kernel, IB, DK, DV, EMAX,
                      CHAN ? "chan" : "head", de ? "delta" : "rwkv6");
        t.tag = b;
        for (int w = 0; w < WARPS; ++w) {
            const std::string p = "w" + std::to_string(w) + ".";
            const size_t base = (size_t)w * P::BYTES;
            t.add(p + "sk", base + P::K_OFF, (size_t)EMAX * P::ROWB);
            if (CHAN) t.add(p + "sa", base + P::A_OFF, (size_t)EMAX * P::ROWB);
            const size_t F = base + P::F_OFF;
            t.add(p + "as", F + P::AS * 4, EMAX * 4);
            t.add(p + "beta", F + P::BETA * 4, EMAX * 4);
            t.add(p + "d", F + P::D * 4, EMAX * 4);
            t.add(p + "cn", F + P::CN * 4, EMAX * 4);
            t.add(p + "s", F + P::S * 4, EMAX * 4);
            t.add(p + "xrow", F + P::XROW * 4, (size_t)EMAX * EMAX * 4);
        }
    }
    void f(const std::string &reg, long idx, int n, size_t align, const char *what) {
        t.acc(reg, idx * 4, (size_t)n * 4, align, what);
    }
    void layout() {
        const size_t smem = (size_t)WARPS * P::BYTES;
        if (smem > SMEM_LIMIT) fail("prep request above 227 KiB", t.tag);
        if (P::F_OFF % 16) fail("float arrays not 16-byte aligned", t.tag);
        if (P::BYTES % 16) fail("warp areas not 16-byte aligned", t.tag);
        t.no_overlap(smem);
    }
    void run(int n, int L) {
        if (n >= L || L > EMAX) fail("fill beyond the staging capacity", t.tag);
        for (int w = 0; w < WARPS; ++w) {
            const std::string p = "w" + std::to_string(w) + ".";
            for (int lane = 0; lane < 32; ++lane) {
                const int c0 = lane * CW;
                // staging of keys and decays of entries 0..n
                for (int u = lane; u < (n + 1) * (DK / E); u += 32) {
                    const int e = u / (DK / E), col = (u % (DK / E)) * E;
                    t.acc(p + "sk", ((long)e * DK + col) * IB, 16, 16, "cp.async key");
                    if (CHAN) t.acc(p + "sa", ((long)e * DK + col) * IB, 16, 16, "cp.async decay");
                }
                for (int i = 0; i < SBN; ++i) {
                    const int e = lane + 32 * i;
                    if (e <= n) {
                        if (delta) f(p + "beta", e, 1, 4, "beta");
                        if (!CHAN) f(p + "as", e, 1, 4, "head decay");
                    }
                }
                for (int base = 0; base == 0 || (delta && base < n * EMAX); base += 32 * XB)
                    for (int i = 0; i < XB; ++i) {
                        const int u = base + i * 32 + lane, j = u / EMAX, e = u % EMAX;
                        if (delta && u < n * EMAX && e <= j) {
                            if (j >= L) fail("X read outside the head's block", t.tag);
                            f(p + "xrow", (long)j * EMAX + e, 1, 4, "X rows of the log");
                        }
                    }
                // dots, newest first
                const size_t vw = (size_t)CW * IB;  // one lane's key slice
                t.acc(p + "sk", ((long)n * DK + c0) * IB, vw, vw, "the new key");
                for (int top = n; top >= 0; top -= CH) {
                    for (int jj = 0; jj < CH; ++jj) {
                        const int e = top - jj;
                        if (e < 0) continue;
                        t.acc(p + "sk", ((long)e * DK + c0) * IB, vw, vw, "key slice");
                        if (CHAN) t.acc(p + "sa", ((long)e * DK + c0) * IB, vw, vw, "decay slice");
                        else f(p + "as", e, 1, 4, "head decay");
                    }
                    const int shift = CH == 32 ? 0 : CH == 16 ? 1 : CH == 8 ? 2 : 3;
                    const int e = top - (lane >> shift);
                    if ((lane & ((1 << shift) - 1)) == 0 && e >= 0) {
                        f(p + "d", e, 1, 4, "d");
                        f(p + "cn", e, 1, 4, "C row");
                    }
                }
                // X row n, then s
                for (int j = lane; delta && j <= n; j += 32) {
                    for (int m = j; m < n; ++m) {
                        f(p + "cn", m, 1, 4, "C read");
                        f(p + "xrow", (long)m * EMAX + j, 1, 4, "X read");
                    }
                    f(p + "xrow", (long)n * EMAX + j, 1, 4, "X row n");
                }
                if (delta) f(p + "beta", n, 1, 4, "beta_n");
                for (int e = lane; e <= n; e += 32) {
                    if (delta)
                        for (int i = e; i <= n; ++i) {
                            f(p + "xrow", (long)i * EMAX + e, 1, 4, "X column");
                            f(p + "d", i, 1, 4, "d read");
                        }
                    else
                        f(p + "d", e, 1, 4, "d read");
                    f(p + "s", e, 1, 4, "s");
                }
                for (int e = 0; e <= n; ++e) {
                    t.acc(p + "sk", ((long)e * DK + c0) * IB, vw, vw, "key slice (x_0)");
                    f(p + "s", e, 1, 4, "s read");
                }
            }
        }
    }
};

template <int IB, int DK, int DV, int EMAX, bool CHAN>
int prep_cases() {
    int cases = 0;
    for (int delta = 0; delta < 2; ++delta) {
        if (!delta && !CHAN) continue;
        PrepReplay<IB, DK, DV, EMAX, CHAN> rp(delta);
        rp.layout();
        for (int L : {1, 2, 5, 15, 16, 17, 31, 32, 33, 63, 64}) {  // every staging capacity, at and beside its edges
            if (prep_emax(L) != EMAX) continue;
            for (int n = 0; n < L; ++n) {
                rp.run(n, L);
                ++cases;
            }
        }
    }
    return cases;
}

template <int IB, int DK, int DV>
int prep_all() {
    return prep_cases<IB, DK, DV, 16, false>() + prep_cases<IB, DK, DV, 16, true>() +
           prep_cases<IB, DK, DV, 32, false>() + prep_cases<IB, DK, DV, 32, true>() +
           prep_cases<IB, DK, DV, 64, false>() + prep_cases<IB, DK, DV, 64, true>();
}

// ---------------------------------------------------------------- fused append-read (deferred_read.cu)

template <int IB, int SB, int DK, int DV, bool CHAN>
struct FusedReplay {
    using LY = fused::Layout<IB, SB, DK, DV, CHAN>;
    static constexpr int VEC = 16 / SB, G = DK / VEC, RPW = 32 / G, R = 8, CW = DK / 32, RV = DV / 32;
    PrepReplay<IB, DK, DV, fused::EMAX, CHAN> rp;
    FusedReplay(bool de) : rp(de, LY::NP, "fused") {
        Table &t = rp.t;
        for (int s = 0; s < LY::NSLOT; ++s) t.add("slot" + std::to_string(s), LY::slot(s), LY::SLOT_BYTES);
        for (int d = 0; d < fused::ND; ++d)
            for (int b = 0; b < fused::NBUF; ++b)
                t.add("ring" + std::to_string(d) + "." + std::to_string(b), LY::ring(d, b), fused::UNIT_BYTES);
        t.add("full", LY::BAR_FULL, 8 * LY::NSLOT);
        t.add("free", LY::BAR_FREE, 8 * LY::NSLOT);
        t.add("ringbar", LY::BAR_RING, 8 * fused::ND * fused::NBUF);
        t.add("abort", LY::ABORT_OFF, 4);
    }
    void layout() {
        Table &t = rp.t;
        if (LY::UNIT_ROWS != R * RPW) fail("a bulk copy is not one decode unit", t.tag);
        if (DV % LY::UNIT_ROWS) fail("units do not tile a head", t.tag);
        if (LY::NP < 1 || LY::NSLOT % LY::NP) fail("each slot must belong to one prep warp", t.tag);
        if ((size_t)LY::REQUEST > SMEM_LIMIT) fail("fused request above 227 KiB", t.tag);
        if (LY::BYTES + 127 > LY::REQUEST) fail("no room to align the base to 128 bytes", t.tag);
        if (LY::RING_OFF % 16 || fused::UNIT_BYTES % 16) fail("bulk-copy buffers not 16-byte aligned", t.tag);
        if (LY::BAR_OFF % 8) fail("mbarriers not 8-byte aligned", t.tag);
        t.no_overlap(LY::BYTES);
    }
    // the decode side, the same at every fill: (x_0, w) stored into each slot
    // and read back by a decode unit, and every buffer read as a unit's tile
    void decode() {
        Table &t = rp.t;
        for (int s = 0; s < LY::NSLOT; ++s) {
            const std::string sl = "slot" + std::to_string(s);
            for (int lane = 0; lane < 32; ++lane) {
                for (int c = 0; c < CW; ++c) t.acc(sl, (long)(lane * CW + c) * 4, 4, 4, "x_0 store");
                for (int r = 0; r < RV; ++r) t.acc(sl, (long)(DK + lane * RV + r) * 4, 4, 4, "w store");
                const int sub = lane / G, col = (lane % G) * VEC;
                for (int e = 0; e < VEC; ++e) t.acc(sl, (long)(col + e) * 4, 4, 4, "x_0 read");
                for (int j = 0; j < LY::UPH; ++j)
                    for (int r = 0; r < R; ++r)
                        t.acc(sl, (long)(DK + j * LY::UNIT_ROWS + r * RPW + sub) * 4, 4, 4, "w read");
            }
        }
        for (int d = 0; d < fused::ND; ++d)
            for (int b = 0; b < fused::NBUF; ++b) {
                const std::string rg = "ring" + std::to_string(d) + "." + std::to_string(b);
                for (int lane = 0; lane < 32; ++lane) {
                    const int sub = lane / G, col = (lane % G) * VEC;
                    for (int r = 0; r < R; ++r) t.acc(rg, ((long)(r * RPW + sub) * DK + col) * SB, 16, 16, "base slice");
                }
            }
    }
    // one fill n: ReplayPrep of every prep warp, and the base copies of
    // `heads` heads checked against the base's extent
    void run(int n, int L, long long heads) {
        Table &t = rp.t;
        rp.run(n, L);
        // bulk-copy sources: every unit of every head inside the base, 16-byte aligned
        const unsigned long long total = (unsigned long long)heads * DV * DK * SB;
        for (long long h = 0; h < heads; ++h)
            for (int j = 0; j < LY::UPH; ++j) {
                const unsigned long long off = ((unsigned long long)h * DV + (unsigned long long)j * LY::UNIT_ROWS) * DK * SB;
                if (off + fused::UNIT_BYTES > total || off % 16) fail("base copy outside the base", t.tag);
            }
        if (shrink.count("unit")) {  // a base believed one row shorter per head
            const unsigned long long short_total = total - (unsigned long long)heads * DK * SB;
            const unsigned long long last = ((unsigned long long)(heads - 1) * DV + (DV - LY::UNIT_ROWS)) * DK * SB;
            if (last + fused::UNIT_BYTES > short_total) fail("out of region", t.tag + " base copy");
        }
    }
};

template <int IB, int SB, int DK, int DV, bool CHAN>
int fused_cases() {
    int cases = 0;
    for (int delta = 0; delta < 2; ++delta) {
        if (!delta && !CHAN) continue;
        FusedReplay<IB, SB, DK, DV, CHAN> fr(delta);
        fr.layout();
        fr.decode();
        for (int L : {1, 2, 5, 15, 16}) {
            for (int n = 0; n < L; ++n) {
                fr.run(n, L, 3 + 7 * n);
                ++cases;
            }
        }
    }
    return cases;
}

template <int IB, int SB>
int fused_all() {
    int c = 0;
    c += fused_cases<IB, SB, 64, 64, false>() + fused_cases<IB, SB, 64, 64, true>();
    c += fused_cases<IB, SB, 64, 128, false>() + fused_cases<IB, SB, 64, 128, true>();
    c += fused_cases<IB, SB, 64, 256, false>() + fused_cases<IB, SB, 64, 256, true>();
    c += fused_cases<IB, SB, 128, 64, false>() + fused_cases<IB, SB, 128, 64, true>();
    c += fused_cases<IB, SB, 128, 128, false>() + fused_cases<IB, SB, 128, 128, true>();
    c += fused_cases<IB, SB, 128, 256, false>() + fused_cases<IB, SB, 128, 256, true>();
    return c;
}

}  // namespace

int main(int argc, char **argv) {
    bool do_merge = true, do_prep = true, do_fused = true;
    for (int i = 1; i < argc; ++i) {
        if (std::strcmp(argv[i], "shrink") == 0 && i + 2 < argc) {
            shrink[argv[i + 1]] = std::atol(argv[i + 2]);
            i += 2;
        } else if (std::strcmp(argv[i], "merge") == 0) {
            do_prep = do_fused = false;
        } else if (std::strcmp(argv[i], "prep") == 0) {
            do_merge = do_fused = false;
        } else if (std::strcmp(argv[i], "fused") == 0) {
            do_merge = do_prep = false;
        }
    }
    int cases = 0;
    // merge: state fp32, bf16, int8 (widened into a float tile); d_k 64, 128; 8 or 16 entries per block
    if (do_merge) {
        cases += merge_cases<4, false, 64, 8>() + merge_cases<4, false, 64, 16>();
        cases += merge_cases<4, false, 128, 8>() + merge_cases<4, false, 128, 16>();
        cases += merge_cases<2, false, 64, 8>() + merge_cases<2, false, 64, 16>();
        cases += merge_cases<2, false, 128, 8>() + merge_cases<2, false, 128, 16>();
        cases += merge_cases<1, true, 64, 8>() + merge_cases<1, true, 64, 16>();
        cases += merge_cases<1, true, 128, 8>() + merge_cases<1, true, 128, 16>();
    }
    // prep: bf16 and fp32 inputs, d_k 64 and 128, d_v 64 .. 256
    if (do_prep) {
        cases += prep_all<2, 64, 64>() + prep_all<2, 128, 128>() + prep_all<2, 128, 256>();
        cases += prep_all<4, 64, 64>() + prep_all<4, 128, 128>() + prep_all<4, 128, 256>();
    }
    // fused append-read: bf16 and fp32 inputs, fp32 and bf16 bases, every d_k x d_v
    if (do_fused) cases += fused_all<2, 4>() + fused_all<2, 2>() + fused_all<4, 4>() + fused_all<4, 2>();
    std::printf("%d cases, %d failures\n", cases, failures);
    return failures ? 1 : 0;
}
