// Host-side check of the tensor-core epilogue's storage plan, using the
// library's own per-leaf operation codes (leaf_ops / seq_leaf_ops /
// encode_leaf_ops from device_common.cuh).  For every leaf count n it replays
// the epilogue's decisions on symbolic values: a pending single leaf stays in
// its TMEM accumulator and must be taken by the very next leaf; a pending
// 2-leaf value sits in the one TMEM slot, a 3-4-leaf value in the one
// shared-memory slot; values of >= 5 leaves go to the L2 stack, popped from
// its top.  The replay must rebuild exactly the halving tree (or the
// left-to-right chain), keep at most one value per on-chip class, push only
// values of the class's size, and never hold more L2 values than the host's
// bound (max_big_pending, restated below).  check_wide replays the plan of
// the 192-column tile, which keeps the 2-leaf value in registers and may park
// a single leaf in the 3-4 leaf slot.
#include <cstdio>
#include <string>
#include <vector>

#include "device_common.cuh"

using namespace tbik;

static std::string tree_expr(int lo, int n) {
    if (n == 1) return "L" + std::to_string(lo);
    const int h = (n + 1) / 2;
    return "(" + tree_expr(lo, h) + "+" + tree_expr(lo + h, n - h) + ")";
}
static std::string seq_expr(int n) {
    std::string e = "L0";
    for (int j = 1; j < n; ++j) e = "(" + e + "+L" + std::to_string(j) + ")";
    return e;
}
static int bound(int n) {  // pending left subtrees of >= 5 leaves
    if (n <= 1) return 0;
    const int h = (n + 1) / 2;
    const int l = bound(h), r = bound(n - h) + (h >= 5 ? 1 : 0);
    return l > r ? l : r;
}
struct Val {
    std::string e;
    int leaves;
};

static int check(int n, bool seq) {
    Val single{"", 0}, slot2{"", 0}, slot34{"", 0};
    bool have_single = false, have2 = false, have34 = false;
    std::vector<Val> l2;
    for (int j = 0; j < n; ++j) {
        const uint32_t code = encode_leaf_ops(seq ? seq_leaf_ops(n, j) : leaf_ops(n, j));
        const bool p1 = code & 1, p2 = (code >> 1) & 1, pm = (code >> 2) & 1;
        const int nb = (code >> 3) & 31;
        const int cls = (code >> 8) & 3;
        const bool fin = (code >> 10) & 1;
        Val v{"L" + std::to_string(j), 1};
        if (!fin && cls == 0) {
            if (have_single) return 1;  // a single left waiting
            single = v;
            have_single = true;
            continue;
        }
        if (have_single && !p1) return 2;  // a pending single must be taken by the next leaf
        // pops, smallest first: the single, the 2-leaf slot, the 3-4 slot, the L2 stack from its top
        if (p1) {
            if (!have_single) return 3;
            v = {"(" + single.e + "+" + v.e + ")", single.leaves + v.leaves};
            have_single = false;
        }
        if (p2) {
            if (!have2) return 4;
            v = {"(" + slot2.e + "+" + v.e + ")", slot2.leaves + v.leaves};
            have2 = false;
        }
        if (pm) {
            if (!have34) return 5;
            v = {"(" + slot34.e + "+" + v.e + ")", slot34.leaves + v.leaves};
            have34 = false;
        }
        for (int i = 0; i < nb; ++i) {
            if (l2.empty()) return 6;
            v = {"(" + l2.back().e + "+" + v.e + ")", l2.back().leaves + v.leaves};
            l2.pop_back();
        }
        if (fin) {
            if (j != n - 1 || have_single || have2 || have34 || !l2.empty()) return 7;
            if (v.e != (seq ? seq_expr(n) : tree_expr(0, n))) return 8;
            if (v.leaves != n) return 9;
            return 0;
        }
        const int want = v.leaves == 1 ? 0 : (v.leaves == 2 ? 1 : (v.leaves <= 4 ? 2 : 3));
        if (cls != want) return 10;
        if (cls == 1) {
            if (have2) return 11;
            slot2 = v;
            have2 = true;
        } else if (cls == 2) {
            if (have34) return 12;
            slot34 = v;
            have34 = true;
        } else {
            l2.push_back(v);
        }
    }
    return 13;  // no final leaf
}

// The storage plan of the 192-column tile (two TMEM accumulators): a pending
// 2-leaf value lives in the epilogue's registers R.  A single leaf goes to R
// when R is free (bit 11 clear: no 2-leaf value pending); otherwise to the 3-4
// leaf slot when that is free (bit 12 clear), else it stays in its
// accumulator.  The leaf that pops a single held outside R must pop the 2-leaf
// value of R in the same step.  Every popping leaf leaves its working value in
// R, so R must be free or consumed; a pushed 2-leaf value stays there.
static int check_wide(int n, bool seq) {
    Val R{"", 0}, tsingle{"", 0}, slot{"", 0};
    bool haveR = false, have_ts = false, have_slot = false;
    std::vector<Val> l2;
    for (int j = 0; j < n; ++j) {
        const uint32_t code = encode_leaf_ops(seq ? seq_leaf_ops(n, j) : leaf_ops(n, j));
        const bool p1 = code & 1, p2 = (code >> 1) & 1, pm = (code >> 2) & 1;
        const int nb = (code >> 3) & 31;
        const int cls = (code >> 8) & 3;
        const bool fin = (code >> 10) & 1, c2p = (code >> 11) & 1, mp = (code >> 12) & 1;
        if (c2p != (haveR && R.leaves == 2)) return 21;  // bit 11 states what R holds
        if (mp != (have_slot && slot.leaves >= 3)) return 36;  // bit 12 states what the slot holds
        if (have_ts && !p1) return 22;  // a TMEM single is taken by the next leaf
        if (have_slot && slot.leaves == 1 && !p1) return 37;  // so is a single in the slot
        Val v{"L" + std::to_string(j), 1};
        if (!fin && cls == 0) {  // a single leaf
            if (!c2p) {
                if (haveR) return 24;
                R = v;
                haveR = true;
            } else if (!mp) {
                if (have_slot) return 38;
                slot = v;
                have_slot = true;
            } else {
                if (have_ts) return 23;
                tsingle = v;
                have_ts = true;
            }
            continue;
        }
        if (p1 && c2p) {  // single (TMEM when bit 12, else the slot) + leaf, then the 2-leaf value of R
            if (!haveR || R.leaves != 2 || !p2) return 25;
            if (mp) {
                if (!have_ts) return 39;
                v = {"(" + tsingle.e + "+" + v.e + ")", 2};
                have_ts = false;
            } else {
                if (!have_slot || slot.leaves != 1) return 40;
                v = {"(" + slot.e + "+" + v.e + ")", 2};
                have_slot = false;
            }
            v = {"(" + R.e + "+" + v.e + ")", R.leaves + 2};
            haveR = false;
        } else if (p1) {  // the single held in R
            if (have_ts || !haveR || R.leaves != 1 || p2) return 26;
            v = {"(" + R.e + "+" + v.e + ")", 2};
            haveR = false;
        } else if (p2) {  // the 2-leaf value of R
            if (!haveR || R.leaves != 2) return 27;
            v = {"(" + R.e + "+" + v.e + ")", 3};
            haveR = false;
        } else if (haveR) {
            return 28;  // the working value would overwrite a pending value
        }
        if (pm) {
            if (!have_slot || slot.leaves < 3) return 29;
            v = {"(" + slot.e + "+" + v.e + ")", slot.leaves + v.leaves};
            have_slot = false;
        }
        for (int i = 0; i < nb; ++i) {
            if (l2.empty()) return 30;
            v = {"(" + l2.back().e + "+" + v.e + ")", l2.back().leaves + v.leaves};
            l2.pop_back();
        }
        if (fin) {
            if (j != n - 1 || haveR || have_ts || have_slot || !l2.empty()) return 31;
            if (v.e != (seq ? seq_expr(n) : tree_expr(0, n))) return 32;
            return 0;
        }
        const int want = v.leaves == 1 ? 0 : (v.leaves == 2 ? 1 : (v.leaves <= 4 ? 2 : 3));
        if (cls != want) return 33;
        if (cls == 1) {
            R = v;
            haveR = true;
        } else if (cls == 2) {
            if (have_slot) return 34;
            slot = v;
            have_slot = true;
        } else {
            l2.push_back(v);
        }
    }
    return 35;
}

int main() {
    int bad = 0;
    for (int n = 1; n <= 1100 && bad < 10; ++n) {
        for (int seq = 0; seq < 2; ++seq) {
            const int w = check_wide(n, seq != 0);
            if (w) {
                std::printf("%s n=%d (192-column plan): rule %d violated\n", seq ? "chain" : "tree", n, w);
                ++bad;
            }
        }
        const int r = check(n, false);
        if (r) {
            std::printf("tree n=%d: rule %d violated\n", n, r);
            ++bad;
        }
        const int q = check(n, true);
        if (q) {
            std::printf("chain n=%d: rule %d violated\n", n, q);
            ++bad;
        }
    }
    // the host's L2 bound is never exceeded and is reached (it is tight)
    for (int n = 1; n <= 1100 && bad < 10; ++n) {
        size_t depth = 0, cur = 0;
        for (int j = 0; j < n; ++j) {
            const uint32_t code = encode_leaf_ops(leaf_ops(n, j));
            const int nb = (code >> 3) & 31;
            const int cls = (code >> 8) & 3;
            const bool fin = (code >> 10) & 1;
            if (!fin && cls == 0) continue;
            cur -= nb;
            if (!fin && cls == 3) ++cur;
            if (cur > depth) depth = cur;
        }
        if ((int)depth != bound(n)) {
            std::printf("n=%d: L2 depth %zu, host bound %d\n", n, depth, bound(n));
            ++bad;
        }
    }
    if (!bad) std::printf("tree walk ok\n");
    return bad ? 1 : 0;
}
