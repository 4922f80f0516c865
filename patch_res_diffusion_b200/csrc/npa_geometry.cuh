// npa_geometry.cuh - the work decomposition of patch-restricted attention,
// shared by the host launcher and the kernel.
//
// Both geometries are one rectangle scheme: query patches of Ph x Pw tokens
// whose key/value window is the patch grown by mh rows and mw columns and
// clipped to the H x W grid.
//   * NPA (ScaleDiff summary, "Approach"): Ph = Pw = patch, mh = mw = margin.
//   * PCPP (PCPP review, "What carries the argument"): strips of s = H/n rows
//     spanning the grid, Ph = s, Pw = W, mh = r = ceil(p*s), mw = 0. The grown
//     window of strip i is rows [i*s - r, (i+1)*s + r) clipped, all columns:
//     the strip plus the r adjacent rows of each neighbouring strip.
//
// Work unit = (batch*head, patch, group of tiles_per_unit 128-row query
// tiles); a persistent CTA walks the units blockIdx.x, blockIdx.x + gridDim.x,
// ... A query tile is a box of qr patch rows x qc patch columns (qr*qc <=
// 128); a key/value block is a box of kr rows x kc columns (kr*kc = kb = 128
// keys) inside the window, followed by ceil(G/kb) blocks of global
// tokens. Every quantity is recomputed from the unit index with integer
// arithmetic; the only table is the host-built patch order.
#pragma once

#include <cstdint>
#include <cuda.h>

namespace npa {

// Up to this many patches are visited largest window first; beyond it, in
// natural order.
constexpr int kMaxPatchOrder = 256;
constexpr int kMaxCostClasses = 16;
// A host-built per-CTA unit list covers launches of up to this many units and
// CTAs (it travels in the kernel parameters); larger launches run the units
// round robin.
constexpr int kMaxSchedUnits = 7168;
constexpr int kMaxSchedCtas = 160;
// Scheduling cost of a unit beyond its key blocks (query load, pipeline
// refill, epilogue), in key blocks.
constexpr int kUnitOverheadBlocks = 2;

struct FwdParams {
    CUtensorMap tm_q;   // 4D {d, W, H, B*heads}, box {64, qc, qr, 1}, 128B swizzle
    CUtensorMap tm_k;   // 4D, box {64, kc, kr, 1}
    CUtensorMap tm_v;   // 4D, box {64, kc, kr, 1}
    CUtensorMap tm_gk;  // 3D {d, G, B*heads}, box {64, kb, 1} (unused when G == 0)
    CUtensorMap tm_gv;
    CUtensorMap tm_ks;  // previous step's K / V for the borrowed rows (two_source only)
    CUtensorMap tm_vs;
    CUtensorMap tm_gq;  // global-token queries: 3D {d, G, B*heads}, box {64, 128, 1}
    void *o;            // bf16 [B, heads, H*W, d]
    int H, W, G;
    int Ph, Pw, mh, mw;
    int nPh, nPw;                    // patches along rows / columns
    int qc, qr, tiles_c, tiles_r;    // query tile box and tiles per patch
    int kb;                          // keys per key block (128)
    int kc_log2, kr;                 // key block box: (1 << kc_log2) columns x kr rows
    int tiles_per_unit;              // query tiles per work unit (2)
    int n_qblocks;                   // query-tile groups per patch
    float scale_log2;                // log2(e) / sqrt(d)
    unsigned long long wait_limit_ns;
    int BH;                          // batch * heads
    int n_units;                     // work units in execution order
    int two_source;                  // 1: rows outside the patch come from tm_ks / tm_vs
    int patch_begin, patch_count;    // patches computed (natural order when n_perm == 0)
    int n_splits;                    // global-token queries: key-range splits per query tile group
    int gq_tiles;                    // global-token queries: ceil(G / 128)
    float *o_part;                   // splits > 1: [n_splits][B*heads][G][d] unnormalised O
    float *ml;                       // splits > 1: [n_splits][B*heads][G][2] reference max, row sum
    int n_perm;                      // entries of patch_order (0: natural order)
    unsigned short patch_order[kMaxPatchOrder];  // patches by decreasing window area
    int n_cls;                       // runs of equal cost in patch_order (0: none recorded)
    int cls_rank0[kMaxCostClasses + 1];  // first patch_order index of each run; [n_cls] = n_perm
    // Overlapping-window mode (MultiDiffusion-style comparator): the queries
    // of a unit are its whole window, and the normalised float32 output of
    // every window is written to md_part, window-major: window (pi, pj)
    // starts at row md_axis_offset(pi) of a [md_rows, md_tw] token plane per
    // batch*head and column md_axis_offset(pj) within it.
    int md;
    int md_rows, md_tw;              // sum of window heights / widths over the patch rows / columns
    float *md_part;                  // [B*heads][md_rows][md_tw][d]
    // Per-CTA unit lists (n_sched > 0): CTA c runs units sched[cta_first[c]],
    // ..., sched[cta_first[c + 1] - 1] in that order. n_sched == 0: CTA c
    // runs units c, c + gridDim.x, c + 2 gridDim.x, ...
    int debug_stall;  // bounds-checking build: CTA 0 withholds one P_full arrival (abort-path test)
    int n_sched;
    unsigned short cta_first[kMaxSchedCtas + 1];
    unsigned short sched[kMaxSchedUnits];
};

// The window's rows are walked as three segments: [seg[0], seg[1]) and
// [seg[2], seg[3]) are read from the previous step's keys/values (two-source
// PCPP: the borrowed neighbour rows) and [seg[1], seg[2]) from the current
// ones. With one source the outer segments are empty.
struct Work {
    int bh;
    int pr0, pr1, pc0, pc1;   // clipped patch
    int wr0, wr1, wc0, wc1;   // clipped window
    int seg[4];               // row segment boundaries (see above)
    int nb0, nb01;            // key blocks of segment 0, of segments 0 and 1
    int tile0;                // first query tile of the unit's group within the patch
    int wtc;                  // window blocks along the columns
    int n_win, n_blocks;      // window blocks, window + global blocks
    int jb, je;               // the unit's key blocks [jb, je) (a key-range split)
    int split;
};

// Where key block j (< n_win) of a unit lies: first row and column of its box,
// how many of its rows and columns are inside its segment and the window, and
// whether it is read from the previous step's buffers.
struct BlockGeom {
    int row, col, vr, vc;
    bool stale;
};

__host__ __device__ inline int imin_(int a, int b) { return a < b ? a : b; }
__host__ __device__ inline int imax_(int a, int b) { return a > b ? a : b; }
__host__ __device__ inline int cdiv_(int a, int b) { return (a + b - 1) / b; }

// Sum of the clipped window extents of the first i patches along an axis of
// length L (patch side P, margin m).
__host__ __device__ inline int md_axis_offset(int L, int P, int m, int i) {
    int s = 0;
    for (int k = 0; k < i; ++k) s += imin_(L, (k + 1) * P + m) - imax_(0, k * P - m);
    return s;
}

__host__ __device__ inline int floor_div_(int a, int b) { return a >= 0 ? a / b : -((-a + b - 1) / b); }

// Overlapping-window mode: the patches (along one axis of n patches of side
// P, margin m) whose windows contain coordinate x are [*lo, *hi]: window i
// spans [i*P - m, (i+1)*P + m) clipped, so it contains x exactly when
// (x - m)/P - 1 < i <= (x + m)/P.
__host__ __device__ inline void md_cover_range(int n, int P, int m, int x, int *lo, int *hi) {
    *lo = imax_(0, floor_div_(x - m, P));
    *hi = imin_(n - 1, floor_div_(x + m, P));
}

// Host: key blocks a patch's clipped window needs (the scheduling cost of
// each of its units).
inline int patch_cost(const FwdParams &p, int patch) {
    const int kc = 1 << p.kc_log2;
    const int pi = patch / p.nPw, pj = patch % p.nPw;
    const int r0 = pi * p.Ph, r1 = imin_(p.H, r0 + p.Ph);
    const int c0 = pj * p.Pw, c1 = imin_(p.W, c0 + p.Pw);
    const int wh = imin_(p.H, r1 + p.mh) - imax_(0, r0 - p.mh);
    const int ww = imin_(p.W, c1 + p.mw) - imax_(0, c0 - p.mw);
    return cdiv_(ww, kc) * cdiv_(wh, p.kr);
}

// Host: the predicted cost of one unit of a patch, in key blocks: its
// window's blocks, the global-token blocks and kUnitOverheadBlocks.
inline long long unit_cost(const FwdParams &p, int patch) {
    return patch_cost(p, patch) + cdiv_(p.G, p.kb) + kUnitOverheadBlocks;
}

// Host: fills patch_order with the patches [patch_begin, patch_begin +
// patch_count) by decreasing cost (ties in natural order), so a persistent
// CTA's last units are its cheapest, and cls_rank0 with the runs of equal
// cost. Needs H, W, Ph, Pw, mh, mw, nPw, kc_log2, kr, patch_begin and
// patch_count set; leaves n_perm = 0 (natural order) past kMaxPatchOrder
// patches and n_cls = 0 past kMaxCostClasses runs.
inline void order_patches(FwdParams &prm) {
    const int np = prm.patch_count;
    prm.n_perm = 0;
    prm.n_cls = 0;
    if (np > kMaxPatchOrder) return;
    int cost[kMaxPatchOrder];  // indexed by position in the patch range
    unsigned short idx[kMaxPatchOrder];
    for (int i = 0; i < np; ++i) {
        cost[i] = patch_cost(prm, prm.patch_begin + i);
        idx[i] = (unsigned short)i;
    }
    // insertion sort, stable, descending cost (np <= 256)
    for (int i = 1; i < np; ++i) {
        const unsigned short x = idx[i];
        int j = i - 1;
        while (j >= 0 && cost[idx[j]] < cost[x]) {
            idx[j + 1] = idx[j];
            --j;
        }
        idx[j + 1] = x;
    }
    for (int i = 0; i < np; ++i) prm.patch_order[i] = (unsigned short)(prm.patch_begin + idx[i]);
    prm.n_perm = np;
    int n_cls = 0;
    for (int i = 0; i < np; ++i) {
        if (i > 0 && cost[idx[i]] == cost[idx[i - 1]]) continue;
        if (n_cls == kMaxCostClasses) {
            n_cls = 0;
            break;
        }
        prm.cls_rank0[n_cls++] = i;
    }
    prm.n_cls = n_cls;
    if (n_cls) prm.cls_rank0[n_cls] = np;
}

// Work units are ordered by cost class (patches with the same number of key
// blocks, largest first), then batch*head, then patch within the class, then
// query-tile group. The cheapest units come last, and the units running at the
// same time are the neighbouring patches of a few heads, whose overlapping
// key/value windows are then read from L2 rather than DRAM (one launch of
// B2 h10 256x256 patch 64 margin 32 read 0.84 GB from DRAM in this order,
// 1.13 GB with batch*head varying fastest). Without classes (more than
// kMaxCostClasses distinct costs) batch*head varies fastest.
// The (batch*head, patch) of a unit, in the order above.
__host__ __device__ inline int unit_patch(const FwdParams &p, int unit, int *bh) {
    const int rest = unit / p.n_qblocks;
    int rank;
    if (p.n_cls > 0) {
        int c = 0;
        while (c + 1 < p.n_cls && rest >= p.BH * p.cls_rank0[c + 1]) ++c;
        const int r = rest - p.BH * p.cls_rank0[c];
        const int cnt = p.cls_rank0[c + 1] - p.cls_rank0[c];
        *bh = r / cnt;
        rank = p.cls_rank0[c] + r % cnt;
    } else {
        *bh = rest % p.BH;
        rank = rest / p.BH;
    }
    return p.n_perm ? int(p.patch_order[rank]) : p.patch_begin + rank;
}

// Host: the per-CTA unit lists, on the predicted unit costs (unit_cost).
//  * head_major (the keys and values of all heads do not fit in L2): units
//    are taken batch*head first, then cost class, patch and query-tile
//    group, and each goes to the CTA that becomes free first (list
//    scheduling), so the CTAs finish together and the units running at one
//    moment share one or two heads' keys and values (a head's windows stay
//    in L2 instead of being read again for every cost class).
//  * otherwise (everything fits in L2): the split of every cost class over
//    the CTAs is chosen for the smallest largest CTA cost - longest units
//    first, then moves and swaps of single units off the busiest CTA while
//    they lower it - and each CTA runs its units costliest class first, the
//    units of a class dealt round robin in the unit numbering.
// Needs order_patches() done with a class table; leaves n_sched = 0 (round
// robin) otherwise or past the table sizes.
inline void build_schedule(FwdParams &p, int grid, bool head_major) {
    p.n_sched = 0;
    if (p.n_cls == 0 || p.n_units > kMaxSchedUnits || grid > kMaxSchedCtas || grid < 1) return;
    const int nq = p.n_qblocks;
    const int ncls = p.n_cls;
    long long ccost[kMaxCostClasses];
    for (int k = 0; k < ncls; ++k)
        ccost[k] = unit_cost(p, p.n_perm ? int(p.patch_order[p.cls_rank0[k]]) : p.patch_begin + p.cls_rank0[k]);
    long long load[kMaxSchedCtas];
    int count[kMaxSchedCtas];
    for (int c = 0; c < grid; ++c) load[c] = count[c] = 0;
    if (head_major) {
        static thread_local unsigned short order[kMaxSchedUnits];
        static thread_local unsigned short owner[kMaxSchedUnits];
        int n = 0;
        for (int bh = 0; bh < p.BH; ++bh)
            for (int c = 0; c < ncls; ++c) {
                const int cnt = p.cls_rank0[c + 1] - p.cls_rank0[c];
                for (int k = 0; k < cnt; ++k)
                    for (int qb = 0; qb < nq; ++qb)
                        order[n++] = (unsigned short)((p.BH * p.cls_rank0[c] + bh * cnt + k) * nq + qb);
            }
        // binary min-heap of (finish time, cta), ties to the lower CTA index
        int heap[kMaxSchedCtas];
        for (int c = 0; c < grid; ++c) heap[c] = c;
        auto less = [&](int a, int b) { return load[a] < load[b] || (load[a] == load[b] && a < b); };
        for (int i = 0; i < n; ++i) {
            int bh;
            const int c = heap[0];
            owner[i] = (unsigned short)c;
            ++count[c];
            load[c] += unit_cost(p, unit_patch(p, order[i], &bh));
            for (int k = 0;;) {  // sift the root down
                const int l = 2 * k + 1, r = l + 1;
                int m = k;
                if (l < grid && less(heap[l], heap[m])) m = l;
                if (r < grid && less(heap[r], heap[m])) m = r;
                if (m == k) break;
                const int t = heap[k];
                heap[k] = heap[m];
                heap[m] = t;
                k = m;
            }
        }
        p.cta_first[0] = 0;
        for (int c = 0; c < grid; ++c) p.cta_first[c + 1] = (unsigned short)(p.cta_first[c] + count[c]);
        int fill[kMaxSchedCtas];
        for (int c = 0; c < grid; ++c) fill[c] = p.cta_first[c];
        for (int i = 0; i < n; ++i) p.sched[fill[owner[i]]++] = order[i];
        p.n_sched = n;
        return;
    }
    // units of class k: numbers [BH * cls_rank0[k] * nq, BH * cls_rank0[k+1] * nq)
    static thread_local int cnt[kMaxSchedCtas][kMaxCostClasses];
    for (int c = 0; c < grid; ++c)
        for (int k = 0; k < ncls; ++k) cnt[c][k] = 0;
    for (int k = 0; k < ncls; ++k) {  // longest units first, each to the least loaded CTA
        const int units_k = p.BH * (p.cls_rank0[k + 1] - p.cls_rank0[k]) * nq;
        for (int i = 0; i < units_k; ++i) {
            int c = 0;
            for (int d = 1; d < grid; ++d)
                if (load[d] < load[c]) c = d;
            ++cnt[c][k];
            load[c] += ccost[k];
        }
    }
    for (int it = 0; it < 64 * grid; ++it) {  // improve the busiest CTA while possible
        int cm = 0;
        for (int d = 1; d < grid; ++d)
            if (load[d] > load[cm]) cm = d;
        long long best = load[cm];
        int bk = -1, bc = -1, bm = -1;  // class moved off cm, receiving CTA, class moved back (-1: none)
        for (int k = 0; k < ncls; ++k) {
            if (!cnt[cm][k]) continue;
            for (int c = 0; c < grid; ++c) {
                if (c == cm) continue;
                const long long mv = load[c] + ccost[k] > load[cm] - ccost[k] ? load[c] + ccost[k] : load[cm] - ccost[k];
                if (mv < best) {
                    best = mv;
                    bk = k;
                    bc = c;
                    bm = -1;
                }
                for (int m = 0; m < ncls; ++m) {
                    if (!cnt[c][m] || ccost[m] >= ccost[k]) continue;
                    const long long a = load[cm] - ccost[k] + ccost[m], b2 = load[c] + ccost[k] - ccost[m];
                    const long long sw = a > b2 ? a : b2;
                    if (sw < best) {
                        best = sw;
                        bk = k;
                        bc = c;
                        bm = m;
                    }
                }
            }
        }
        if (bk < 0) break;
        --cnt[cm][bk];
        ++cnt[bc][bk];
        load[cm] -= ccost[bk];
        load[bc] += ccost[bk];
        if (bm >= 0) {
            --cnt[bc][bm];
            ++cnt[cm][bm];
            load[bc] -= ccost[bm];
            load[cm] += ccost[bm];
        }
    }
    p.cta_first[0] = 0;
    for (int c = 0; c < grid; ++c) {
        int t = 0;
        for (int k = 0; k < ncls; ++k) t += cnt[c][k];
        p.cta_first[c + 1] = (unsigned short)(p.cta_first[c] + t);
    }
    int fill[kMaxSchedCtas];
    for (int c = 0; c < grid; ++c) fill[c] = p.cta_first[c];
    for (int k = 0; k < ncls; ++k) {  // deal class k's units round robin to the CTAs that take some
        int left[kMaxSchedCtas];
        for (int c = 0; c < grid; ++c) left[c] = cnt[c][k];
        const int u0 = p.BH * p.cls_rank0[k] * nq, u1 = p.BH * p.cls_rank0[k + 1] * nq;
        int c = 0;
        for (int u = u0; u < u1; ++u) {
            while (left[c] == 0) c = c + 1 == grid ? 0 : c + 1;
            p.sched[fill[c]++] = (unsigned short)u;
            --left[c];
            c = c + 1 == grid ? 0 : c + 1;
        }
    }
    p.n_sched = p.n_units;
}

// The i-th unit of this CTA's work, or -1 past its last.
__device__ __forceinline__ int cta_unit(const FwdParams &p, int i) {
#ifdef __CUDA_ARCH__
    if (p.n_sched) {
        const int k = p.cta_first[blockIdx.x] + i;
        return k < p.cta_first[blockIdx.x + 1] ? int(p.sched[k]) : -1;
    }
    const int u = blockIdx.x + i * gridDim.x;
    return u < p.n_units ? u : -1;
#else
    return -1;
#endif
}

__host__ __device__ inline Work decode_work(const FwdParams &p, int unit) {
    Work w;
    const int qb = unit % p.n_qblocks;
    const int patch = unit_patch(p, unit, &w.bh);
    const int pi = patch / p.nPw, pj = patch % p.nPw;
    w.pr0 = pi * p.Ph;
    w.pr1 = imin_(p.H, w.pr0 + p.Ph);
    w.pc0 = pj * p.Pw;
    w.pc1 = imin_(p.W, w.pc0 + p.Pw);
    w.wr0 = imax_(0, w.pr0 - p.mh);
    w.wr1 = imin_(p.H, w.pr1 + p.mh);
    w.wc0 = imax_(0, w.pc0 - p.mw);
    w.wc1 = imin_(p.W, w.pc1 + p.mw);
    if (p.md) {  // overlapping windows: every token of the window is a query
        w.pr0 = w.wr0;
        w.pr1 = w.wr1;
        w.pc0 = w.wc0;
        w.pc1 = w.wc1;
    }
    w.tile0 = p.tiles_per_unit * qb;
    const int kc = 1 << p.kc_log2;
    w.wtc = cdiv_(w.wc1 - w.wc0, kc);
    if (p.two_source) {
        w.seg[0] = w.wr0;
        w.seg[1] = w.pr0;
        w.seg[2] = w.pr1;
        w.seg[3] = w.wr1;
    } else {
        w.seg[0] = w.seg[1] = w.wr0;
        w.seg[2] = w.seg[3] = w.wr1;
    }
    w.nb0 = w.wtc * cdiv_(w.seg[1] - w.seg[0], p.kr);
    w.nb01 = w.nb0 + w.wtc * cdiv_(w.seg[2] - w.seg[1], p.kr);
    w.n_win = w.nb01 + w.wtc * cdiv_(w.seg[3] - w.seg[2], p.kr);
    w.n_blocks = w.n_win + cdiv_(p.G, p.kb);
    w.jb = 0;
    w.je = w.n_blocks;
    w.split = 0;
    return w;
}

// Global-token queries (the text-query half of joint attention): a unit is
// (batch*head, key-range split, group of 128-token query tiles); the window is
// the whole grid followed by the global tokens, and split s covers key
// blocks [s*n/S, (s+1)*n/S).
__host__ __device__ inline Work decode_work_gq(const FwdParams &p, int unit) {
    Work w;
    const int qb = unit % p.n_qblocks;
    const int rest = unit / p.n_qblocks;
    w.split = rest % p.n_splits;
    w.bh = rest / p.n_splits;
    w.pr0 = w.pc0 = 0;
    w.pr1 = p.H;
    w.pc1 = p.W;
    w.wr0 = w.wc0 = 0;
    w.wr1 = p.H;
    w.wc1 = p.W;
    w.seg[0] = w.seg[1] = 0;
    w.seg[2] = w.seg[3] = p.H;
    w.tile0 = p.tiles_per_unit * qb;
    w.wtc = cdiv_(p.W, 1 << p.kc_log2);
    w.nb0 = 0;
    w.nb01 = w.n_win = w.wtc * cdiv_(p.H, p.kr);
    w.n_blocks = w.n_win + cdiv_(p.G, p.kb);
    w.jb = (int)((long long)w.split * w.n_blocks / p.n_splits);
    w.je = (int)((long long)(w.split + 1) * w.n_blocks / p.n_splits);
    return w;
}

template <bool GQ>
__host__ __device__ inline Work decode(const FwdParams &p, int unit) {
    return GQ ? decode_work_gq(p, unit) : decode_work(p, unit);
}

__host__ __device__ inline BlockGeom block_geom(const FwdParams &p, const Work &w, int j) {
    const int sg = j < w.nb0 ? 0 : (j < w.nb01 ? 1 : 2);
    const int l = j - (sg == 0 ? 0 : (sg == 1 ? w.nb0 : w.nb01));
    const int tr = l / w.wtc, tc = l - tr * w.wtc;
    // selects, not a runtime index, so the segment bounds stay in registers
    const int lo = sg == 0 ? w.seg[0] : (sg == 1 ? w.seg[1] : w.seg[2]);
    const int hi = sg == 0 ? w.seg[1] : (sg == 1 ? w.seg[2] : w.seg[3]);
    BlockGeom b;
    b.row = lo + tr * p.kr;
    b.col = w.wc0 + (tc << p.kc_log2);
    b.vr = imin_(p.kr, hi - b.row);
    b.vc = imin_(1 << p.kc_log2, w.wc1 - b.col);
    b.stale = sg != 1;
    return b;
}

// Origin (first row, first column) of query tile t of the unit's patch.
__host__ __device__ inline void q_tile_origin(const FwdParams &p, const Work &w, int t, int *row0, int *col0) {
    const int tr = t / p.tiles_c, tc = t % p.tiles_c;
    *row0 = w.pr0 + tr * p.qr;
    *col0 = w.pc0 + tc * p.qc;
}

__host__ __device__ inline bool q_tile_valid(const FwdParams &p, const Work &w, int t) {
    if (t >= p.tiles_c * p.tiles_r) return false;
    int r0, c0;
    q_tile_origin(p, w, t, &r0, &c0);
    return r0 < w.pr1 && c0 < w.pc1;
}

}  // namespace npa
