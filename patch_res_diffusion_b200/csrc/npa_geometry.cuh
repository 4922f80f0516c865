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
// Work unit = (batch*head, patch, pair of 128-row query tiles); a persistent
// CTA walks the units blockIdx.x, blockIdx.x + gridDim.x, ... A query tile is
// a box of qr patch rows x qc patch columns (qr*qc <= 128); a key/value block
// is a box of kr rows x kc columns (kr*kc = 128) inside the window, followed
// by ceil(G/128) blocks of global tokens. Every quantity is recomputed from
// the unit index with integer arithmetic; there are no index tables.
#pragma once

#include <cstdint>
#include <cuda.h>

namespace npa {

// Up to this many patches are visited largest window first; beyond it, in
// natural order.
constexpr int kMaxPatchOrder = 256;

struct FwdParams {
    CUtensorMap tm_q;   // 4D {d, W, H, B*heads}, box {64, qc, qr, 1}, 128B swizzle
    CUtensorMap tm_k;   // 4D, box {64, kc, kr, 1}
    CUtensorMap tm_v;   // 4D, box {64, kc, kr, 1}
    CUtensorMap tm_gk;  // 3D {d, G, B*heads}, box {64, 128, 1} (unused when G == 0)
    CUtensorMap tm_gv;
    void *o;            // bf16 [B, heads, H*W, d]
    int H, W, G;
    int Ph, Pw, mh, mw;
    int nPh, nPw;                    // patches along rows / columns
    int qc, qr, tiles_c, tiles_r;    // query tile box and tiles per patch
    int kc_log2, kr;                 // key block box: (1 << kc_log2) columns x kr rows
    int n_qblocks;                   // query-tile pairs per patch
    float scale_log2;                // log2(e) / sqrt(d)
    unsigned long long wait_limit_ns;
    int BH;                          // batch * heads
    int n_units;                     // work units in execution order
    int n_perm;                      // entries of patch_order (0: natural order)
    unsigned short patch_order[kMaxPatchOrder];  // patches by decreasing window area
};

struct Work {
    int bh;
    int pr0, pr1, pc0, pc1;   // clipped patch
    int wr0, wr1, wc0, wc1;   // clipped window
    int tile0;                // first query tile (of two) within the patch
    int wtc;                  // window blocks along the columns
    int n_win, n_blocks;      // window blocks, window + global blocks
};

__host__ __device__ inline int imin_(int a, int b) { return a < b ? a : b; }
__host__ __device__ inline int imax_(int a, int b) { return a > b ? a : b; }
__host__ __device__ inline int cdiv_(int a, int b) { return (a + b - 1) / b; }

// Work units are ordered query-tile pair fastest, then batch*head, then
// patch (largest window first), so the units that run at the same time share
// few key/value windows (they stay in L2) and the cheapest units come last.
__host__ __device__ inline Work decode_work(const FwdParams &p, int unit) {
    Work w;
    const int qb = unit % p.n_qblocks;
    const int rest = unit / p.n_qblocks;
    w.bh = rest % p.BH;
    const int rank = rest / p.BH;
    const int patch = rank < p.n_perm ? int(p.patch_order[rank]) : rank;
    const int pi = patch / p.nPw, pj = patch % p.nPw;
    w.pr0 = pi * p.Ph;
    w.pr1 = imin_(p.H, w.pr0 + p.Ph);
    w.pc0 = pj * p.Pw;
    w.pc1 = imin_(p.W, w.pc0 + p.Pw);
    w.wr0 = imax_(0, w.pr0 - p.mh);
    w.wr1 = imin_(p.H, w.pr1 + p.mh);
    w.wc0 = imax_(0, w.pc0 - p.mw);
    w.wc1 = imin_(p.W, w.pc1 + p.mw);
    w.tile0 = 2 * qb;
    const int kc = 1 << p.kc_log2;
    w.wtc = cdiv_(w.wc1 - w.wc0, kc);
    w.n_win = w.wtc * cdiv_(w.wr1 - w.wr0, p.kr);
    w.n_blocks = w.n_win + cdiv_(p.G, 128);
    return w;
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
