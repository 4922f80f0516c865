// md_combine.cuh - second pass of the overlapping-window comparator: the mean,
// over the windows containing each token, of the windows' normalised float32
// outputs (written window-major by npa_fwd_kernel's comparator epilogue),
// rounded to bf16. md_cover_range gives the windows along each axis.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "npa_geometry.cuh"
#include "sm100.cuh"

namespace npa {

constexpr int kMaxMdAxis = 256;

struct MdCombineParams {
    const float *part;
    __nv_bfloat16 *o;
    int H, W, Ph, Pw, mh, mw, nPh, nPw, BH, md_rows, md_tw;
    int rh[kMaxMdAxis], cw[kMaxMdAxis];  // row / column offsets of the windows in the partials
};

// D / 4 lanes per token, each holding four channels (16-byte loads), so a
// warp averages 32 * 4 / D tokens; 256 threads per block.
template <int D>
__global__ void __launch_bounds__(256) md_combine_kernel(const __grid_constant__ MdCombineParams p) {
    constexpr int kLanes = D / 4;
    constexpr int kTokPerBlock = 256 / kLanes;
    const long long tok = (long long)blockIdx.x * kTokPerBlock + threadIdx.x / kLanes;
    const long long N = (long long)p.H * p.W;
    if (tok >= (long long)p.BH * N) return;
    const int lane = threadIdx.x % kLanes;
    const int bh = (int)(tok / N), t = (int)(tok - (long long)bh * N);
    const int r = t / p.W, c = t - (t / p.W) * p.W;
    int pi0, pi1, pj0, pj1;
    md_cover_range(p.nPh, p.Ph, p.mh, r, &pi0, &pi1);
    md_cover_range(p.nPw, p.Pw, p.mw, c, &pj0, &pj1);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int pi = pi0; pi <= pi1; ++pi) {
        const int wr0 = imax_(0, pi * p.Ph - p.mh);
        for (int pj = pj0; pj <= pj1; ++pj) {
            const int wc0 = imax_(0, pj * p.Pw - p.mw);
            const size_t prow = ((size_t)bh * p.md_rows + (p.rh[pi] + r - wr0)) * p.md_tw + (p.cw[pj] + c - wc0);
            const float4 v = __ldcs(reinterpret_cast<const float4 *>(p.part + prow * D) + lane);
            acc.x += v.x;
            acc.y += v.y;
            acc.z += v.z;
            acc.w += v.w;
        }
    }
    const float inv = 1.f / float((pi1 - pi0 + 1) * (pj1 - pj0 + 1));
    uint2 out;
    out.x = sm100::pack_bf16x2(acc.x * inv, acc.y * inv);
    out.y = sm100::pack_bf16x2(acc.z * inv, acc.w * inv);
    *reinterpret_cast<uint2 *>(p.o + (size_t)tok * D + lane * 4) = out;
}

}  // namespace npa
