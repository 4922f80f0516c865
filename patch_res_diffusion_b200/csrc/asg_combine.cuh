// asg_combine.cuh - the asynchronous structure guidance (ASG) combine:
//   out[i, b, c, s] = eps[i, b, c, s] + w_t * M[i, b, s] * (ref[b, c, s] - eps[i, b, c, s])
// ASGDiffusion (pith.science review), "core_discovery" and "key_machinery":
// each patch's noise prediction is pulled toward the reference patch's
// prediction from the previous step, weighted per pixel by the normalised
// mask. One pass over HBM: every element of eps is read once and written
// once; the mask is read once per (patch, batch element, pixel) and reused
// across the channels; the reference is shared by all patches (read from L2
// after the first patch). One thread per 8-pixel chunk of one (patch, batch
// element): 16-byte vector loads and stores along the pixels.
//
// Arithmetic: the bf16 inputs are widened to float32, the result is
// fma(w_t * M, ref - eps, eps) rounded to bf16 (nearest even).
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

namespace npa {

struct AsgParams {
    const __nv_bfloat16 *eps;   // [n, B, C, S]
    const __nv_bfloat16 *ref;   // [B, C, S]
    const __nv_bfloat16 *mask;  // [n, B, S]
    __nv_bfloat16 *out;         // [n, B, C, S] (may be eps itself)
    long long n_items;          // n * B * ceil(S / 8): 8-pixel chunks of one (patch, batch element)
    int B, C, S, chunks;        // chunks = ceil(S / 8)
    float w;
    int vec;                    // 1: S % 8 == 0, every chunk is one 16-byte vector per channel
};

__device__ __forceinline__ float bf16_lo(uint32_t x) { return __uint_as_float(x << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t x) { return __uint_as_float(x & 0xffff0000u); }

__device__ __forceinline__ uint32_t pack_rn(float a, float b) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<const uint32_t *>(&h);
}

// eps and out stream through once (evict-first cache policy), so the
// reference and the masks, which every patch reads, stay in L2.
__device__ __forceinline__ uint4 ld_eps(const __nv_bfloat16 *a) { return __ldcs(reinterpret_cast<const uint4 *>(a)); }
__device__ __forceinline__ void st_out(__nv_bfloat16 *a, uint4 v) { __stcs(reinterpret_cast<uint4 *>(a), v); }

// Eight pixels of one channel: fma(w_t * M, ref - eps, eps), bf16 pairs.
__device__ __forceinline__ uint4 combine8(const float (&wm)[8], uint4 ev, uint4 rv) {
    const uint32_t e[4] = {ev.x, ev.y, ev.z, ev.w}, r[4] = {rv.x, rv.y, rv.z, rv.w};
    uint32_t o[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const float e0 = bf16_lo(e[k]), e1 = bf16_hi(e[k]);
        o[k] = pack_rn(fmaf(wm[2 * k], bf16_lo(r[k]) - e0, e0), fmaf(wm[2 * k + 1], bf16_hi(r[k]) - e1, e1));
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
}

__global__ void __launch_bounds__(256) asg_combine_kernel(const __grid_constant__ AsgParams p) {
    for (long long item = (long long)blockIdx.x * blockDim.x + threadIdx.x; item < p.n_items;
         item += (long long)gridDim.x * blockDim.x) {
        const int chunk = (int)(item % p.chunks);
        const long long ib = item / p.chunks;  // patch * B + batch element
        const int b = (int)(ib % p.B);
        const int s0 = chunk * 8;
        const size_t eps_base = (size_t)ib * p.C * p.S + s0;
        const size_t ref_base = (size_t)b * p.C * p.S + s0;
        if (p.vec) {
            const uint4 mv = *reinterpret_cast<const uint4 *>(p.mask + (size_t)ib * p.S + s0);
            float wm[8];
            const uint32_t mw[4] = {mv.x, mv.y, mv.z, mv.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                wm[2 * k] = p.w * bf16_lo(mw[k]);
                wm[2 * k + 1] = p.w * bf16_hi(mw[k]);
            }
            // groups of kG channels: all their loads are issued before any of
            // their stores (out may be eps itself, so without this each load
            // would wait for the previous channel's store). On 570 MB: 4,709
            // GB/s one channel at a time, 5,665 in groups of 4, 5,898 with the
            // streaming cache policy; groups of 8 were no faster.
            constexpr int kG = 4;
            int c = 0;
            for (; c + kG <= p.C; c += kG) {
                uint4 ev[kG], rv[kG];
#pragma unroll
                for (int g = 0; g < kG; ++g) {
                    ev[g] = ld_eps(p.eps + eps_base + (size_t)(c + g) * p.S);
                    rv[g] = __ldg(reinterpret_cast<const uint4 *>(p.ref + ref_base + (size_t)(c + g) * p.S));
                }
#pragma unroll
                for (int g = 0; g < kG; ++g) st_out(p.out + eps_base + (size_t)(c + g) * p.S, combine8(wm, ev[g], rv[g]));
            }
            for (; c < p.C; ++c) {
                const uint4 ev = ld_eps(p.eps + eps_base + (size_t)c * p.S);
                const uint4 rv = __ldg(reinterpret_cast<const uint4 *>(p.ref + ref_base + (size_t)c * p.S));
                st_out(p.out + eps_base + (size_t)c * p.S, combine8(wm, ev, rv));
            }
        } else {
            const int n = p.S - s0 < 8 ? p.S - s0 : 8;
            for (int k = 0; k < n; ++k) {
                const float wm = p.w * __bfloat162float(p.mask[(size_t)ib * p.S + s0 + k]);
                for (int c = 0; c < p.C; ++c) {
                    const size_t ie = eps_base + (size_t)c * p.S + k;
                    const float e = __bfloat162float(p.eps[ie]);
                    const float r = __bfloat162float(p.ref[ref_base + (size_t)c * p.S + k]);
                    p.out[ie] = __float2bfloat16_rn(fmaf(wm, r - e, e));
                }
            }
        }
    }
}

}  // namespace npa
