// npa_fwd_kernel.cuh - the sm_100a forward kernel for patch-restricted
// self-attention (NPA and PCPP share it through npa_geometry.cuh).
//
// One CTA per work unit: two 128-query tiles of one patch that share the
// patch's key/value window. Ten warps, each with one role:
//   warps 0-3  softmax + epilogue for query tile 0 (TMEM lanes 0..127)
//   warps 4-7  softmax + epilogue for query tile 1
//   warp  8    TMA producer (Q once, then K and V blocks through a ring of
//              kStages shared-memory stages); owns the TMEM allocation
//   warp  9    MMA issuer (one thread issues every tcgen05.mma)
//
// Per key block j and tile q the MMA warp issues S_q = Q_q K_j^T into TMEM
// (M=128, N=128, K=d, both operands K-major in 128-byte-swizzled shared
// memory); the softmax warps read S_q from TMEM (one thread per query row),
// update the running maximum and sum, and write P_q = exp2(S*log2e/sqrt(d) -
// m) as bf16 back into the first 64 columns of the same TMEM region; the MMA
// warp then issues O_q += P_q V_j with A = P_q read from TMEM and B = V_j
// (MN-major, 128-byte swizzle). The issue order PV_q(j-1) -> S_q(j) lets the
// two tiles ping-pong: the tensor core works on one tile while the softmax
// warps of the other run. Because tcgen05 operations of one thread complete
// in order, the commit that announces S_q(j) also guarantees that PV_q(j-1)
// has finished, so the softmax warps may rescale O_q and overwrite P_q as
// soon as S_q(j) is visible.
//
// The running maximum is rescaled lazily: O and the row sum are rescaled only
// when the block maximum exceeds the reference maximum by more than 8 (log2
// units), which keeps P <= 256 and leaves the final O / l exact.
//
// Every wait is bounded (FwdParams::wait_limit_ns). On expiry the CTA records
// NPA_ERR_DEVICE_TIMEOUT in the device status word, stops issuing work,
// drains what is in flight and frees its tensor memory.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "npa_geometry.cuh"
#include "sm100.cuh"

namespace npa {

__device__ unsigned int g_npa_status;  // first device-side error since last read

__device__ __forceinline__ void record_error(unsigned int code) { atomicCAS(&g_npa_status, 0u, code); }

constexpr unsigned int kErrDeviceTimeout = 5u;  // NPA_ERR_DEVICE_TIMEOUT

template <int D>
struct KCfg {
    static_assert(D == 64 || D == 128, "head dim");
    static constexpr int kChunks = D / 64;              // 64-element (128-byte) column blocks
    static constexpr int kChunkBytes = 128 * 128;       // 128 rows x 128 bytes
    static constexpr int kTileBytes = kChunks * kChunkBytes;
    static constexpr int kStages = (D == 64) ? 4 : 2;
    static constexpr int kThreads = 320;
    static constexpr int kOffQ = 0;
    static constexpr int kOffK = 2 * kTileBytes;
    static constexpr int kOffV = kOffK + kStages * kTileBytes;
    static constexpr int kOffBar = kOffV + kStages * kTileBytes;
    // barrier indices
    static constexpr int bQFull = 0;
    static constexpr int bKFull = 1;
    static constexpr int bKEmpty = bKFull + kStages;
    static constexpr int bVFull = bKEmpty + kStages;
    static constexpr int bVEmpty = bVFull + kStages;
    static constexpr int bSFull = bVEmpty + kStages;   // [2]
    static constexpr int bPFull = bSFull + 2;          // [2]
    static constexpr int bOFinal = bPFull + 2;         // [2]
    static constexpr int bDrain = bOFinal + 2;
    static constexpr int kNumBars = bDrain + 1;
    static constexpr int kOffMisc = kOffBar + kNumBars * 8;
    static constexpr int kSmemBytes = kOffMisc + 16 + 1024;  // + slack for 1024-byte alignment
    // tensor memory columns
    static constexpr uint32_t kTmemCols = 512;
    __device__ static constexpr uint32_t col_s(int q) { return q ? 128u : 0u; }
    __device__ static constexpr uint32_t col_o(int q) { return 256u + (q ? uint32_t(D) : 0u); }
};

// ---------------------------------------------------------------------------
// Producer: one thread of warp 8.
// ---------------------------------------------------------------------------
template <int D>
__device__ __forceinline__ void load_block(const FwdParams &p, const Work &w, int j, bool is_v, uint8_t *dst,
                                           uint64_t *bar) {
    using C = KCfg<D>;
    if (j < w.n_win) {
        const int tr = j / w.wtc, tc = j - tr * w.wtc;
        const int col = w.wc0 + (tc << p.kc_log2), row = w.wr0 + tr * p.kr;
        const CUtensorMap *m = is_v ? &p.tm_v : &p.tm_k;
#pragma unroll
        for (int c = 0; c < C::kChunks; ++c)
            sm100::tma_load_4d(dst + c * C::kChunkBytes, m, bar, c * 64, col, row, w.bh);
    } else {
        const int g0 = (j - w.n_win) * 128;
        const CUtensorMap *m = is_v ? &p.tm_gv : &p.tm_gk;
#pragma unroll
        for (int c = 0; c < C::kChunks; ++c)
            sm100::tma_load_3d(dst + c * C::kChunkBytes, m, bar, c * 64, g0, w.bh);
    }
}

template <int D>
__device__ void run_producer(const FwdParams &p, const Work &w, uint8_t *smem, uint64_t *bars,
                             volatile uint32_t *abort_flag) {
    using C = KCfg<D>;
    const uint64_t lim = p.wait_limit_ns;
    sm100::tma_prefetch_desc(&p.tm_q);
    sm100::tma_prefetch_desc(&p.tm_k);
    sm100::tma_prefetch_desc(&p.tm_v);
    if (p.G > 0) {
        sm100::tma_prefetch_desc(&p.tm_gk);
        sm100::tma_prefetch_desc(&p.tm_gv);
    }
    const uint32_t q_bytes = uint32_t(C::kChunks * p.qc * p.qr * 128);
    sm100::mbar_arrive_expect_tx(&bars[C::bQFull], 2 * q_bytes);
#pragma unroll
    for (int t = 0; t < 2; ++t) {
        int row0, col0;
        q_tile_origin(p, w, w.tile0 + t, &row0, &col0);
#pragma unroll
        for (int c = 0; c < C::kChunks; ++c)
            sm100::tma_load_4d(smem + C::kOffQ + t * C::kTileBytes + c * C::kChunkBytes, &p.tm_q,
                               &bars[C::bQFull], c * 64, col0, row0, w.bh);
    }
    int nk = 0, nv = 0;  // K / V blocks issued
    for (int j = 0; j < w.n_blocks; ++j) {
        if (*abort_flag) break;
        const int s = j % C::kStages, use = j / C::kStages;
        if (use > 0 && !sm100::mbar_wait(&bars[C::bKEmpty + s], (use - 1) & 1, lim)) {
            record_error(kErrDeviceTimeout);
            *abort_flag = 1;
            break;
        }
        sm100::mbar_arrive_expect_tx(&bars[C::bKFull + s], C::kTileBytes);
        load_block<D>(p, w, j, false, smem + C::kOffK + s * C::kTileBytes, &bars[C::bKFull + s]);
        ++nk;
        if (use > 0 && !sm100::mbar_wait(&bars[C::bVEmpty + s], (use - 1) & 1, lim)) {
            record_error(kErrDeviceTimeout);
            *abort_flag = 1;
            break;
        }
        sm100::mbar_arrive_expect_tx(&bars[C::bVFull + s], C::kTileBytes);
        load_block<D>(p, w, j, true, smem + C::kOffV + s * C::kTileBytes, &bars[C::bVFull + s]);
        ++nv;
    }
    // Drain: every issued copy must have landed before the CTA may exit
    // (immediate on the normal path, where the consumers already saw them).
    sm100::mbar_wait(&bars[C::bQFull], 0, lim);
    for (int s = 0; s < C::kStages; ++s) {
        if (nk > s) sm100::mbar_wait(&bars[C::bKFull + s], ((nk - 1 - s) / C::kStages) & 1, lim);
        if (nv > s) sm100::mbar_wait(&bars[C::bVFull + s], ((nv - 1 - s) / C::kStages) & 1, lim);
    }
}

// ---------------------------------------------------------------------------
// MMA issuer: one thread of warp 9.
// ---------------------------------------------------------------------------
template <int D>
__device__ void run_mma(const FwdParams &p, const Work &w, uint8_t *smem, uint64_t *bars, uint32_t tmem,
                        volatile uint32_t *abort_flag) {
    using C = KCfg<D>;
    constexpr uint32_t kIdS = sm100::idesc_bf16_f32(128, 128, false, false);  // S = Q K^T
    constexpr uint32_t kIdO = sm100::idesc_bf16_f32(128, D, false, true);     // O += P V, V MN-major
    const uint64_t lim = p.wait_limit_ns;
    const uint32_t sQ = sm100::smem_u32(smem + C::kOffQ);
    const uint32_t sK = sm100::smem_u32(smem + C::kOffK);
    const uint32_t sV = sm100::smem_u32(smem + C::kOffV);
    const int n = w.n_blocks;
    bool ok = sm100::mbar_wait(&bars[C::bQFull], 0, lim);
    sm100::tc_fence_after();
    for (int j = 0; ok && j <= n; ++j) {
        if (*abort_flag) break;
        if (j < n) {
            ok = sm100::mbar_wait(&bars[C::bKFull + j % C::kStages], (j / C::kStages) & 1, lim);
            if (!ok) break;
        }
        if (j > 0) {
            ok = sm100::mbar_wait(&bars[C::bVFull + (j - 1) % C::kStages], ((j - 1) / C::kStages) & 1, lim);
            if (!ok) break;
        }
        sm100::tc_fence_after();
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            if (j > 0) {
                ok = sm100::mbar_wait(&bars[C::bPFull + q], (j - 1) & 1, lim);
                if (!ok) break;
                sm100::tc_fence_after();
                const uint32_t vbase = sV + ((j - 1) % C::kStages) * C::kTileBytes;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    // V block: 16 keys x D, MN-major; LBO = next 64-column block,
                    // SBO = next group of 8 keys.
                    const uint64_t bdesc = sm100::sdesc_sw128(vbase + kk * 2048, C::kChunkBytes, 1024);
                    sm100::mma_ts(tmem + C::col_o(q), tmem + C::col_s(q) + kk * 8, bdesc, kIdO,
                                  (j > 1 || kk > 0) ? 1u : 0u);
                }
                if (j == n) sm100::tc_commit(&bars[C::bOFinal + q]);
            }
            if (j < n) {
                const uint32_t kbase = sK + (j % C::kStages) * C::kTileBytes;
                const uint32_t qbase = sQ + q * C::kTileBytes;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * C::kChunkBytes + (kk & 3) * 32;
                    const uint64_t adesc = sm100::sdesc_sw128(qbase + off, 16, 1024);
                    const uint64_t bdesc = sm100::sdesc_sw128(kbase + off, 16, 1024);
                    sm100::mma_ss(tmem + C::col_s(q), adesc, bdesc, kIdS, kk > 0 ? 1u : 0u);
                }
                sm100::tc_commit(&bars[C::bSFull + q]);
            }
        }
        if (!ok) break;
        if (j < n) sm100::tc_commit(&bars[C::bKEmpty + j % C::kStages]);
        if (j > 0) sm100::tc_commit(&bars[C::bVEmpty + (j - 1) % C::kStages]);
    }
    if (!ok) {
        record_error(kErrDeviceTimeout);
        *abort_flag = 1;
    }
    // Drain: no MMA may still be running when the tensor memory is freed.
    sm100::tc_commit(&bars[C::bDrain]);
    sm100::mbar_wait(&bars[C::bDrain], 0, lim);
}

// ---------------------------------------------------------------------------
// Softmax + epilogue: one warpgroup (128 threads) per query tile.
// ---------------------------------------------------------------------------
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, uint64_t lim) {
    const bool got = sm100::mbar_wait(bar, parity, lim);
    return __all_sync(0xffffffffu, got);
}

template <int D>
__device__ void run_softmax(const FwdParams &p, const Work &w, uint64_t *bars, uint32_t tmem,
                            volatile uint32_t *abort_flag, int q) {
    using C = KCfg<D>;
    const uint64_t lim = p.wait_limit_ns;
    const int row = threadIdx.x & 127;
    const uint32_t lane_off = uint32_t((threadIdx.x >> 5) & 3) * 32u << 16;
    const uint32_t tS = tmem + lane_off + C::col_s(q);
    const uint32_t tO = tmem + lane_off + C::col_o(q);
    const float sl2 = p.scale_log2;
    const int kc = 1 << p.kc_log2;
    float m_ref = -INFINITY;  // reference maximum, already scaled to log2 units
    float l = 0.f;
    bool ok = true;
    for (int j = 0; j < w.n_blocks; ++j) {
        if (__any_sync(0xffffffffu, *abort_flag != 0u)) {
            ok = false;
            break;
        }
        if (!warp_wait(&bars[C::bSFull + q], j & 1, lim)) {
            record_error(kErrDeviceTimeout);
            *abort_flag = 1;
            ok = false;
            break;
        }
        sm100::tc_fence_after();
        uint32_t sa[64], sb[64];
        sm100::tmem_ld64(tS, sa);
        sm100::tmem_ld64(tS + 64, sb);
        float s[128];
#pragma unroll
        for (int i = 0; i < 64; ++i) {
            s[i] = __uint_as_float(sa[i]);
            s[64 + i] = __uint_as_float(sb[i]);
        }
        // keys of this block that lie outside the window (or past the last
        // global token) get -inf
        if (j < w.n_win) {
            const int tr = j / w.wtc, tc = j - tr * w.wtc;
            const int vc = w.wc1 - (w.wc0 + (tc << p.kc_log2));
            const int vr = w.wr1 - (w.wr0 + tr * p.kr);
            if (vc < kc || vr < p.kr) {
#pragma unroll
                for (int i = 0; i < 128; ++i)
                    if ((i & (kc - 1)) >= vc || (i >> p.kc_log2) >= vr) s[i] = -INFINITY;
            }
        } else {
            const int vg = p.G - (j - w.n_win) * 128;
            if (vg < 128) {
#pragma unroll
                for (int i = 0; i < 128; ++i)
                    if (i >= vg) s[i] = -INFINITY;
            }
        }
        float mx = s[0];
#pragma unroll
        for (int i = 1; i < 128; ++i) mx = fmaxf(mx, s[i]);
        const float m_new = fmaxf(m_ref, mx * sl2);
        const bool rescale = m_new > m_ref + 8.0f;
        float alpha = 1.f;
        if (rescale) {
            alpha = sm100::ex2_approx(m_ref - m_new);  // 0 on the first block
            m_ref = m_new;
        }
        if (j > 0 && __any_sync(0xffffffffu, rescale)) {
#pragma unroll 1
            for (int c = 0; c < D / 32; ++c) {
                uint32_t o[32];
                sm100::tmem_ld32(tO + c * 32, o);
#pragma unroll
                for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
                sm100::tmem_st32(tO + c * 32, o);
            }
        }
        l *= alpha;
        const float neg_m = (m_ref == -INFINITY) ? 0.f : -m_ref;
        uint32_t pk[64];
#pragma unroll
        for (int i = 0; i < 64; ++i) {
            const float p0 = sm100::ex2_approx(fmaf(s[2 * i], sl2, neg_m));
            const float p1 = sm100::ex2_approx(fmaf(s[2 * i + 1], sl2, neg_m));
            l += p0 + p1;
            pk[i] = sm100::pack_bf16x2(p0, p1);
        }
        sm100::tmem_st64(tS, pk);
        sm100::tc_fence_before();
        sm100::mbar_arrive(&bars[C::bPFull + q]);
    }
    if (!ok) return;
    if (!warp_wait(&bars[C::bOFinal + q], 0, lim)) {
        record_error(kErrDeviceTimeout);
        *abort_flag = 1;
        return;
    }
    sm100::tc_fence_after();
    // epilogue: O / l -> bf16 -> the query's token position
    const float inv_l = l > 0.f ? 1.f / l : 0.f;
    const int t = w.tile0 + q;
    int row0, col0;
    q_tile_origin(p, w, t, &row0, &col0);
    const int rr = row / p.qc, cc = row - rr * p.qc;
    const int grow = row0 + rr, gcol = col0 + cc;
    const bool valid = t < p.tiles_c * p.tiles_r && row < p.qc * p.qr && grow < w.pr1 && gcol < w.pc1;
    uint4 *dst = reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(p.o) +
                                           ((size_t)w.bh * p.H * p.W + (size_t)grow * p.W + gcol) * D);
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        sm100::tmem_ld32(tO + c * 32, o);
        if (valid) {
#pragma unroll
            for (int v = 0; v < 4; ++v) {
                uint4 pkt;
                pkt.x = sm100::pack_bf16x2(__uint_as_float(o[8 * v + 0]) * inv_l, __uint_as_float(o[8 * v + 1]) * inv_l);
                pkt.y = sm100::pack_bf16x2(__uint_as_float(o[8 * v + 2]) * inv_l, __uint_as_float(o[8 * v + 3]) * inv_l);
                pkt.z = sm100::pack_bf16x2(__uint_as_float(o[8 * v + 4]) * inv_l, __uint_as_float(o[8 * v + 5]) * inv_l);
                pkt.w = sm100::pack_bf16x2(__uint_as_float(o[8 * v + 6]) * inv_l, __uint_as_float(o[8 * v + 7]) * inv_l);
                dst[c * 4 + v] = pkt;
            }
        }
    }
}

// ---------------------------------------------------------------------------
// The kernel
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(320, 1) npa_fwd_kernel(const __grid_constant__ FwdParams p) {
    using C = KCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = sm100::smem_u32(smem_raw);
    uint8_t *smem = smem_raw + ((1024u - (raw & 1023u)) & 1023u);

    const Work w = decode_work(p, blockIdx.x);
    if (!q_tile_valid(p, w, w.tile0) && !q_tile_valid(p, w, w.tile0 + 1)) return;

    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::kOffBar);
    uint32_t *misc = reinterpret_cast<uint32_t *>(smem + C::kOffMisc);  // [0] TMEM base, [1] abort flag
    const int warp = threadIdx.x >> 5;

    if (threadIdx.x == 0) {
        sm100::mbar_init(&bars[C::bQFull], 1);
        for (int s = 0; s < C::kStages; ++s) {
            sm100::mbar_init(&bars[C::bKFull + s], 1);
            sm100::mbar_init(&bars[C::bKEmpty + s], 1);
            sm100::mbar_init(&bars[C::bVFull + s], 1);
            sm100::mbar_init(&bars[C::bVEmpty + s], 1);
        }
        for (int q = 0; q < 2; ++q) {
            sm100::mbar_init(&bars[C::bSFull + q], 1);
            sm100::mbar_init(&bars[C::bPFull + q], 128);
            sm100::mbar_init(&bars[C::bOFinal + q], 1);
        }
        sm100::mbar_init(&bars[C::bDrain], 1);
        misc[1] = 0;
        sm100::fence_barrier_init();
    }
    if (warp == 8) {
        sm100::tmem_alloc(&misc[0], C::kTmemCols);
        sm100::tmem_relinquish();
    }
    sm100::tc_fence_before();
    __syncthreads();
    sm100::tc_fence_after();
    const uint32_t tmem = misc[0];
    volatile uint32_t *abort_flag = &misc[1];

    if (warp == 8) {
        if ((threadIdx.x & 31) == 0) run_producer<D>(p, w, smem, bars, abort_flag);
    } else if (warp == 9) {
        if ((threadIdx.x & 31) == 0) run_mma<D>(p, w, smem, bars, tmem, abort_flag);
    } else {
        run_softmax<D>(p, w, bars, tmem, abort_flag, warp >> 2);
    }

    sm100::tc_fence_before();
    __syncthreads();
    sm100::tc_fence_after();
    if (warp == 8) {
        __syncwarp();
        sm100::tmem_dealloc(tmem, C::kTmemCols);
    }
}

// One block, one thread waiting on a barrier nothing arrives at: exercises the
// bounded-wait path and the status word without touching the GPU's health.
__global__ void npa_wait_selftest_kernel(unsigned long long limit_ns) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        sm100::mbar_init(&bar, 1);
        sm100::fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0 && !sm100::mbar_wait(&bar, 0, limit_ns)) record_error(kErrDeviceTimeout);
}

}  // namespace npa
