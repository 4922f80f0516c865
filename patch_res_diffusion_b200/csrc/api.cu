// api.cu - host side of the C ABI declared in include/npa.h: argument
// validation, geometry resolution, TMA tensor-map encoding and the launches of
// the sm_100a kernels. Nothing here computes attention or the combines.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <climits>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "npa.h"
#include "asg_combine.cuh"
#include "md_combine.cuh"
#include "npa_fwd_kernel.cuh"

namespace {

using npa::FwdParams;

// The kernel's bounded waits give up after this long (a healthy wait is far
// below a millisecond).
constexpr unsigned long long kWaitLimitNs = 2000000000ull;

#ifdef NPA_DEBUG_BOUNDS
// Bounds-checking build: wait limit (microseconds) of the next attention
// launch whose CTA 0 withholds one arrival; 0 = none pending.
std::atomic<unsigned> g_debug_stall_us{0};
#endif

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

std::mutex g_mu;
EncodeTiledFn g_encode = nullptr;
constexpr int kMaxDevices = 64;
struct DeviceState {
    bool checked = false;
    npa_status status = NPA_ERR_UNSUPPORTED;
    int sm_count = 0;
    int l2_bytes = 0;
};
DeviceState g_dev[kMaxDevices];

// Sets an attention kernel's shared-memory limit and checks that it was
// compiled with the register count its warp roles redistribute: the softmax
// warpgroups' setmaxnreg.inc draws on the registers the block was launched
// with, and would never complete if the launch held fewer.
template <int D, bool GQ, bool MD = false>
bool prepare_kernel() {
    using C = npa::KCfg<D, 2, 128>;
    void (*kernel)(FwdParams) = npa::npa_fwd_kernel<D, 2, 128, GQ, MD>;
    cudaFuncAttributes attr;
    if (cudaFuncGetAttributes(&attr, kernel) != cudaSuccess || attr.numRegs != (int)C::kRegsLaunch) return false;
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes) == cudaSuccess;
}

// Resolves the tensor-map encoder and checks (once per device) that the
// current device is an sm_100 part; sets the kernels' shared-memory limits.
// On success *sm_count holds the device's multiprocessor count.
npa_status ensure_ready(int *sm_count = nullptr, int *l2_bytes = nullptr) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return NPA_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return NPA_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_encode) {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult qres;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &qres) != cudaSuccess ||
            qres != cudaDriverEntryPointSuccess || fn == nullptr)
            return NPA_ERR_CUDA;
        g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    }
    DeviceState &ds = g_dev[dev];
    if (!ds.checked) {
        int major = 0, minor = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
            return NPA_ERR_CUDA;
        if (cudaDeviceGetAttribute(&ds.sm_count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            ds.sm_count < 1 || cudaDeviceGetAttribute(&ds.l2_bytes, cudaDevAttrL2CacheSize, dev) != cudaSuccess)
            return NPA_ERR_CUDA;
        if (major != 10 || minor != 0) {
            ds.status = NPA_ERR_UNSUPPORTED;
        } else if (!prepare_kernel<64, false>() || !prepare_kernel<128, false>() ||
                   !prepare_kernel<64, false, true>() || !prepare_kernel<128, false, true>() ||
                   !prepare_kernel<64, true>() || !prepare_kernel<128, true>()) {
            ds.status = NPA_ERR_UNSUPPORTED;  // a kernel's compiled shape does not match its launch plan
        } else {
            ds.status = NPA_OK;
        }
        ds.checked = true;
    }
    if (sm_count) *sm_count = ds.sm_count;
    if (l2_bytes) *l2_bytes = ds.l2_bytes;
    return ds.status;
}

// The per-CTA unit lists take 0.1-0.5 ms to build on the host, so the last
// few are kept, keyed by everything they depend on.
struct SchedKey {
    int BH, H, W, G, Ph, Pw, mh, mw, kc_log2, kr, n_qblocks, patch_begin, patch_count, grid, head_major;
    bool operator==(const SchedKey &o) const { return std::memcmp(this, &o, sizeof(SchedKey)) == 0; }
};
struct SchedEntry {
    SchedKey key;
    unsigned long long used = 0;  // 0: empty
    int n_sched = 0;
    unsigned short cta_first[npa::kMaxSchedCtas + 1];
    unsigned short sched[npa::kMaxSchedUnits];
};
constexpr int kSchedCacheEntries = 8;
std::mutex g_sched_mu;
SchedEntry g_sched_cache[kSchedCacheEntries];
unsigned long long g_sched_clock = 0;

// Fills prm's per-CTA lists (npa::build_schedule), from the cache when the
// same geometry was scheduled recently.
void schedule_units(FwdParams &prm, int grid, bool head_major) {
    SchedKey key;
    std::memset(&key, 0, sizeof(key));
    key = SchedKey{prm.BH, prm.H,      prm.W,  prm.G,         prm.Ph,          prm.Pw,          prm.mh,          prm.mw,
                   prm.kc_log2, prm.kr, prm.n_qblocks, prm.patch_begin, prm.patch_count, grid, head_major ? 1 : 0};
    std::lock_guard<std::mutex> lock(g_sched_mu);
    SchedEntry *victim = &g_sched_cache[0];
    for (SchedEntry &e : g_sched_cache) {
        if (e.used && e.key == key) {
            e.used = ++g_sched_clock;
            prm.n_sched = e.n_sched;
            std::memcpy(prm.cta_first, e.cta_first, sizeof(e.cta_first));
            std::memcpy(prm.sched, e.sched, sizeof(unsigned short) * (size_t)e.n_sched);
            return;
        }
        if (e.used < victim->used) victim = &e;
    }
    npa::build_schedule(prm, grid, head_major);
    victim->key = key;
    victim->used = ++g_sched_clock;
    victim->n_sched = prm.n_sched;
    std::memcpy(victim->cta_first, prm.cta_first, sizeof(prm.cta_first));
    std::memcpy(victim->sched, prm.sched, sizeof(unsigned short) * (size_t)prm.n_sched);
}

// Rectangle form of both geometries (see npa_geometry.cuh).
struct Geo {
    int H, W, Ph, Pw, mh, mw;
};

// Sum over the patches along one axis of (patch extent) x (window extent).
long long axis_pair_sum(int L, int P, int m) {
    long long s = 0;
    for (int p0 = 0; p0 < L; p0 += P) {
        const int p1 = p0 + P < L ? p0 + P : L;
        const int w0 = p0 - m > 0 ? p0 - m : 0;
        const int w1 = p1 + m < L ? p1 + m : L;
        s += (long long)(p1 - p0) * (w1 - w0);
    }
    return s;
}

// Sum over the patches along one axis of the window extent padded to `tile`.
long long axis_window_sum(int L, int P, int m, int tile, bool padded) {
    long long s = 0;
    for (int p0 = 0; p0 < L; p0 += P) {
        const int p1 = p0 + P < L ? p0 + P : L;
        const int w0 = p0 - m > 0 ? p0 - m : 0;
        const int w1 = p1 + m < L ? p1 + m : L;
        const int e = w1 - w0;
        s += padded ? (long long)((e + tile - 1) / tile) * tile : e;
    }
    return s;
}

// Key block shape for blocks of kb keys: 2^lg columns x kb/2^lg rows, chosen
// to waste the fewest key slots over all windows (ties go to the wider box:
// longer contiguous runs).
int choose_kc_log2(const Geo &g, int kb) {
    const int top = kb == 128 ? 7 : 6;
    int best_lg = top;
    long long best_waste = LLONG_MAX;
    const long long exact = axis_window_sum(g.W, g.Pw, g.mw, 1, false) * axis_window_sum(g.H, g.Ph, g.mh, 1, false);
    for (int lg = top; lg >= top - 3; --lg) {
        const int kc = 1 << lg, kr = kb >> lg;
        const long long padded =
            axis_window_sum(g.W, g.Pw, g.mw, kc, true) * axis_window_sum(g.H, g.Ph, g.mh, kr, true);
        if (padded - exact < best_waste) {
            best_waste = padded - exact;
            best_lg = lg;
        }
    }
    return best_lg;
}

// Query tile shape: qc patch columns x qr patch rows (qc*qr <= 128), chosen to
// need the fewest tiles per patch.
void choose_q_tile(int Ph, int Pw, int *qc_out, int *qr_out) {
    const int cands[6] = {Pw < 128 ? Pw : 128, 128, 64, 32, 16, 8};
    long long best = LLONG_MAX;
    int bc = 128, br = 1;
    for (int i = 0; i < 6; ++i) {
        const int c = cands[i];
        if (c < 1 || c > 128) continue;
        int r = 128 / c;
        if (r > Ph) r = Ph;
        if (r < 1) r = 1;
        const long long tiles = (long long)((Pw + c - 1) / c) * ((Ph + r - 1) / r);
        if (tiles < best) {
            best = tiles;
            bc = c;
            br = r;
        }
    }
    *qc_out = bc;
    *qr_out = br;
}

// Overlapping-window mode: the query tile box (qc columns x qr rows, qc*qr <=
// 128) that needs the fewest tiles over all windows; windows form a grid, so
// the count is (sum over column windows of ceil(width/qc)) x (sum over row
// windows of ceil(height/qr)). tiles_c / tiles_r cover the largest window.
void choose_q_tile_md(const Geo &g, int *qc_out, int *qr_out, int *tiles_c, int *tiles_r) {
    const int nph = (g.H + g.Ph - 1) / g.Ph, npw = (g.W + g.Pw - 1) / g.Pw;
    long long best = LLONG_MAX;
    for (int qc = 128; qc >= 8; qc /= 2) {
        const int qr = 128 / qc;
        long long sc = 0, sr = 0;
        int mc = 0, mr = 0;
        for (int j = 0; j < npw; ++j) {
            const int ww = std::min(g.W, (j + 1) * g.Pw + g.mw) - std::max(0, j * g.Pw - g.mw);
            sc += (ww + qc - 1) / qc;
            mc = std::max(mc, (ww + qc - 1) / qc);
        }
        for (int i = 0; i < nph; ++i) {
            const int wh = std::min(g.H, (i + 1) * g.Ph + g.mh) - std::max(0, i * g.Ph - g.mh);
            sr += (wh + qr - 1) / qr;
            mr = std::max(mr, (wh + qr - 1) / qr);
        }
        if (sc * sr < best) {
            best = sc * sr;
            *qc_out = qc;
            *qr_out = qr;
            *tiles_c = mc;
            *tiles_r = mr;
        }
    }
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool overlaps(const void *a, size_t na, const void *b, size_t nb) {
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return x < y + nb && y < x + na;
}

bool encode(CUtensorMap *m, const void *base, cuuint32_t rank, const cuuint64_t *dims, const cuuint64_t *strides,
            const cuuint32_t *box) {
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void *>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

npa_status validate_common(const void *q, const void *k, const void *v, void *o, int B, int heads, int H, int W,
                           int d, const npa_global_kv *gkv, int *G_out) {
    if (!q || !k || !v || !o) return NPA_ERR_INVALID_ARG;
    if (B < 1 || heads < 1 || H < 1 || W < 1 || d < 1) return NPA_ERR_INVALID_ARG;
    int G = 0;
    if (gkv && gkv->n_tokens != 0) {
        if (gkv->n_tokens < 0 || !gkv->k || !gkv->v) return NPA_ERR_INVALID_ARG;
        G = gkv->n_tokens;
    }
    if (d != 64 && d != 128) return NPA_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return NPA_ERR_MISALIGNED;
    if (G && (!aligned16(gkv->k) || !aligned16(gkv->v))) return NPA_ERR_MISALIGNED;
    const long long N = (long long)H * W;
    const long long BH = (long long)B * heads;
    // tensor-map limits (strides < 2^40 bytes) and 32-bit unit/coordinate math
    if (N * d * 2 >= (1LL << 40) || BH > INT_MAX / 4 || N > INT_MAX || (long long)G * d * 2 >= (1LL << 40))
        return NPA_ERR_UNSUPPORTED;
    const size_t bytes = (size_t)(BH * N * d * 2);
    const size_t gbytes = (size_t)(BH * G * d * 2);
    if (overlaps(o, bytes, q, bytes) || overlaps(o, bytes, k, bytes) || overlaps(o, bytes, v, bytes))
        return NPA_ERR_INVALID_ARG;
    if (G && (overlaps(o, bytes, gkv->k, gbytes) || overlaps(o, bytes, gkv->v, gbytes))) return NPA_ERR_INVALID_ARG;
    *G_out = G;
    return NPA_OK;
}

// ks / vs (both or neither): previous-step keys/values for the rows of a
// window outside its patch. [patch_begin, patch_begin + patch_count): the
// patches computed, in natural numbering; patch_count < 0 means all.
npa_status launch(const void *q, const void *k, const void *v, const void *ks, const void *vs, void *o, int B,
                  int heads, int d, const Geo &g, int G, const npa_global_kv *gkv, int patch_begin, int patch_count,
                  npa_stream_t stream, float *md_part = nullptr) {
    int sm_count = 0, l2_bytes = 0;
    npa_status st = ensure_ready(&sm_count, &l2_bytes);
    if (st != NPA_OK) return st;
    const int nt = 2;  // query tiles per work unit

    FwdParams prm;
    std::memset(&prm, 0, sizeof(prm));
    prm.o = o;
    prm.H = g.H;
    prm.W = g.W;
    prm.G = G;
    prm.Ph = g.Ph;
    prm.Pw = g.Pw;
    prm.mh = g.mh;
    prm.mw = g.mw;
    prm.nPh = (g.H + g.Ph - 1) / g.Ph;
    prm.nPw = (g.W + g.Pw - 1) / g.Pw;
    if (md_part) {
        if (prm.nPh > npa::kMaxMdAxis || prm.nPw > npa::kMaxMdAxis) return NPA_ERR_UNSUPPORTED;
        choose_q_tile_md(g, &prm.qc, &prm.qr, &prm.tiles_c, &prm.tiles_r);
        prm.md = 1;
        prm.md_part = md_part;
        prm.md_rows = npa::md_axis_offset(g.H, g.Ph, g.mh, prm.nPh);
        prm.md_tw = npa::md_axis_offset(g.W, g.Pw, g.mw, prm.nPw);
    } else {
        choose_q_tile(g.Ph, g.Pw, &prm.qc, &prm.qr);
        prm.tiles_c = (g.Pw + prm.qc - 1) / prm.qc;
        prm.tiles_r = (g.Ph + prm.qr - 1) / prm.qr;
    }
    prm.kb = 128;
    prm.tiles_per_unit = nt;
    prm.kc_log2 = choose_kc_log2(g, prm.kb);
    prm.kr = prm.kb >> prm.kc_log2;
    prm.n_qblocks = (prm.tiles_c * prm.tiles_r + nt - 1) / nt;
    prm.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)d));
    prm.wait_limit_ns = kWaitLimitNs;
#ifdef NPA_DEBUG_BOUNDS
    if (const unsigned stall_us = g_debug_stall_us.exchange(0)) {
        prm.debug_stall = 1;
        prm.wait_limit_ns = stall_us * 1000ull;
    }
#endif

    if ((long long)prm.nPh * prm.nPw > INT_MAX / 4) return NPA_ERR_UNSUPPORTED;
    prm.patch_begin = patch_begin;
    prm.patch_count = patch_count < 0 ? prm.nPh * prm.nPw : patch_count;
    prm.two_source = ks != nullptr;
    const long long units = (long long)B * heads * prm.patch_count * prm.n_qblocks;
    if (units > INT_MAX / 2) return NPA_ERR_UNSUPPORTED;

    const int BH = B * heads;
    prm.BH = BH;
    prm.n_units = (int)units;
    npa::order_patches(prm);
    // persistent grid: one CTA per multiprocessor (shared memory and TMEM
    // admit one), each walking its host-built list of units (or every
    // gridDim.x-th unit); when the keys and values of all heads do not fit in
    // L2, the lists run head by head
    const unsigned grid = (unsigned)(units < sm_count ? units : sm_count);
    if (!md_part) {
        const double kv_bytes = 4.0 * BH * (double)g.H * g.W * d + 4.0 * BH * (double)G * d;
        schedule_units(prm, (int)grid, kv_bytes > (double)l2_bytes);
    }
    const cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)g.W, (cuuint64_t)g.H, (cuuint64_t)BH};
    const cuuint64_t strides[3] = {(cuuint64_t)d * 2, (cuuint64_t)g.W * d * 2, (cuuint64_t)g.H * g.W * d * 2};
    const cuuint32_t qbox[4] = {64, (cuuint32_t)prm.qc, (cuuint32_t)prm.qr, 1};
    const cuuint32_t kbox[4] = {64, (cuuint32_t)(1 << prm.kc_log2), (cuuint32_t)prm.kr, 1};
    if (!encode(&prm.tm_q, q, 4, dims, strides, qbox) || !encode(&prm.tm_k, k, 4, dims, strides, kbox) ||
        !encode(&prm.tm_v, v, 4, dims, strides, kbox))
        return NPA_ERR_CUDA;
    if (ks && (!encode(&prm.tm_ks, ks, 4, dims, strides, kbox) || !encode(&prm.tm_vs, vs, 4, dims, strides, kbox)))
        return NPA_ERR_CUDA;
    if (G > 0) {
        const cuuint64_t gdims[3] = {(cuuint64_t)d, (cuuint64_t)G, (cuuint64_t)BH};
        const cuuint64_t gstrides[2] = {(cuuint64_t)d * 2, (cuuint64_t)G * d * 2};
        const cuuint32_t gbox[3] = {64, (cuuint32_t)prm.kb, 1};
        if (!encode(&prm.tm_gk, gkv->k, 3, gdims, gstrides, gbox) ||
            !encode(&prm.tm_gv, gkv->v, 3, gdims, gstrides, gbox))
            return NPA_ERR_CUDA;
    }

    void *args[1] = {&prm};
    cudaError_t e;
    const void *kernel;
    unsigned threads, smem;
    if (d == 64 && md_part) {
        kernel = (const void *)npa::npa_fwd_kernel<64, 2, 128, false, true>;
        threads = npa::KCfg<64, 2, 128>::kThreads;
        smem = npa::KCfg<64, 2, 128>::kSmemBytes;
    } else if (d == 128 && md_part) {
        kernel = (const void *)npa::npa_fwd_kernel<128, 2, 128, false, true>;
        threads = npa::KCfg<128, 2, 128>::kThreads;
        smem = npa::KCfg<128, 2, 128>::kSmemBytes;
    } else if (d == 64) {
        kernel = (const void *)npa::npa_fwd_kernel<64, 2, 128, false>;
        threads = npa::KCfg<64, 2, 128>::kThreads;
        smem = npa::KCfg<64, 2, 128>::kSmemBytes;
    } else {
        kernel = (const void *)npa::npa_fwd_kernel<128, 2, 128, false>;
        threads = npa::KCfg<128, 2, 128>::kThreads;
        smem = npa::KCfg<128, 2, 128>::kSmemBytes;
    }
    e = cudaLaunchKernel(kernel, dim3(grid), dim3(threads), args, smem, (cudaStream_t)stream);
    if (e != cudaSuccess) return NPA_ERR_CUDA;
    if (md_part) {
        npa::MdCombineParams cp;
        std::memset(&cp, 0, sizeof(cp));
        cp.part = md_part;
        cp.o = static_cast<__nv_bfloat16 *>(o);
        cp.H = g.H;
        cp.W = g.W;
        cp.Ph = g.Ph;
        cp.Pw = g.Pw;
        cp.mh = g.mh;
        cp.mw = g.mw;
        cp.nPh = prm.nPh;
        cp.nPw = prm.nPw;
        cp.BH = BH;
        cp.md_rows = prm.md_rows;
        cp.md_tw = prm.md_tw;
        for (int i = 0; i < prm.nPh; ++i) cp.rh[i] = npa::md_axis_offset(g.H, g.Ph, g.mh, i);
        for (int j = 0; j < prm.nPw; ++j) cp.cw[j] = npa::md_axis_offset(g.W, g.Pw, g.mw, j);
        void *cargs[1] = {&cp};
        const long long tokens = (long long)BH * g.H * g.W;
        const long long per_block = 256 / (d / 4);  // tokens per 256-thread block
        const dim3 cgrid((unsigned)((tokens + per_block - 1) / per_block));
        if (d == 64)
            e = cudaLaunchKernel((const void *)npa::md_combine_kernel<64>, cgrid, dim3(256), cargs, 0,
                                 (cudaStream_t)stream);
        else
            e = cudaLaunchKernel((const void *)npa::md_combine_kernel<128>, cgrid, dim3(256), cargs, 0,
                                 (cudaStream_t)stream);
        if (e != cudaSuccess) return NPA_ERR_CUDA;
    }
    return NPA_OK;
}

// ---------------------------------------------------------------------------
// Global-token queries (text-query half of joint attention)
// ---------------------------------------------------------------------------
struct GqPlan {
    int kc_log2, kr, n_blocks, n_qblocks, base_units, splits;
    size_t split_bytes;  // workspace bytes per key-range split
};

GqPlan plan_gq(int B, int heads, int H, int W, int d, int G, int sm_count) {
    GqPlan pl;
    const Geo g{H, W, H, W, 0, 0};
    pl.kc_log2 = choose_kc_log2(g, 128);
    pl.kr = 128 >> pl.kc_log2;
    pl.n_blocks = ((W + (1 << pl.kc_log2) - 1) >> pl.kc_log2) * ((H + pl.kr - 1) / pl.kr) + (G + 127) / 128;
    const int tiles = (G + 127) / 128;
    pl.n_qblocks = (tiles + 1) / 2;
    pl.base_units = B * heads * pl.n_qblocks;
    // split the key range until the units roughly fill the GPU once
    int s = (sm_count + pl.base_units / 2) / pl.base_units;
    if (s < 1) s = 1;
    if (s > 16) s = 16;
    if (s > pl.n_blocks) s = pl.n_blocks;
    pl.splits = s;
    pl.split_bytes = (size_t)B * heads * G * (d + 2) * sizeof(float);
    return pl;
}

npa_status launch_gq(const void *gq, const void *k, const void *v, const void *gk, const void *gv, void *go, int B,
                     int heads, int H, int W, int d, int G, float *o_part, float *ml, int splits, int sm_count,
                     npa_stream_t stream) {
    const GqPlan pl = plan_gq(B, heads, H, W, d, G, sm_count);
    FwdParams prm;
    std::memset(&prm, 0, sizeof(prm));
    prm.o = go;
    prm.H = H;
    prm.W = W;
    prm.G = G;
    prm.Ph = H;
    prm.Pw = W;
    prm.nPh = prm.nPw = 1;
    prm.kb = 128;
    prm.tiles_per_unit = 2;
    prm.kc_log2 = pl.kc_log2;
    prm.kr = pl.kr;
    prm.n_qblocks = pl.n_qblocks;
    prm.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)d));
    prm.wait_limit_ns = kWaitLimitNs;
    prm.BH = B * heads;
    prm.n_splits = splits;
    prm.gq_tiles = (G + 127) / 128;
    prm.o_part = o_part;
    prm.ml = ml;
    const long long units = (long long)prm.BH * pl.n_qblocks * splits;
    if (units > INT_MAX / 2) return NPA_ERR_UNSUPPORTED;
    prm.n_units = (int)units;
    const cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)W, (cuuint64_t)H, (cuuint64_t)prm.BH};
    const cuuint64_t strides[3] = {(cuuint64_t)d * 2, (cuuint64_t)W * d * 2, (cuuint64_t)H * W * d * 2};
    const cuuint32_t kbox[4] = {64, (cuuint32_t)(1 << pl.kc_log2), (cuuint32_t)pl.kr, 1};
    const cuuint64_t gdims[3] = {(cuuint64_t)d, (cuuint64_t)G, (cuuint64_t)prm.BH};
    const cuuint64_t gstrides[2] = {(cuuint64_t)d * 2, (cuuint64_t)G * d * 2};
    const cuuint32_t gbox[3] = {64, 128, 1};
    if (!encode(&prm.tm_k, k, 4, dims, strides, kbox) || !encode(&prm.tm_v, v, 4, dims, strides, kbox) ||
        !encode(&prm.tm_gk, gk, 3, gdims, gstrides, gbox) || !encode(&prm.tm_gv, gv, 3, gdims, gstrides, gbox) ||
        !encode(&prm.tm_gq, gq, 3, gdims, gstrides, gbox))
        return NPA_ERR_CUDA;
    const unsigned grid = (unsigned)(units < sm_count ? units : sm_count);
    void *args[1] = {&prm};
    cudaError_t e;
    if (d == 64) {
        using C = npa::KCfg<64, 2, 128>;
        e = cudaLaunchKernel((const void *)npa::npa_fwd_kernel<64, 2, 128, true>, dim3(grid), dim3(C::kThreads),
                             args, C::kSmemBytes, (cudaStream_t)stream);
    } else {
        using C = npa::KCfg<128, 2, 128>;
        e = cudaLaunchKernel((const void *)npa::npa_fwd_kernel<128, 2, 128, true>, dim3(grid), dim3(C::kThreads),
                             args, C::kSmemBytes, (cudaStream_t)stream);
    }
    if (e != cudaSuccess) return NPA_ERR_CUDA;
    if (splits > 1) {
        const int rows = prm.BH * G;
        const float *op = o_part, *mlp = ml;
        __nv_bfloat16 *gop = static_cast<__nv_bfloat16 *>(go);
        int ns = splits, nr = rows;
        void *cargs[5] = {&op, &mlp, &gop, &ns, &nr};
        const dim3 cgrid((unsigned)((rows + 7) / 8));
        if (d == 64)
            e = cudaLaunchKernel((const void *)npa::gq_combine_kernel<64>, cgrid, dim3(256), cargs, 0,
                                 (cudaStream_t)stream);
        else
            e = cudaLaunchKernel((const void *)npa::gq_combine_kernel<128>, cgrid, dim3(256), cargs, 0,
                                 (cudaStream_t)stream);
        if (e != cudaSuccess) return NPA_ERR_CUDA;
    }
    return NPA_OK;
}

npa_status validate_gq(const void *gq, const void *k, const void *v, const void *gk, const void *gv, void *go,
                       int B, int heads, int H, int W, int d, int G) {
    if (!gq || !k || !v || !gk || !gv || !go) return NPA_ERR_INVALID_ARG;
    if (B < 1 || heads < 1 || H < 1 || W < 1 || G < 1) return NPA_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return NPA_ERR_UNSUPPORTED;
    if (!aligned16(gq) || !aligned16(k) || !aligned16(v) || !aligned16(gk) || !aligned16(gv) || !aligned16(go))
        return NPA_ERR_MISALIGNED;
    const long long N = (long long)H * W, BH = (long long)B * heads;
    if (N * d * 2 >= (1LL << 40) || BH > INT_MAX / 64 || N > INT_MAX || (long long)G * d * 2 >= (1LL << 40) ||
        BH * G > INT_MAX / 2)
        return NPA_ERR_UNSUPPORTED;
    const size_t gbytes = (size_t)(BH * G * d * 2), ibytes = (size_t)(BH * N * d * 2);
    if (overlaps(go, gbytes, gq, gbytes) || overlaps(go, gbytes, gk, gbytes) || overlaps(go, gbytes, gv, gbytes) ||
        overlaps(go, gbytes, k, ibytes) || overlaps(go, gbytes, v, ibytes))
        return NPA_ERR_INVALID_ARG;
    return NPA_OK;
}

// ---------------------------------------------------------------------------
// Fixed scratch for npa_global_query_attention_fwd_noalloc: the key-range
// split partials live in this file-scope device array instead of caller
// memory. Every GPU that loads the library holds it until the process exits.
// In host code g_noalloc_scratch only stands for the symbol; its device
// address is fetched once per device with cudaGetSymbolAddress (with that
// device current) and passed to the kernels.
// ---------------------------------------------------------------------------
constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];
void *g_noalloc_addr[kMaxDevices] = {};

int neighbor_rows(int s, double p) {
    if (s < 1 || !(p >= 0.0) || !(p <= 1.0)) return -1;
    int r = (int)std::ceil(p * (double)s - 1e-9);
    if (r < 0) r = 0;
    if (r > s) r = s;
    return r;
}

// Overlapping-window mode: bytes of float32 window partials.
size_t md_workspace_bytes(int B, int heads, int H, int W, int d, int patch, int margin) {
    const long long rows = npa::md_axis_offset(H, patch, margin, (H + patch - 1) / patch);
    const long long cols = npa::md_axis_offset(W, patch, margin, (W + patch - 1) / patch);
    return (size_t)B * heads * rows * cols * d * sizeof(float);
}

double useful_flops(int B, int heads, int d, const Geo &g, int G) {
    const double pairs = (double)axis_pair_sum(g.H, g.Ph, g.mh) * (double)axis_pair_sum(g.W, g.Pw, g.mw) +
                         (double)g.H * g.W * G;
    return 4.0 * d * (double)B * heads * pairs;
}

}  // namespace

extern "C" {

npa_status npa_attention_fwd(const void *q, const void *k, const void *v, void *o, int B, int heads, int H, int W,
                             int d, int patch, int margin, const npa_global_kv *global_kv, npa_stream_t stream) {
    int G = 0;
    npa_status st = validate_common(q, k, v, o, B, heads, H, W, d, global_kv, &G);
    if (st != NPA_OK) return st;
    if (patch < 1 || margin < 0) return NPA_ERR_INVALID_ARG;
    const Geo g{H, W, patch, patch, margin, margin};
    return launch(q, k, v, nullptr, nullptr, o, B, heads, d, g, G, global_kv, 0, -1, stream);
}

npa_status pcpp_attention_fwd(const void *q, const void *k, const void *v, void *o, int B, int heads, int H, int W,
                              int d, int n_strips, double p, const npa_global_kv *global_kv, npa_stream_t stream) {
    int G = 0;
    npa_status st = validate_common(q, k, v, o, B, heads, H, W, d, global_kv, &G);
    if (st != NPA_OK) return st;
    if (n_strips < 1 || H % n_strips != 0 || !(p >= 0.0) || !(p <= 1.0)) return NPA_ERR_INVALID_ARG;
    const int s = H / n_strips;
    const Geo g{H, W, s, W, neighbor_rows(s, p), 0};
    return launch(q, k, v, nullptr, nullptr, o, B, heads, d, g, G, global_kv, 0, -1, stream);
}

npa_status pcpp_attention_fwd_stale(const void *q, const void *k, const void *v, const void *k_stale,
                                    const void *v_stale, void *o, int B, int heads, int H, int W, int d, int n_strips,
                                    double p, int strip_begin, int strip_count, const npa_global_kv *global_kv,
                                    npa_stream_t stream) {
    int G = 0;
    npa_status st = validate_common(q, k, v, o, B, heads, H, W, d, global_kv, &G);
    if (st != NPA_OK) return st;
    if (!k_stale || !v_stale) return NPA_ERR_INVALID_ARG;
    if (!aligned16(k_stale) || !aligned16(v_stale)) return NPA_ERR_MISALIGNED;
    const size_t bytes = (size_t)B * heads * H * W * d * 2;
    if (overlaps(o, bytes, k_stale, bytes) || overlaps(o, bytes, v_stale, bytes)) return NPA_ERR_INVALID_ARG;
    if (n_strips < 1 || H % n_strips != 0 || !(p >= 0.0) || !(p <= 1.0)) return NPA_ERR_INVALID_ARG;
    if (strip_begin < 0 || strip_count < 1 || strip_begin > n_strips - strip_count) return NPA_ERR_INVALID_ARG;
    const int s = H / n_strips;
    const Geo g{H, W, s, W, neighbor_rows(s, p), 0};
    return launch(q, k, v, k_stale, v_stale, o, B, heads, d, g, G, global_kv, strip_begin, strip_count, stream);
}

size_t npa_global_query_workspace_size(int B, int heads, int H, int W, int d, int G) {
    if (B < 1 || heads < 1 || H < 1 || W < 1 || G < 1 || (d != 64 && d != 128)) return 0;
    int dev = 0, sm = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return 0;
    const GqPlan pl = plan_gq(B, heads, H, W, d, G, sm);
    return pl.splits > 1 ? (size_t)pl.splits * pl.split_bytes : 0;
}

npa_status npa_global_query_attention_fwd(const void *gq, const void *k, const void *v, const void *gk,
                                          const void *gv, void *go, int B, int heads, int H, int W, int d, int G,
                                          void *workspace, size_t workspace_bytes, npa_stream_t stream) {
    npa_status st = validate_gq(gq, k, v, gk, gv, go, B, heads, H, W, d, G);
    if (st != NPA_OK) return st;
    if (workspace && !aligned16(workspace)) return NPA_ERR_MISALIGNED;
    int sm_count = 0;
    st = ensure_ready(&sm_count);
    if (st != NPA_OK) return st;
    const GqPlan pl = plan_gq(B, heads, H, W, d, G, sm_count);
    // as many splits as planned and as the workspace holds (one needs none)
    int splits = workspace ? (int)(workspace_bytes / pl.split_bytes) : 1;
    if (splits > pl.splits) splits = pl.splits;
    if (splits < 2) splits = 1;
    float *o_part = static_cast<float *>(workspace);
    float *ml = splits > 1 ? o_part + (size_t)splits * B * heads * G * d : nullptr;
    if (splits > 1) {
        const size_t wsz = (size_t)splits * pl.split_bytes;
        const size_t gbytes = (size_t)B * heads * G * d * 2;
        if (overlaps(workspace, wsz, go, gbytes) || overlaps(workspace, wsz, gq, gbytes)) return NPA_ERR_INVALID_ARG;
    }
    return launch_gq(gq, k, v, gk, gv, go, B, heads, H, W, d, G, o_part, ml, splits, sm_count, stream);
}

npa_status npa_global_query_attention_fwd_noalloc(const void *gq, const void *k, const void *v, const void *gk,
                                                  const void *gv, void *go, int B, int heads, int H, int W, int d,
                                                  int G, npa_stream_t stream) {
    npa_status st = validate_gq(gq, k, v, gk, gv, go, B, heads, H, W, d, G);
    if (st != NPA_OK) return st;
    // the array must hold at least two partial results (the smallest split);
    // the limit does not depend on the device, so it is checked first
    const size_t per_split = (size_t)B * heads * G * (d + 2) * sizeof(float);
    if (2 * per_split > kNoAllocScratchBytes) return NPA_ERR_UNSUPPORTED;
    int sm_count = 0;
    st = ensure_ready(&sm_count);
    if (st != NPA_OK) return st;
    const GqPlan pl = plan_gq(B, heads, H, W, d, G, sm_count);
    int splits = 1;
    if (pl.splits > 1) {
        splits = (int)(kNoAllocScratchBytes / per_split);
        if (splits > pl.splits) splits = pl.splits;
    }
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return NPA_ERR_CUDA;
    void *base = nullptr;
    {
        std::lock_guard<std::mutex> lock(g_mu);
        if (!g_noalloc_addr[dev]) {
            void *ptr = nullptr;
            if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || ptr == nullptr) return NPA_ERR_CUDA;
            g_noalloc_addr[dev] = ptr;
        }
        base = g_noalloc_addr[dev];
    }
    float *o_part = splits > 1 ? static_cast<float *>(base) : nullptr;
    float *ml = splits > 1 ? o_part + (size_t)splits * B * heads * G * d : nullptr;
    return launch_gq(gq, k, v, gk, gv, go, B, heads, H, W, d, G, o_part, ml, splits, sm_count, stream);
}

size_t npa_multidiffusion_workspace_size(int B, int heads, int H, int W, int d, int patch, int margin) {
    if (B < 1 || heads < 1 || H < 1 || W < 1 || patch < 1 || margin < 0 || (d != 64 && d != 128)) return 0;
    return md_workspace_bytes(B, heads, H, W, d, patch, margin);
}

npa_status npa_multidiffusion_attention_fwd(const void *q, const void *k, const void *v, void *o, int B, int heads,
                                            int H, int W, int d, int patch, int margin,
                                            const npa_global_kv *global_kv, void *workspace,
                                            size_t workspace_bytes, npa_stream_t stream) {
    int G = 0;
    npa_status st = validate_common(q, k, v, o, B, heads, H, W, d, global_kv, &G);
    if (st != NPA_OK) return st;
    if (patch < 1 || margin < 0 || !workspace) return NPA_ERR_INVALID_ARG;
    if (!aligned16(workspace)) return NPA_ERR_MISALIGNED;
    const long long nph = (H + patch - 1) / patch, npw = (W + patch - 1) / patch;
    if (nph > npa::kMaxMdAxis || npw > npa::kMaxMdAxis) return NPA_ERR_UNSUPPORTED;
    const size_t need = md_workspace_bytes(B, heads, H, W, d, patch, margin);
    if (workspace_bytes < need) return NPA_ERR_INVALID_ARG;
    const size_t bytes = (size_t)B * heads * H * W * d * 2, gbytes = (size_t)B * heads * G * d * 2;
    if (overlaps(workspace, need, q, bytes) || overlaps(workspace, need, k, bytes) ||
        overlaps(workspace, need, v, bytes) || overlaps(workspace, need, o, bytes))
        return NPA_ERR_INVALID_ARG;
    if (G && (overlaps(workspace, need, global_kv->k, gbytes) || overlaps(workspace, need, global_kv->v, gbytes)))
        return NPA_ERR_INVALID_ARG;
    const Geo g{H, W, patch, patch, margin, margin};
    return launch(q, k, v, nullptr, nullptr, o, B, heads, d, g, G, global_kv, 0, -1, stream,
                  static_cast<float *>(workspace));
}

double npa_multidiffusion_useful_flops(int B, int heads, int H, int W, int d, int patch, int margin, int G) {
    if (B < 1 || heads < 1 || H < 1 || W < 1 || d < 1 || patch < 1 || margin < 0 || G < 0) return -1.0;
    double s1r = 0, s2r = 0, s1c = 0, s2c = 0;
    for (int i = 0; i < (H + patch - 1) / patch; ++i) {
        const double w = std::min(H, (i + 1) * patch + margin) - std::max(0, i * patch - margin);
        s1r += w;
        s2r += w * w;
    }
    for (int j = 0; j < (W + patch - 1) / patch; ++j) {
        const double w = std::min(W, (j + 1) * patch + margin) - std::max(0, j * patch - margin);
        s1c += w;
        s2c += w * w;
    }
    return 4.0 * d * (double)B * heads * (s2r * s2c + G * s1r * s1c);
}

npa_status asg_guidance_combine(const void *eps, const void *eps_ref, const void *mask, void *out, int n_patches,
                                int B, int C, int S, float w_t, npa_stream_t stream) {
    if (!eps || !eps_ref || !mask || !out) return NPA_ERR_INVALID_ARG;
    if (n_patches < 1 || B < 1 || C < 1 || S < 1 || !std::isfinite(w_t)) return NPA_ERR_INVALID_ARG;
    if (!aligned16(eps) || !aligned16(eps_ref) || !aligned16(mask) || !aligned16(out)) return NPA_ERR_MISALIGNED;
    const long long nb = (long long)n_patches * B;
    if (nb * C > (1LL << 40) / S || nb > INT_MAX) return NPA_ERR_UNSUPPORTED;
    const size_t e_bytes = (size_t)nb * C * S * 2, r_bytes = (size_t)B * C * S * 2, m_bytes = (size_t)nb * S * 2;
    if (out != eps && overlaps(out, e_bytes, eps, e_bytes)) return NPA_ERR_INVALID_ARG;
    if (overlaps(out, e_bytes, eps_ref, r_bytes) || overlaps(out, e_bytes, mask, m_bytes)) return NPA_ERR_INVALID_ARG;
    int sm_count = 0;
    const npa_status st = ensure_ready(&sm_count);
    if (st != NPA_OK) return st;
    npa::AsgParams prm;
    prm.eps = static_cast<const __nv_bfloat16 *>(eps);
    prm.ref = static_cast<const __nv_bfloat16 *>(eps_ref);
    prm.mask = static_cast<const __nv_bfloat16 *>(mask);
    prm.out = static_cast<__nv_bfloat16 *>(out);
    prm.B = B;
    prm.C = C;
    prm.S = S;
    prm.chunks = (S + 7) / 8;
    prm.n_items = nb * prm.chunks;
    prm.w = w_t;
    prm.vec = S % 8 == 0;
    // enough blocks for every chunk, at most 8 resident 256-thread blocks per
    // multiprocessor (the kernel strides over the rest)
    const long long blocks = (prm.n_items + 255) / 256;
    const unsigned grid = (unsigned)(blocks < 8LL * sm_count ? blocks : 8LL * sm_count);
    void *args[1] = {&prm};
    const cudaError_t e =
        cudaLaunchKernel((const void *)npa::asg_combine_kernel, dim3(grid), dim3(256), args, 0, (cudaStream_t)stream);
    return e == cudaSuccess ? NPA_OK : NPA_ERR_CUDA;
}

int pcpp_neighbor_rows(int strip_rows, double p) { return neighbor_rows(strip_rows, p); }

double npa_useful_flops(int B, int heads, int H, int W, int d, int patch, int margin, int G) {
    if (B < 1 || heads < 1 || H < 1 || W < 1 || d < 1 || patch < 1 || margin < 0 || G < 0) return -1.0;
    return useful_flops(B, heads, d, Geo{H, W, patch, patch, margin, margin}, G);
}

double pcpp_useful_flops(int B, int heads, int H, int W, int d, int n_strips, double p, int G) {
    if (B < 1 || heads < 1 || H < 1 || W < 1 || d < 1 || n_strips < 1 || H % n_strips != 0 || G < 0) return -1.0;
    const int s = H / n_strips;
    const int r = neighbor_rows(s, p);
    if (r < 0) return -1.0;
    return useful_flops(B, heads, d, Geo{H, W, s, W, r, 0}, G);
}

npa_status npa_device_status(npa_stream_t stream) {
    if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return NPA_ERR_CUDA;
    unsigned int v = 0;
    if (cudaMemcpyFromSymbol(&v, npa::g_npa_status, sizeof(v)) != cudaSuccess) return NPA_ERR_CUDA;
    if (v != 0) {
        const unsigned int zero = 0;
        if (cudaMemcpyToSymbol(npa::g_npa_status, &zero, sizeof(zero)) != cudaSuccess) return NPA_ERR_CUDA;
    }
    return (npa_status)v;
}

npa_status npa_selftest_wait_timeout(uint32_t limit_us, npa_stream_t stream) {
    if (limit_us < 1 || limit_us > 1000000) return NPA_ERR_INVALID_ARG;
    npa_status st = ensure_ready();
    if (st != NPA_OK) return st;
    unsigned long long ns = (unsigned long long)limit_us * 1000ull;
    void *args[1] = {&ns};
    cudaError_t e = cudaLaunchKernel((const void *)npa::npa_wait_selftest_kernel, dim3(1), dim3(32), args, 0,
                                     (cudaStream_t)stream);
    return e == cudaSuccess ? NPA_OK : NPA_ERR_CUDA;
}

#ifdef NPA_DEBUG_BOUNDS
npa_status npa_debug_withhold_arrival_once(uint32_t wait_limit_us) {
    if (wait_limit_us < 1 || wait_limit_us > 1000000) return NPA_ERR_INVALID_ARG;
    g_debug_stall_us.store(wait_limit_us);
    return NPA_OK;
}
#endif

const char *npa_status_string(npa_status status) {
    switch (status) {
        case NPA_OK: return "NPA_OK";
        case NPA_ERR_INVALID_ARG: return "NPA_ERR_INVALID_ARG";
        case NPA_ERR_UNSUPPORTED: return "NPA_ERR_UNSUPPORTED";
        case NPA_ERR_MISALIGNED: return "NPA_ERR_MISALIGNED";
        case NPA_ERR_CUDA: return "NPA_ERR_CUDA";
        case NPA_ERR_DEVICE_TIMEOUT: return "NPA_ERR_DEVICE_TIMEOUT";
        case NPA_ERR_DEVICE_BOUNDS: return "NPA_ERR_DEVICE_BOUNDS";
    }
    return "NPA_ERR_UNKNOWN";
}

}  // extern "C"
