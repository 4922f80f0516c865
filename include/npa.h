/*
 * npa.h - C ABI of the B200 (sm_100a) patch-restricted self-attention library.
 *
 * The library computes the forward pass of softmax self-attention in which
 * every query token sees only a restricted, geometry-defined set of keys:
 *
 *  - Neighborhood Patch Attention (NPA). ScaleDiff: Higher-Resolution Image
 *    Synthesis via Efficient and Model-Agnostic Diffusion (atlas.scime.ai
 *    summary), opening summary and "Approach": the latent token grid is cut
 *    into non-overlapping square query patches; each patch attends to an
 *    overlapping key/value neighbourhood. Here the neighbourhood is the patch
 *    grown by `margin` tokens on every side and clipped to the grid (border
 *    windows are smaller; they are not shifted inward). When `patch` does not
 *    divide H or W the last patch row/column is smaller.
 *
 *  - Partially conditioned attention (PCPP). Partially Conditioned Patch
 *    Parallelism for Accelerated Diffusion Model Inference (pith.science
 *    review), "What carries the argument" and "Core claim": the grid is cut
 *    into `n_strips` horizontal strips of s = H / n_strips rows; a strip
 *    attends to its own rows plus the p-fraction of each adjacent strip's
 *    height that touches it (the bottom rows of the strip above, the top rows
 *    of the strip below). The row count is r = ceil(p * s) evaluated in double
 *    with a 1e-9 allowance (so 0.3 * 10 gives 3), limited to s.
 *
 *  - Either geometry may append G global tokens (for example joint text
 *    tokens) to every key/value set. Global tokens produce no output rows.
 *
 * Around these it provides the stale-row form of PCPP that runs across
 * devices, the text-query half of joint attention (global tokens as queries),
 * the overlapping-window attention NPA is compared with, and the ASG guidance
 * combine; each declaration below cites its passage.
 *
 * Arithmetic: bfloat16 inputs, float32 accumulation of Q.K^T and P.V on the
 * tensor cores, float32 online softmax with scale 1/sqrt(d), bfloat16 output
 * rounded to nearest even. Softmax probabilities are rounded to bfloat16
 * before the P.V product.
 *
 * Layouts (all row-major, contiguous, little endian, 16-byte aligned):
 *   q, k, v, o : bfloat16 [B, heads, H*W, d], token t = row*W + col
 *   global k, v: bfloat16 [B, heads, G, d]
 *
 * Ownership and ordering: the caller owns every buffer. Calls are
 * asynchronous and ordered on `stream` (NULL = the legacy default stream);
 * buffers must stay valid until the stream reaches the call. The compute
 * entry points allocate no device memory; the library's device state is one
 * status word per device (see npa_device_status) and the fixed scratch array
 * of npa_global_query_attention_fwd_noalloc. Host-side state is
 * limited to per-device capability checks, kernel attributes, that array's
 * device address (set up under a lock on first use) and a small cache of the
 * per-CTA work lists of recently launched geometries (under its own lock), so
 * the entry points are safe to call from several host threads. The first call
 * of a new geometry builds its work lists on the host (0.1-0.5 ms); later
 * calls take them from the cache.
 *
 * CUDA graphs: after a first call on a device (which checks the device and
 * sets kernel attributes), npa_attention_fwd, pcpp_attention_fwd,
 * pcpp_attention_fwd_stale, npa_global_query_attention_fwd,
 * npa_multidiffusion_attention_fwd and asg_guidance_combine may be captured in
 * a stream capture. The tensor maps are encoded on the host when the call is
 * captured, so the graph replays on the same buffers (their contents may
 * change between replays); npa_device_status synchronises and must not be
 * captured.
 *
 * Errors: every entry point validates its arguments on the host and returns a
 * status code; nothing aborts, prints or throws across this boundary. A
 * failed launch returns NPA_ERR_CUDA. Device-side waits are bounded; if one
 * runs out, the kernel stops early, leaves the output undefined and records
 * NPA_ERR_DEVICE_TIMEOUT in the device status word.
 */
#ifndef NPA_B200_H
#define NPA_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t / CUstream. */
typedef struct CUstream_st *npa_stream_t;

typedef enum {
    NPA_OK = 0,
    NPA_ERR_INVALID_ARG = 1,     /* null pointer, size < 1, bad p, overlap, H % n_strips != 0 */
    NPA_ERR_UNSUPPORTED = 2,     /* d not in {64,128}, size beyond limits, device not sm_100 */
    NPA_ERR_MISALIGNED = 3,      /* a pointer is not 16-byte aligned */
    NPA_ERR_CUDA = 4,            /* a CUDA runtime/driver call failed */
    NPA_ERR_DEVICE_TIMEOUT = 5,  /* a bounded device-side wait ran out */
    NPA_ERR_DEVICE_BOUNDS = 6    /* bounds-checking build only: a device-side bounds check failed */
} npa_status;

/* Optional global tokens appended to every key/value set.
 * k, v: bfloat16 [B, heads, n_tokens, d], device memory.
 * Pass NULL, or n_tokens = 0, for none. */
typedef struct {
    const void *k;
    const void *v;
    int n_tokens;
} npa_global_kv;

/* Neighborhood Patch Attention forward (ScaleDiff summary, "Approach").
 * q, k, v, o: device pointers, layout above; o must not overlap q, k, v or the
 * global tokens. patch >= 1 (query patch side in tokens), margin >= 0 (window
 * growth in tokens on each side). d must be 64 or 128. */
npa_status npa_attention_fwd(const void *q, const void *k, const void *v, void *o,
                             int B, int heads, int H, int W, int d, int patch, int margin,
                             const npa_global_kv *global_kv, npa_stream_t stream);

/* Partially conditioned attention forward (PCPP review, "What carries the
 * argument"). n_strips >= 1 must divide H; 0 <= p <= 1 is the partial value.
 * Other arguments as for npa_attention_fwd. */
npa_status pcpp_attention_fwd(const void *q, const void *k, const void *v, void *o,
                              int B, int heads, int H, int W, int d, int n_strips, double p,
                              const npa_global_kv *global_kv, npa_stream_t stream);

/* Partially conditioned attention with stale neighbour rows, the form PCPP
 * runs across devices (PCPP review, "Core claim": a patch is updated from its
 * own activation plus the top or bottom p-fraction of the neighbouring
 * patches from the previous denoising step). For the queries of strips
 * [strip_begin, strip_begin + strip_count) the keys/values of the query's own
 * strip are read from k, v (current step) and the borrowed neighbour rows
 * from k_stale, v_stale (previous step; same layout and size as k, v; only
 * the r rows next to each computed strip are read). Output rows of other
 * strips are left untouched. Other arguments and errors as for
 * pcpp_attention_fwd; 0 <= strip_begin, 1 <= strip_count,
 * strip_begin + strip_count <= n_strips, and o must not overlap k_stale or
 * v_stale. */
npa_status pcpp_attention_fwd_stale(const void *q, const void *k, const void *v, const void *k_stale,
                                    const void *v_stale, void *o, int B, int heads, int H, int W, int d,
                                    int n_strips, double p, int strip_begin, int strip_count,
                                    const npa_global_kv *global_kv, npa_stream_t stream);

/* Text-query half of joint (MM-DiT) attention: the G global tokens as
 * queries, each attending to all H*W image tokens and all G global tokens
 * (full attention). The pages restrict only the image-token queries
 * (ScaleDiff summary, "Approach": NPA replaces the image self-attention; it
 * extends to FLUX, whose text tokens join that attention), so the text
 * queries are left unrestricted here.
 * gq, go: bfloat16 [B, heads, G, d]; k, v: [B, heads, H*W, d]; gk, gv:
 * [B, heads, G, d] (device). The key range is split across CTAs when the
 * query tiles alone would leave most of the GPU idle; the partial results go
 * to `workspace` (caller-owned device memory, 16-byte aligned, at least
 * npa_global_query_workspace_size() bytes for the full split count; a
 * smaller or NULL workspace gives fewer or no splits - same result, less
 * parallelism) and are merged by a second kernel on the same stream. go must
 * not overlap the inputs or the workspace. */
npa_status npa_global_query_attention_fwd(const void *gq, const void *k, const void *v, const void *gk,
                                          const void *gv, void *go, int B, int heads, int H, int W, int d,
                                          int G, void *workspace, size_t workspace_bytes, npa_stream_t stream);

/* npa_global_query_attention_fwd for callers that cannot hand the library
 * device memory: for example a plugin whose host framework owns every device
 * allocation and exposes no allocator to it, or a service that forbids
 * device allocation after start-up because cudaMalloc can synchronise the
 * device and stall other work. The pages have no counterpart to this; it
 * is a deployment variant of the same computation.
 * The key-range split partials go to a fixed 16 MiB array inside the library
 * (allocated when the library is loaded, held by every GPU that loads it
 * until the process exits); nothing is allocated per call. The array must
 * hold at least two partial results, 2 * B * heads * G * (d + 2) * 4 bytes
 * <= 16 MiB, else the call returns NPA_ERR_UNSUPPORTED before touching the
 * device. This is stricter than npa_global_query_attention_fwd, which runs
 * such a problem unsplit when its workspace is too small: a caller of the
 * fixed array learns its limit from the status instead of getting a call
 * that silently loses the split's parallelism. The split count is also
 * limited by the array (FLUX's 24 heads x 512 text tokens at d = 128 run
 * with 2 splits). The
 * first call on each device looks up the array's device address (with that
 * device current) and should come before any stream capture. Every call
 * shares the array and overwrites it; nothing in it needs to start at zero.
 * Calls that overlap on the GPU (other streams, other host threads) race on
 * the array: order them on one stream. Other arguments, results and errors
 * as for npa_global_query_attention_fwd. */
npa_status npa_global_query_attention_fwd_noalloc(const void *gq, const void *k, const void *v, const void *gk,
                                                  const void *gv, void *go, int B, int heads, int H, int W,
                                                  int d, int G, npa_stream_t stream);

/* Overlapping-window attention, the comparator NPA is measured against
 * (ScaleDiff summary, "Problem" and "Approach": MultiDiffusion processes
 * overlapping patches and averages them, which inflates the attention cost;
 * NPA keeps the query patches disjoint). The overlapping patches are the NPA
 * windows: window (pi, pj) is patch (pi, pj) grown by `margin` and clipped to
 * the grid; every token of a window attends to every token of that window
 * (plus the global tokens), and a token's output is the mean, over the windows
 * that contain it, of its attention output in each. This reading of the
 * comparison at the level of one attention layer is the library's; the pages
 * compare whole pipelines.
 * Runs the attention kernel over all windows, writing each window's
 * normalised float32 output to `workspace` (caller-owned device memory,
 * 16-byte aligned, at least npa_multidiffusion_workspace_size() bytes, not
 * overlapping any other buffer), then a second kernel on the same stream that
 * averages them into o. At most 256 patches along each axis
 * (NPA_ERR_UNSUPPORTED beyond). A NULL or short workspace gives
 * NPA_ERR_INVALID_ARG. Other arguments and errors as for npa_attention_fwd. */
npa_status npa_multidiffusion_attention_fwd(const void *q, const void *k, const void *v, void *o, int B, int heads,
                                            int H, int W, int d, int patch, int margin,
                                            const npa_global_kv *global_kv, void *workspace,
                                            size_t workspace_bytes, npa_stream_t stream);

/* Workspace bytes of npa_multidiffusion_attention_fwd: 4 * d * B * heads *
 * (sum of window heights) * (sum of window widths); 0 for invalid arguments. */
size_t npa_multidiffusion_workspace_size(int B, int heads, int H, int W, int d, int patch, int margin);

/* Useful floating-point work of one npa_multidiffusion_attention_fwd call:
 * 4 * d * B * heads * sum over windows of |window| * (|window| + G). Negative
 * for invalid arguments. */
double npa_multidiffusion_useful_flops(int B, int heads, int H, int W, int d, int patch, int margin, int G);

/* Asynchronous structure guidance combine (ASGDiffusion review,
 * "core_discovery" and "key_machinery"): every patch's noise prediction is
 * pulled toward the reference patch's prediction from the previous step,
 *   out[i, b, c, s] = eps[i, b, c, s] + w_t * mask[i, b, s] * (eps_ref[b, c, s] - eps[i, b, c, s]).
 * The pages leave the mask's layout open; here it is one spatial map per
 * patch and batch element, shared by the channels. eps, out: bfloat16
 * [n_patches, B, C, S] (S = latent pixels of a patch); eps_ref: [B, C, S];
 * mask: [n_patches, B, S]; all device memory, 16-byte aligned. out may be eps
 * itself (in place) but must not otherwise overlap an input. Arithmetic in
 * float32 (one fused multiply-add), bf16 result rounded to nearest even.
 * NPA_ERR_INVALID_ARG for null pointers, sizes < 1, a non-finite w_t or an
 * overlap; NPA_ERR_MISALIGNED; NPA_ERR_UNSUPPORTED past 2^40 elements. */
npa_status asg_guidance_combine(const void *eps, const void *eps_ref, const void *mask, void *out, int n_patches,
                                int B, int C, int S, float w_t, npa_stream_t stream);

/* Workspace bytes npa_global_query_attention_fwd uses for its full split
 * count on the current device (0: no split needed, or invalid arguments). */
size_t npa_global_query_workspace_size(int B, int heads, int H, int W, int d, int G);

/* Rows a strip borrows from each adjacent strip (PCPP review, "What carries
 * the argument": p is the fraction of each neighbour patch's height that is
 * concatenated into the local key/value set; "Core claim": the top or bottom
 * p-fraction). The pages do not say how p * strip_rows is rounded; the reading
 * taken is r = ceil(p * strip_rows - 1e-9) in double, so that a product that
 * is an integer up to rounding (0.3 * 10) is not rounded up, limited to
 * [0, strip_rows]. Returns -1 if strip_rows < 1 or p is outside [0, 1]. */
int pcpp_neighbor_rows(int strip_rows, double p);

/* Useful floating-point work of one call, the numerator of the library's
 * throughput figure: 4 * d * B * heads * (sum over queries of the key-set
 * size, global keys included), i.e. two multiply-adds per (query, key,
 * channel), one for Q.K^T and one for P.V; softmax work is not counted. It
 * counts only the entries of the restricted attention matrix - the work that
 * remains once the key set is restricted (ScaleDiff summary, "Approach": the
 * neighbourhood restriction keeps the self-attention cost from growing with
 * overlapping patches; PCPP review, "What carries the argument": partial
 * conditioning shrinks the attention matrix) - not the full-attention work
 * avoided. Key-set sizes follow the geometry of npa_attention_fwd and
 * pcpp_attention_fwd. Returns a negative value for invalid geometry
 * arguments. */
double npa_useful_flops(int B, int heads, int H, int W, int d, int patch, int margin, int G);
double pcpp_useful_flops(int B, int heads, int H, int W, int d, int n_strips, double p, int G);

/* Waits for `stream`, then reads and clears the current device's status word:
 * NPA_OK, or the first device-side error recorded since the last read. */
npa_status npa_device_status(npa_stream_t stream);

/* Diagnostic: launches one block that waits on a barrier nothing ever
 * arrives at, with a bounded wait of `limit_us` microseconds (1..1000000),
 * so the bounded-wait path can be exercised without hanging a GPU. The
 * expected outcome is that npa_device_status() then returns
 * NPA_ERR_DEVICE_TIMEOUT. Returns NPA_ERR_INVALID_ARG for a bad limit. */
npa_status npa_selftest_wait_timeout(uint32_t limit_us, npa_stream_t stream);

/* Bounds-checking build (libnpa_b200_debug.so, compiled with
 * NPA_DEBUG_BOUNDS; the pages have no counterpart, this is a debugging aid
 * standing in for a memory checker). Every kernel checks each TMA box origin
 * against its tensor's extent and each output row against the output's row
 * count; a failed check records NPA_ERR_DEVICE_BOUNDS in the status word,
 * clamps the load into the tensor or skips the store, and the kernel carries
 * on. The normal library has no checks and does not export the function
 * below.
 *
 * npa_debug_withhold_arrival_once: the next npa_attention_fwd,
 * pcpp_attention_fwd, pcpp_attention_fwd_stale or
 * npa_multidiffusion_attention_fwd launch runs with bounded waits of
 * `wait_limit_us` microseconds (1..1000000), and its first CTA withholds the
 * arrival that announces the second key block's P of its last query tile.
 * That wait runs out, the CTA records NPA_ERR_DEVICE_TIMEOUT, stops issuing,
 * waits for the copies and products already issued, frees its tensor memory
 * and exits; the call's output is undefined. It exercises the kernel's abort
 * path without faulting or hanging the GPU; the next call runs normally.
 * Returns NPA_ERR_INVALID_ARG for a bad limit. */
npa_status npa_debug_withhold_arrival_once(uint32_t wait_limit_us);

/* Static, human-readable name of a status code. */
const char *npa_status_string(npa_status status);

#ifdef __cplusplus
}
#endif

#endif /* NPA_B200_H */
