/*
 * svg.h -- C ABI of libsvgattn: block-sparse spatio-temporal attention forward on B200.
 *
 * The operation ("Accelerating Spatio-Temporal Attention for Video Diffusion on TPUs",
 * Google Developers Blog case study, as summarised on the three pages on the subject):
 * video-diffusion attention heads are routed either to a SPATIAL mask (keys in the same or
 * nearby frames) or to a TEMPORAL mask (keys in a narrow spatial region across all frames),
 * both keeping full attention to the first frame as a sink ("Sparse Attention Patterns";
 * "Interesting facts"). The kernel tiles the query x key plane, skips empty tiles, runs full
 * tiles without evaluating the mask and masks only boundary tiles ("Efficient Kernel
 * Implementation", tile-aware masking). Temporal heads are reordered space-major first so
 * their mask becomes regular ("Interesting facts": token ordering). An optional tile-aligned
 * variant rounds the mask to whole tiles (summary; "What changed").
 *
 * Mask, on ORIGINAL token identities (token i = t*S + s, frame t, flattened patch
 * s = y*grid_w + x, S = grid_h*grid_w, N = frames*S):
 *   spatial:  keep(i,j) <=> |t(i)-t(j)| <= frame_window  or  t(j) < sink_frames
 *   temporal: keep(i,j) <=> |s(i)-s(j)| <= spatial_band  or  t(j) < sink_frames
 * Token order (position of token (t,s)) used by a head's Q/K/V/O rows on the device:
 *   spatial heads:  t*S + s                                   (frame-major, unchanged)
 *   temporal heads, SVG_LAYOUT_SINK_PREFIX (F0 = sink_frames):
 *                   t <  F0: t*S + s ;  t >= F0: F0*S + s*(frames-F0) + (t-F0)
 *   temporal heads, SVG_LAYOUT_FULL_SPACE_MAJOR: s*frames + t
 * Tiles are bq x bk blocks of the (query position, key position) plane; a tile is FULL if
 * every in-range pair is kept, EMPTY if none is, BOUNDARY otherwise. The rounded variant
 * keeps a whole tile iff 2*kept >= in-range area, and drops it otherwise.
 *
 * Conventions for every entry point:
 *   - Tensors are contiguous [heads, tokens, d] bf16 (raw 16-bit patterns), device memory,
 *     16-byte aligned. The caller owns and allocates every buffer; the library allocates no
 *     device memory on any call.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream). All device
 *     work is enqueued asynchronously on it; only svg_tilemap_summary and svg_read_status
 *     synchronise (that stream only), and svg_attention_fwd_host, which works on host buffers
 *     through streams of its own, returns when its result is on the host.
 *   - Host arrays (`h_route`) are read during the call and may be freed when it returns.
 *   - Return value: SVG_OK (0) or a negative SVG_ERR_* code; nothing is enqueued when an
 *     argument check fails. Errors detected on the device (a wait that timed out, a tile map
 *     built for other parameters) are written to the status word (see svg_read_status).
 *   - Requires a compute capability 10.0 device (B200, sm_100a); otherwise
 *     SVG_ERR_UNSUPPORTED.
 *   - Environment (read once per process by the host code): SVG_KERNEL=ps makes the attention
 *     kernel stage P in shared memory instead of tensor memory (the same results up to
 *     rounding), for every attention entry point.
 *   - Per-device state (the streams of svg_attention_fwd_host, device attributes) is created on
 *     first use and belongs to the device's primary context: do not reset a device
 *     (cudaDeviceReset) while the library is in use on it.
 */
#ifndef SVG_H_
#define SVG_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define SVG_OK 0
#define SVG_ERR_ARG (-1)          /* bad pointer, size, shape or parameter combination */
#define SVG_ERR_UNSUPPORTED (-2)  /* not an sm_100 device, or d / tile shape not supported */
#define SVG_ERR_CUDA (-3)         /* a CUDA runtime/driver call failed */
#define SVG_ERR_TIMEOUT (-4)      /* device status: a pipeline wait exceeded its time limit */
#define SVG_ERR_WORKSPACE (-5)    /* workspace too small, or built for other parameters */

enum { SVG_ROUTE_SPATIAL = 0, SVG_ROUTE_TEMPORAL = 1 };
enum { SVG_MASK_EXACT = 0, SVG_MASK_ROUNDED = 1 };
enum { SVG_LAYOUT_SINK_PREFIX = 0, SVG_LAYOUT_FULL_SPACE_MAJOR = 1 };
/* SPLIT: full tiles unmasked, boundary tiles element-masked (the pages' fast path).
 * NAIVE: every visited tile element-masked (the pages' slower first sparse kernel). */
enum { SVG_MODE_SPLIT = 0, SVG_MODE_NAIVE = 1 };

typedef struct { int32_t frames, grid_h, grid_w; } svg_geom;

typedef struct {
    int32_t frame_window;  /* k >= 0: spatial heads keep key frames with |t_q - t_k| <= k   */
    int32_t spatial_band;  /* b >= 0: temporal heads keep keys with |s_q - s_k| <= b        */
    int32_t sink_frames;   /* F0 in [0, frames]: keys of frames [0, F0) are always kept      */
    int32_t variant;       /* SVG_MASK_EXACT or SVG_MASK_ROUNDED                            */
    int32_t layout;        /* token order of temporal heads (SVG_LAYOUT_*)                  */
} svg_mask;

typedef struct { int32_t bq, bk; } svg_tile;   /* bq in {64,128,256,512}, bk in {64,128} */

/* Byte offsets of the arrays inside a tile-map workspace (see svg_build_tilemap). */
typedef struct {
    uint64_t total_bytes;
    uint64_t cls;         /* uint8  [nq*nk]   class per tile: 0 empty, 1 full, 2 boundary   */
    uint64_t cnt;         /* uint32 [nq*nk]   EXACT retained pairs per tile                 */
    uint64_t row_ptr;     /* uint32 [nq+1]    CSR offsets of visited tiles per q-tile        */
    uint64_t cols;        /* uint32 [...]     kt | class << 30, ascending kt                 */
    uint64_t pair_ptr;    /* uint32 [np+1]    offsets of the 256-row execution lists         */
    uint64_t pair_ent;    /* uint32 [...]     kt | flagA << 28 | flagB << 30                  */
    uint64_t pair_cnt;    /* uint32 [2*np]    active entries of half 0 / half 1 of each pair  */
    uint64_t pair_order;  /* uint32 [np]      pairs by descending work, ties by index         */
    uint64_t pair_grp;    /* uint32 [2*np]    per position of pair_order: [start, end) of its run
                                              of positions with equal work                      */
    int32_t nq, nk, npairs;
} svg_tilemap_layout;

/* Totals of one built tile map (svg_tilemap_summary). */
typedef struct {
    uint64_t retained_exact;  /* kept pairs of the exact mask (layout-independent)        */
    uint64_t retained_map;    /* kept pairs of the map's own mask (= exact, or rounded)    */
    uint64_t n_full, n_boundary, n_empty;   /* tile classes of the map                      */
    uint64_t visited_area;    /* in-range pairs inside non-empty tiles                     */
    uint64_t pair_entries;    /* entries of all 256-row execution lists                    */
    uint64_t pair_half_tiles; /* active (entry, half) combinations: MMA work units          */
} svg_tilemap_summary_t;

/*
 * Size of the tile-map workspace for ONE route class (all heads of a class share it):
 * the largest the map can need for this geometry and tile shape. Returns 0 on bad args.
 */
size_t svg_tilemap_bytes(svg_geom geom, svg_tile tile);

/* Fills *out with the byte offsets used by svg_build_tilemap. Host-only, no device work. */
int svg_tilemap_get_layout(svg_geom geom, svg_tile tile, svg_tilemap_layout *out);

/*
 * Classifies every (query tile, key tile) pair of one route class as full / boundary /
 * empty (rounded variant: full / empty), counts retained pairs per tile exactly, and
 * builds: the per-q-tile CSR list of visited tiles; the execution lists used by
 * svg_attention_fwd, one per pair of 128-row query blocks (256 rows, the kernel's work item),
 * with a flag per block: 0 skip, 1 full, 2 masked, 3 full but key range past the sequence end;
 * and the pairs in descending order of work, with the runs of equal work, for the persistent
 * scheduler. Integer work only.
 *   d_ws: device buffer of at least svg_tilemap_bytes(geom, tile) bytes, 256-B aligned;
 *         written entirely by this call (also records the parameters it was built for).
 * Errors: SVG_ERR_ARG (bad geometry/mask/route), SVG_ERR_UNSUPPORTED (tile shape),
 *         SVG_ERR_WORKSPACE (ws_bytes too small), SVG_ERR_CUDA (launch failure).
 */
int svg_build_tilemap(svg_geom geom, svg_mask mask, svg_tile tile, int32_t route,
                      void *d_ws, size_t ws_bytes, void *stream);

/* Copies the totals of a built map to *h_out. Synchronises `stream`. */
int svg_tilemap_summary(const void *d_ws, svg_tilemap_summary_t *h_out, void *stream);

/*
 * Token permutation of a [heads, tokens, d] bf16 tensor (d_in != d_out, no overlap).
 * inverse = 0: out[h][pi_h(i)] = in[h][i]   (original order -> the head's order)
 * inverse = 1: out[h][i] = in[h][pi_h(i)]   (the head's order -> original order)
 * pi_h is the identity for spatial heads (rows are still copied) and the temporal order
 * selected by mask.layout / mask.sink_frames for temporal heads. h_route: host uint8
 * [heads], SVG_ROUTE_*. tokens must equal frames*grid_h*grid_w; d in {64, 128};
 * heads <= 4096. Pure data movement (HBM-bound).
 */
int svg_permute(const void *d_in, void *d_out, int32_t heads, int64_t tokens, int32_t d,
                const uint8_t *h_route, svg_geom geom, svg_mask mask, int32_t inverse,
                void *stream);

/* Bytes of scratch svg_attention_fwd / svg_dense_attention_fwd need (scheduler counter
 * and status word). The calls clear it themselves. */
size_t svg_attention_scratch_bytes(void);

/*
 * Block-sparse attention forward, flash-style (online softmax), tensor cores (tcgen05).
 *   q, k, v: [heads, tokens, d] bf16, each head's rows in that head's token order
 *            (svg_permute, inverse = 0, for temporal heads).
 *   o:       [heads, tokens, d] bf16 output in the same order (svg_permute inverse = 1
 *            restores original order for temporal heads).
 *   lse:     nullable fp32 [heads, tokens]: natural-log sum of exp of the kept scaled
 *            scores per row (-inf and O = 0 for a row with no kept key).
 *   scale:   softmax scale; <= 0 selects 1/sqrt(d).
 *   h_route: host uint8 [heads] route per head; heads <= 4096.
 *   d_ws_spatial / d_ws_temporal: tile maps built by svg_build_tilemap for the route class
 *            with the same geom, mask and tile (may be NULL if no head uses that class).
 *   mode:    SVG_MODE_SPLIT or SVG_MODE_NAIVE.
 *   d_scratch: device buffer of svg_attention_scratch_bytes() bytes (cleared by the call).
 *   d_status:  nullable device int32; receives 0 or a negative SVG_ERR_* code detected on
 *              the device. When NULL, the status word inside d_scratch is used.
 * d in {64, 128}; tile.bk selects the key-tile width the kernel streams.
 */
int svg_attention_fwd(const void *q, const void *k, const void *v, void *o, float *lse,
                      int32_t heads, int64_t tokens, int32_t d, float scale,
                      const uint8_t *h_route, const void *d_ws_spatial, const void *d_ws_temporal,
                      svg_geom geom, svg_mask mask, svg_tile tile, int32_t mode,
                      void *d_scratch, size_t scratch_bytes, int32_t *d_status, void *stream);

/*
 * Scheduling and tracing options of svg_attention_fwd_ex.
 *   order: SVG_ORDER_HEAD_MAJOR hands the persistent CTAs the work items (256 query rows of one head)
 *          head by head, each head's items heaviest first -- the order of svg_attention_fwd.
 *          SVG_ORDER_WORK hands them out by descending work over ALL heads (longest processing time
 *          first): every head of a route class has the same items, so each class's items are taken
 *          run by run of equal work, head by head within a run, and the two classes are merged by
 *          work. Results are identical; only which CTA computes which rows, and when, changes.
 *   d_cta_trace: nullable device uint64 [trace_ctas][4]; when given, the call clears it and each CTA
 *          i < trace_ctas of the launch writes {start ns, end ns (%globaltimer), items it ran, 128-row
 *          half-tiles of those items}. Give trace_ctas >= the device's SM count to see every CTA;
 *          entries of CTAs that did not run stay 0. 8-byte aligned.
 */
enum { SVG_ORDER_HEAD_MAJOR = 0, SVG_ORDER_WORK = 1 };
typedef struct {
    int32_t order;
    uint64_t *d_cta_trace;
    int32_t trace_ctas;
} svg_launch_opts;

/* svg_attention_fwd with the options above (opts must not be NULL: SVG_ERR_ARG). */
int svg_attention_fwd_ex(const void *q, const void *k, const void *v, void *o, float *lse,
                         int32_t heads, int64_t tokens, int32_t d, float scale,
                         const uint8_t *h_route, const void *d_ws_spatial, const void *d_ws_temporal,
                         svg_geom geom, svg_mask mask, svg_tile tile, int32_t mode,
                         void *d_scratch, size_t scratch_bytes, int32_t *d_status,
                         const svg_launch_opts *opts, void *stream);

/*
 * svg_attention_fwd with QK^T on the tensor core's 8-bit path: q8 and k8 are e4m3 (one byte per
 * element, [heads, tokens, d], d = 128, each head's rows in its token order -- svg_permute moves
 * e4m3 rows when called with d = 64, since a 128-byte row is 64 bf16-sized elements); v, o, lse and
 * every other argument as in svg_attention_fwd. `scale` multiplies the e4m3 dot products, so it
 * carries any quantisation scales of Q and K (<= 0: 1/sqrt(d)). The scores are the exact fp32 sums of
 * the e4m3 products; softmax, P (bf16) and P V are those of svg_attention_fwd, so the result is the
 * attention of the dequantised Q and K. Not a counterpart of anything on the pages: an opt-in
 * variant that halves the QK^T work and its shared-memory traffic. SVG_ERR_UNSUPPORTED for d != 128.
 */
int svg_attention_fwd_qk8(const void *q8, const void *k8, const void *v, void *o, float *lse,
                          int32_t heads, int64_t tokens, int32_t d, float scale,
                          const uint8_t *h_route, const void *d_ws_spatial, const void *d_ws_temporal,
                          svg_geom geom, svg_mask mask, svg_tile tile, int32_t mode,
                          void *d_scratch, size_t scratch_bytes, int32_t *d_status, void *stream);

/* Dense attention forward (every pair kept) with the same kernel and scheduler; the
 * in-repo baseline. Arguments as in svg_attention_fwd; bk in {64, 128}. */
int svg_dense_attention_fwd(const void *q, const void *k, const void *v, void *o, float *lse,
                            int32_t heads, int64_t tokens, int32_t d, float scale, int32_t bk,
                            void *d_scratch, size_t scratch_bytes, int32_t *d_status,
                            void *stream);

/*
 * Allocation-free variant of svg_attention_fwd. The case study has no counterpart; it exists for
 * callers that cannot allocate device memory themselves, e.g. a plugin inside a host
 * framework that hands it only the input and output buffers, or a server that forbids
 * device allocation after start-up because cudaMalloc may synchronise the device and
 * fragment a fixed memory budget.
 * Instead of a caller-provided scratch buffer it uses a static device array of
 * SVG_NOALLOC_SCRATCH_BYTES bytes inside the library (every device that loads the library
 * holds it until the process exits). Arguments are those of svg_attention_fwd without
 * d_scratch / scratch_bytes.
 *   - Every call looks up the array's device address (cudaGetSymbolAddress, with the caller's
 *     device current); the first lookup on a device may load the library's device code there,
 *     so make the first call on each device before any stream capture.
 *   - Every call on a device shares the one array and clears it on `stream` before its
 *     kernel runs; calls that overlap on the GPU (other streams, other host threads) race on
 *     it and must be serialised by the caller.
 *   - d_status (nullable) receives the device status as in svg_attention_fwd; without it,
 *     device-side errors are written only to the shared array and cannot be read back.
 *   - Returns SVG_ERR_ARG when the scratch the call needs exceeds SVG_NOALLOC_SCRATCH_BYTES
 *     (it needs svg_attention_scratch_bytes(), independent of the problem size), plus every
 *     error svg_attention_fwd returns. Allocates nothing (no cudaMalloc / cudaFree).
 */
#define SVG_NOALLOC_SCRATCH_BYTES 256
int svg_attention_fwd_noalloc(const void *q, const void *k, const void *v, void *o, float *lse,
                              int32_t heads, int64_t tokens, int32_t d, float scale,
                              const uint8_t *h_route, const void *d_ws_spatial,
                              const void *d_ws_temporal, svg_geom geom, svg_mask mask,
                              svg_tile tile, int32_t mode, int32_t *d_status, void *stream);

/*
 * Head routing by sampling: Sparse VideoGen profiles heads at inference time and routes each to
 * the spatial or the temporal mask based on sampled rows ("Sparse Attention Patterns"; summary of
 * the case study). For every head, the query rows listed in d_rows (ORIGINAL token indices,
 * frame-major) attend to all keys under the dense mask, the spatial mask and the temporal mask of
 * `mask` (exact variant, original token order; layout and variant are ignored): scores and the
 * three P V products on the tensor cores (bf16 operands, fp32 accumulation; P rounded to bf16 as in
 * the attention kernel), one online softmax per mask in fp32. With E_m = sum over the rows of
 * |O_m - O_dense|^2 and E_d = sum of |O_dense|^2:
 *   d_route[h] = E_spatial <= E_temporal ? SVG_ROUTE_SPATIAL : SVG_ROUTE_TEMPORAL
 *   d_err[2h], d_err[2h+1] = E_spatial / E_d, E_temporal / E_d   (d_err nullable)
 *   q, k, v:  [heads, tokens, d] bf16 in ORIGINAL order (before any permutation).
 *   d_rows:   device int32 [n_rows]; entries outside [0, tokens) are ignored.
 *   d_work:   device buffer of svg_route_work_bytes(heads, tokens, d, n_rows) bytes, 256-byte
 *             aligned: a device status word first (0, or SVG_ERR_TIMEOUT when a pipeline wait ran
 *             out; svg_read_status(d_work) reads it), then the per-row errors and the softmax
 *             state of each key chunk of each row.
 *   d_route:  device uint8 [heads].
 * The sums over rows run in a fixed order, so the decision is deterministic.
 * Errors: SVG_ERR_ARG (null or misaligned pointer, bad geometry/mask, tokens != frames*H*W),
 *   SVG_ERR_UNSUPPORTED (d not 64 or 128), SVG_ERR_WORKSPACE (work_bytes too small), SVG_ERR_CUDA.
 */
size_t svg_route_work_bytes(int32_t heads, int64_t tokens, int32_t d, int32_t n_rows);
int svg_route_heads(const void *q, const void *k, const void *v, int32_t heads, int64_t tokens,
                    int32_t d, float scale, svg_geom geom, svg_mask mask, const int32_t *d_rows,
                    int32_t n_rows, void *d_work, size_t work_bytes, uint8_t *d_route,
                    float *d_err, void *stream);

/*
 * End-to-end attention on HOST buffers: copies Q/K/V to the device, takes temporal heads to
 * their token order, runs svg_attention_fwd, takes O back to the original order and copies it
 * to the host; the same computation as svg_permute + svg_attention_fwd + svg_permute(inverse)
 * on device buffers, with bitwise-identical results. Heads go through in chunks of
 * `chunk_heads`, on three streams owned by the library (copies in, compute, copies out) and three
 * device slots, so that one chunk's copies overlap the neighbouring chunks' compute
 * ("Sources & evidence" of the case study: the pages time the attention kernel alone and leave
 * out host transfers; this call is what a user without device buffers runs).
 *   h_q, h_k, h_v: host [heads, tokens, d] bf16, ORIGINAL order. Page-locked memory
 *                  (cudaHostAlloc / cudaHostRegister) lets the copies overlap compute; pageable
 *                  memory works but serialises them.
 *   h_o:           host [heads, tokens, d] bf16 out, original order.
 *   h_route, d_ws_spatial, d_ws_temporal, geom, mask, tile, mode: as for svg_attention_fwd.
 *   chunk_heads:   heads per chunk (>= 1; values above `heads` act as `heads`).
 *   d_buf:         device buffer, 256-byte aligned, of
 *                  svg_attention_host_buffer_bytes(tokens, d, min(chunk_heads, heads)) bytes.
 * Synchronous: returns once h_o holds the result. Calls on one device are serialised (the
 * streams are shared). Returns SVG_OK, an argument error before any device work, SVG_ERR_CUDA,
 * or the first device status a chunk reported (SVG_ERR_TIMEOUT / SVG_ERR_WORKSPACE).
 */
size_t svg_attention_host_buffer_bytes(int64_t tokens, int32_t d, int32_t chunk_heads);
int svg_attention_fwd_host(const void *h_q, const void *h_k, const void *h_v, void *h_o,
                           int32_t heads, int64_t tokens, int32_t d, float scale,
                           const uint8_t *h_route, const void *d_ws_spatial,
                           const void *d_ws_temporal, svg_geom geom, svg_mask mask,
                           svg_tile tile, int32_t mode, int32_t chunk_heads, void *d_buf,
                           size_t buf_bytes);

/*
 * svg_attention_fwd with the token permutation fused into the kernel: q, k, v, o (and lse) are
 * all in the ORIGINAL frame-major order for every head, and no svg_permute pass is needed. The
 * pages' kernel runs temporal heads on permuted tokens and leaves the reordering out of its
 * timings ("routing, token permutation" excluded, "Sources & evidence"); here temporal heads
 * read each K/V/Q tile's rows where they lie (one patch's run of frames as one strided TMA box,
 * 4-row TMA gathers for the partial runs at tile edges) and write each O row back to its
 * original index, so the arithmetic, tile by tile, is that of
 * svg_permute + svg_attention_fwd + svg_permute(inverse) and the results are bitwise equal.
 * Arguments as svg_attention_fwd; lse (nullable) is [heads, tokens] in original order.
 * SVG_ERR_UNSUPPORTED when heads * tokens exceeds 2^31 - 1 (rows are gathered through a
 * [heads * tokens, d] view whose row coordinate is a signed 32-bit number).
 */
int svg_attention_fwd_fused(const void *q, const void *k, const void *v, void *o, float *lse,
                            int32_t heads, int64_t tokens, int32_t d, float scale,
                            const uint8_t *h_route, const void *d_ws_spatial,
                            const void *d_ws_temporal, svg_geom geom, svg_mask mask,
                            svg_tile tile, int32_t mode, void *d_scratch, size_t scratch_bytes,
                            int32_t *d_status, void *stream);

/*
 * Test hook, not a counterpart of anything on the pages: svg_attention_fwd whose softmax warps
 * first wait on a barrier that nothing completes. That wait gives up after its limit (2 s); the
 * launch then drains its copies and MMAs, frees its tensor memory, returns early and leaves
 * SVG_ERR_TIMEOUT in the status word. It lets the failure path run on a GPU without a fault.
 * Arguments and argument errors as svg_attention_fwd.
 */
int svg_test_attention_fwd_stall(const void *q, const void *k, const void *v, void *o, float *lse,
                                 int32_t heads, int64_t tokens, int32_t d, float scale,
                                 const uint8_t *h_route, const void *d_ws_spatial,
                                 const void *d_ws_temporal, svg_geom geom, svg_mask mask,
                                 svg_tile tile, int32_t mode, void *d_scratch, size_t scratch_bytes,
                                 int32_t *d_status, void *stream);

/* Reads the device status word of a scratch buffer (or d_status). Synchronises `stream`. */
int svg_read_status(const void *d_scratch_or_status, int32_t *h_status, void *stream);

/* Static description of an error code. */
const char *svg_error_string(int code);

/* Which CUDA call last failed on the calling thread and why (after an SVG_ERR_CUDA return);
 * "none" if none has. The string stays valid until the next failing call on that thread. */
const char *svg_last_cuda_error(void);

/*
 * Checked build (libsvgattn_checked.so, compiled with -DSVG_CHECKED=1): every kernel checks the
 * indexes it computes for global memory, tile-map arrays and TMA coordinates; a failed check is
 * counted in a device counter and the access is skipped or clamped into range (no trap). For debug
 * runs on small cases; the release build compiles the checks away.
 *   svg_checked_build(): 1 in the checked build, 0 in the release build.
 *   svg_checks_failed(): failed checks since the last reset into *h_count, cleared when reset != 0;
 *     synchronises the device. The release build sets *h_count = 0 without touching the device.
 */
int svg_checked_build(void);
int svg_checks_failed(uint32_t *h_count, int32_t reset);

/* Library version (major*10000 + minor*100 + patch). */
int svg_version(void);

#ifdef __cplusplus
}
#endif
#endif /* SVG_H_ */
