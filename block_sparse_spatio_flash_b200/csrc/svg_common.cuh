// svg_common.cuh -- shared definitions of the libsvgattn CUDA sources (sm_100a only).
//
//  * MaskGeom: the spatial / temporal masks of the Sparse-VideoGen routing as described in
//    "Accelerating Spatio-Temporal Attention for Video Diffusion on TPUs" ("Sparse Attention
//    Patterns": spatial heads look at the same or nearby frames, temporal heads at a narrow
//    spatial region across frames; "Interesting facts": both keep the first frame as a sink,
//    temporal heads need their own token order), expressed in POSITION space: for a query at
//    position p the kept keys are [0, sink_end) U [lo(p), hi(p)) U (periodic sink), a form that
//    makes tile classification O(1) per row and boundary masking a few compares per element.
//  * TmHeader: the record at the start of a tile-map workspace.
//  * Thin inline-PTX wrappers for mbarrier, TMA (cp.async.bulk.tensor) and tcgen05.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/svg.h"

namespace svg {

constexpr uint32_t kTmMagic = 0x53564731u;  // "SVG1"
constexpr int kMaxHeads = 4096;
constexpr int64_t kMaxTokens = 1 << 22;
constexpr int kPairRows = 256;  // query rows per item of the attention kernel: two 128-row halves
constexpr int kHalfRows = 128;

// Checked build (-DSVG_CHECKED=1, the library libsvgattn_checked.so): device-side bounds checks on
// the indexes the kernels compute for global memory, tile-map arrays and TMA coordinates. A failed
// check adds one to a device counter (svg_checks_failed reads it) and the access is skipped or its
// index clamped into range; nothing traps. In the release build every check compiles away.
#ifndef SVG_CHECKED
#define SVG_CHECKED 0
#endif

// ---------------------------------------------------------------------------------------
// Mask geometry in position space.
struct MaskGeom {
  int T, S, N;        // frames, tokens per frame, tokens
  int k, b, F0;       // frame window, spatial band, sink frames
  int route, layout;  // SVG_ROUTE_*, SVG_LAYOUT_* (layout only matters for temporal heads)
};

__host__ __device__ inline MaskGeom make_geom(const svg_geom& g, const svg_mask& m, int route) {
  MaskGeom r;
  r.T = g.frames;
  r.S = g.grid_h * g.grid_w;
  r.N = r.T * r.S;
  r.k = m.frame_window;
  r.b = m.spatial_band;
  r.F0 = m.sink_frames;
  r.route = route;
  r.layout = m.layout;
  return r;
}

// True when the head's sink is the periodic set {c : c mod T < F0} (fully space-major order).
__host__ __device__ inline bool periodic_sink(const MaskGeom& g) {
  return g.route == SVG_ROUTE_TEMPORAL && g.layout == SVG_LAYOUT_FULL_SPACE_MAJOR && g.F0 > 0;
}

// End of the contiguous sink prefix [0, sink_end) of key positions.
__host__ __device__ inline int sink_end(const MaskGeom& g) {
  if (g.route == SVG_ROUTE_TEMPORAL && g.layout == SVG_LAYOUT_FULL_SPACE_MAJOR) return 0;
  return g.F0 * g.S;
}

// (frame, patch) of the token at position p of this head's order.
__host__ __device__ inline void pos_to_ts(const MaskGeom& g, int p, int& t, int& s) {
  if (g.route == SVG_ROUTE_SPATIAL) {
    t = p / g.S;
    s = p - t * g.S;
    return;
  }
  if (g.layout == SVG_LAYOUT_FULL_SPACE_MAJOR) {
    s = p / g.T;
    t = p - s * g.T;
    return;
  }
  const int pre = g.F0 * g.S;
  if (p < pre) {
    t = p / g.S;
    s = p - t * g.S;
    return;
  }
  const int q = p - pre, tr = g.T - g.F0;
  s = q / tr;
  t = g.F0 + (q - s * tr);
}

// Position of token (t, s) in this head's order.
// Original (frame-major) index of the token at position p of the head's order.
__host__ __device__ inline int orig_index(const MaskGeom& g, int p) {
  int t, s;
  pos_to_ts(g, p, t, s);
  return t * g.S + s;
}

__host__ __device__ inline int ts_to_pos(const MaskGeom& g, int t, int s) {
  if (g.route == SVG_ROUTE_SPATIAL) return t * g.S + s;
  if (g.layout == SVG_LAYOUT_FULL_SPACE_MAJOR) return s * g.T + t;
  if (t < g.F0) return t * g.S + s;
  return g.F0 * g.S + s * (g.T - g.F0) + (t - g.F0);
}

// Window / band part of the kept key positions of the query at position p: [lo, hi).
// Spatial: frames [t-k, t+k] are contiguous in frame-major order. Temporal: patches
// [s-b, s+b] are contiguous in the space-major part of the order (and the sink-frame copies
// of those patches are inside the sink anyway).
__host__ __device__ inline void row_interval(const MaskGeom& g, int p, int& lo, int& hi) {
  int t, s;
  pos_to_ts(g, p, t, s);
  if (g.route == SVG_ROUTE_SPATIAL) {
    const int f0 = t - g.k < 0 ? 0 : t - g.k;
    const int f1 = t + g.k > g.T - 1 ? g.T - 1 : t + g.k;
    lo = f0 * g.S;
    hi = (f1 + 1) * g.S;
    return;
  }
  const int s0 = s - g.b < 0 ? 0 : s - g.b;
  const int s1 = s + g.b > g.S - 1 ? g.S - 1 : s + g.b;
  if (g.layout == SVG_LAYOUT_FULL_SPACE_MAJOR) {
    lo = s0 * g.T;
    hi = (s1 + 1) * g.T;
  } else {
    const int pre = g.F0 * g.S, tr = g.T - g.F0;
    lo = pre + s0 * tr;
    hi = pre + (s1 + 1) * tr;
  }
}

__host__ __device__ inline int ilen(int a0, int a1) { return a1 > a0 ? a1 - a0 : 0; }

// #{c in [0, x) : c mod T < F0}
__host__ __device__ inline int periodic_prefix(const MaskGeom& g, int x) {
  const int q = x / g.T, r = x - q * g.T;
  return q * g.F0 + (r < g.F0 ? r : g.F0);
}

// Kept keys of a query row (interval [lo, hi)) inside key positions [c0, c1).
__host__ __device__ inline int row_kept_in(const MaskGeom& g, int lo, int hi, int c0, int c1) {
  const int b0 = lo > c0 ? lo : c0, b1 = hi < c1 ? hi : c1;
  int n = ilen(b0, b1);
  const int se = sink_end(g);
  if (se > 0) n += ilen(c0, se < c1 ? se : c1) - ilen(b0, se < b1 ? se : b1);
  if (periodic_sink(g)) {
    n += periodic_prefix(g, c1) - periodic_prefix(g, c0);
    if (b1 > b0) n -= periodic_prefix(g, b1) - periodic_prefix(g, b0);
  }
  return n;
}

// ---------------------------------------------------------------------------------------
// Tile-map workspace record (offset 0 of the workspace, 256 bytes).
struct TmHeader {
  uint32_t magic, version;
  int32_t T, H, W, route, k, b, F0, variant, layout, bq, bk, nq, nk, npairs, N;
  unsigned long long retained_exact, retained_map, n_full, n_boundary, n_empty, visited_area,
      pair_entries, pair_half_tiles;
};
static_assert(sizeof(TmHeader) <= 256, "header must fit in 256 bytes");

struct TmLayout {
  uint64_t total, cls, cnt, row_ptr, cols, pair_ptr, pair_ent, pair_cnt, pair_order;
  uint64_t pair_grp;
  int nq, nk, npairs;
};

// Division of 32-bit unsigned numbers by a divisor d >= 1 fixed per launch, by one multiply-high,
// an add and two shifts (Granlund and Montgomery, "Division by Invariant Integers using
// Multiplication", 1994, the round-up method for N = 32): with l = ceil(log2 d),
// m = floor(2^32 (2^l - d) / d) + 1, t = hi32(m n), the quotient is (t + ((n - t) >> min(l, 1)))
// >> max(l - 1, 0), exact for every 32-bit n.
struct FastDiv {
  uint32_t m, s1, s2, d;
};
inline FastDiv make_fastdiv(uint32_t d) {
  uint32_t l = 0;
  while (l < 32 && (1ull << l) < d) ++l;
  FastDiv f;
  f.m = (uint32_t)((((1ull << 32) * ((1ull << l) - d)) / d) + 1);
  f.s1 = l < 1 ? l : 1;
  f.s2 = l > 0 ? l - 1 : 0;
  f.d = d;
  return f;
}
__host__ __device__ inline uint32_t fastdiv(uint32_t n, const FastDiv& f) {
#if defined(__CUDA_ARCH__)
  const uint32_t t = __umulhi(n, f.m);
#else
  const uint32_t t = (uint32_t)(((uint64_t)n * f.m) >> 32);
#endif
  return (t + ((n - t) >> f.s1)) >> f.s2;
}

// Records a failed CUDA call (what + error) for svg_last_cuda_error; returns SVG_ERR_CUDA.
int record_cuda_error(const char* what, int cuda_error);

inline uint64_t align_up(uint64_t x, uint64_t a) { return (x + a - 1) / a * a; }

inline TmLayout tm_layout(int64_t N, int bq, int bk) {
  TmLayout L;
  L.nq = (int)((N + bq - 1) / bq);
  L.nk = (int)((N + bk - 1) / bk);
  L.npairs = (int)((N + kPairRows - 1) / kPairRows);
  const uint64_t tiles = (uint64_t)L.nq * L.nk;
  uint64_t off = 256;
  L.cls = off;        off = align_up(off + tiles, 256);
  L.cnt = off;        off = align_up(off + 4 * tiles, 256);
  L.row_ptr = off;    off = align_up(off + 4 * (uint64_t)(L.nq + 1), 256);
  L.cols = off;       off = align_up(off + 4 * tiles, 256);
  L.pair_ptr = off;   off = align_up(off + 4 * (uint64_t)(L.npairs + 1), 256);
  L.pair_ent = off;   off = align_up(off + 4 * (uint64_t)L.npairs * L.nk, 256);
  L.pair_cnt = off;   off = align_up(off + 8 * (uint64_t)L.npairs, 256);
  L.pair_order = off; off = align_up(off + 4 * (uint64_t)L.npairs, 256);
  L.pair_grp = off;   off = align_up(off + 8 * (uint64_t)L.npairs, 256);
  L.total = off;
  return L;
}

// Execution-list entry of a pair of 128-row blocks (a 256-row item): kt in the low 28 bits, then
// one 2-bit flag per block, block i at bit 28 + 2i.
enum : uint32_t { kFlagSkip = 0, kFlagFull = 1, kFlagMasked = 2, kFlagBounds = 3 };
__host__ __device__ inline uint32_t ent_kt(uint32_t e) { return e & 0x0FFFFFFFu; }
__host__ __device__ inline uint32_t ent_flag(uint32_t e, int half) { return (e >> (28 + 2 * half)) & 3u; }

// Scratch of the attention entry points: [0] status, [1] reserved, [2] work counter (head-major
// order), bytes [16, 24): the two class positions of the work-ordered scheduler (low / high word).
constexpr size_t kScratchBytes = 256;
constexpr size_t kCounter64Off = 16;

// Scheduling orders of the persistent attention kernel's work items.
enum : int { kOrderHeadMajor = 0, kOrderWork = 1 };

// Launch parameters of the attention kernel (filled on the host, read on the device).
struct AttnParams {
  CUtensorMap tm_q, tm_k, tm_v;
  // Fused token order (fused = 1): Q/K/V/O stay in the original order; temporal heads read
  // their rows with 4-row gathers through these 2-D maps ([heads * N] rows x d, box 64 x 1)
  // and write O rows back to their original index.
  CUtensorMap tm_q2, tm_k2, tm_v2;
  // ... and through these 4-D maps (d, patch, frame, head) with a box of one patch x run_len frames:
  // a whole run of one patch's frames (consecutive positions of a temporal head's order, rows S
  // apart in the original order) in one tiled copy; run_len = 0 when runs are not copied as boxes
  CUtensorMap tm_q4, tm_k4, tm_v4;
  int run_len, run_t0;
  // fused order: division by the length of a patch's run of frames (T in the fully space-major
  // order, T - F0 after the sink prefix; d = 1 when there is none), and the number of runs
  FastDiv run_div;
  int runs;
  int fused;
  // QK^T operands in e4m3 (one byte per element): tm_q / tm_k then describe 1-byte tensors
  int qk8;
  // Test hook: the softmax warps first wait on a barrier that nothing completes, so that the
  // bounded-wait / abort / drain path runs and the launch ends with SVG_ERR_TIMEOUT.
  int inject_stall;
  __nv_bfloat16* o;
  float* lse;
  int H, N, npairs, nk, n_items;
  float sl2;  // scale * log2(e)
  int dense, naive, variant, bq;
  int bkm;  // key-tile width of the entries (tile map's bk, or the dense call's bk)
  MaskGeom g[2];
  const TmHeader* hdr[2];
  const uint8_t* cls[2];
  const uint32_t* pair_ptr[2];
  const uint32_t* pair_ent[2];
  const uint32_t* pair_cnt[2];
  const uint32_t* pair_order[2];
  // work-ordered scheduler: per position of pair_order, the [start, end) of its run of equal work
  const uint32_t* pair_grp[2];
  int order;  // kOrderHeadMajor or kOrderWork
  int hc[2];  // heads of each route class
  unsigned long long* counter64;
  // nullable per-CTA trace, [trace_ctas][4]: start ns, end ns, items, 128-row half-tiles
  unsigned long long* cta_trace;
  int trace_ctas;
  int uses[2];
  int exp_T, exp_H, exp_W, exp_k, exp_b, exp_F0, exp_variant, exp_layout, exp_bq, exp_bk;
  int* status;
  unsigned int* counter;
  unsigned int* checks;  // failed-check counter of the checked build (null in the release build)
  uint32_t route_bits[kMaxHeads / 32];
};

// ---------------------------------------------------------------------------------------
// PTX wrappers.
#if defined(__CUDACC__)
// True when `ok` (always true in the release build); a false check is counted in *failed.
__device__ __forceinline__ bool check_ok(bool ok, unsigned int* failed) {
#if SVG_CHECKED
  if (!ok && failed) atomicAdd(failed, 1u);
  return ok;
#else
  (void)failed;
  return true;
#endif
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, uint32_t bar, int c0, int c1,
                                            int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], "
      "[%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// 3-D tiled TMA load global -> shared of this CTA, completion counted on `bar` (bytes).
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1,
                                            int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], "
      "[%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}
// 4-D tiled TMA load global -> shared of this CTA, completion counted on `bar` (bytes).
__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap* map, uint32_t bar, int c0, int c1,
                                            int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5, "
      "%6}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}
// Four rows r0..r3 (any order, any rows) of 64 columns starting at column c0 of a 2-D tensor
// map with a one-row box, to 4 x 128 bytes at dst (128-byte swizzle as a tiled load of those
// rows would place them).
__device__ __forceinline__ void tma_gather4(uint32_t dst, const CUtensorMap* map, uint32_t bar, int c0, int r0, int r1,
                                            int r2, int r3) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, "
      "%5, %6, %7}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(r0), "r"(r1), "r"(r2), "r"(r3)
      : "memory");
}
__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// tcgen05 (5th-generation tensor cores, TMEM accumulators), CTA group 1.
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// D[tmem] (+)= A[smem] * B[smem]
__device__ __forceinline__ void umma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                        uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// D[tmem] (+)= A[smem] * B[smem]^T, both e4m3 (kind::f8f6f4, K = 32 per instruction)
__device__ __forceinline__ void umma_ss_f8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                           uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// D[tmem] (+)= A[tmem] * B[smem]
__device__ __forceinline__ void umma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                        uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// mbarrier arrives once every tcgen05 op issued so far by this thread has completed.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

#define SVG_R8(i) "=r"(r[i + 0]), "=r"(r[i + 1]), "=r"(r[i + 2]), "=r"(r[i + 3]), "=r"(r[i + 4]), "=r"(r[i + 5]), \
                  "=r"(r[i + 6]), "=r"(r[i + 7])
#define SVG_W8(i) "r"(r[i + 0]), "r"(r[i + 1]), "r"(r[i + 2]), "r"(r[i + 3]), "r"(r[i + 4]), "r"(r[i + 5]), \
                  "r"(r[i + 6]), "r"(r[i + 7])
#define SVG_D8(i) "+r"(r[i + 0]), "+r"(r[i + 1]), "+r"(r[i + 2]), "+r"(r[i + 3]), "+r"(r[i + 4]), "+r"(r[i + 5]), \
                  "+r"(r[i + 6]), "+r"(r[i + 7])

// 32 lanes x 32 columns of 32 bits: thread i of the warp receives lane (base_lane + i),
// columns [col, col+32). Results are valid only after tmem_ld_fence32 on the same array.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : SVG_R8(0), SVG_R8(8), SVG_R8(16), SVG_R8(24)
      : "r"(taddr)
      : "memory");
}
// Orders later uses of r[0..32) after the completion wait (a data dependency through asm).
__device__ __forceinline__ void tmem_ld_fence32(uint32_t* r) {
  asm volatile("" : SVG_D8(0), SVG_D8(8), SVG_D8(16), SVG_D8(24) : : "memory");
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      SVG_W8(0), SVG_W8(8), SVG_W8(16), SVG_W8(24)
      : "memory");
}

// Shared-memory matrix descriptor (tcgen05 format): start>>4 [0,14), LBO>>4 [16,30),
// SBO>>4 [32,46), version 1 at bit 46, layout type [61,64) (2 = 128-byte swizzle).
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);
  d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}

// Instruction descriptor, kind::f16: D fp32, A and B bf16, M = 128.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int n, bool b_mn_major, int m = 128) {
  return (1u << 4)                      // D format fp32
         | (1u << 7)                    // A format bf16
         | (1u << 10)                   // B format bf16
         | ((b_mn_major ? 1u : 0u) << 16)
         | ((uint32_t)(n >> 3) << 17)   // N / 8
         | ((uint32_t)(m >> 4) << 24);  // M / 16
}

// Instruction descriptor, kind::f8f6f4: D fp32, A and B e4m3 (format code 0), both K-major.
__host__ __device__ constexpr uint32_t idesc_e4m3_f32(int n, int m = 128) {
  return (1u << 4)                      // D format fp32
         | ((uint32_t)(n >> 3) << 17)   // N / 8
         | ((uint32_t)(m >> 4) << 24);  // M / 16
}

// ---- bounded waits and shared-memory stores of the pipelined kernels ----
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s per wait

__device__ __forceinline__ int ld_shared_volatile(uint32_t addr) {
  int v;
  asm volatile("ld.volatile.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
  return v;
}
__device__ __forceinline__ void st_shared(uint32_t addr, int v) {
  asm volatile("st.volatile.shared.b32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

// Bounded wait on an mbarrier phase. Returns false on timeout or when another role aborted.
// abort_addr: shared address of the abort flag; status: global status word.
static __device__ __noinline__ bool wait_bar_slow(uint32_t bar, uint32_t parity, uint32_t abort_addr, int* status) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 15u) == 0) {
      if (ld_shared_volatile(abort_addr)) return false;
      if (globaltimer_ns() - t0 > kWaitLimitNs) {
        st_shared(abort_addr, 1);
        atomicCAS(status, 0, SVG_ERR_TIMEOUT);
        return false;
      }
    }
  }
}

// Fast path inline (an already-completed phase costs one try_wait), the bounded loop out of line.
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, uint32_t abort_addr, int* status) {
  return mbar_try_wait(bar, parity) || wait_bar_slow(bar, parity, abort_addr, status);
}

// Drain wait: ignores the abort flag, short limit; used only on the error path.
static __device__ __noinline__ void drain_bar(uint32_t a, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(a, parity))
    if (globaltimer_ns() - t0 > 200000000ull) return;
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}
// Makes this thread's shared-memory stores visible to the tensor core (the async proxy).
__device__ __forceinline__ void fence_proxy_async_shared() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// One P row (BK bf16, packed in pairs in r[0, BK/2)) into a K-major 128-byte-swizzle tile of
// 128 rows: keys [64c, 64c + 64) in chunk c (128 rows x 128 bytes), row lr at byte lr * 128 of the
// chunk, its 16-byte unit u at position u ^ (lr % 8). A warp's 32 rows cover all banks in four
// passes per store.
template <int BK>
__device__ __forceinline__ void store_p_sw128(uint32_t base, int lr, const uint32_t* r) {
  const uint32_t row = base + (uint32_t)lr * 128u, sw = (uint32_t)lr & 7u;
#pragma unroll
  for (int ch = 0; ch < BK / 64; ++ch)
#pragma unroll
    for (uint32_t u = 0; u < 8; ++u) {
      const uint32_t* w = r + ch * 32 + 4 * u;
      st_shared_v4(row + ch * (128u * 128u) + ((u ^ sw) << 4), w[0], w[1], w[2], w[3]);
    }
}

// ---- softmax arithmetic shared by the attention kernels ----
__device__ __forceinline__ float ex2f(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 2^x on the FMA / integer pipes, to take part of the exponentials off the MUFU unit (used two
// lanes at a time by exp2_poly2 below).
// Cody-Waite style range reduction: n = round(x) (by the 1.5*2^23 rounding trick), f = x - n in
// [-1/2, 1/2]; 2^f by a degree-3 polynomial whose coefficients minimise the maximum relative
// error on [-1/2, 1/2] (fitted by linear programming, max rel. error 7.5e-5, far below the bf16
// rounding of P); 2^n is added to the exponent field by one integer multiply-add. Inputs below
// -125 (masked scores are -inf) give 2^-125 times the polynomial's value at 0, a normal number
// too small to move any finite sum; a row whose every score is masked is zeroed by its caller.
constexpr float kExpC0 = 9.999280572e-01f, kExpC1 = 6.932609677e-01f, kExpC2 = 2.426111251e-01f,
                kExpC3 = 5.517166853e-02f;

// Column pairs (mod 8) whose exponentials are computed by exp2_poly2 instead of ex2.approx.
#ifndef SVG_POLY_MASK
#define SVG_POLY_MASK 0x00u
#endif
constexpr uint32_t kPolyMask = SVG_POLY_MASK;


__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 v = __floats2bfloat162_rn(a, b);  // .x = a (low 16 bits)
  return *reinterpret_cast<uint32_t*>(&v);
}

// 2^x of two lanes on the packed fp32x2 pipe, by the method above: the rounding adds, the reduced argument
// and the three polynomial steps are one FADD2 / FFMA2 each for both lanes; the clamp and the
// exponent insertion (one integer multiply-add) stay per lane.
__device__ __forceinline__ float2 exp2_poly2(float2 x) {
  const float2 xc = make_float2(fmaxf(x.x, -125.f), fmaxf(x.y, -125.f));
  const float2 r = __fadd2_rn(xc, make_float2(12582912.f, 12582912.f));
  const float2 n = __fadd2_rn(r, make_float2(-12582912.f, -12582912.f));
  const float2 f = __ffma2_rn(n, make_float2(-1.f, -1.f), xc);  // xc - n, exact
  float2 p = __ffma2_rn(make_float2(kExpC3, kExpC3), f, make_float2(kExpC2, kExpC2));
  p = __ffma2_rn(p, f, make_float2(kExpC1, kExpC1));
  p = __ffma2_rn(p, f, make_float2(kExpC0, kExpC0));
  return make_float2(__uint_as_float(__float_as_uint(r.x) * 8388608u + __float_as_uint(p.x)),
                     __uint_as_float(__float_as_uint(r.y) * 8388608u + __float_as_uint(p.y)));
}

// Columns [J0, J0 + 64) of one score row, in place: p_j = 2^(s_j * sl2 - base), packed to bf16
// pairs into r[J0/2, J0/2 + 32) (the scores there are already consumed); the fp32 p_j are added
// to four running sums. The scale-subtract uses the packed fp32x2 FMA (two columns per
// instruction); column pairs (j, j+1) with bit (j/2) % 8 of kPolyMask set take exp2_poly2, the
// rest ex2.approx.
template <int J0>
__device__ __forceinline__ void exp_pack_64(uint32_t* r, float2 sc, float2 nb, float2 (&acc)[2]) {
  const float* s = reinterpret_cast<const float*>(r);
#pragma unroll
  for (int j = J0; j < J0 + 64; j += 2) {
    const float2 x = __ffma2_rn(make_float2(s[j], s[j + 1]), sc, nb);
    const float2 p = ((kPolyMask >> ((j / 2) & 7)) & 1u) ? exp2_poly2(x) : make_float2(ex2f(x.x), ex2f(x.y));
    acc[(j / 2) & 1].x += p.x;
    acc[(j / 2) & 1].y += p.y;
    r[j / 2] = pack_bf16(p.x, p.y);
  }
}

// A row maximum may grow by up to 2^kRescaleLog2 before O and l are rescaled (log2 units).
constexpr float kRescaleLog2 = 8.0f;
constexpr float kRescaleBound = 256.0f;  // 2^kRescaleLog2: the largest P taken without a rescale
static_assert(kRescaleBound == (float)(1 << (int)kRescaleLog2), "rescale bound");

// ---------------------------------------------------------------------------------------
// Softmax steps of one score row (one thread per query row, BK scores in registers).

// The row's BK fp32 scores from TMEM.
template <int BK>
__device__ __forceinline__ void load_scores(uint32_t tS, uint32_t* r) {
#pragma unroll
  for (int q = 0; q < BK / 32; ++q) tmem_ld32(tS + q * 32, r + q * 32);
  tmem_ld_wait();
#pragma unroll
  for (int q = 0; q < BK / 32; ++q) tmem_ld_fence32(r + q * 32);
}

// Sets to -inf the scores the mask drops: boundary tiles element by element (kept keys of the
// row are [0, se) U [lo, hi), or the periodic sink of the fully space-major order), the ragged
// key tail, every visited tile in naive mode, and rows without a kept tile under rounded masks.
template <int BK>
__device__ __forceinline__ void mask_scores(const AttnParams& P, int cls, uint32_t f, int c0, int prow, uint32_t ent,
                                            int lo, int hi, int se, bool per, uint32_t* r) {
  float* s = reinterpret_cast<float*>(r);
  const bool elem = (f == kFlagMasked) || (P.naive && !P.dense);
  if (!(elem || f == kFlagBounds)) return;
  const int nn = P.N - c0;
  if (!elem) {
#pragma unroll
    for (int j = 0; j < BK; ++j)
      if (j >= nn) s[j] = -INFINITY;
  } else if (P.variant == SVG_MASK_ROUNDED) {
    const uint8_t* rcls = P.cls[cls] + (size_t)(prow / P.bq) * P.nk;
    const bool in_map = check_ok(prow >= 0 && prow < P.N && ent_kt(ent) < (uint32_t)P.nk, P.checks);
    const bool rowkept = in_map && __ldg(rcls + ent_kt(ent)) == 1;
#pragma unroll
    for (int j = 0; j < BK; ++j)
      if (!(rowkept && j < nn)) s[j] = -INFINITY;
  } else {
    const int a = lo - c0;
    const uint32_t w = (uint32_t)(hi - lo);
    const int sk = se - c0;
    if (!per) {
#pragma unroll
      for (int j = 0; j < BK; ++j) {
        const bool keep = (j < nn) && ((j < sk) || ((uint32_t)(j - a) < w));
        if (!keep) s[j] = -INFINITY;
      }
    } else {
      const MaskGeom& g = P.g[cls];
      int rr = c0 % g.T;
#pragma unroll
      for (int j = 0; j < BK; ++j) {
        const bool keep = (j < nn) && ((rr < g.F0) || ((uint32_t)(j - a) < w));
        if (!keep) s[j] = -INFINITY;
        rr = (rr + 1 == g.T) ? 0 : rr + 1;
      }
    }
  }
}

// Row maximum first, then the rescale decision: the warp rescales (returns true) when any row's
// maximum grew by more than 2^kRescaleLog2 or had none yet; l is corrected here, O by the
// caller after P is stored.
template <int BK>
__device__ __forceinline__ bool max_first(const uint32_t* r, float sl2, float& m, float& l, float& alpha) {
  const float* s = reinterpret_cast<const float*>(r);
  float mx4[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) mx4[i] = s[i];
#pragma unroll
  for (int j = 4; j < BK; j += 4)
#pragma unroll
    for (int i = 0; i < 4; ++i) mx4[i] = fmaxf(mx4[i], s[j + i]);
  const float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
  const float m_new = fmaxf(m, mx);
  const bool need = (m_new > m) && (m == -INFINITY || (m_new - m) * sl2 > kRescaleLog2);
  const bool rescale = __any_sync(0xffffffffu, need);
  if (rescale) {
    alpha = (m_new == -INFINITY) ? 1.f : ex2f((m - m_new) * sl2);
    l *= alpha;
    m = m_new;
  }
  return rescale;
}

// P = 2^(S * sl2 - m * sl2) packed to bf16 into r[0, BK/2), fp32 partial row sums in acc.
template <int BK>
__device__ __forceinline__ void exp_tile(uint32_t* r, float sl2, float m, float2 (&acc)[2]) {
  const float base = (m == -INFINITY) ? 0.f : m * sl2;
  const float2 sc = make_float2(sl2, sl2), nb = make_float2(-base, -base);
  acc[0] = make_float2(0.f, 0.f);
  acc[1] = make_float2(0.f, 0.f);
  exp_pack_64<0>(r, sc, nb, acc);
  if (BK == 128) exp_pack_64<64 % BK>(r, sc, nb, acc);
}


#endif  // __CUDACC__

}  // namespace svg
