// svg_attention.cu -- persistent block-sparse flash-attention forward for sm_100a.
//
// What it computes: softmax attention restricted to the kept (query, key) pairs of each
// head's spatial or temporal mask, visiting only non-empty key tiles, with a mask-free path
// for full tiles and element masking only in boundary tiles ("Efficient Kernel
// Implementation", tile-aware masking, of "Accelerating Spatio-Temporal Attention for Video
// Diffusion on TPUs"; the summary's full/boundary split). Online (flash-style) softmax keeps
// memory O(N d).
//
// How (B200-specific, not the TPU design):
//  * one CTA per SM, 352 threads, persistent; work items are (head, 256 query rows) taken
//    from a global atomic counter in head-major order, each head's items heaviest first (or,
//    as an option, longest processing time first over all heads);
//  * warp 8 issues TMA loads (128-byte swizzle) of Q once per item and of the K tiles, warp 10
//    those of the V tiles, into a shared-memory ring; warp 9 issues tcgen05 MMAs: S = Q K^T
//    into TMEM, then O += P V with P read straight from TMEM;
//  * warps 0-3 and 4-7 are two softmax groups, one per 128-row half, one thread per query
//    row (= TMEM lane). While one group turns its S into P, the tensor core computes the
//    other half's S and P V, so MMA and exponentials overlap;
//  * option PS: P goes to shared memory instead, so the next tile's S is computed while the
//    softmax of this tile runs (measured slower on B200; kept selectable);
//  * O is rescaled (in TMEM) only when a row maximum grows by more than 2^8, which keeps
//    the result exact while making the correction rare; after a row's first tile the
//    exponentials are taken against the running maximum, and the tile's own maximum only when
//    a row's P sums past 2^8 (the tile is then read again from TMEM);
//  * every wait is bounded by a wall-clock limit; a timeout sets the status word and all
//    roles drain their in-flight copies / MMAs and return.
//  * fused token order: temporal heads read their tiles where the rows lie in the original order
//    (whole runs of one patch's frames as 4-D boxes, edge rows gathered) and write O rows back to
//    their original index.
#include <cuda_bf16.h>
#include <string.h>

#include "svg_common.cuh"

namespace svg {

constexpr int kThreads = 352;
constexpr int kProducerWarp = 8;   // claims the items, loads Q and the K tiles
constexpr int kMmaWarp = 9;
constexpr int kProducer2Warp = 10;  // loads the V tiles of the items warp 8 publishes


// QK8: Q and K in e4m3 (one byte per element, d = 128: one 128-byte swizzle chunk per row), QK^T on
// the tensor core's 8-bit path; V, P and O as in the bf16 path.
// PS: P goes to shared memory (same 128-byte swizzle layout as a Q half) instead of TMEM, and P V
// reads it from there. S_h's TMEM columns are then free as soon as the softmax has loaded them,
// so the next tile's S_h is computed while the softmax of this tile runs.
template <int D, int BK, bool QK8 = false, bool PS = false>
struct Cfg {
  static constexpr int kChunks = D / 64;            // 128-byte swizzle chunks per bf16 row (V)
  static constexpr int kQKChunks = QK8 ? D / 128 : D / 64;  // the same for a Q or K row
  static constexpr int kQKColsPerChunk = QK8 ? 128 : 64;
  static constexpr int kQHalfBytes = 128 * D * (QK8 ? 1 : 2);
  static constexpr int kQBytes = 2 * kQHalfBytes;
  static constexpr int kPHalfBytes = PS ? 128 * BK * 2 : 0;
  static constexpr int kPBytes = 2 * kPHalfBytes;
  static constexpr int kKBytes = BK * D * (QK8 ? 1 : 2);
  static constexpr int kVBytes = BK * D * 2;
  static constexpr int kTileBytes = BK * D * 2;     // ring slot: one K or one V tile
  static constexpr int kStages = PS ? (224 * 1024 - kQBytes - kPBytes) / kTileBytes : (160 * 1024) / kTileBytes;
  static constexpr int kDataBytes = kQBytes + kPBytes + kStages * kTileBytes;
  static constexpr int kSmemBytes = kDataBytes + 1024 /*control*/ + 1024 /*alignment slack*/;
  // TMEM columns: S (and P) of half h at 128*h, P (bf16 pairs) aliases the upper half of
  // S, O accumulators of half h at 256 + D*h.
  __host__ __device__ static constexpr uint32_t s_col(int h) { return 128u * h; }
  static constexpr uint32_t kPCol = BK / 2;
  __host__ __device__ static constexpr uint32_t o_col(int h) { return 256u + (uint32_t)D * h; }
  static_assert(kStages >= (PS ? 3 : 2), "ring too small");
  static_assert(kSmemBytes <= 232448, "shared memory budget");
};

struct ItemInfo {
  int valid, head, pair, cls, count, nA, nB, pad;
  const uint32_t* ents;
};

// Shared-memory control block, addressed by 32-bit shared addresses so that the roles keep
// a single base register instead of one generic pointer per barrier.
//   [0, NS)        kv_full[s]    TMA K/V tile landed in ring slot s
//   [NS, 2NS)      kv_empty[s]   MMAs done reading ring slot s
//   2NS + 0 / 1    q_full / q_free
//   2NS + 2 + h    s_full[h]     S_h = Q_h K^T (and every earlier MMA) complete
//   2NS + 4 + h    p_ready[h]    P_h in TMEM, O_h corrected (128 arrivals)
//   2NS + 6 + h    o_done[h]     last P V of half h complete (PS: every P V of half h, pv_done)
//   2NS + 8 + h    o_free[h]     epilogue finished reading O_h (128 arrivals)
//   2NS + 10 + i   item_full[i]  work item published in slot i
//   2NS + 12 + i   item_empty[i] slot i read by the MMA warp, the 8 softmax warps and the V producer
//   2NS + 14       drain         final MMA completion
//   2NS + 15       never         completed by nothing (test hook: a wait that runs out)
//   2NS + 16 + h   s_free[h]     (PS) S_h loaded by the softmax, its TMEM columns free (128 arrivals)
//   2NS + 18 ...   two ItemInfo slots, TMEM base, abort flag, workspace check, trace counts
template <int NS>
struct Ctl {
  uint32_t base;  // shared address of the control block
  int* status;
  __device__ __forceinline__ uint32_t kv_full(uint32_t s) const { return base + 8u * s; }
  __device__ __forceinline__ uint32_t kv_empty(uint32_t s) const { return base + 8u * (NS + s); }
  __device__ __forceinline__ uint32_t q_full() const { return base + 8u * (2 * NS + 0); }
  __device__ __forceinline__ uint32_t q_free() const { return base + 8u * (2 * NS + 1); }
  __device__ __forceinline__ uint32_t s_full(int h) const { return base + 8u * (2 * NS + 2 + h); }
  __device__ __forceinline__ uint32_t p_ready(int h) const { return base + 8u * (2 * NS + 4 + h); }
  __device__ __forceinline__ uint32_t o_done(int h) const { return base + 8u * (2 * NS + 6 + h); }
  __device__ __forceinline__ uint32_t o_free(int h) const { return base + 8u * (2 * NS + 8 + h); }
  __device__ __forceinline__ uint32_t item_full(uint32_t i) const { return base + 8u * (2 * NS + 10 + i); }
  __device__ __forceinline__ uint32_t item_empty(uint32_t i) const { return base + 8u * (2 * NS + 12 + i); }
  __device__ __forceinline__ uint32_t drain() const { return base + 8u * (2 * NS + 14); }
  __device__ __forceinline__ uint32_t never() const { return base + 8u * (2 * NS + 15); }
  __device__ __forceinline__ uint32_t s_free(int h) const { return base + 8u * (2 * NS + 16 + h); }
  static constexpr uint32_t kItemsOff = 8u * (2 * NS + 18);  // 2 x 40 bytes
  static constexpr uint32_t kTmemOff = kItemsOff + 96;
  static constexpr uint32_t kAbortOff = kTmemOff + 8;
  static constexpr uint32_t kBadWsOff = kAbortOff + 8;
  static constexpr uint32_t kTraceOff = kBadWsOff + 8;  // items, half-tiles of this CTA (producer)
  static constexpr uint32_t kBytes = kTraceOff + 8;
};

// O_h *= alpha in TMEM, 32 columns at a time (one thread per row).
template <int D>
__device__ __forceinline__ void rescale_o(uint32_t tO, float alpha) {
#pragma unroll 1
  for (int q = 0; q < D / 32; ++q) {
    uint32_t o[32];
    tmem_ld32(tO + q * 32, o);
    tmem_ld_wait();
    tmem_ld_fence32(o);
#pragma unroll
    for (int x = 0; x < 32; ++x) o[x] = __float_as_uint(__uint_as_float(o[x]) * alpha);
    tmem_st32(tO + q * 32, o);
  }
}

template <int BK>
__device__ __forceinline__ uint32_t dense_entry(const AttnParams& P, const ItemInfo& it, int e) {
  const bool ragged = (e == P.nk - 1) && (P.N % BK != 0);
  const uint32_t f = ragged ? kFlagBounds : kFlagFull;
  const uint32_t fa = it.nA ? f : 0u, fb = it.nB ? f : 0u;
  return (uint32_t)e | (fa << 28) | (fb << 30);
}

template <int BK>
__device__ __forceinline__ uint32_t get_entry(const AttnParams& P, const ItemInfo& it, int e) {
  if (P.dense) return dense_entry<BK>(P, it, e);
  if (!check_ok(e >= 0 && e < it.count, P.checks)) return 0u;
  const uint32_t ent = __ldg(it.ents + e);
  return check_ok(ent_kt(ent) < (uint32_t)P.nk, P.checks) ? ent : (ent & ~0x0FFFFFFFu);
}

__device__ __forceinline__ int route_of(const AttnParams& P, int h) {
  return (P.route_bits[h >> 5] >> (h & 31)) & 1;
}

// The item's execution list: pair `pair` of route class it.cls.
__device__ __forceinline__ void fill_sparse_item(const AttnParams& P, ItemInfo& it) {
  const int c = it.cls;
  if (!check_ok((unsigned)it.pair < (unsigned)P.npairs, P.checks)) it.pair = 0;
  const uint32_t b0 = __ldg(P.pair_ptr[c] + it.pair), b1 = __ldg(P.pair_ptr[c] + it.pair + 1);
  it.count = (int)(b1 - b0);
  it.ents = P.pair_ent[c] + b0;
  it.nA = (int)__ldg(P.pair_cnt[c] + 2 * it.pair);
  it.nB = (int)__ldg(P.pair_cnt[c] + 2 * it.pair + 1);
  if (!check_ok(b0 <= b1 && (uint64_t)b1 <= (uint64_t)P.npairs * (uint64_t)P.nk && it.nA <= it.count &&
                    it.nB <= it.count && it.count <= P.nk,
                P.checks))
    it.count = it.nA = it.nB = 0;
}

// Head-major order: counter value idx -> head idx / npairs, that head's items heaviest first.
template <int BK>
__device__ ItemInfo decode_item(const AttnParams& P, uint32_t idx) {
  ItemInfo it;
  memset(&it, 0, sizeof(it));
  if (idx >= (uint32_t)P.n_items) return it;
  it.valid = 1;
  it.head = (int)(idx / (uint32_t)P.npairs);
  const int j = (int)(idx - (uint32_t)it.head * (uint32_t)P.npairs);
  it.cls = route_of(P, it.head);
  if (P.dense) {
    it.pair = j;
    it.count = P.nk;
    it.nA = (j * kPairRows < P.N) ? P.nk : 0;
    it.nB = (j * kPairRows + kHalfRows < P.N) ? P.nk : 0;
    it.ents = nullptr;
  } else {
    it.pair = (int)__ldg(P.pair_order[it.cls] + j);
    fill_sparse_item(P, it);
  }
  return it;
}

// ---- work-ordered scheduler -------------------------------------------------------------
// Every head of a route class has the same items with the same work, so the items of a class in
// descending work, taken head by head within each run of equal work, form the class's sequence;
// the two classes' sequences are merged by work (ties to the spatial class) through one 64-bit
// counter holding both positions. This is longest-processing-time-first over all (head, item)
// pairs, with the heads of one run kept together so that items in flight share K / V rows in L2.

// Work (active 128-row half-tiles) of position p of class c's order.
__device__ __forceinline__ int work_at(const AttnParams& P, int c, uint32_t p) {
  const uint32_t g = __ldg(P.pair_order[c] + p);
  return (int)(__ldg(P.pair_cnt[c] + 2 * g) + __ldg(P.pair_cnt[c] + 2 * g + 1));
}

// The r-th head (0-based, ascending) whose route is c.
__device__ int head_of_rank(const AttnParams& P, int c, int r) {
  const int words = (P.H + 31) >> 5;
  for (int w = 0; w < words; ++w) {
    uint32_t bits = c ? P.route_bits[w] : ~P.route_bits[w];
    if (w == words - 1 && (P.H & 31)) bits &= (1u << (P.H & 31)) - 1u;
    const int n = __popc(bits);
    if (r < n) {
      for (int i = 0; i < r; ++i) bits &= bits - 1u;
      return w * 32 + __ffs(bits) - 1;
    }
    r -= n;
  }
  return 0;  // unreachable for r < heads of class c
}

// Claims the next (class, position) in merged work order; false when both sequences are done.
// A failed compare-and-swap means another CTA claimed an item, so the retries of one CTA are
// bounded by the number of items; the cap only guards against a corrupted counter.
__device__ bool claim_work_item(const AttnParams& P, int& cls, uint32_t& pos) {
  const uint64_t n0 = (uint64_t)P.hc[0] * (uint64_t)P.npairs, n1 = (uint64_t)P.hc[1] * (uint64_t)P.npairs;
  unsigned long long cur = atomicAdd(P.counter64, 0ull);
  for (uint32_t tries = 0; tries < (1u << 28); ++tries) {
    const uint32_t i0 = (uint32_t)cur, i1 = (uint32_t)(cur >> 32);
    const int w0 = i0 < n0 ? work_at(P, 0, i0 / (uint32_t)P.hc[0]) : -1;
    const int w1 = i1 < n1 ? work_at(P, 1, i1 / (uint32_t)P.hc[1]) : -1;
    if (w0 < 0 && w1 < 0) return false;
    const int c = w0 >= w1 ? 0 : 1;
    const unsigned long long nxt = cur + (c ? (1ull << 32) : 1ull);
    const unsigned long long prev = atomicCAS(P.counter64, cur, nxt);
    if (prev == cur) {
      cls = c;
      pos = c ? i1 : i0;
      return true;
    }
    cur = prev;
  }
  atomicCAS(P.status, 0, SVG_ERR_TIMEOUT);
  return false;
}

// Position pos of class c's sequence -> (head, item).
__device__ ItemInfo decode_work_item(const AttnParams& P, int c, uint32_t pos) {
  ItemInfo it;
  memset(&it, 0, sizeof(it));
  const uint32_t hc = (uint32_t)P.hc[c];
  const uint32_t p = pos / hc;
  const uint32_t s = __ldg(P.pair_grp[c] + 2 * p), e = __ldg(P.pair_grp[c] + 2 * p + 1);
  const uint32_t len = e - s, o = pos - hc * s;
  if (!check_ok(p < (uint32_t)P.npairs && s <= p && p < e && e <= (uint32_t)P.npairs && o < hc * len, P.checks))
    return it;  // not valid: this CTA stops taking items
  it.valid = 1;
  it.cls = c;
  it.head = head_of_rank(P, c, (int)(o / len));
  it.pair = (int)__ldg(P.pair_order[c] + s + o % len);
  fill_sparse_item(P, it);
  return it;
}

// ---- fused token order: the rows of a temporal head's tile, read where they lie ------------
// Positions [p0, p0 + ROWS) of a temporal head's token order go to a ROWS-row tile (64-column chunks
// ROWS * 128 bytes apart, 128-byte swizzle). Rows of the sink prefix are contiguous in the original
// order: one tiled copy per chunk. Past the prefix the order runs through one patch's frames at a
// time (run_len positions whose rows are S apart in the original order): every run lying wholly
// inside the tile is one 4-D box copy per chunk, and the 4-row groups that hold rows of the partial
// runs at the tile's edges (or rows past the sequence end, clamped to the last row) are gathered
// row by row. A gathered group may also hold rows of a whole run; both copies then write the same
// bytes there. The byte count covers every copy, duplicates included.
struct FusedPlan {
  int kind;        // 0: inside the sink prefix, 1: gather every group, 2: runs and edge groups
  int n_box, u_a;  // whole runs u_a .. u_a + n_box - 1 (patch index = run index)
  uint32_t gmask;  // 4-row groups to gather (bit = group = lane)
  int rr[4];       // this lane's gathered rows (original indices in the [heads * N, d] view)
};

template <int ROWS>
__device__ __forceinline__ FusedPlan fused_plan(const AttnParams& P, int p0, int lane) {
  const MaskGeom& g = P.g[SVG_ROUTE_TEMPORAL];
  const int pre = sink_end(g), R = P.run_len;
  FusedPlan f;
  f.n_box = 0;
  f.u_a = 0;
  f.gmask = 0;
  f.rr[0] = f.rr[1] = f.rr[2] = f.rr[3] = 0;
  constexpr uint32_t kAll = ROWS / 4 >= 32 ? 0xFFFFFFFFu : ((1u << (ROWS / 4)) - 1u);
  if (p0 + ROWS <= pre) {
    f.kind = 0;
    return f;
  }
  if (p0 < pre || R == 0) {
    f.kind = 1;
    f.gmask = kAll;
    return f;
  }
  f.kind = 2;
  const int q0 = p0 - pre;
  const int u_a = (int)fastdiv((uint32_t)(q0 + R - 1), P.run_div);  // first run that starts inside the tile
  int u_end = (int)fastdiv((uint32_t)(q0 + ROWS), P.run_div);       // runs [u_a, u_end) end inside the tile
  if (u_end > P.runs) u_end = P.runs;
  f.u_a = u_a;
  f.n_box = u_end > u_a ? u_end - u_a : 0;
  const int c0 = f.n_box ? u_a * R - q0 : 0, c1 = f.n_box ? u_end * R - q0 : 0;  // rows the boxes cover
  const int r0 = 4 * lane;
  const bool need = r0 < ROWS && !(r0 >= c0 && r0 + 4 <= c1);
  f.gmask = __ballot_sync(0xFFFFFFFFu, need) & kAll;
  return f;
}

// Original index of the token at position p of a temporal head's order (orig_index with the run
// division done by fastdiv).
__device__ __forceinline__ int temporal_orig_index(const AttnParams& P, const MaskGeom& g, int p) {
  if (g.layout == SVG_LAYOUT_FULL_SPACE_MAJOR) {
    const int s = (int)fastdiv((uint32_t)p, P.run_div);
    return (p - s * g.T) * g.S + s;
  }
  const int pre = g.F0 * g.S;
  if (p < pre) return p;
  const int q = p - pre;
  const int s = (int)fastdiv((uint32_t)q, P.run_div);
  return (g.F0 + q - s * (g.T - g.F0)) * g.S + s;
}

// The plan and this lane's gathered rows for head `head`, tile rows [p0, p0 + ROWS).
template <int ROWS>
__device__ __forceinline__ FusedPlan fused_plan_rows(const AttnParams& P, int head, int p0, int lane) {
  FusedPlan f = fused_plan<ROWS>(P, p0, lane);
  if ((f.gmask >> lane) & 1u) {
    const MaskGeom& g = P.g[SVG_ROUTE_TEMPORAL];
    const int hrow = head * P.N;  // first row of the head in the [heads * N, d] view (fits: checked on the host)
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      f.rr[i] = hrow + temporal_orig_index(P, g, min(p0 + 4 * lane + i, P.N - 1));
      if (!check_ok(f.rr[i] >= hrow && f.rr[i] < hrow + P.N, P.checks)) f.rr[i] = hrow;
    }
  }
  return f;
}

template <int ROWS, int CHUNKS>
__device__ __forceinline__ uint32_t fused_bytes(const AttnParams& P, const FusedPlan& f) {
  if (f.kind == 0) return (uint32_t)(ROWS * 128 * CHUNKS);
  return ((uint32_t)f.n_box * (uint32_t)P.run_len * 128u + (uint32_t)__popc(f.gmask) * 512u) * CHUNKS;
}

template <int ROWS, int CHUNKS>
__device__ __forceinline__ void fused_issue(const AttnParams& P, const FusedPlan& f, const CUtensorMap* tile_map,
                                            const CUtensorMap* box_map, const CUtensorMap* row_map, uint32_t dst,
                                            uint32_t bar, int head, int p0, int lane) {
  if (f.kind == 0) {
    if (lane == 0)
      for (int ch = 0; ch < CHUNKS; ++ch) tma_load_3d(dst + ch * (ROWS * 128), tile_map, bar, ch * 64, p0, head);
    return;
  }
  const MaskGeom& g = P.g[SVG_ROUTE_TEMPORAL];
  if (lane < f.n_box) {
    const int u = f.u_a + lane;
    const uint32_t row = (uint32_t)(sink_end(g) + u * P.run_len - p0);
    check_ok(u >= 0 && u < g.S && P.run_t0 + P.run_len <= g.T && row + (uint32_t)P.run_len <= (uint32_t)ROWS,
             P.checks);
    for (int ch = 0; ch < CHUNKS; ++ch)
      tma_load_4d(dst + ch * (ROWS * 128) + row * 128u, box_map, bar, ch * 64, u, P.run_t0, head);
  }
  if ((f.gmask >> lane) & 1u) {
    for (int ch = 0; ch < CHUNKS; ++ch)
      tma_gather4(dst + ch * (ROWS * 128) + (uint32_t)lane * 512u, row_map, bar, ch * 64, f.rr[0], f.rr[1], f.rr[2],
                  f.rr[3]);
  }
}

// ---------------------------------------------------------------------------------------
template <int D, int BK, bool QK8 = false, bool PS = false>
__global__ void __launch_bounds__(kThreads, 1) attn_kernel(const __grid_constant__ AttnParams P) {
  using C = Cfg<D, BK, QK8, PS>;
  constexpr int NS = C::kStages;
  using K = Ctl<NS>;
  static_assert(K::kBytes <= 1024, "control block");
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte alignment for the 128-byte swizzle atoms
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = raw + ((1024u - (raw & 1023u)) & 1023u);
  const uint32_t sQ = sbase, sP = sbase + C::kQBytes, sRing = sP + C::kPBytes;
  K c;
  c.base = sbase + C::kDataBytes;
  c.status = P.status;
  uint8_t* ctl_gen = smem_raw + (c.base - raw);  // generic pointer to the control block
  ItemInfo* items = reinterpret_cast<ItemInfo*>(ctl_gen + K::kItemsOff);
  const uint32_t abort_addr = c.base + K::kAbortOff;
  int* status = P.status;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint64_t t_start = P.cta_trace ? globaltimer_ns() : 0ull;

  if (threadIdx.x == 0) {
    *reinterpret_cast<uint64_t*>(ctl_gen + K::kTraceOff) = 0ull;
    for (int st = 0; st < NS; ++st) {
      mbar_init(reinterpret_cast<uint64_t*>(ctl_gen) + st, 1);       // kv_full
      mbar_init(reinterpret_cast<uint64_t*>(ctl_gen) + NS + st, 1);  // kv_empty
    }
    uint64_t* b = reinterpret_cast<uint64_t*>(ctl_gen) + 2 * NS;
    mbar_init(b + 0, 1);  // q_full
    mbar_init(b + 1, 1);  // q_free
    for (int h = 0; h < 2; ++h) {
      mbar_init(b + 2 + h, 1);     // s_full
      mbar_init(b + 4 + h, 128);   // p_ready
      mbar_init(b + 6 + h, 1);     // o_done
      mbar_init(b + 8 + h, 128);   // o_free
      mbar_init(b + 10 + h, 1);    // item_full
      mbar_init(b + 12 + h, 10);   // item_empty
    }
    mbar_init(b + 14, 1);  // drain
    mbar_init(b + 15, 1);  // never
    mbar_init(b + 16, 128);  // s_free[0]
    mbar_init(b + 17, 128);  // s_free[1]
    *reinterpret_cast<volatile int*>(ctl_gen + K::kAbortOff) = 0;
    // the tile maps must have been built for exactly these parameters
    int bad = 0;
    if (!P.dense) {
      for (int k = 0; k < 2; ++k) {
        if (!P.uses[k]) continue;
        const TmHeader* h = P.hdr[k];
        bad |= h->magic != kTmMagic || h->route != k || h->T != P.exp_T || h->H != P.exp_H ||
               h->W != P.exp_W || h->k != P.exp_k || h->b != P.exp_b || h->F0 != P.exp_F0 ||
               h->variant != P.exp_variant || h->layout != P.exp_layout || h->bq != P.exp_bq ||
               h->bk != P.exp_bk || h->nk != P.nk || h->npairs != P.npairs;
      }
    }
    *reinterpret_cast<int*>(ctl_gen + K::kBadWsOff) = bad;
    if (bad) atomicCAS(P.status, 0, SVG_ERR_WORKSPACE);
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(reinterpret_cast<uint32_t*>(ctl_gen + K::kTmemOff), 512);
    tmem_relinquish();
  }
  if (warp == kProducerWarp && lane == 0) {
    prefetch_tmap(&P.tm_q);
    prefetch_tmap(&P.tm_k);
    prefetch_tmap(&P.tm_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<uint32_t*>(ctl_gen + K::kTmemOff);
  const bool skip_all = *reinterpret_cast<int*>(ctl_gen + K::kBadWsOff) != 0;

  if (!skip_all && (warp == kProducerWarp || warp == kProducer2Warp)) {
    // ------------------------------------------------------------------ producer
    // Lane 0 takes the waits, the work counter and the transaction counts; the results are
    // broadcast so that the whole warp follows the same control flow. Tiled loads are issued by
    // lane 0; in fused token order a temporal item's tiles are read where their rows lie
    // (fused_plan / fused_issue: whole runs as boxes by lanes 0.., edge groups gathered by lane L
    // for rows 4L .. 4L + 3).
    // Two producer warps share the ring: warp 8 claims and publishes the items, loads Q and every K
    // tile; warp 10 reads the published items and loads every V tile. Both count the ring positions
    // of every tile, so each tile keeps the position (slot and phase) the MMA warp reads it at.
    const bool vw = warp == kProducer2Warp;
    const int my_w = vw ? 1 : 0;
    uint32_t kv_pos = 0, q_iter = 0, tr_items = 0, tr_tiles = 0;
    uint32_t mine = 0;  // bit i: this warp filled ring position kv_pos - 1 - i
    bool q_issued = false;
    for (uint32_t it = 0;; ++it) {
      const uint32_t slot = it & 1u, ph = (it >> 1) & 1u;
      ItemInfo inf;
      if (vw) {  // the item warp 8 published in this slot
        if (!__shfl_sync(0xffffffffu, lane == 0 ? (int)wait_bar(c.item_full(slot), ph, abort_addr, status) : 0, 0))
          break;
        inf = items[slot];
        __syncwarp();
        if (lane == 0) mbar_arrive(c.item_empty(slot));
        if (!inf.valid) break;
      } else {
      if (!__shfl_sync(0xffffffffu, lane == 0 ? (int)wait_bar(c.item_empty(slot), ph ^ 1u, abort_addr, status) : 0,
                       0))
        break;
      if (P.order == kOrderWork) {
        int wc = 0;
        uint32_t wpos = 0;
        const bool got = lane == 0 ? claim_work_item(P, wc, wpos) : false;
        const uint32_t code = __shfl_sync(0xffffffffu, got ? ((uint32_t)wc << 31) | wpos : 0xFFFFFFFFu, 0);
        if (code == 0xFFFFFFFFu) {
          memset(&inf, 0, sizeof(inf));
        } else {
          inf = decode_work_item(P, (int)(code >> 31), code & 0x7FFFFFFFu);
        }
      } else {
        const uint32_t idx = __shfl_sync(0xffffffffu, lane == 0 ? atomicAdd(P.counter, 1u) : 0u, 0);
        inf = decode_item<BK>(P, idx);
      }
      if (lane == 0) {
        items[slot] = inf;
        mbar_arrive(c.item_full(slot));
        if (inf.valid) {
          ++tr_items;
          tr_tiles += (uint32_t)(inf.nA + inf.nB);
        }
      }
      if (!inf.valid) break;
      }
      const bool gat = P.fused && inf.cls == SVG_ROUTE_TEMPORAL;
      if (!vw && inf.nA + inf.nB > 0) {
        if (!__shfl_sync(0xffffffffu, lane == 0 ? (int)wait_bar(c.q_free(), (q_iter & 1u) ^ 1u, abort_addr, status) : 0,
                         0))
          break;
        ++q_iter;
        FusedPlan qpl[2];
        uint32_t qbytes = 0;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          if ((h == 0 ? inf.nA : inf.nB) == 0) continue;
          if (gat) {
            qpl[h] = fused_plan_rows<kHalfRows>(P, inf.head, inf.pair * kPairRows + h * kHalfRows, lane);
            qbytes += fused_bytes<kHalfRows, C::kChunks>(P, qpl[h]);
          } else {
            qbytes += (uint32_t)C::kQHalfBytes;
          }
        }
        if (lane == 0) mbar_expect_tx(c.q_full(), qbytes);
        __syncwarp();
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          if ((h == 0 ? inf.nA : inf.nB) == 0) continue;
          const int p0 = inf.pair * kPairRows + h * kHalfRows;
          if (gat) {
            fused_issue<kHalfRows, C::kChunks>(P, qpl[h], &P.tm_q, &P.tm_q4, &P.tm_q2, sQ + h * C::kQHalfBytes,
                                               c.q_full(), inf.head, p0, lane);
          } else if (lane == 0) {
            for (int ch = 0; ch < C::kQKChunks; ++ch)
              tma_load_3d(sQ + h * C::kQHalfBytes + ch * (128 * 128), &P.tm_q, c.q_full(), ch * C::kQKColsPerChunk, p0,
                          inf.head);
          }
        }
        q_issued = true;
      }
      // K / V loads in the order the MMA warp consumes them: K(e), V(e) per entry; with P in
      // shared memory S(e+1) comes before P V(e): K(0), then K(e+1), V(e) per entry.
      // the last two entries' key-tile rows, {entry, row0} by entry parity, and in fused order their
      // copy plans: each entry's are worked out once, for its K and its V tile
      int ca[2] = {-1, 0}, cb[2] = {-1, 0};
      FusedPlan pa, pb;
      auto fill = [&](int (&cc)[2], FusedPlan& pl, int e) {
        cc[0] = e;
        cc[1] = (int)ent_kt(get_entry<BK>(P, inf, e)) * BK;
        if (gat) pl = fused_plan_rows<BK>(P, inf.head, cc[1], lane);
      };
      bool ok = true;
      for (int n = 0; n < 2 * inf.count && ok; ++n) {
        int e, w;
        if (!PS) {
          e = n >> 1;
          w = n & 1;
        } else if (n == 0) {
          e = 0;
          w = 0;
        } else if (n == 2 * inf.count - 1) {
          e = inf.count - 1;
          w = 1;
        } else {
          const int m = n - 1;
          e = (m >> 1) + ((m & 1) ^ 1);
          w = m & 1;
        }
        if (w != my_w) {  // the other producer's tile: its position only
          ++kv_pos;
          mine <<= 1;
          continue;
        }
        int row0;
        FusedPlan kpl;
        if ((e & 1) == 0) {
          if (ca[0] != e) fill(ca, pa, e);
          row0 = ca[1];
          kpl = pa;
        } else {
          if (cb[0] != e) fill(cb, pb, e);
          row0 = cb[1];
          kpl = pb;
        }
        const uint32_t st = kv_pos % NS, phs = (kv_pos / NS) & 1u;
        if (!__shfl_sync(0xffffffffu, lane == 0 ? (int)wait_bar(c.kv_empty(st), phs ^ 1u, abort_addr, status) : 0,
                         0)) {
          ok = false;
          break;
        }
        if (lane == 0)
          mbar_expect_tx(c.kv_full(st), gat ? fused_bytes<BK, C::kChunks>(P, kpl) : (w == 0 ? C::kKBytes : C::kVBytes));
        __syncwarp();
        const uint32_t dst = sRing + st * C::kTileBytes;
        if (gat) {
          fused_issue<BK, C::kChunks>(P, kpl, w == 0 ? &P.tm_k : &P.tm_v, w == 0 ? &P.tm_k4 : &P.tm_v4,
                                      w == 0 ? &P.tm_k2 : &P.tm_v2, dst, c.kv_full(st), inf.head, row0, lane);
        } else if (lane == 0) {
          if (w == 0) {
            for (int ch = 0; ch < C::kQKChunks; ++ch)
              tma_load_3d(dst + ch * (BK * 128), &P.tm_k, c.kv_full(st), ch * C::kQKColsPerChunk, row0, inf.head);
          } else {
            for (int ch = 0; ch < C::kChunks; ++ch)
              tma_load_3d(dst + ch * (BK * 128), &P.tm_v, c.kv_full(st), ch * 64, row0, inf.head);
          }
        }
        ++kv_pos;
        mine = (mine << 1) | 1u;
      }
      if (!ok) break;
    }
    if (lane == 0 && ld_shared_volatile(abort_addr)) {  // let issued copies land before the CTA may exit
      // (each producer drains the positions it filled among the last NS)
      const uint32_t n = kv_pos < (uint32_t)NS ? kv_pos : (uint32_t)NS;
      for (uint32_t i = 0; i < n; ++i) {
        if (!((mine >> i) & 1u)) continue;
        const uint32_t pos = kv_pos - 1 - i;
        drain_bar(c.kv_full(pos % NS), (pos / NS) & 1u);
      }
      if (q_issued) drain_bar(c.q_full(), (q_iter - 1) & 1u);
    }
    if (lane == 0 && !vw) {  // this CTA's share of the work, for the optional trace
      *reinterpret_cast<uint32_t*>(ctl_gen + K::kTraceOff) = tr_items;
      *reinterpret_cast<uint32_t*>(ctl_gen + K::kTraceOff + 4) = tr_tiles;
    }
  } else if (!skip_all && warp == kMmaWarp) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = QK8 ? idesc_e4m3_f32(BK) : idesc_bf16_f32(BK, false);
      constexpr uint32_t idesc_o = idesc_bf16_f32(D, true);
      // Descriptors are built once; per k-step and per ring slot only the start-address
      // field (bits [0,14), address >> 4) moves, and no address exceeds 256 KB, so a plain add
      // on the low word never carries out of the field.
      const uint64_t qdesc = smem_desc_sw128(sQ, 16, 1024);
      const uint64_t kdesc = smem_desc_sw128(sRing, 16, 1024);
      const uint64_t vdesc = smem_desc_sw128(sRing, BK * 128, 1024);
      // S_h = Q_h K^T from the K tile at descriptor kd, then s_full[h]
      auto issue_s = [&](int h, uint64_t kd) {
        const uint64_t qd = qdesc + ((h * C::kQHalfBytes) >> 4);
        if constexpr (QK8) {
#pragma unroll
          for (int kk = 0; kk < D / 32; ++kk) {
            // 32 e4m3 = 32 bytes along K inside a 128-byte swizzle atom; 128 columns per atom
            const uint32_t qoff = ((kk >> 2) * (128 * 128) + (kk & 3) * 32) >> 4;
            const uint32_t koff = ((kk >> 2) * (BK * 128) + (kk & 3) * 32) >> 4;
            umma_ss_f8(tmem + C::s_col(h), qd + qoff, kd + koff, idesc_s, kk > 0 ? 1u : 0u);
          }
        } else {
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            // 16 bf16 = 32 bytes along K inside a 128-byte swizzle atom; 64 columns per atom
            const uint32_t qoff = ((kk >> 2) * (128 * 128) + (kk & 3) * 32) >> 4;
            const uint32_t koff = ((kk >> 2) * (BK * 128) + (kk & 3) * 32) >> 4;
            umma_ss(tmem + C::s_col(h), qd + qoff, kd + koff, idesc_s, kk > 0 ? 1u : 0u);
          }
        }
        umma_commit(c.s_full(h));
      };
      uint32_t kv_pos = 0, q_iter = 0, p_cnt0 = 0, p_cnt1 = 0, of_cnt0 = 0, of_cnt1 = 0;
      bool ok = true;
      if constexpr (PS) {
        // P in shared memory. Per entry e: S_h(e+1) as soon as the softmax has loaded S_h(e)
        // (s_free), then O_h += P_h(e) V(e) once P_h(e) is stored (p_ready); every P V commits
        // pv_done[h] (the o_done barrier), which frees P_h's buffer and orders O_h for the softmax.
        const uint64_t pdesc = smem_desc_sw128(sP, 16, 1024);
        uint32_t sf_cnt0 = 0, sf_cnt1 = 0;
        // S(e) of the entry's active halves from ring position kpos, then the K slot's release
        auto s_entry = [&](uint32_t ent, uint32_t kpos, bool last_s) -> bool {
          bool k_ready = false;
          const uint64_t kd = kdesc + (((kpos % NS) * C::kTileBytes) >> 4);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            if (ent_flag(ent, h) == kFlagSkip) continue;
            uint32_t& sc = h == 0 ? sf_cnt0 : sf_cnt1;
            if (sc > 0 && !wait_bar(c.s_free(h), (sc - 1) & 1u, abort_addr, status)) return false;
            ++sc;
            if (!k_ready) {
              if (!wait_bar(c.kv_full(kpos % NS), (kpos / NS) & 1u, abort_addr, status)) return false;
              k_ready = true;
            }
            tc_fence_after();  // after the softmax's loads of the previous S_h
            issue_s(h, kd);
          }
          if (!k_ready && !wait_bar(c.kv_full(kpos % NS), (kpos / NS) & 1u, abort_addr, status)) return false;
          umma_commit(c.kv_empty(kpos % NS));  // K read by the S MMAs
          if (last_s) umma_commit(c.q_free());  // Q read by the item's last S MMA
          return true;
        };
        for (uint32_t it = 0; ok; ++it) {
          const uint32_t slot = it & 1u, ph = (it >> 1) & 1u;
          if (!wait_bar(c.item_full(slot), ph, abort_addr, status)) break;
          const ItemInfo inf = items[slot];
          mbar_arrive(c.item_empty(slot));
          if (!inf.valid) break;
          if (inf.nA + inf.nB > 0) {
            if (!wait_bar(c.q_full(), q_iter & 1u, abort_addr, status)) break;
            ++q_iter;
          }
          uint32_t has_o = 0;
          uint32_t ent_n = inf.count > 0 ? get_entry<BK>(P, inf, 0) : 0u;
          if (inf.count > 0) ok = s_entry(ent_n, kv_pos++, inf.count == 1);
          for (int e = 0; e < inf.count && ok; ++e) {
            const uint32_t ent = ent_n;
            if (e + 1 < inf.count) {
              ent_n = get_entry<BK>(P, inf, e + 1);
              ok = s_entry(ent_n, kv_pos++, e + 2 == inf.count);
              if (!ok) break;
            }
            const uint32_t vpos = kv_pos++;
            bool v_ready = false;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              if (ent_flag(ent, h) == kFlagSkip) continue;
              uint32_t& pc = h == 0 ? p_cnt0 : p_cnt1;
              uint32_t& oc = h == 0 ? of_cnt0 : of_cnt1;
              ok = wait_bar(c.p_ready(h), pc & 1u, abort_addr, status);
              ++pc;
              if (ok && !((has_o >> h) & 1u)) {
                ok = wait_bar(c.o_free(h), (oc & 1u) ^ 1u, abort_addr, status);
                ++oc;
              }
              if (ok && !v_ready) {
                ok = wait_bar(c.kv_full(vpos % NS), (vpos / NS) & 1u, abort_addr, status);
                v_ready = true;
              }
              if (!ok) break;
              tc_fence_after();
              const uint64_t vd = vdesc + (((vpos % NS) * C::kTileBytes) >> 4);
              const uint64_t pd = pdesc + ((h * C::kPHalfBytes) >> 4);
              const uint32_t acc0 = (has_o >> h) & 1u;
#pragma unroll
              for (int kk = 0; kk < BK / 16; ++kk) {
                const uint32_t poff = ((kk >> 2) * (128 * 128) + (kk & 3) * 32) >> 4;
                umma_ss(tmem + C::o_col(h), pd + poff, vd + ((kk * 2048) >> 4), idesc_o,
                        (acc0 || kk > 0) ? 1u : 0u);
              }
              umma_commit(c.o_done(h));
              has_o |= 1u << h;
            }
            if (!ok) break;
            if (!v_ready) {
              ok = wait_bar(c.kv_full(vpos % NS), (vpos / NS) & 1u, abort_addr, status);
              if (!ok) break;
            }
            umma_commit(c.kv_empty(vpos % NS));  // V read by the P V MMAs
          }
        }
      }
      for (uint32_t it = 0; ok && !PS; ++it) {
        const uint32_t slot = it & 1u, ph = (it >> 1) & 1u;
        if (!wait_bar(c.item_full(slot), ph, abort_addr, status)) break;
        const ItemInfo inf = items[slot];
        mbar_arrive(c.item_empty(slot));
        if (!inf.valid) break;
        if (inf.nA + inf.nB > 0) {  // (TMA data: the barrier alone orders it for the tensor core)
          if (!wait_bar(c.q_full(), q_iter & 1u, abort_addr, status)) break;
          ++q_iter;
        }
        int rem0 = inf.nA, rem1 = inf.nB;   // active entries left per half
        uint32_t prev_act = 0, has_o = 0;    // bit h: half h active at the previous entry / O_h written
        uint32_t prev_v = 0;
        for (int e = 0; e <= inf.count && ok; ++e) {
          // entry e (or, at e == count, only the trailing P V of the last entry)
          const bool last = e == inf.count;
          const uint32_t ent = last ? 0u : get_entry<BK>(P, inf, e);
          const uint32_t kpos = kv_pos, vpos = kv_pos + 1;
          bool k_ready = false;
          const uint64_t kd = kdesc + (((kpos % NS) * C::kTileBytes) >> 4);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            if (!ok) break;
            if ((prev_act >> h) & 1u) {  // O_h += P_h V(e-1): needs P_h and, first time, a free O_h
              uint32_t& pc = h == 0 ? p_cnt0 : p_cnt1;
              uint32_t& oc = h == 0 ? of_cnt0 : of_cnt1;
              ok = wait_bar(c.p_ready(h), pc & 1u, abort_addr, status);
              ++pc;
              if (ok && !((has_o >> h) & 1u)) {
                ok = wait_bar(c.o_free(h), (oc & 1u) ^ 1u, abort_addr, status);
                ++oc;
              }
              if (ok) ok = wait_bar(c.kv_full(prev_v % NS), (prev_v / NS) & 1u, abort_addr, status);
              if (!ok) break;
              tc_fence_after();
              const uint64_t vd = vdesc + (((prev_v % NS) * C::kTileBytes) >> 4);
              const uint32_t acc0 = (has_o >> h) & 1u;
#pragma unroll
              for (int kk = 0; kk < BK / 16; ++kk)
                umma_ts(tmem + C::o_col(h), tmem + C::s_col(h) + C::kPCol + kk * 8, vd + ((kk * 2048) >> 4),
                        idesc_o, (acc0 || kk > 0) ? 1u : 0u);
              has_o |= 1u << h;
              int& rem = h == 0 ? rem0 : rem1;
              if (--rem == 0) umma_commit(c.o_done(h));
            }
            const bool act = !last && ent_flag(ent, h) != kFlagSkip;
            if (act) {
              if (!k_ready) {  // TMA data: no tcgen05 fence needed; S_h's order against the softmax's
                               // TMEM reads comes from the fence after the last P_h wait
                ok = wait_bar(c.kv_full(kpos % NS), (kpos / NS) & 1u, abort_addr, status);
                if (!ok) break;
                k_ready = true;
              }
              issue_s(h, kd);
            }
            prev_act = (prev_act & ~(1u << h)) | ((act ? 1u : 0u) << h);
          }
          if (!ok) break;
          if (e > 0) umma_commit(c.kv_empty(prev_v % NS));  // V(e-1) read by the P V MMAs
          if (last) break;
          if (!k_ready) {  // (an entry always has an active half; never release a slot still loading)
            ok = wait_bar(c.kv_full(kpos % NS), (kpos / NS) & 1u, abort_addr, status);
            if (!ok) break;
          }
          umma_commit(c.kv_empty(kpos % NS));            // K(e) read by the S MMAs
          if (e == inf.count - 1) umma_commit(c.q_free());  // Q read by the last S MMA
          prev_v = vpos;
          kv_pos += 2;
        }
      }
      // all issued MMAs complete before TMEM is released
      umma_commit(c.drain());
      drain_bar(c.drain(), 0);
    }
    __syncwarp();
  } else if (!skip_all && warp < 8) {
    // ------------------------------------------------------------------ softmax groups
    const int h = warp >> 2;
    const int lr = threadIdx.x & 127;                    // row within the half = TMEM lane
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_off + C::s_col(h);
    const uint32_t tP = tS + C::kPCol;
    const uint32_t tO = tmem + lane_off + C::o_col(h);
    const uint32_t sPh = sP + h * C::kPHalfBytes;
    const float sl2 = P.sl2;
    uint32_t s_cnt = 0, od_cnt = 0, pv_cnt = 0;
    // (test hook) a wait that nothing satisfies: it gives up after the limit, raises the abort
    // flag and the timeout status, and every role drains and leaves
    const bool stalled = P.inject_stall && !__all_sync(0xffffffffu, wait_bar(c.never(), 0, abort_addr, status));
    for (uint32_t it = 0; !stalled; ++it) {
      const uint32_t slot = it & 1u, ph = (it >> 1) & 1u;
      if (!__all_sync(0xffffffffu, wait_bar(c.item_full(slot), ph, abort_addr, status))) break;
      const ItemInfo inf = items[slot];
      __syncwarp();
      if (lane == 0) mbar_arrive(c.item_empty(slot));
      if (!inf.valid) break;
      const int row = inf.pair * kPairRows + h * kHalfRows + lr;
      const bool in_range = row < P.N;
      const int nmine = h == 0 ? inf.nA : inf.nB;
      const int prow = in_range ? row : P.N - 1;
      // where the row lives in Q / O / LSE: its position, or its original index in fused order
      const int orow_idx = (P.fused && inf.cls == SVG_ROUTE_TEMPORAL) ? orig_index(P.g[SVG_ROUTE_TEMPORAL], prow) : prow;
      const bool store_ok = check_ok(orow_idx >= 0 && orow_idx < P.N && inf.head >= 0 && inf.head < P.H, P.checks);
      if (nmine == 0) {  // no kept key for any row of this half (rounded masks only)
        if (in_range && store_ok) {
          __nv_bfloat16* orow = P.o + ((size_t)inf.head * P.N + orow_idx) * D;
          const uint4 z = make_uint4(0, 0, 0, 0);
          for (int x = 0; x < D / 8; ++x) reinterpret_cast<uint4*>(orow)[x] = z;
          if (P.lse) P.lse[(size_t)inf.head * P.N + orow_idx] = -INFINITY;
        }
        continue;
      }
      // kept keys of this row: [0, se) U [lo, hi) U (periodic sink), see svg_common.cuh
      int lo = 0, hi = 0, se = 0;
      bool per = false;
      if (!P.dense) {
        const MaskGeom& g = P.g[inf.cls];
        row_interval(g, prow, lo, hi);
        se = sink_end(g);
        per = periodic_sink(g);
      }
      float m = -INFINITY, l = 0.f;
      bool first = true;
      bool ok = true;
      uint32_t ent_next = inf.count > 0 ? get_entry<BK>(P, inf, 0) : 0u;
      for (int e = 0; e < inf.count; ++e) {
        const uint32_t ent = ent_next;
        if (e + 1 < inf.count) ent_next = get_entry<BK>(P, inf, e + 1);  // hide the load latency
        const uint32_t f = ent_flag(ent, h);
        if (f == kFlagSkip) continue;
        const int c0 = (int)ent_kt(ent) * BK;
        if (!__all_sync(0xffffffffu, wait_bar(c.s_full(h), s_cnt & 1u, abort_addr, status))) {
          ok = false;
          break;
        }
        ++s_cnt;
        tc_fence_after();
        uint32_t r[BK];
        float alpha = 1.f;
        float2 acc[2];
        load_scores<BK>(tS, r);
        if constexpr (PS) {  // S_h's columns are free for the next tile's S_h
          tc_fence_before();
          mbar_arrive(c.s_free(h));
        }
        mask_scores<BK>(P, inf.cls, f, c0, prow, ent, lo, hi, se, per, r);
        bool rescale = false;
        // Exponentials against the running maximum first, without the tile's maximum: when every
        // row's P sums to at most 2^kRescaleLog2, no P exceeds it, which is exactly when the
        // maximum-first step would not rescale, so the result is the same bit for bit. Otherwise
        // (rare) the tile is read again from TMEM, where S still is, and taken maximum first. With
        // P in shared memory S may already be overwritten, so that schedule always takes the maximum.
        bool max_step = PS || !__all_sync(0xffffffffu, m != -INFINITY);
#pragma unroll 1
        for (int pass = 0;; ++pass) {
          if (max_step) {
            if (pass > 0) {
              load_scores<BK>(tS, r);
              mask_scores<BK>(P, inf.cls, f, c0, prow, ent, lo, hi, se, per, r);
            }
            rescale = max_first<BK>(r, sl2, m, l, alpha);
          }
          exp_tile<BK>(r, sl2, m, acc);
          if (max_step) break;
          const float lt = (acc[0].x + acc[1].x) + (acc[0].y + acc[1].y);
          if (!__any_sync(0xffffffffu, !(lt <= kRescaleBound))) break;
          max_step = true;
        }
        l += (acc[0].x + acc[1].x) + (acc[0].y + acc[1].y);
        if constexpr (PS) {
          // the previous P_h V is complete: P_h's buffer is free and O_h holds every earlier P V
          if (pv_cnt > 0 &&
              !__all_sync(0xffffffffu, wait_bar(c.o_done(h), (pv_cnt - 1) & 1u, abort_addr, status))) {
            ok = false;
            break;
          }
          ++pv_cnt;
          if (rescale && !first) {
            tc_fence_after();
            rescale_o<D>(tO, alpha);
            tmem_st_wait();
          }
          store_p_sw128<BK>(sPh, lr, r);
          fence_proxy_async_shared();
          tc_fence_before();
          mbar_arrive(c.p_ready(h));
        } else {
#pragma unroll
          for (int q = 0; q < BK / 64; ++q) tmem_st32(tP + q * 32, r + q * 32);
          if (rescale && !first) rescale_o<D>(tO, alpha);  // O_h holds every earlier P V (S_h's commit covered them)
          tmem_st_wait();
          tc_fence_before();
          mbar_arrive(c.p_ready(h));
        }
        first = false;
      }
      if (!ok) break;
      // ---- epilogue: O / l -> bf16
      if constexpr (PS) {
        if (!__all_sync(0xffffffffu, wait_bar(c.o_done(h), (pv_cnt - 1) & 1u, abort_addr, status))) break;
      } else {
        if (!__all_sync(0xffffffffu, wait_bar(c.o_done(h), od_cnt & 1u, abort_addr, status))) break;
        ++od_cnt;
      }
      tc_fence_after();
      const float inv_l = (l > 0.f && m != -INFINITY) ? 1.f / l : 0.f;  // a row with no kept key gives 0
      __nv_bfloat16* orow = P.o + ((size_t)inf.head * P.N + orow_idx) * D;
#pragma unroll 1
      for (int q = 0; q < D / 32; ++q) {
        uint32_t o[32];
        tmem_ld32(tO + q * 32, o);
        tmem_ld_wait();
        tmem_ld_fence32(o);
        if (in_range && store_ok) {
          uint4* dst = reinterpret_cast<uint4*>(orow + q * 32);
#pragma unroll
          for (int x = 0; x < 4; ++x) {
            uint4 v;
            v.x = pack_bf16(__uint_as_float(o[8 * x + 0]) * inv_l, __uint_as_float(o[8 * x + 1]) * inv_l);
            v.y = pack_bf16(__uint_as_float(o[8 * x + 2]) * inv_l, __uint_as_float(o[8 * x + 3]) * inv_l);
            v.z = pack_bf16(__uint_as_float(o[8 * x + 4]) * inv_l, __uint_as_float(o[8 * x + 5]) * inv_l);
            v.w = pack_bf16(__uint_as_float(o[8 * x + 6]) * inv_l, __uint_as_float(o[8 * x + 7]) * inv_l);
            dst[x] = v;
          }
        }
      }
      tc_fence_before();
      mbar_arrive(c.o_free(h));
      if (in_range && store_ok && P.lse)
        P.lse[(size_t)inf.head * P.N + orow_idx] =
            (l > 0.f && m != -INFINITY) ? (m * sl2 + log2f(l)) * 0.69314718055994531f : -INFINITY;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) tmem_dealloc(tmem, 512);
  if (P.cta_trace && threadIdx.x == 0 && (int)blockIdx.x < P.trace_ctas) {
    unsigned long long* tr = P.cta_trace + 4 * (size_t)blockIdx.x;
    tr[0] = t_start;
    tr[1] = globaltimer_ns();
    tr[2] = *reinterpret_cast<const uint32_t*>(ctl_gen + K::kTraceOff);
    tr[3] = *reinterpret_cast<const uint32_t*>(ctl_gen + K::kTraceOff + 4);
  }
}

// ---------------------------------------------------------------------------------------
template <int D, int BK, bool QK8, bool PS>
static int launch_t(const AttnParams& P, int grid, cudaStream_t st) {
  using C = Cfg<D, BK, QK8, PS>;
  auto kern = attn_kernel<D, BK, QK8, PS>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
  if (e != cudaSuccess) return record_cuda_error("cudaFuncSetAttribute(attn_kernel)", e);
  kern<<<grid, kThreads, C::kSmemBytes, st>>>(P);
  e = cudaGetLastError();
  return e == cudaSuccess ? SVG_OK : record_cuda_error("launch attn_kernel", e);
}

template <bool PS>
static int launch_ps(const AttnParams& P, int d, int bk, int grid, cudaStream_t st) {
  if (P.qk8) {  // e4m3 Q and K: d = 128
    if (d == 128 && bk == 128) return launch_t<128, 128, true, PS>(P, grid, st);
    if (d == 128 && bk == 64) return launch_t<128, 64, true, PS>(P, grid, st);
    return SVG_ERR_UNSUPPORTED;
  }
  if (d == 128 && bk == 128) return launch_t<128, 128, false, PS>(P, grid, st);
  if (d == 128 && bk == 64) return launch_t<128, 64, false, PS>(P, grid, st);
  if (d == 64 && bk == 128) return launch_t<64, 128, false, PS>(P, grid, st);
  if (d == 64 && bk == 64) return launch_t<64, 64, false, PS>(P, grid, st);
  return SVG_ERR_UNSUPPORTED;
}

// p_smem: P staged in shared memory (the decoupled schedule) instead of TMEM.
int launch_attention(const AttnParams& P, int d, int bk, int grid, bool p_smem, cudaStream_t st) {
  return p_smem ? launch_ps<true>(P, d, bk, grid, st) : launch_ps<false>(P, d, bk, grid, st);
}

size_t attn_params_size() { return sizeof(AttnParams); }

}  // namespace svg
