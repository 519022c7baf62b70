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
//  * one CTA per SM, 320 threads, persistent; work items are (head, 256 query rows) taken
//    from a global atomic counter in head-major order, each head's items heaviest first;
//  * warp 8 issues TMA loads (128-byte swizzle) of Q once per item and of K / V tiles into a
//    shared-memory ring; warp 9 issues tcgen05 MMAs: S = Q K^T into TMEM, then O += P V with
//    P read straight from TMEM;
//  * warps 0-3 and 4-7 are two softmax groups, one per 128-row half, one thread per query
//    row (= TMEM lane). While one group turns its S into P, the tensor core computes the
//    other half's S and P V, so MMA and exponentials overlap;
//  * O is rescaled (in TMEM) only when a row maximum grows by more than 2^8, which keeps
//    the result exact while making the correction rare;
//  * every wait is bounded by a wall-clock limit; a timeout sets the status word and all
//    roles drain their in-flight copies / MMAs and return.
#include <cuda_bf16.h>
#include <string.h>

#include "svg_common.cuh"

namespace svg {

constexpr int kThreads = 320;
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s per wait
constexpr float kRescaleThreshold = 8.0f;        // log2 units


template <int D, int BK>
struct Cfg {
  static constexpr int kChunks = D / 64;            // 128-byte swizzle chunks per row
  static constexpr int kQHalfBytes = 128 * D * 2;
  static constexpr int kQBytes = 2 * kQHalfBytes;
  static constexpr int kTileBytes = BK * D * 2;     // one K or one V tile
  static constexpr int kStages = (160 * 1024) / kTileBytes;
  static constexpr int kDataBytes = kQBytes + kStages * kTileBytes;
  static constexpr int kSmemBytes = kDataBytes + 1024 /*control*/ + 1024 /*alignment slack*/;
  // TMEM columns: S (and P) of half h at 128*h, P (bf16 pairs) aliases the upper half of
  // S, O accumulators of half h at 256 + D*h.
  __host__ __device__ static constexpr uint32_t s_col(int h) { return 128u * h; }
  static constexpr uint32_t kPCol = BK / 2;
  __host__ __device__ static constexpr uint32_t o_col(int h) { return 256u + (uint32_t)D * h; }
  static_assert(kStages >= 2, "ring too small");
  static_assert((2 * kStages + 31) * 8 <= 1024, "control block");
  static_assert(kSmemBytes <= 232448, "shared memory budget");
};

struct ItemInfo {
  int valid, head, pair, cls, count, nA, nB, pad;
  const uint32_t* ents;
};

struct Ctl {
  uint64_t* kv_full;
  uint64_t* kv_empty;
  uint64_t *q_full, *q_free, *s_full, *p_ready, *o_done, *o_free, *item_full, *item_empty, *drain;
  ItemInfo* items;
  volatile int* abort_flag;
  int* status;
};

__device__ __forceinline__ void raise_error(const Ctl& c, int code) {
  *c.abort_flag = 1;
  atomicCAS(c.status, 0, code);
}

// Bounded wait on an mbarrier phase. Returns false on timeout or when another role aborted.
__device__ __noinline__ bool wait_bar(const Ctl& c, uint64_t* bar, uint32_t parity) {
  const uint32_t a = smem_u32(bar);
  if (mbar_try_wait(a, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(a, parity)) return true;
    if ((it & 15u) == 0) {
      if (*c.abort_flag) return false;
      if (globaltimer_ns() - t0 > kWaitLimitNs) {
        raise_error(c, SVG_ERR_TIMEOUT);
        return false;
      }
    }
  }
}

// Drain wait: ignores the abort flag, short limit; used only on the error path.
__device__ __noinline__ void drain_bar(uint64_t* bar, uint32_t parity) {
  const uint32_t a = smem_u32(bar);
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(a, parity))
    if (globaltimer_ns() - t0 > 200000000ull) return;
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
  return P.dense ? dense_entry<BK>(P, it, e) : __ldg(it.ents + e);
}

__device__ __forceinline__ int route_of(const AttnParams& P, int h) {
  return (P.route_bits[h >> 5] >> (h & 31)) & 1;
}

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
    const int c = it.cls;
    it.pair = (int)__ldg(P.pair_order[c] + j);
    const uint32_t b0 = __ldg(P.pair_ptr[c] + it.pair), b1 = __ldg(P.pair_ptr[c] + it.pair + 1);
    it.count = (int)(b1 - b0);
    it.ents = P.pair_ent[c] + b0;
    it.nA = (int)__ldg(P.pair_cnt[c] + 2 * it.pair);
    it.nB = (int)__ldg(P.pair_cnt[c] + 2 * it.pair + 1);
  }
  return it;
}

__device__ __forceinline__ float ex2f(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 v = __floats2bfloat162_rn(a, b);  // .x = a (low 16 bits)
  return *reinterpret_cast<uint32_t*>(&v);
}

// ---------------------------------------------------------------------------------------
template <int D, int BK>
__global__ void __launch_bounds__(kThreads, 1) attn_kernel(const __grid_constant__ AttnParams P) {
  using C = Cfg<D, BK>;
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte alignment for the 128-byte swizzle atoms
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
  uint8_t* sQ = smem;
  uint8_t* sRing = smem + C::kQBytes;
  uint8_t* ctl_base = smem + C::kDataBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(ctl_base);
  Ctl c;
  c.kv_full = bars;
  c.kv_empty = bars + C::kStages;
  uint64_t* b = bars + 2 * C::kStages;
  c.q_full = b + 0;
  c.q_free = b + 1;
  c.s_full = b + 2;      // [2]
  c.p_ready = b + 4;     // [2]
  c.o_done = b + 6;      // [2]
  c.o_free = b + 8;      // [2]
  c.item_full = b + 10;  // [2]
  c.item_empty = b + 12; // [2]
  c.drain = b + 14;
  static_assert(sizeof(ItemInfo) == 40, "item slot size");
  c.items = reinterpret_cast<ItemInfo*>(b + 16);            // 2 x 40 bytes: b[16..26)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(b + 28);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(b + 29);
  int* bad_ws = reinterpret_cast<int*>(b + 30);
  c.abort_flag = abort_flag;
  c.status = P.status;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(c.kv_full + s, 1);
      mbar_init(c.kv_empty + s, 1);
    }
    mbar_init(c.q_full, 1);
    mbar_init(c.q_free, 1);
    for (int h = 0; h < 2; ++h) {
      mbar_init(c.s_full + h, 1);
      mbar_init(c.p_ready + h, 128);
      mbar_init(c.o_done + h, 1);
      mbar_init(c.o_free + h, 128);
      mbar_init(c.item_full + h, 1);
      mbar_init(c.item_empty + h, 9);
    }
    mbar_init(c.drain, 1);
    *abort_flag = 0;
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
    *bad_ws = bad;
    if (bad) atomicCAS(P.status, 0, SVG_ERR_WORKSPACE);
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, 512);
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
  const uint32_t tmem = *tmem_slot;
  const bool skip_all = *bad_ws != 0;

  if (!skip_all && warp == kProducerWarp) {
    // ------------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t kv_pos = 0, q_iter = 0;
      bool q_issued = false;
      for (uint32_t it = 0;; ++it) {
        const uint32_t slot = it & 1u, ph = (it >> 1) & 1u;
        if (!wait_bar(c, c.item_empty + slot, ph ^ 1u)) break;
        const uint32_t idx = atomicAdd(P.counter, 1u);
        const ItemInfo inf = decode_item<BK>(P, idx);
        c.items[slot] = inf;
        mbar_arrive(c.item_full + slot);
        if (!inf.valid) break;
        if (inf.nA + inf.nB > 0) {
          if (!wait_bar(c, c.q_free, (q_iter & 1u) ^ 1u)) break;
          ++q_iter;
          const uint32_t bytes = (uint32_t)C::kQHalfBytes * ((inf.nA > 0) + (inf.nB > 0));
          mbar_expect_tx(c.q_full, bytes);
          for (int h = 0; h < 2; ++h) {
            if ((h == 0 ? inf.nA : inf.nB) == 0) continue;
            for (int ch = 0; ch < C::kChunks; ++ch)
              tma_load_3d(sQ + h * C::kQHalfBytes + ch * (128 * 128), &P.tm_q, c.q_full, ch * 64,
                          inf.pair * kPairRows + h * kHalfRows, inf.head);
          }
          q_issued = true;
        }
        bool ok = true;
        for (int e = 0; e < inf.count && ok; ++e) {
          const uint32_t ent = get_entry<BK>(P, inf, e);
          const int row0 = (int)ent_kt(ent) * BK;
          for (int w = 0; w < 2; ++w) {
            const uint32_t s = kv_pos % C::kStages, phs = (kv_pos / C::kStages) & 1u;
            if (!wait_bar(c, c.kv_empty + s, phs ^ 1u)) {
              ok = false;
              break;
            }
            mbar_expect_tx(c.kv_full + s, C::kTileBytes);
            uint8_t* dst = sRing + s * C::kTileBytes;
            for (int ch = 0; ch < C::kChunks; ++ch)
              tma_load_3d(dst + ch * (BK * 128), w == 0 ? &P.tm_k : &P.tm_v, c.kv_full + s, ch * 64, row0,
                          inf.head);
            ++kv_pos;
          }
        }
        if (!ok) break;
      }
      if (*abort_flag) {  // let issued copies land before the CTA may exit
        const uint32_t n = kv_pos < (uint32_t)C::kStages ? kv_pos : (uint32_t)C::kStages;
        for (uint32_t i = 0; i < n; ++i) {
          const uint32_t pos = kv_pos - 1 - i;
          drain_bar(c.kv_full + pos % C::kStages, (pos / C::kStages) & 1u);
        }
        if (q_issued) drain_bar(c.q_full, (q_iter - 1) & 1u);
      }
    }
    __syncwarp();
  } else if (!skip_all && warp == kMmaWarp) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(BK, false);
      constexpr uint32_t idesc_o = idesc_bf16_f32(D, true);
      const uint32_t q_base = smem_u32(sQ), ring_base = smem_u32(sRing);
      uint32_t kv_pos = 0, q_iter = 0, p_cnt[2] = {0, 0}, of_cnt[2] = {0, 0};
      bool ok = true;
      for (uint32_t it = 0; ok; ++it) {
        const uint32_t slot = it & 1u, ph = (it >> 1) & 1u;
        if (!wait_bar(c, c.item_full + slot, ph)) break;
        const ItemInfo inf = c.items[slot];
        mbar_arrive(c.item_empty + slot);
        if (!inf.valid) break;
        const bool has_q = inf.nA + inf.nB > 0;
        if (has_q) {
          if (!wait_bar(c, c.q_full, q_iter & 1u)) break;
          ++q_iter;
          tc_fence_after();
        }
        int remaining[2] = {inf.nA, inf.nB};
        bool prev_act[2] = {false, false}, has_o[2] = {false, false};
        uint32_t prev_v = 0;
        // O_h += P_h V(prev): waits for P and (first time) for the epilogue to free O_h.
        auto issue_pv = [&](int h, uint32_t vpos) -> bool {
          if (!wait_bar(c, c.p_ready + h, p_cnt[h] & 1u)) return false;
          ++p_cnt[h];
          if (!has_o[h]) {
            if (!wait_bar(c, c.o_free + h, (of_cnt[h] & 1u) ^ 1u)) return false;
            ++of_cnt[h];
          }
          if (!wait_bar(c, c.kv_full + vpos % C::kStages, (vpos / C::kStages) & 1u)) return false;
          tc_fence_after();
          const uint32_t vaddr = ring_base + (vpos % C::kStages) * C::kTileBytes;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t bdesc = smem_desc_sw128(vaddr + kk * 2048, BK * 128, 1024);
            umma_ts(tmem + C::o_col(h), tmem + C::s_col(h) + C::kPCol + kk * 8, bdesc, idesc_o,
                    (has_o[h] || kk > 0) ? 1u : 0u);
          }
          has_o[h] = true;
          if (--remaining[h] == 0) umma_commit(c.o_done + h);
          return true;
        };
        for (int e = 0; e < inf.count; ++e) {
          const uint32_t ent = get_entry<BK>(P, inf, e);
          const uint32_t kpos = kv_pos, vpos = kv_pos + 1;
          kv_pos += 2;
          if (!wait_bar(c, c.kv_full + kpos % C::kStages, (kpos / C::kStages) & 1u)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t kaddr = ring_base + (kpos % C::kStages) * C::kTileBytes;
          for (int h = 0; h < 2 && ok; ++h) {
            if (prev_act[h] && !issue_pv(h, prev_v)) {
              ok = false;
              break;
            }
            const bool act = ent_flag(ent, h) != kFlagSkip;
            if (act) {
              const uint32_t qaddr = q_base + h * C::kQHalfBytes;
#pragma unroll
              for (int kk = 0; kk < D / 16; ++kk) {
                const uint32_t off = (kk & 3) * 32;  // 16 bf16 = 32 bytes along K inside the swizzle atom
                const uint64_t adesc = smem_desc_sw128(qaddr + (kk >> 2) * (128 * 128) + off, 16, 1024);
                const uint64_t bdesc = smem_desc_sw128(kaddr + (kk >> 2) * (BK * 128) + off, 16, 1024);
                umma_ss(tmem + C::s_col(h), adesc, bdesc, idesc_s, kk > 0 ? 1u : 0u);
              }
              umma_commit(c.s_full + h);
            }
            prev_act[h] = act;
          }
          if (!ok) break;
          umma_commit(c.kv_empty + kpos % C::kStages);               // K(e) read by the S MMAs
          if (e > 0) umma_commit(c.kv_empty + (vpos - 2) % C::kStages);  // V(e-1) read by the PVs
          if (e == inf.count - 1) umma_commit(c.q_free);              // Q read by the last S MMA
          prev_v = vpos;
        }
        if (!ok) break;
        for (int h = 0; h < 2; ++h)
          if (prev_act[h] && !issue_pv(h, prev_v)) {
            ok = false;
            break;
          }
        if (!ok) break;
        if (inf.count > 0) umma_commit(c.kv_empty + prev_v % C::kStages);
      }
      // all issued MMAs complete before TMEM is released
      umma_commit(c.drain);
      drain_bar(c.drain, 0);
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
    const float sl2 = P.sl2;
    uint32_t s_cnt = 0, od_cnt = 0;
    for (uint32_t it = 0;; ++it) {
      const uint32_t slot = it & 1u, ph = (it >> 1) & 1u;
      if (!__all_sync(0xffffffffu, wait_bar(c, c.item_full + slot, ph))) break;  // warp-uniform exit
      const ItemInfo inf = c.items[slot];
      __syncwarp();
      if (lane == 0) mbar_arrive(c.item_empty + slot);
      if (!inf.valid) break;
      const int row = inf.pair * kPairRows + h * kHalfRows + lr;
      const bool in_range = row < P.N;
      const int nmine = h == 0 ? inf.nA : inf.nB;
      __nv_bfloat16* orow = P.o + ((size_t)inf.head * P.N + (in_range ? row : 0)) * D;
      if (nmine == 0) {  // no kept key for any row of this half (rounded masks only)
        if (in_range) {
          uint4 z = make_uint4(0, 0, 0, 0);
          for (int x = 0; x < D / 8; ++x) reinterpret_cast<uint4*>(orow)[x] = z;
          if (P.lse) P.lse[(size_t)inf.head * P.N + row] = -INFINITY;
        }
        continue;
      }
      const MaskGeom& g = P.g[inf.cls];
      const int prow = in_range ? row : P.N - 1;
      int lo = 0, hi = 0;
      if (!P.dense) row_interval(g, prow, lo, hi);
      const int se = P.dense ? 0 : sink_end(g);
      const bool per = !P.dense && periodic_sink(g);
      const uint8_t* rcls = P.cls[inf.cls] + (size_t)(prow / (P.bq > 0 ? P.bq : 1)) * P.nk;
      float m = -INFINITY, l = 0.f;
      bool first = true;
      bool ok = true;
      for (int e = 0; e < inf.count; ++e) {
        const uint32_t ent = get_entry<BK>(P, inf, e);
        const uint32_t f = ent_flag(ent, h);
        if (f == kFlagSkip) continue;
        const int c0 = (int)ent_kt(ent) * BK;
        if (!__all_sync(0xffffffffu, wait_bar(c, c.s_full + h, s_cnt & 1u))) {
          ok = false;
          break;
        }
        ++s_cnt;
        tc_fence_after();
        uint32_t r[BK];
#pragma unroll
        for (int q = 0; q < BK / 32; ++q) tmem_ld32(tS + q * 32, r + q * 32);
        tmem_ld_wait();
#pragma unroll
        for (int q = 0; q < BK / 32; ++q) tmem_ld_fence32(r + q * 32);
        float* s = reinterpret_cast<float*>(r);
        // ---- masking
        const bool elem = (f == kFlagMasked) || (P.naive && !P.dense);
        if (elem || f == kFlagBounds) {
          const int nn = P.N - c0;
          if (!elem) {
#pragma unroll
            for (int j = 0; j < BK; ++j)
              if (j >= nn) s[j] = -INFINITY;
          } else if (P.variant == SVG_MASK_ROUNDED) {
            const bool rowkept = __ldg(rcls + ent_kt(ent)) == 1;
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
        // ---- online softmax
        float mx = s[0];
#pragma unroll
        for (int j = 1; j < BK; ++j) mx = fmaxf(mx, s[j]);
        const float m_new = fmaxf(m, mx);
        const bool need = (m_new > m) && (m == -INFINITY || (m_new - m) * sl2 > kRescaleThreshold);
        if (__any_sync(0xffffffffu, need)) {
          const float alpha = (m_new == -INFINITY) ? 1.f : ex2f((m - m_new) * sl2);
          if (!first) {
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
          l *= alpha;
          m = m_new;
        }
        const float base = (m == -INFINITY) ? 0.f : m * sl2;
        uint32_t pk[BK / 2];
        float lsum = 0.f;
#pragma unroll
        for (int j = 0; j < BK; j += 2) {
          const float p0 = ex2f(fmaf(s[j], sl2, -base));
          const float p1 = ex2f(fmaf(s[j + 1], sl2, -base));
          lsum += p0 + p1;
          pk[j / 2] = pack_bf16(p0, p1);
        }
        l += lsum;
#pragma unroll
        for (int q = 0; q < BK / 64; ++q) tmem_st32(tP + q * 32, pk + q * 32);
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(c.p_ready + h);
        first = false;
      }
      if (!ok) break;
      // ---- epilogue: O / l -> bf16
      if (!__all_sync(0xffffffffu, wait_bar(c, c.o_done + h, od_cnt & 1u))) break;
      ++od_cnt;
      tc_fence_after();
      const float inv_l = l > 0.f ? 1.f / l : 0.f;
#pragma unroll 1
      for (int q = 0; q < D / 32; ++q) {
        uint32_t o[32];
        tmem_ld32(tO + q * 32, o);
        tmem_ld_wait();
        tmem_ld_fence32(o);
        if (in_range) {
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
      mbar_arrive(c.o_free + h);
      if (in_range && P.lse)
        P.lse[(size_t)inf.head * P.N + row] =
            l > 0.f ? (m * sl2 + log2f(l)) * 0.69314718055994531f : -INFINITY;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) tmem_dealloc(tmem, 512);
}

// ---------------------------------------------------------------------------------------
template <int D, int BK>
static int launch_t(const AttnParams& P, int grid, cudaStream_t st) {
  using C = Cfg<D, BK>;
  auto kern = attn_kernel<D, BK>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes) != cudaSuccess)
    return SVG_ERR_CUDA;
  kern<<<grid, kThreads, C::kSmemBytes, st>>>(P);
  return cudaGetLastError() == cudaSuccess ? SVG_OK : SVG_ERR_CUDA;
}

int launch_attention(const AttnParams& P, int d, int bk, int grid, cudaStream_t st) {
  if (d == 128 && bk == 128) return launch_t<128, 128>(P, grid, st);
  if (d == 128 && bk == 64) return launch_t<128, 64>(P, grid, st);
  if (d == 64 && bk == 128) return launch_t<64, 128>(P, grid, st);
  if (d == 64 && bk == 64) return launch_t<64, 64>(P, grid, st);
  return SVG_ERR_UNSUPPORTED;
}

size_t attn_params_size() { return sizeof(AttnParams); }

}  // namespace svg
