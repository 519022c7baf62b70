// svg_attention2.cu -- block-sparse flash-attention forward on SM pairs (d = 128).
//
// Same computation as svg_attention.cu (softmax attention restricted to the kept pairs of each
// head's spatial or temporal mask, visiting only non-empty key tiles, full tiles unmasked and
// boundary tiles element-masked: "Efficient Kernel Implementation", tile-aware masking, of
// "Accelerating Spatio-Temporal Attention for Video Diffusion on TPUs"), arranged for B200's
// two-SM tensor-core instructions:
//  * a cluster of two CTAs on two SMs handles 512 query rows of one head; each CTA owns 256
//    rows as two 128-row halves (TMEM lanes), and both halves of index h form one MMA phase;
//  * the even CTA issues tcgen05.mma.cta_group::2 (M = 256): each SM supplies its own 128 Q
//    rows and HALF of every K tile (BK/2 keys) and HALF of every V tile (64 of the 128 head
//    dimensions), so each SM moves half the K/V bytes of the one-SM kernel from L2 into shared
//    memory while receiving its full 128 x BK scores and 128 x 128 outputs in its own TMEM;
//  * per CTA: warp 8 loads (TMA, each CTA its own copy) Q halves and its K/V halves; warps 0-3 / 4-7
//    are the softmax groups of the two halves; warp 9 of the even CTA issues the MMAs;
//  * completion of every TMA copy of both CTAs is counted on the even CTA's barriers; MMA
//    completion is signalled to the barriers of both CTAs (one commit per CTA); the odd CTA's
//    softmax threads arrive on the even CTA's barriers through their cluster addresses;
//  * every wait is bounded; a timeout aborts both CTAs of the pair.
#include <cuda_bf16.h>
#include <string.h>

#include "svg_common.cuh"

namespace svg {
namespace pair2 {

constexpr int kThreads = 320;
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s per wait
constexpr float kRescaleThreshold = 8.0f;        // log2 units

template <int BK>
struct Cfg {
  static constexpr int D = 128;
  static constexpr int kQHalfBytes = 128 * D * 2;        // 32 KB: 128 rows x 128 dims
  static constexpr int kQBytes = 2 * kQHalfBytes;
  static constexpr int kKRows = BK / 2;                  // keys of a K tile held by one SM
  static constexpr int kKBytes = kKRows * D * 2;         // two 64-dim swizzle chunks
  static constexpr int kVBytes = BK * 64 * 2;            // BK keys x 64 dims (one chunk)
  static constexpr int kSlotBytes = kKBytes;
  static_assert(kKBytes == kVBytes, "ring slots hold either half tile");
  static constexpr int kStages = (160 * 1024) / kSlotBytes;
  static constexpr int kDataBytes = kQBytes + kStages * kSlotBytes;
  static constexpr int kSmemBytes = kDataBytes + 1024 /*control*/ + 1024 /*alignment slack*/;
  __host__ __device__ static constexpr uint32_t s_col(int h) { return 128u * h; }
  static constexpr uint32_t kPCol = BK / 2;
  __host__ __device__ static constexpr uint32_t o_col(int h) { return 256u + 128u * h; }
  static_assert(kSmemBytes <= 232448, "shared memory budget");
};

struct ItemInfo {
  int valid, head, quad, cls, count, nA, nB, pad;  // nA / nB: entries in which phase 0 / 1 runs
  const uint32_t* ents;
};
static_assert(sizeof(ItemInfo) == 40, "item slot size");

// Control block (same shared offsets in both CTAs), 8-byte slots:
//   [0, NS) kv_full   [NS, 2NS) kv_empty   2NS+0 q_full   2NS+1 q_free
//   2NS+2+h s_full    2NS+4+h p_ready      2NS+6+h o_done 2NS+8+h o_free
//   2NS+10+i item_full  2NS+12+i item_empty  2NS+14 drain ; then 2 items, TMEM base, abort, check.
// kv_full, q_full, p_ready, o_free, item_empty and drain are used in the even CTA only.
template <int NS>
struct Ctl {
  uint32_t base;  // this CTA's control block (shared::cta address == its own cluster address)
  uint32_t lead;  // the even CTA's control block (shared::cluster address)
  uint32_t peer;  // the other CTA's control block (shared::cluster address)
  __device__ __forceinline__ uint32_t kv_full(uint32_t b, uint32_t s) const { return b + 8u * s; }
  __device__ __forceinline__ uint32_t kv_empty(uint32_t b, uint32_t s) const { return b + 8u * (NS + s); }
  __device__ __forceinline__ uint32_t q_full(uint32_t b) const { return b + 8u * (2 * NS + 0); }
  __device__ __forceinline__ uint32_t q_free(uint32_t b) const { return b + 8u * (2 * NS + 1); }
  __device__ __forceinline__ uint32_t s_full(uint32_t b, int h) const { return b + 8u * (2 * NS + 2 + h); }
  __device__ __forceinline__ uint32_t p_ready(uint32_t b, int h) const { return b + 8u * (2 * NS + 4 + h); }
  __device__ __forceinline__ uint32_t o_done(uint32_t b, int h) const { return b + 8u * (2 * NS + 6 + h); }
  __device__ __forceinline__ uint32_t o_free(uint32_t b, int h) const { return b + 8u * (2 * NS + 8 + h); }
  __device__ __forceinline__ uint32_t item_full(uint32_t b, uint32_t i) const { return b + 8u * (2 * NS + 10 + i); }
  __device__ __forceinline__ uint32_t item_empty(uint32_t b, uint32_t i) const { return b + 8u * (2 * NS + 12 + i); }
  __device__ __forceinline__ uint32_t drain(uint32_t b) const { return b + 8u * (2 * NS + 14); }
  static constexpr uint32_t kItemsOff = 8u * (2 * NS + 16);  // 2 x 40 bytes
  static constexpr uint32_t kTmemOff = kItemsOff + 96;
  static constexpr uint32_t kAbortOff = kTmemOff + 8;
  static constexpr uint32_t kBadWsOff = kAbortOff + 8;
  static constexpr uint32_t kBytes = kBadWsOff + 8;
};

__device__ __forceinline__ int ld_volatile_shared(uint32_t addr) {
  int v;
  asm volatile("ld.volatile.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
  return v;
}

struct Abort {
  uint32_t local;   // shared address of this CTA's abort flag
  uint32_t remote;  // cluster address of the other CTA's abort flag
  int* status;
};

// Bounded wait (acquire at cluster scope). On timeout both CTAs of the pair are told to stop.
__device__ __noinline__ bool wait_bar(uint32_t bar, uint32_t parity, const Abort& ab) {
  if (mbar_try_wait_cluster(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    if ((it & 15u) == 0) {
      if (ld_volatile_shared(ab.local)) return false;
      if (globaltimer_ns() - t0 > kWaitLimitNs) {
        asm volatile("st.volatile.shared.b32 [%0], %1;" ::"r"(ab.local), "r"(1) : "memory");
        st_cluster_u32(ab.remote, 1u);
        atomicCAS(ab.status, 0, SVG_ERR_TIMEOUT);
        return false;
      }
    }
  }
}

__device__ __noinline__ void drain_bar(uint32_t a, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait_cluster(a, parity))
    if (globaltimer_ns() - t0 > 200000000ull) return;
}

__device__ __forceinline__ int route_of(const AttnParams& P, int h) {
  return (P.route_bits[h >> 5] >> (h & 31)) & 1;
}

template <int BK>
__device__ __forceinline__ uint32_t get_entry(const AttnParams& P, const ItemInfo& it, int e) {
  if (!P.dense) return __ldg(it.ents + e);
  const bool ragged = (e == P.nk - 1) && (P.N % BK != 0);
  const uint32_t f = ragged ? kFlagBounds : kFlagFull;
  uint32_t ent = (uint32_t)e;
#pragma unroll
  for (int r = 0; r < 2; ++r)
#pragma unroll
    for (int h = 0; h < 2; ++h)
      if (it.quad * kQuadRows + r * kPairRows + h * kHalfRows < P.N) ent |= f << (24 + 4 * r + 2 * h);
  return ent;
}

__device__ __forceinline__ bool phase_active(uint32_t ent, int h) {
  return (qent_flag(ent, 0, h) | qent_flag(ent, 1, h)) != 0;
}

__device__ ItemInfo decode_item(const AttnParams& P, uint32_t idx) {
  ItemInfo it;
  memset(&it, 0, sizeof(it));
  if (idx >= (uint32_t)P.n_items) return it;
  it.valid = 1;
  it.head = (int)(idx / (uint32_t)P.nquads);
  const int j = (int)(idx - (uint32_t)it.head * (uint32_t)P.nquads);
  it.cls = route_of(P, it.head);
  if (P.dense) {
    it.quad = j;
    it.count = P.nk;
    it.nA = P.nk;
    it.nB = (j * kQuadRows + kHalfRows < P.N) ? P.nk : 0;
    it.ents = nullptr;
  } else {
    const int c = it.cls;
    it.quad = (int)__ldg(P.quad_order[c] + j);
    const uint32_t b0 = __ldg(P.quad_ptr[c] + it.quad), b1 = __ldg(P.quad_ptr[c] + it.quad + 1);
    it.count = (int)(b1 - b0);
    it.ents = P.quad_ent[c] + b0;
    it.nA = (int)__ldg(P.quad_cnt[c] + 2 * it.quad);
    it.nB = (int)__ldg(P.quad_cnt[c] + 2 * it.quad + 1);
  }
  return it;
}

// ---------------------------------------------------------------------------------------
template <int BK>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    attn2_kernel(const __grid_constant__ AttnParams P) {
  using C = Cfg<BK>;
  constexpr int NS = C::kStages;
  constexpr int D = C::D;
  using K = Ctl<NS>;
  static_assert(K::kBytes <= 1024, "control block");
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = raw + ((1024u - (raw & 1023u)) & 1023u);  // same offset in both CTAs
  const uint32_t sQ = sbase, sRing = sbase + C::kQBytes;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  K c;
  c.base = sbase + C::kDataBytes;
  c.lead = mapa_shared(c.base, 0);
  c.peer = mapa_shared(c.base, rank ^ 1u);
  uint8_t* ctl_gen = smem_raw + (c.base - raw);
  ItemInfo* items = reinterpret_cast<ItemInfo*>(ctl_gen + K::kItemsOff);
  Abort ab;
  ab.local = c.base + K::kAbortOff;
  ab.remote = c.peer + K::kAbortOff;
  ab.status = P.status;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    uint64_t* b = reinterpret_cast<uint64_t*>(ctl_gen);
    for (int st = 0; st < NS; ++st) {
      mbar_init(b + st, 1);       // kv_full: the even CTA's expect_tx arrival + both CTAs' bytes
      mbar_init(b + NS + st, 1);  // kv_empty: one commit
    }
    b += 2 * NS;
    mbar_init(b + 0, 1);  // q_full
    mbar_init(b + 1, 1);  // q_free
    for (int h = 0; h < 2; ++h) {
      mbar_init(b + 2 + h, 1);    // s_full
      mbar_init(b + 4 + h, 256);  // p_ready: 128 rows in each CTA
      mbar_init(b + 6 + h, 1);    // o_done
      mbar_init(b + 8 + h, 256);  // o_free
      mbar_init(b + 10 + h, 1);   // item_full
      mbar_init(b + 12 + h, 18);  // item_empty: MMA + 8 + 8 softmax warps + the odd CTA's producer
    }
    mbar_init(b + 14, 1);  // drain
    *reinterpret_cast<volatile int*>(ctl_gen + K::kAbortOff) = 0;
    int bad = 0;
    if (!P.dense) {
      for (int k = 0; k < 2; ++k) {
        if (!P.uses[k]) continue;
        const TmHeader* h = P.hdr[k];
        bad |= h->magic != kTmMagic || h->route != k || h->T != P.exp_T || h->H != P.exp_H ||
               h->W != P.exp_W || h->k != P.exp_k || h->b != P.exp_b || h->F0 != P.exp_F0 ||
               h->variant != P.exp_variant || h->layout != P.exp_layout || h->bq != P.exp_bq ||
               h->bk != P.exp_bk || h->nk != P.nk || h->nquads != P.nquads;
      }
    }
    *reinterpret_cast<int*>(ctl_gen + K::kBadWsOff) = bad;
    if (bad) atomicCAS(P.status, 0, SVG_ERR_WORKSPACE);
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {  // same warp in both CTAs
    tmem_alloc_pair(c.base + K::kTmemOff, 512);
    tmem_relinquish_pair();
  }
  if (warp == kProducerWarp && lane == 0) {
    prefetch_tmap(&P.tm_q);
    prefetch_tmap(&P.tm_k);
    prefetch_tmap(&P.tm_v);
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // both CTAs' barriers exist before any cross-CTA arrival
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(ctl_gen + K::kTmemOff);
  // both CTAs check the same parameters, so they agree on skipping
  const bool skip_all = *reinterpret_cast<volatile int*>(ctl_gen + K::kBadWsOff) != 0;

  if (!skip_all && warp == kProducerWarp) {
    // ------------------------------------------------------------------ producers (both CTAs)
    if (lane == 0) {
      uint32_t kv_pos = 0, q_iter = 0;
      for (uint32_t it = 0;; ++it) {
        const uint32_t slot = it & 1u, ph = (it >> 1) & 1u;
        ItemInfo inf;
        if (leader) {
          if (!wait_bar(c.item_empty(c.base, slot), ph ^ 1u, ab)) break;
          const uint32_t idx = atomicAdd(P.counter, 1u);
          inf = decode_item(P, idx);
          items[slot] = inf;
          const uint32_t* w = reinterpret_cast<const uint32_t*>(&inf);
          const uint32_t rslot = c.peer + K::kItemsOff + slot * (uint32_t)sizeof(ItemInfo);
#pragma unroll
          for (int x = 0; x < (int)(sizeof(ItemInfo) / 4); ++x) st_cluster_u32(rslot + 4 * x, w[x]);
          mbar_arrive_cluster(c.item_full(c.base, slot));
          mbar_arrive_cluster(c.item_full(c.peer, slot));  // release: orders the copy above
        } else {
          if (!wait_bar(c.item_full(c.base, slot), ph, ab)) break;
          inf = items[slot];
          mbar_arrive_cluster(c.item_empty(c.lead, slot));
        }
        if (!inf.valid) break;
        if (inf.nA + inf.nB > 0) {
          if (!wait_bar(c.q_free(c.base), (q_iter & 1u) ^ 1u, ab)) break;
          ++q_iter;
          if (leader)
            mbar_expect_tx(c.q_full(c.base), 2u * (uint32_t)C::kQHalfBytes * ((inf.nA > 0) + (inf.nB > 0)));
          for (int h = 0; h < 2; ++h) {
            if ((h == 0 ? inf.nA : inf.nB) == 0) continue;
            for (int ch = 0; ch < 2; ++ch)
              tma_load_3d_pair(sQ + h * C::kQHalfBytes + ch * (128 * 128), &P.tm_q, c.q_full(c.lead), ch * 64,
                               inf.quad * kQuadRows + (int)rank * kPairRows + h * kHalfRows, inf.head);
          }
        }
        bool ok = true;
        for (int e = 0; e < inf.count && ok; ++e) {
          const uint32_t ent = get_entry<BK>(P, inf, e);
          const int key0 = (int)qent_kt(ent) * BK;
          for (int w = 0; w < 2; ++w) {  // K half, then V half
            const uint32_t st = kv_pos % NS, phs = (kv_pos / NS) & 1u;
            if (!wait_bar(c.kv_empty(c.base, st), phs ^ 1u, ab)) {
              ok = false;
              break;
            }
            if (leader) mbar_expect_tx(c.kv_full(c.base, st), 2u * (uint32_t)C::kSlotBytes);
            const uint32_t dst = sRing + st * C::kSlotBytes;
            const uint32_t bar = c.kv_full(c.lead, st);
            if (w == 0) {
              for (int ch = 0; ch < 2; ++ch)
                tma_load_3d_pair(dst + ch * (C::kKRows * 128), &P.tm_k, bar, ch * 64, key0 + (int)rank * C::kKRows,
                                 inf.head);
            } else {
              tma_load_3d_pair(dst, &P.tm_v, bar, (int)rank * 64, key0, inf.head);
            }
            ++kv_pos;
          }
        }
        if (!ok) break;
      }
      if (ld_volatile_shared(ab.local)) {  // let issued copies land before the pair may exit
        const uint64_t t0 = globaltimer_ns();
        while (globaltimer_ns() - t0 < 2000000ull) {
        }
      }
    }
    __syncwarp();
  } else if (!skip_all && warp == kMmaWarp) {
    // ------------------------------------------------------------------ MMA issuer (even CTA)
    if (leader && lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(BK, false, 256);
      constexpr uint32_t idesc_o = idesc_bf16_f32(D, true, 256);
      const uint64_t qdesc = smem_desc_sw128(sQ, 16, 1024);
      const uint64_t kdesc = smem_desc_sw128(sRing, 16, 1024);
      const uint64_t vdesc = smem_desc_sw128(sRing, BK * 128, 1024);
      uint32_t kv_pos = 0, q_iter = 0, p_cnt0 = 0, p_cnt1 = 0, of_cnt0 = 0, of_cnt1 = 0;
      bool ok = true;
      for (uint32_t it = 0; ok; ++it) {
        const uint32_t slot = it & 1u, ph = (it >> 1) & 1u;
        if (!wait_bar(c.item_full(c.base, slot), ph, ab)) break;
        const ItemInfo inf = items[slot];
        mbar_arrive_cluster(c.item_empty(c.base, slot));
        if (!inf.valid) break;
        if (inf.nA + inf.nB > 0) {
          if (!wait_bar(c.q_full(c.base), q_iter & 1u, ab)) break;
          ++q_iter;
          tc_fence_after();
        }
        int rem0 = inf.nA, rem1 = inf.nB;
        uint32_t prev_act = 0, has_o = 0, prev_v = 0;
        for (int e = 0; e <= inf.count && ok; ++e) {
          const bool last = e == inf.count;
          const uint32_t ent = last ? 0u : get_entry<BK>(P, inf, e);
          const uint32_t kpos = kv_pos, vpos = kv_pos + 1;
          bool k_ready = false;
          const uint64_t kd = kdesc + (((kpos % NS) * C::kSlotBytes) >> 4);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            if (!ok) break;
            if ((prev_act >> h) & 1u) {  // O_h += P_h V(e-1) on both SMs
              uint32_t& pc = h == 0 ? p_cnt0 : p_cnt1;
              uint32_t& oc = h == 0 ? of_cnt0 : of_cnt1;
              ok = wait_bar(c.p_ready(c.base, h), pc & 1u, ab);
              ++pc;
              if (ok && !((has_o >> h) & 1u)) {
                ok = wait_bar(c.o_free(c.base, h), (oc & 1u) ^ 1u, ab);
                ++oc;
              }
              if (ok) ok = wait_bar(c.kv_full(c.base, prev_v % NS), (prev_v / NS) & 1u, ab);
              if (!ok) break;
              tc_fence_after();
              const uint64_t vd = vdesc + (((prev_v % NS) * C::kSlotBytes) >> 4);
              const uint32_t acc0 = (has_o >> h) & 1u;
#pragma unroll
              for (int kk = 0; kk < BK / 16; ++kk)
                umma_ts_pair(tmem + C::o_col(h), tmem + C::s_col(h) + C::kPCol + kk * 8, vd + ((kk * 2048) >> 4),
                             idesc_o, (acc0 || kk > 0) ? 1u : 0u);
              has_o |= 1u << h;
              int& rem = h == 0 ? rem0 : rem1;
              if (--rem == 0) {
                umma_commit_pair(c.o_done(c.base, h));
                umma_commit_pair(c.o_done(c.peer, h));
              }
            }
            const bool act = !last && phase_active(ent, h);
            if (act) {
              if (!k_ready) {
                ok = wait_bar(c.kv_full(c.base, kpos % NS), (kpos / NS) & 1u, ab);
                if (!ok) break;
                tc_fence_after();
                k_ready = true;
              }
              const uint64_t qd = qdesc + ((h * C::kQHalfBytes) >> 4);
#pragma unroll
              for (int kk = 0; kk < D / 16; ++kk) {
                const uint32_t qoff = ((kk >> 2) * (128 * 128) + (kk & 3) * 32) >> 4;
                const uint32_t koff = ((kk >> 2) * (C::kKRows * 128) + (kk & 3) * 32) >> 4;
                umma_ss_pair(tmem + C::s_col(h), qd + qoff, kd + koff, idesc_s, kk > 0 ? 1u : 0u);
              }
              umma_commit_pair(c.s_full(c.base, h));
              umma_commit_pair(c.s_full(c.peer, h));
            }
            prev_act = (prev_act & ~(1u << h)) | ((act ? 1u : 0u) << h);
          }
          if (!ok) break;
          if (e > 0) {  // V(e-1) read by the P V MMAs
            umma_commit_pair(c.kv_empty(c.base, prev_v % NS));
            umma_commit_pair(c.kv_empty(c.peer, prev_v % NS));
          }
          if (last) break;
          if (!k_ready) {
            ok = wait_bar(c.kv_full(c.base, kpos % NS), (kpos / NS) & 1u, ab);
            if (!ok) break;
          }
          umma_commit_pair(c.kv_empty(c.base, kpos % NS));  // K(e) read by the S MMAs
          umma_commit_pair(c.kv_empty(c.peer, kpos % NS));
          if (e == inf.count - 1) {
            umma_commit_pair(c.q_free(c.base));
            umma_commit_pair(c.q_free(c.peer));
          }
          prev_v = vpos;
          kv_pos += 2;
        }
      }
      umma_commit_pair(c.drain(c.base));
      drain_bar(c.drain(c.base), 0);
    }
    __syncwarp();
  } else if (!skip_all && warp < 8) {
    // ------------------------------------------------------------------ softmax groups (both CTAs)
    const int h = warp >> 2;
    const int lr = threadIdx.x & 127;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_off + C::s_col(h);
    const uint32_t tP = tS + C::kPCol;
    const uint32_t tO = tmem + lane_off + C::o_col(h);
    const float sl2 = P.sl2;
    uint32_t s_cnt = 0, od_cnt = 0;
    for (uint32_t it = 0;; ++it) {
      const uint32_t slot = it & 1u, ph = (it >> 1) & 1u;
      if (!__all_sync(0xffffffffu, wait_bar(c.item_full(c.base, slot), ph, ab))) break;
      const ItemInfo inf = items[slot];
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(c.item_empty(c.lead, slot));
      if (!inf.valid) break;
      const int row = inf.quad * kQuadRows + (int)rank * kPairRows + h * kHalfRows + lr;
      const bool in_range = row < P.N;
      const int nphase = h == 0 ? inf.nA : inf.nB;
      if (nphase == 0) {  // no tile at all for this half (rounded masks only)
        if (in_range) {
          __nv_bfloat16* orow = P.o + ((size_t)inf.head * P.N + row) * D;
          const uint4 z = make_uint4(0, 0, 0, 0);
          for (int x = 0; x < D / 8; ++x) reinterpret_cast<uint4*>(orow)[x] = z;
          if (P.lse) P.lse[(size_t)inf.head * P.N + row] = -INFINITY;
        }
        continue;
      }
      const int prow = in_range ? row : P.N - 1;
      int lo = 0, hi = 0, se = 0;
      bool per = false;
      if (!P.dense) {
        const MaskGeom& g = P.g[inf.cls];
        row_interval(g, prow, lo, hi);
        se = sink_end(g);
        per = periodic_sink(g);
      }
      float m = -INFINITY, l = 0.f;
      bool first = true, ok = true;
      uint32_t ent_next = inf.count > 0 ? get_entry<BK>(P, inf, 0) : 0u;
      for (int e = 0; e < inf.count; ++e) {
        const uint32_t ent = ent_next;
        if (e + 1 < inf.count) ent_next = get_entry<BK>(P, inf, e + 1);
        if (!phase_active(ent, h)) continue;
        const uint32_t f = qent_flag(ent, (int)rank, h);
        const int c0 = (int)qent_kt(ent) * BK;
        if (!__all_sync(0xffffffffu, wait_bar(c.s_full(c.base, h), s_cnt & 1u, ab))) {
          ok = false;
          break;
        }
        ++s_cnt;
        tc_fence_after();
        uint32_t r[BK];
        if (f == kFlagSkip) {
          // the other SM's rows need this tile, ours keep nothing in it: P = 0
#pragma unroll
          for (int j = 0; j < BK / 2; ++j) r[j] = 0u;
#pragma unroll
          for (int q = 0; q < BK / 64; ++q) tmem_st32(tP + q * 32, r + q * 32);
          tmem_st_wait();
          tc_fence_before();
          mbar_arrive_cluster(c.p_ready(c.lead, h));
          first = false;
          continue;
        }
#pragma unroll
        for (int q = 0; q < BK / 32; ++q) tmem_ld32(tS + q * 32, r + q * 32);
        tmem_ld_wait();
#pragma unroll
        for (int q = 0; q < BK / 32; ++q) tmem_ld_fence32(r + q * 32);
        float* s = reinterpret_cast<float*>(r);
        const bool elem = (f == kFlagMasked) || (P.naive && !P.dense);
        if (elem || f == kFlagBounds) {
          const int nn = P.N - c0;
          if (!elem) {
#pragma unroll
            for (int j = 0; j < BK; ++j)
              if (j >= nn) s[j] = -INFINITY;
          } else if (P.variant == SVG_MASK_ROUNDED) {
            const uint8_t* rcls = P.cls[inf.cls] + (size_t)(prow / P.bq) * P.nk;
            const bool rowkept = __ldg(rcls + qent_kt(ent)) == 1;
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
              const MaskGeom& g = P.g[inf.cls];
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
        float mx4[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) mx4[i] = s[i];
#pragma unroll
        for (int j = 4; j < BK; j += 4)
#pragma unroll
          for (int i = 0; i < 4; ++i) mx4[i] = fmaxf(mx4[i], s[j + i]);
        const float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
        const float m_new = fmaxf(m, mx);
        const bool need = (m_new > m) && (m == -INFINITY || (m_new - m) * sl2 > kRescaleThreshold);
        const bool rescale = __any_sync(0xffffffffu, need);
        float alpha = 1.f;
        if (rescale) {
          alpha = (m_new == -INFINITY) ? 1.f : ex2f((m - m_new) * sl2);
          l *= alpha;
          m = m_new;
        }
        const float base = (m == -INFINITY) ? 0.f : m * sl2;
        {
          const float2 sc = make_float2(sl2, sl2), nb = make_float2(-base, -base);
          float2 acc[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
          exp_pack_64<0>(r, sc, nb, acc);
          if (BK == 128) exp_pack_64<64 % BK>(r, sc, nb, acc);
#pragma unroll
          for (int q = 0; q < BK / 64; ++q) tmem_st32(tP + q * 32, r + q * 32);
          l += (acc[0].x + acc[1].x) + (acc[0].y + acc[1].y);
        }
        if (rescale && !first) {
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
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive_cluster(c.p_ready(c.lead, h));
        first = false;
      }
      if (!ok) break;
      if (!__all_sync(0xffffffffu, wait_bar(c.o_done(c.base, h), od_cnt & 1u, ab))) break;
      ++od_cnt;
      tc_fence_after();
      const float inv_l = (l > 0.f && m != -INFINITY) ? 1.f / l : 0.f;  // a row with no kept key gives 0
      __nv_bfloat16* orow = P.o + ((size_t)inf.head * P.N + prow) * D;
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
      mbar_arrive_cluster(c.o_free(c.lead, h));
      if (in_range && P.lse)
        P.lse[(size_t)inf.head * P.N + row] =
            (l > 0.f && m != -INFINITY) ? (m * sl2 + log2f(l)) * 0.69314718055994531f : -INFINITY;
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // no CTA leaves while the pair's MMAs or arrivals may still touch it
  tc_fence_after();
  if (warp == kMmaWarp) tmem_dealloc_pair(tmem, 512);
}

template <int BK>
static int launch_t(const AttnParams& P, int grid, cudaStream_t st) {
  using C = Cfg<BK>;
  auto kern = attn2_kernel<BK>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
  if (e != cudaSuccess) return record_cuda_error("cudaFuncSetAttribute(attn2_kernel)", e);
  kern<<<grid, kThreads, C::kSmemBytes, st>>>(P);
  e = cudaGetLastError();
  return e == cudaSuccess ? SVG_OK : record_cuda_error("launch attn2_kernel", e);
}

}  // namespace pair2

namespace pair2 {
// Clusters of this kernel that fit on the device at once (GPC boundaries can leave an SM
// without a partner), cached per device and tile width.
template <int BK>
static int max_clusters() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  if (cached[dev] > 0) return cached[dev];
  using C = Cfg<BK>;
  cudaFuncSetAttribute(attn2_kernel<BK>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = C::kSmemBytes;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, attn2_kernel<BK>, &cfg) != cudaSuccess || n <= 0) return 0;
  cached[dev] = n;
  return n;
}
}  // namespace pair2

// Launches the SM-pair kernel with one resident cluster per work item in flight, at most
// `max_clusters` and at most as many as fit on the device at once.
int launch_attention_pair(const AttnParams& P, int bk, int max_clusters, cudaStream_t st) {
  int fit = bk == 128 ? pair2::max_clusters<128>() : bk == 64 ? pair2::max_clusters<64>() : 0;
  if (fit <= 0) return record_cuda_error("cudaOccupancyMaxActiveClusters(attn2_kernel)", (int)cudaErrorInvalidConfiguration);
  const int clusters = max_clusters < fit ? max_clusters : fit;
  if (bk == 128) return pair2::launch_t<128>(P, 2 * clusters, st);
  if (bk == 64) return pair2::launch_t<64>(P, 2 * clusters, st);
  return SVG_ERR_UNSUPPORTED;
}

}  // namespace svg
