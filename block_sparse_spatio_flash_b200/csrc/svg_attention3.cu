// svg_attention3.cu -- block-sparse flash-attention forward on SM pairs, one 128-row half per SM,
// scores double-buffered (d = 128).
//
// Same computation as svg_attention.cu (softmax attention restricted to the kept pairs of each
// head's spatial or temporal mask, visiting only non-empty key tiles, full tiles unmasked and
// boundary tiles element-masked: "Efficient Kernel Implementation", tile-aware masking, of
// "Accelerating Spatio-Temporal Attention for Video Diffusion on TPUs"), arranged so that the
// scores of the next key tile are computed while the softmax works on the current one:
//  * a cluster of two CTAs on two SMs takes one item = 256 query rows of one head; CTA r owns
//    rows [256 i + 128 r, +128) (its TMEM lanes). The even CTA issues tcgen05.mma.cta_group::2
//    (M = 256): each SM supplies its 128 Q rows, half of every K tile (BK/2 keys) and half of
//    every V tile (64 of the 128 head dimensions), so each SM moves half the K/V bytes of the
//    one-SM kernel from L2 into shared memory;
//  * the item's key tiles alternate between two softmax groups per SM (warps 0-3: tiles 0, 2, 4
//    ..., warps 4-7: tiles 1, 3, 5 ...). Group g owns TMEM columns S_g = [128 g, +128) (P_g in
//    its upper half) and an output accumulator O_g = [256 + 128 g, +128), and keeps its own
//    running maximum and sum; the epilogue merges the two partial outputs;
//  * the MMA order per item is S(0), S(1), PV(0), S(2), PV(1), S(3), ... : S(e + 2) reuses S_g
//    only after PV(e) has read P(e) from it (the tensor core runs MMAs in issue order), and while
//    group g turns S(e) into P(e) the tensor core is already computing S(e + 1) for the other
//    group. The commit that announces S(e) also covers PV(e - 2), the last update of O_g, so a
//    group may rescale O_g as soon as it sees its scores;
//  * per CTA: warp 8 loads (TMA, no cluster copies) its Q half and its K / V halves; warp 9 of
//    the even CTA issues the MMAs; completion of every TMA copy of both CTAs is counted on the even
//    CTA's barriers, MMA completion is signalled to the barriers of both CTAs;
//  * every wait is bounded; a timeout aborts both CTAs of the pair.
#include <cuda_bf16.h>
#include <string.h>

#include "svg_common.cuh"

namespace svg {
namespace pair1 {

constexpr int kThreads = 320;
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s per wait

template <int BK>
struct Cfg {
  static constexpr int D = 128;
  static constexpr int kQBytes = 128 * D * 2;            // this SM's 128 rows x 128 dims
  static constexpr int kKRows = BK / 2;                  // keys of a K tile held by one SM
  static constexpr int kKBytes = kKRows * D * 2;         // two 64-dim swizzle chunks
  static constexpr int kVBytes = BK * 64 * 2;            // BK keys x 64 dims (one chunk)
  static constexpr int kSlotBytes = kKBytes;
  static_assert(kKBytes == kVBytes, "ring slots hold either half tile");
  static constexpr int kStages = (176 * 1024) / kSlotBytes;
  static constexpr int kDataBytes = kQBytes + kStages * kSlotBytes + 2 * 2 * 2 * 128 * 4;  // + exchange
  static constexpr int kSmemBytes = kDataBytes + 1024 /*control*/ + 1024 /*alignment slack*/;
  __host__ __device__ static constexpr uint32_t s_col(int g) { return 128u * g; }
  static constexpr uint32_t kPCol = BK / 2;
  __host__ __device__ static constexpr uint32_t o_col(int g) { return 256u + 128u * g; }
  static_assert(kSmemBytes <= 232448, "shared memory budget");
};

struct ItemInfo {
  int valid, head, pair, cls, count, in0, in1, pad;  // in0 / in1: half 0 / 1 has rows < N
  const uint32_t* ents;
};
static_assert(sizeof(ItemInfo) == 40, "item slot size");

// Control block (same shared offsets in both CTAs), 8-byte slots:
//   [0, NS) kv_full   [NS, 2NS) kv_empty   2NS+0 q_full   2NS+1 q_free
//   2NS+2+g s_full[g]   2NS+4+g p_ready[g] (256)   2NS+6+g o_done[g]   2NS+8+g o_free[g] (512)
//   2NS+10+i item_full   2NS+12+i item_empty (18)   2NS+14 drain   2NS+15 xch (256, per CTA)
//   then 2 items, TMEM base, abort, check.
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
  __device__ __forceinline__ uint32_t s_full(uint32_t b, int g) const { return b + 8u * (2 * NS + 2 + g); }
  __device__ __forceinline__ uint32_t p_ready(uint32_t b, int g) const { return b + 8u * (2 * NS + 4 + g); }
  __device__ __forceinline__ uint32_t o_done(uint32_t b, int g) const { return b + 8u * (2 * NS + 6 + g); }
  __device__ __forceinline__ uint32_t o_free(uint32_t b, int g) const { return b + 8u * (2 * NS + 8 + g); }
  __device__ __forceinline__ uint32_t item_full(uint32_t b, uint32_t i) const { return b + 8u * (2 * NS + 10 + i); }
  __device__ __forceinline__ uint32_t item_empty(uint32_t b, uint32_t i) const { return b + 8u * (2 * NS + 12 + i); }
  __device__ __forceinline__ uint32_t drain(uint32_t b) const { return b + 8u * (2 * NS + 14); }
  __device__ __forceinline__ uint32_t xch(uint32_t b) const { return b + 8u * (2 * NS + 15); }
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
__device__ __noinline__ bool wait_slow(uint32_t bar, uint32_t parity, const Abort& ab) {
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
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, const Abort& ab) {
  return mbar_try_wait_cluster(bar, parity) || wait_slow(bar, parity, ab);
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
  return (uint32_t)e | ((it.in0 ? f : 0u) << 28) | ((it.in1 ? f : 0u) << 30);
}

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
    it.ents = nullptr;
  } else {
    const int c = it.cls;
    it.pair = (int)__ldg(P.pair_order[c] + j);
    const uint32_t b0 = __ldg(P.pair_ptr[c] + it.pair), b1 = __ldg(P.pair_ptr[c] + it.pair + 1);
    it.count = (int)(b1 - b0);
    it.ents = P.pair_ent[c] + b0;
  }
  it.in0 = it.pair * kPairRows < P.N;
  it.in1 = it.pair * kPairRows + kHalfRows < P.N;
  return it;
}

// ---------------------------------------------------------------------------------------
template <int BK>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    attn3_kernel(const __grid_constant__ AttnParams P) {
  using C = Cfg<BK>;
  constexpr int NS = C::kStages;
  constexpr int D = C::D;
  using K = Ctl<NS>;
  static_assert(K::kBytes <= 1024, "control block");
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = raw + ((1024u - (raw & 1023u)) & 1023u);  // same offset in both CTAs
  const uint32_t sQ = sbase, sRing = sbase + C::kQBytes;
  const uint32_t sX = sRing + NS * C::kSlotBytes;  // [parity][m | l][group][row] fp32
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
    for (int g = 0; g < 2; ++g) {
      mbar_init(b + 2 + g, 1);    // s_full
      mbar_init(b + 4 + g, 256);  // p_ready: 128 rows of group g in each CTA
      mbar_init(b + 6 + g, 1);    // o_done
      mbar_init(b + 8 + g, 512);  // o_free: every softmax thread of both CTAs (each reads both O's)
      mbar_init(b + 10 + g, 1);   // item_full
      mbar_init(b + 12 + g, 18);  // item_empty: MMA + 8 + 8 softmax warps + the odd CTA's producer
    }
    mbar_init(b + 14, 1);    // drain
    mbar_init(b + 15, 256);  // xch: both groups of this CTA
    *reinterpret_cast<volatile int*>(ctl_gen + K::kAbortOff) = 0;
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
        if (inf.count == 0) continue;
        if (!wait_bar(c.q_free(c.base), (q_iter & 1u) ^ 1u, ab)) break;
        ++q_iter;
        if (leader) mbar_expect_tx(c.q_full(c.base), 2u * (uint32_t)C::kQBytes);
        for (int ch = 0; ch < 2; ++ch)
          tma_load_3d_pair(sQ + ch * (128 * 128), &P.tm_q, c.q_full(c.lead), ch * 64,
                           inf.pair * kPairRows + (int)rank * kHalfRows, inf.head);
        bool ok = true;
        for (int e = 0; e < inf.count && ok; ++e) {
          const uint32_t ent = get_entry<BK>(P, inf, e);
          const int key0 = (int)ent_kt(ent) * BK;
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
      uint32_t kv_base = 0, q_iter = 0;
      uint32_t pc[2] = {0, 0}, of[2] = {0, 0};
      bool ok = true;
      for (uint32_t it = 0; ok; ++it) {
        const uint32_t slot = it & 1u, ph = (it >> 1) & 1u;
        if (!wait_bar(c.item_full(c.base, slot), ph, ab)) break;
        const ItemInfo inf = items[slot];
        mbar_arrive_cluster(c.item_empty(c.base, slot));
        if (!inf.valid) break;
        const int n = inf.count;
        if (n == 0) continue;
        if (!wait_bar(c.q_full(c.base), q_iter & 1u, ab)) break;  // (TMA data: no tcgen05 fence needed)
        ++q_iter;
        // S(e) = Q K(e)^T into S_{e % 2}; announces S to both CTAs, releases K(e)'s slot and, after
        // the item's last S, Q
        auto issue_s = [&](int e) -> bool {
          const uint32_t kpos = kv_base + 2u * (uint32_t)e;
          if (!wait_bar(c.kv_full(c.base, kpos % NS), (kpos / NS) & 1u, ab)) return false;
          const int g = e & 1;
          const uint64_t kd = kdesc + (((kpos % NS) * C::kSlotBytes) >> 4);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t qoff = ((kk >> 2) * (128 * 128) + (kk & 3) * 32) >> 4;
            const uint32_t koff = ((kk >> 2) * (C::kKRows * 128) + (kk & 3) * 32) >> 4;
            umma_ss_pair(tmem + C::s_col(g), qdesc + qoff, kd + koff, idesc_s, kk > 0 ? 1u : 0u);
          }
          umma_commit_pair(c.s_full(c.base, g));
          umma_commit_pair(c.s_full(c.peer, g));
          umma_commit_pair(c.kv_empty(c.base, kpos % NS));
          umma_commit_pair(c.kv_empty(c.peer, kpos % NS));
          if (e == n - 1) {
            umma_commit_pair(c.q_free(c.base));
            umma_commit_pair(c.q_free(c.peer));
          }
          return true;
        };
        ok = issue_s(0) && (n < 2 || issue_s(1));
        for (int e = 0; e < n && ok; ++e) {
          const int g = e & 1;
          // O_g (+)= P_g V(e): needs P(e) from both CTAs and, for the item's first, a free O_g
          ok = wait_bar(c.p_ready(c.base, g), pc[g] & 1u, ab);
          ++pc[g];
          if (ok && e < 2) {
            ok = wait_bar(c.o_free(c.base, g), (of[g] & 1u) ^ 1u, ab);
            ++of[g];
          }
          const uint32_t vpos = kv_base + 2u * (uint32_t)e + 1u;
          if (ok) ok = wait_bar(c.kv_full(c.base, vpos % NS), (vpos / NS) & 1u, ab);
          if (!ok) break;
          tc_fence_after();
          const uint64_t vd = vdesc + (((vpos % NS) * C::kSlotBytes) >> 4);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            umma_ts_pair(tmem + C::o_col(g), tmem + C::s_col(g) + C::kPCol + kk * 8, vd + ((kk * 2048) >> 4), idesc_o,
                         (e >= 2 || kk > 0) ? 1u : 0u);
          umma_commit_pair(c.kv_empty(c.base, vpos % NS));
          umma_commit_pair(c.kv_empty(c.peer, vpos % NS));
          if (e + 2 >= n) {  // the last P V into O_g
            umma_commit_pair(c.o_done(c.base, g));
            umma_commit_pair(c.o_done(c.peer, g));
          }
          if (e + 2 < n) ok = issue_s(e + 2);
        }
        kv_base += 2u * (uint32_t)n;
      }
      umma_commit_pair(c.drain(c.base));
      drain_bar(c.drain(c.base), 0);
    }
    __syncwarp();
  } else if (!skip_all && warp < 8) {
    // ------------------------------------------------------------------ softmax groups (both CTAs)
    const int g = warp >> 2;                   // group: even (0) or odd (1) key tiles of an item
    const int lr = threadIdx.x & 127;          // row within this SM's half = TMEM lane
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_off + C::s_col(g);
    const uint32_t tP = tS + C::kPCol;
    float* xb = reinterpret_cast<float*>(smem_raw + (sX - raw));
    const float sl2 = P.sl2;
    uint32_t s_cnt = 0, od_cnt[2] = {0, 0}, x_cnt = 0;
    for (uint32_t it = 0;; ++it) {
      const uint32_t slot = it & 1u, ph = (it >> 1) & 1u;
      if (!__all_sync(0xffffffffu, wait_bar(c.item_full(c.base, slot), ph, ab))) break;
      const ItemInfo inf = items[slot];
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(c.item_empty(c.lead, slot));
      if (!inf.valid) break;
      const int row = inf.pair * kPairRows + (int)rank * kHalfRows + lr;
      const bool in_range = row < P.N;
      const int prow = in_range ? row : P.N - 1;
      const int n = inf.count;
      if (n == 0) {  // no tile at all for this item (rounded masks only): O = 0
        if (in_range) {
          __nv_bfloat16* orow = P.o + ((size_t)inf.head * P.N + row) * D + g * 64;
          const uint4 z = make_uint4(0, 0, 0, 0);
          for (int x = 0; x < 8; ++x) reinterpret_cast<uint4*>(orow)[x] = z;
          if (P.lse && g == 0) P.lse[(size_t)inf.head * P.N + row] = -INFINITY;
        }
        continue;
      }
      int lo = 0, hi = 0, se = 0;
      bool per = false;
      if (!P.dense) {
        const MaskGeom& mg = P.g[inf.cls];
        row_interval(mg, prow, lo, hi);
        se = sink_end(mg);
        per = periodic_sink(mg);
      }
      float m = -INFINITY, l = 0.f;
      bool first = true, ok = true;
      for (int e = g; e < n; e += 2) {
        const uint32_t ent = get_entry<BK>(P, inf, e);
        const uint32_t f = ent_flag(ent, (int)rank);
        const int c0 = (int)ent_kt(ent) * BK;
        if (!__all_sync(0xffffffffu, wait_bar(c.s_full(c.base, g), s_cnt & 1u, ab))) {
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
        } else {
          float alpha = 1.f;
          float2 acc[2];
          load_scores<BK>(tS, r);
          mask_scores<BK>(P, inf.cls, f, c0, prow, ent, lo, hi, se, per, r);
          const bool rescale = max_first<BK>(r, sl2, m, l, alpha);
          exp_tile<BK>(r, sl2, m, acc);
          l += (acc[0].x + acc[1].x) + (acc[0].y + acc[1].y);
          if (rescale && !first) {  // O_g holds every earlier P V of this group (S(e)'s commit covers them)
            const uint32_t tO = tmem + lane_off + C::o_col(g);
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
        }
#pragma unroll
        for (int q = 0; q < BK / 64; ++q) tmem_st32(tP + q * 32, r + q * 32);
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive_cluster(c.p_ready(c.lead, g));
        first = false;
      }
      if (!ok) break;
      // ---- epilogue: merge the two groups' partial outputs; group g writes columns [64 g, +64)
      const int n0 = (n + 1) / 2, n1 = n / 2;  // tiles of group 0 / 1
      bool eok = true;
      if (n0 > 0) {
        eok = __all_sync(0xffffffffu, wait_bar(c.o_done(c.base, 0), od_cnt[0] & 1u, ab));
        ++od_cnt[0];
      }
      if (eok && n1 > 0) {
        eok = __all_sync(0xffffffffu, wait_bar(c.o_done(c.base, 1), od_cnt[1] & 1u, ab));
        ++od_cnt[1];
      }
      if (!eok) break;
      tc_fence_after();
      // trade (m, l) with the other group's thread of the same row
      const uint32_t par = x_cnt & 1u;
      xb[((par * 2 + 0) * 2 + g) * 128 + lr] = m;
      xb[((par * 2 + 1) * 2 + g) * 128 + lr] = l;
      mbar_arrive(c.xch(c.base));
      if (!__all_sync(0xffffffffu, wait_bar(c.xch(c.base), par, ab))) break;
      ++x_cnt;
      const float mo = xb[((par * 2 + 0) * 2 + (g ^ 1)) * 128 + lr];
      const float lo_ = xb[((par * 2 + 1) * 2 + (g ^ 1)) * 128 + lr];
      const float m0 = g == 0 ? m : mo, m1 = g == 0 ? mo : m;
      const float l0 = g == 0 ? l : lo_, l1 = g == 0 ? lo_ : l;
      const float M = fmaxf(m0, m1);
      const float a0 = (m0 == -INFINITY) ? 0.f : ex2f((m0 - M) * sl2);
      const float a1 = (m1 == -INFINITY) ? 0.f : ex2f((m1 - M) * sl2);
      const float L = a0 * l0 + a1 * l1;
      const float inv = (L > 0.f && M != -INFINITY) ? 1.f / L : 0.f;  // a row with no kept key gives 0
      const float w0 = a0 * inv, w1 = a1 * inv;
      __nv_bfloat16* orow = P.o + ((size_t)inf.head * P.N + prow) * D + g * 64;
      const bool has1 = n1 > 0;  // (n0 > 0 always here) O_1 of a one-tile item is stale: selected away
#pragma unroll 1
      for (int q = 0; q < 2; ++q) {
        uint32_t o0[32], o1[32];
        const uint32_t col = (uint32_t)(g * 64 + q * 32);
        tmem_ld32(tmem + lane_off + C::o_col(0) + col, o0);
        tmem_ld32(tmem + lane_off + C::o_col(1) + col, o1);
        tmem_ld_wait();
        tmem_ld_fence32(o0);
        tmem_ld_fence32(o1);
        if (in_range) {
          uint4* dst = reinterpret_cast<uint4*>(orow + q * 32);
#pragma unroll
          for (int x = 0; x < 4; ++x) {
            uint32_t pk[4];
#pragma unroll
            for (int y = 0; y < 4; ++y) {
              const int j = 8 * x + 2 * y;
              const float u0 = __uint_as_float(o0[j]) * w0, v0 = __uint_as_float(o0[j + 1]) * w0;
              const float u1 = has1 ? __uint_as_float(o1[j]) * w1 : 0.f;
              const float v1 = has1 ? __uint_as_float(o1[j + 1]) * w1 : 0.f;
              pk[y] = pack_bf16(u0 + u1, v0 + v1);
            }
            dst[x] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          }
        }
      }
      tc_fence_before();
      if (n0 > 0) mbar_arrive_cluster(c.o_free(c.lead, 0));
      if (n1 > 0) mbar_arrive_cluster(c.o_free(c.lead, 1));
      if (in_range && P.lse && g == 0)
        P.lse[(size_t)inf.head * P.N + row] =
            (L > 0.f && M != -INFINITY) ? (M * sl2 + log2f(L)) * 0.69314718055994531f : -INFINITY;
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // no CTA leaves while the pair's MMAs or arrivals may still touch it
  tc_fence_after();
  if (warp == kMmaWarp) tmem_dealloc_pair(tmem, 512);
}

template <int BK>
static int max_clusters() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  if (cached[dev] > 0) return cached[dev];
  using C = Cfg<BK>;
  cudaFuncSetAttribute(attn3_kernel<BK>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = C::kSmemBytes;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, attn3_kernel<BK>, &cfg) != cudaSuccess || n <= 0) return 0;
  cached[dev] = n;
  return n;
}

template <int BK>
static int launch_t(const AttnParams& P, cudaStream_t st) {
  using C = Cfg<BK>;
  auto kern = attn3_kernel<BK>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
  if (e != cudaSuccess) return record_cuda_error("cudaFuncSetAttribute(attn3_kernel)", e);
  const int mc = max_clusters<BK>();
  if (mc <= 0) return record_cuda_error("cudaOccupancyMaxActiveClusters(attn3_kernel)", (int)cudaErrorInvalidConfiguration);
  const int clusters = P.n_items < mc ? P.n_items : mc;
  kern<<<2 * clusters, kThreads, C::kSmemBytes, st>>>(P);
  e = cudaGetLastError();
  return e == cudaSuccess ? SVG_OK : record_cuda_error("launch attn3_kernel", e);
}

}  // namespace pair1

// Items are 256-row pairs (P.npairs per head); d must be 128.
int launch_attention_pair1(const AttnParams& P, int bk, cudaStream_t st) {
  if (bk == 128) return pair1::launch_t<128>(P, st);
  if (bk == 64) return pair1::launch_t<64>(P, st);
  return SVG_ERR_UNSUPPORTED;
}

}  // namespace svg
