// svg_route.cu -- head routing by sampled rows.
//
// Sparse VideoGen profiles heads at inference time and routes each one to the spatial or the
// temporal mask by sampling ("Sparse Attention Patterns": heads are routed dynamically based on
// sampling; summary: SVG profiles heads at inference time). Read here as: attend a few sampled
// query rows of the head under the dense mask and under both sparse masks, and route the head to
// the sparse mask whose outputs are closer to the dense ones (relative squared error over the
// sampled rows; ties go to spatial).
//
// route_tc_kernel (tensor cores, below): one CTA = up to 128 sampled rows of one head x one chunk of
// the keys; per row and mask (dense / spatial / temporal) an online softmax, the scores and the three
// P V products on tcgen05. The unnormalised state (O, running max, running sum) of each chunk is
// written out; route_merge_kernel combines the chunks of a row and writes
// (|O_s - O_d|^2, |O_t - O_d|^2, |O_d|^2); route_reduce_kernel sums those per head in a fixed
// order (deterministic) and sets the route.
#include <cuda_bf16.h>
#include <string.h>

#include "svg_common.cuh"

namespace svg {

constexpr int kRouteKeys = 64;      // keys per tile
constexpr int kRouteMaxChunks = 32;  // at most one chunk per lane of the merge kernel's warp
static_assert(kRouteMaxChunks <= 32, "route_merge_kernel keeps one chunk per lane");
constexpr int kRouteChunkKeys = 2048;

// Key chunks per row block: enough blocks to fill the GPU at the pages' sizes, at most 32.
__host__ __device__ inline int route_chunks(int64_t N) {
  const int64_t c = (N + kRouteChunkKeys - 1) / kRouteChunkKeys;
  return (int)(c < 1 ? 1 : (c > kRouteMaxChunks ? kRouteMaxChunks : c));
}
// Keys per chunk (a multiple of the tile) when the keys are cut into G chunks.
inline int route_chunk_len(int64_t N, int G) {
  const int64_t per = (N + G - 1) / G;
  return (int)((per + kRouteKeys - 1) / kRouteKeys * kRouteKeys);
}
// Chunks for this launch: the count (at most route_chunks(N), the count the work buffer is sized
// for) whose blocks fill the GPU's block slots (blocks_per_sm x SMs) best over whole waves -- a
// last, mostly empty wave costs as much as a full one; among equals the larger count (shorter blocks).
inline int route_launch_chunks(int64_t N, int row_blocks, int heads, int num_sms, int blocks_per_sm) {
  const int64_t per_chunk = (int64_t)row_blocks * heads;
  const int64_t slots = (int64_t)blocks_per_sm * (num_sms > 0 ? num_sms : 1);
  int best = 1;
  double best_fill = -1.0;
  for (int g = 1; g <= route_chunks(N); ++g) {
    const int64_t blocks = per_chunk * g;
    const int64_t waves = (blocks + slots - 1) / slots;
    const double fill = (double)blocks / (double)(waves * slots);
    if (fill >= best_fill - 1e-9) {
      best_fill = fill;
      best = g;
    }
  }
  return best;
}

// Work buffer: a 256-byte status block (int32 status word first), the per-row errors, then the
// per-chunk states.
constexpr size_t kRouteStatusBytes = 256;
size_t route_rowerr_bytes(int heads, int n_rows) {
  return ((size_t)heads * n_rows * 3 * sizeof(float) + 255) / 256 * 256;
}
size_t route_work_bytes(int heads, int64_t N, int d, int n_rows) {
  return kRouteStatusBytes + route_rowerr_bytes(heads, n_rows) +
         (size_t)heads * n_rows * route_chunks(N) * 3 * (size_t)(d + 2) * sizeof(float);
}

struct RouteParams {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  int H, N, D;
  float sl2;             // scale * log2(e): scores are kept in log2 units
  MaskGeom gs, gt;       // spatial / temporal masks on original identities (layout unused)
  const int32_t* rows;   // sampled original query indices
  int n_rows;
  int G, chunk;          // key chunks (all non-empty) and keys per chunk
  float* part;           // [H][n_rows][G][3][D + 2]: O (unnormalised), running max, running sum
  float* rowerr;         // [H][n_rows][3]
  uint8_t* route;        // [H]
  float* err;            // [H][2] nullable: relative errors of spatial / temporal
};

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
  return x;
}
__device__ __forceinline__ double warp_sum(double x) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
  return x;
}
__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, off));
  return x;
}

// ---------------------------------------------------------------------------------------
// Tensor-core form. Sampled rows x keys is a contraction (S = Q_rows K^T, then three P V), so one
// CTA takes up to 128 sampled rows of one head (M = 128; rows past the list are padding) and one
// chunk of the keys, streamed in 64-key tiles by TMA:
//   warps 0-7  two threads per row (warps w and w + 4 share TMEM lanes 32 (w % 4) .. + 31; warp w
//              takes columns [0, 32) of each tile, warp w + 4 columns [32, 64)): load the row's Q
//              into shared memory (128-byte swizzle), then per tile load their half of S from TMEM,
//              and for each mask (dense, spatial, temporal) trade the half-row maxima through
//              shared memory, update that mask's running maximum and sum, compute P = 2^(S sl2 - m)
//              on its kept keys in fp32 and store it into that mask's two P buffers in shared
//              memory as a bf16 pair, P = P_hi + P_lo with P_hi = bf16(P), P_lo = bf16(P - P_hi)
//              (about 16 significant bits, so that the route's error sums keep the fp32 path's
//              accuracy);
//   warp 8     TMA producer of the K / V ring;
//   warp 9     MMA issuer: S(e) = Q K(e)^T into TMEM (N = 64), then O_a += P_hi,a V(e) + P_lo,a V(e)
//              for the three masks into three TMEM accumulators. S(e + 1) is issued as soon as the softmax has
//              loaded S(e) (P lives in shared memory), so it overlaps the softmax of tile e.
// Every wait is bounded; the chunk state written out is the CUDA-core form's, so the same merge
// and reduction kernels finish the route.
constexpr int kRtRows = 128;
constexpr int kRtKeys = kRouteKeys;
constexpr int kRtStages = 4;
constexpr int kRtThreads = 320;
constexpr int kRtSoftmax = 256;  // two threads per row
constexpr int kRtProducer = 8;
constexpr int kRtMma = 9;

template <int D>
struct RtCfg {
  static constexpr int kChunks = D / 64;                   // 128-byte swizzle chunks per Q / K / V row
  static constexpr int kQBytes = kRtRows * D * 2;
  static constexpr int kPBytes = kRtRows * kRtKeys * 2;    // one P buffer: 128 rows x 128 bytes
  static constexpr int kTileBytes = kRtKeys * D * 2;       // one K or V tile
  static constexpr int kDataBytes = kQBytes + 6 * kPBytes + kRtStages * kTileBytes;  // P_hi, P_lo per mask
  static constexpr int kCtlBytes = 512;                    // barriers, abort flag, TMEM base
  static constexpr int kXchBytes = 2 * 3 * 2 * kRtRows * 4;  // half-row maxima, final half-row sums
  static constexpr int kSmemBytes = kDataBytes + kCtlBytes + kXchBytes + 1024 /*alignment*/;
  static constexpr uint32_t kSCol = 0;                     // S: 64 columns
  __host__ __device__ static constexpr uint32_t o_col(int a) { return 128u + (uint32_t)D * a; }
  static_assert(128 + 3 * D <= 512, "TMEM columns");
  static_assert(kSmemBytes <= 232448, "shared memory");
};

struct RouteTcParams {
  CUtensorMap tm_k, tm_v;  // [H, N, d] bf16 as (d, N, H), box 64 columns x 64 keys x 1 head
  const __nv_bfloat16* q;
  int H, N;
  float sl2;
  MaskGeom gs, gt;
  const int32_t* rows;
  int n_rows, G, chunk;
  float* part;
  int* status;
};

// barriers (8 bytes each): kv_full[NS], kv_empty[NS], q_full, s_full, s_free, p_ready[3], pv_done[3],
// drain -- one p_ready / pv_done per mask, so that each mask's P store waits only for that mask's
// previous P V -- then xch[4][3]: the two threads of the rows of lane quarter q traded their half-row
// maxima of mask a (64 arrivals per tile), and fin: every softmax thread wrote its half-row sums
struct RtBar {
  uint32_t base;
  __device__ uint32_t kv_full(uint32_t i) const { return base + 8u * i; }
  __device__ uint32_t kv_empty(uint32_t i) const { return base + 8u * (kRtStages + i); }
  __device__ uint32_t q_full() const { return base + 8u * (2 * kRtStages + 0); }
  __device__ uint32_t s_full() const { return base + 8u * (2 * kRtStages + 1); }
  __device__ uint32_t s_free() const { return base + 8u * (2 * kRtStages + 2); }
  __device__ uint32_t p_ready(int a) const { return base + 8u * (2 * kRtStages + 3 + a); }
  __device__ uint32_t pv_done(int a) const { return base + 8u * (2 * kRtStages + 6 + a); }
  __device__ uint32_t drain() const { return base + 8u * (2 * kRtStages + 9); }
  __device__ uint32_t xch(int q, int a) const { return base + 8u * (2 * kRtStages + 10 + 3 * q + a); }
  __device__ uint32_t fin() const { return base + 8u * (2 * kRtStages + 22); }
  static constexpr int kCount = 2 * kRtStages + 23;
  static constexpr uint32_t kAbortOff = 8u * kCount;       // abort flag
  static constexpr uint32_t kTmemOff = kAbortOff + 8;      // TMEM base
  static_assert(kTmemOff + 8 <= 512, "control block");
};

// Bits [lo - j0, hi - j0) of a 64-key tile starting at key j0 (clamped to the tile).
__device__ __forceinline__ uint64_t rt_range_bits(int j0, int lo, int hi) {
  const int a = max(lo - j0, 0), b = min(hi - j0, kRtKeys);
  if (b <= a) return 0ull;
  const uint64_t upto_b = b >= 64 ? ~0ull : ((1ull << b) - 1ull);
  return upto_b & ~((1ull << a) - 1ull);
}

template <int D>
__global__ void __launch_bounds__(kRtThreads, 1) route_tc_kernel(const __grid_constant__ RouteTcParams P) {
  using C = RtCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = raw + ((1024u - (raw & 1023u)) & 1023u);
  const uint32_t sQ = sbase, sP = sQ + C::kQBytes, sRing = sP + 6 * C::kPBytes;
  RtBar b;
  b.base = sRing + kRtStages * C::kTileBytes;
  const uint32_t sX = b.base + C::kCtlBytes;  // float [3][2][128] half-row maxima, then [3][2][128] sums
  uint8_t* ctl = smem_raw + (b.base - raw);
  const uint32_t abort_addr = b.base + RtBar::kAbortOff;
  int* status = P.status;
  const int h = blockIdx.y, g = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int j_begin = g * P.chunk, j_end = min(P.N, j_begin + P.chunk);
  const int ntiles = (j_end - j_begin + kRtKeys - 1) / kRtKeys;

  if (threadIdx.x == 0) {
    uint64_t* bar = reinterpret_cast<uint64_t*>(ctl);
    for (int i = 0; i < kRtStages; ++i) {
      mbar_init(bar + i, 1);
      mbar_init(bar + kRtStages + i, 1);
    }
    mbar_init(bar + 2 * kRtStages + 0, kRtSoftmax);  // q_full: every softmax thread wrote its part of Q
    mbar_init(bar + 2 * kRtStages + 1, 1);           // s_full
    mbar_init(bar + 2 * kRtStages + 2, kRtSoftmax);  // s_free
    for (int a = 0; a < 3; ++a) {
      mbar_init(bar + 2 * kRtStages + 3 + a, kRtSoftmax);  // p_ready[a]
      mbar_init(bar + 2 * kRtStages + 6 + a, 1);           // pv_done[a]
    }
    mbar_init(bar + 2 * kRtStages + 9, 1);  // drain
    for (int i = 0; i < 12; ++i) mbar_init(bar + 2 * kRtStages + 10 + i, 64);  // xch[q][a]
    mbar_init(bar + 2 * kRtStages + 22, kRtSoftmax);                           // fin
    *reinterpret_cast<volatile int*>(ctl + RtBar::kAbortOff) = 0;
    fence_mbar_init();
  }
  if (warp == kRtMma) {
    tmem_alloc(reinterpret_cast<uint32_t*>(ctl + RtBar::kTmemOff), 512);
    tmem_relinquish();
  }
  if (warp == kRtProducer && lane == 0) {
    prefetch_tmap(&P.tm_k);
    prefetch_tmap(&P.tm_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<uint32_t*>(ctl + RtBar::kTmemOff);

  if (warp == kRtProducer) {
    // ---------------------------------------------------------------- K / V tiles, in the order
    // the MMA warp reads them: K(0), then K(e + 1), V(e) per tile
    if (lane == 0) {
      uint32_t pos = 0;
      for (int n = 0; n < 2 * ntiles; ++n) {
        int e, w;
        if (n == 0) {
          e = 0;
          w = 0;
        } else if (n == 2 * ntiles - 1) {
          e = ntiles - 1;
          w = 1;
        } else {
          const int m = n - 1;
          e = (m >> 1) + ((m & 1) ^ 1);
          w = m & 1;
        }
        const uint32_t st = pos % kRtStages;
        if (!wait_bar(b.kv_empty(st), ((pos / kRtStages) & 1u) ^ 1u, abort_addr, status)) break;
        mbar_expect_tx(b.kv_full(st), C::kTileBytes);
        const uint32_t dst = sRing + st * C::kTileBytes;
        for (int ch = 0; ch < C::kChunks; ++ch)
          tma_load_3d(dst + ch * (kRtKeys * 128), w == 0 ? &P.tm_k : &P.tm_v, b.kv_full(st), ch * 64,
                      j_begin + e * kRtKeys, h);
        ++pos;
      }
      if (ld_shared_volatile(abort_addr)) {  // let issued copies land before the CTA may exit
        const uint32_t n = pos < (uint32_t)kRtStages ? pos : (uint32_t)kRtStages;
        for (uint32_t i = 0; i < n; ++i) {
          const uint32_t q = pos - 1 - i;
          drain_bar(b.kv_full(q % kRtStages), (q / kRtStages) & 1u);
        }
      }
    }
    __syncwarp();
  } else if (warp == kRtMma) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(kRtKeys, false);
      constexpr uint32_t idesc_o = idesc_bf16_f32(D, true);
      const uint64_t qdesc = smem_desc_sw128(sQ, 16, 1024);
      const uint64_t kdesc = smem_desc_sw128(sRing, 16, 1024);
      const uint64_t vdesc = smem_desc_sw128(sRing, kRtKeys * 128, 1024);
      const uint64_t pdesc = smem_desc_sw128(sP, 16, 1024);
      uint32_t pos = 0;
      bool ok = wait_bar(b.q_full(), 0, abort_addr, status);
      tc_fence_after();
      auto issue_s = [&](uint32_t kpos) -> bool {
        const uint32_t st = kpos % kRtStages;
        if (!wait_bar(b.kv_full(st), (kpos / kRtStages) & 1u, abort_addr, status)) return false;
        const uint64_t kd = kdesc + ((st * C::kTileBytes) >> 4);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t qoff = ((kk >> 2) * (kRtRows * 128) + (kk & 3) * 32) >> 4;
          const uint32_t koff = ((kk >> 2) * (kRtKeys * 128) + (kk & 3) * 32) >> 4;
          umma_ss(tmem + C::kSCol, qdesc + qoff, kd + koff, idesc_s, kk > 0 ? 1u : 0u);
        }
        umma_commit(b.s_full());
        umma_commit(b.kv_empty(st));
        return true;
      };
      if (ok && ntiles > 0) ok = issue_s(pos++);
      for (int e = 0; e < ntiles && ok; ++e) {
        if (e + 1 < ntiles) {  // S(e + 1) once the softmax has loaded S(e)
          ok = wait_bar(b.s_free(), (uint32_t)e & 1u, abort_addr, status);
          if (!ok) break;
          tc_fence_after();
          ok = issue_s(pos++);
          if (!ok) break;
        }
        const uint32_t vpos = pos++;
        const uint32_t st = vpos % kRtStages;
        ok = wait_bar(b.kv_full(st), (vpos / kRtStages) & 1u, abort_addr, status);
        const uint64_t vd = vdesc + ((st * C::kTileBytes) >> 4);
#pragma unroll
        for (int a = 0; a < 3 && ok; ++a) {  // each mask's P V as soon as its P is stored
          ok = wait_bar(b.p_ready(a), (uint32_t)e & 1u, abort_addr, status);
          if (!ok) break;
          tc_fence_after();
#pragma unroll
          for (int part = 0; part < 2; ++part) {  // buffer 2a: P_hi, 2a + 1: P_lo
            const uint64_t pd = pdesc + (((2 * a + part) * C::kPBytes) >> 4);
#pragma unroll
            for (int kk = 0; kk < kRtKeys / 16; ++kk)
              umma_ss(tmem + C::o_col(a), pd + (((kk & 3) * 32) >> 4), vd + ((kk * 2048) >> 4), idesc_o,
                      (e > 0 || part > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(b.pv_done(a));
        }
        if (!ok) break;
        umma_commit(b.kv_empty(st));
      }
      umma_commit(b.drain());
      drain_bar(b.drain(), 0);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- rows: Q, softmaxes, state out
    const int qd = warp & 3, half = warp >> 2;  // TMEM lane quarter; column half of each tile
    const int lr = qd * 32 + lane;              // row within the block = TMEM lane
    const uint32_t lane_off = (uint32_t)(qd * 32) << 16;
    constexpr int kHalfCols = kRtKeys / 2;      // 32 score columns per thread
    constexpr int kOCols = D / 2;               // output columns per thread
    const int ridx = blockIdx.x * kRtRows + lr;
    int r = ridx < P.n_rows ? __ldg(P.rows + ridx) : -1;
    if (r < 0 || r >= P.N) r = 0;  // padding and rows outside the sequence: any valid row, unused
    const int S = P.gs.S;
    const int ti = r / S, si = r - ti * S;
    {  // this thread's chunks of the Q row into the 128-byte-swizzle K-major tile: chunk c, row lr,
       // 16-byte unit u at u ^ (lr % 8)
      const uint4* src = reinterpret_cast<const uint4*>(P.q + ((size_t)h * P.N + r) * D);
#pragma unroll
      for (int c = half; c < C::kChunks; c += 2)
#pragma unroll
        for (uint32_t u = 0; u < 8; ++u) {
          const uint4 v = __ldg(src + c * 8 + u);
          st_shared_v4(sQ + c * (kRtRows * 128) + (uint32_t)lr * 128u + ((u ^ ((uint32_t)lr & 7u)) << 4), v.x, v.y,
                       v.z, v.w);
        }
      fence_proxy_async_shared();
      mbar_arrive(b.q_full());
    }
    float* xmax = reinterpret_cast<float*>(smem_raw + (sX - raw));  // [3][2][128]
    float* xsum = xmax + 3 * 2 * kRtRows;                      // [3][2][128]
    float m[3] = {-INFINITY, -INFINITY, -INFINITY}, l[3] = {0.f, 0.f, 0.f};
    bool ok = true;
    for (int e = 0; e < ntiles; ++e) {
      if (!__all_sync(0xffffffffu, wait_bar(b.s_full(), (uint32_t)e & 1u, abort_addr, status))) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t sr[kHalfCols];
      tmem_ld32(tmem + lane_off + C::kSCol + kHalfCols * half, sr);
      tmem_ld_wait();
      tmem_ld_fence32(sr);
      tc_fence_before();
      mbar_arrive(b.s_free());
      float x[kHalfCols];
#pragma unroll
      for (int j = 0; j < kHalfCols; ++j) x[j] = __uint_as_float(sr[j]) * P.sl2;
      // kept keys of each mask in this tile, as bit sets from their ranges of original key index
      // (key j = t * S + s): dense [j0, j_end); sink [0, F0 * S); spatial frames [ti - k, ti + k];
      // temporal, in every frame t the tile touches, patches [si - b, si + b]; this thread's half
      const int j0 = j_begin + e * kRtKeys;
      const int jl = min(j0 + kRtKeys, j_end);  // end of this tile's keys
      uint64_t keep64[3];
      keep64[0] = rt_range_bits(j0, j0, jl);
      const uint64_t sink = rt_range_bits(j0, 0, P.gs.F0 * S) & keep64[0];
      keep64[1] = (rt_range_bits(j0, max(ti - P.gs.k, 0) * S, (min(ti + P.gs.k, P.gs.T - 1) + 1) * S) & keep64[0]) | sink;
      {
        const int s0 = max(si - P.gt.b, 0), s1 = min(si + P.gt.b, S - 1) + 1;
        uint64_t band = 0ull;
        for (int t = j0 / S; t * S < jl; ++t) band |= rt_range_bits(j0, t * S + s0, t * S + s1);
        keep64[2] = (band & keep64[0]) | sink;
      }
#pragma unroll
      for (int a = 0; a < 3; ++a) {
        const uint32_t keep = (uint32_t)(keep64[a] >> (kHalfCols * half));
        // the row's maximum: this half's, traded with the partner thread (bounded wait)
        float hm = -INFINITY;
#pragma unroll
        for (int j = 0; j < kHalfCols; ++j)
          if ((keep >> j) & 1u) hm = fmaxf(hm, x[j]);
        xmax[(a * 2 + half) * kRtRows + lr] = hm;
        mbar_arrive(b.xch(qd, a));
        if (!__all_sync(0xffffffffu, wait_bar(b.xch(qd, a), (uint32_t)e & 1u, abort_addr, status))) {
          ok = false;
          break;
        }
        const float mx = fmaxf(hm, xmax[(a * 2 + (half ^ 1)) * kRtRows + lr]);
        const float mn = fmaxf(m[a], mx);
        const bool need = (mn > m[a]) && (m[a] == -INFINITY || mn - m[a] > kRescaleLog2);
        const bool rescale = __any_sync(0xffffffffu, need);  // the same in both warps: same rows, same maxima
        float alpha = 1.f;
        if (rescale) {
          alpha = (mn == -INFINITY) ? 1.f : ex2f(m[a] - mn);
          l[a] *= alpha;
          m[a] = mn;
        }
        uint32_t hi[kHalfCols / 2], lo[kHalfCols / 2];
        float sum = 0.f;
#pragma unroll
        for (int j = 0; j < kHalfCols; j += 2) {
          const float p0 = ((keep >> j) & 1u) ? ex2f(x[j] - m[a]) : 0.f;
          const float p1 = ((keep >> (j + 1)) & 1u) ? ex2f(x[j + 1] - m[a]) : 0.f;
          sum += p0 + p1;
          hi[j / 2] = pack_bf16(p0, p1);
          const float h0 = __uint_as_float(hi[j / 2] << 16), h1 = __uint_as_float(hi[j / 2] & 0xFFFF0000u);
          lo[j / 2] = pack_bf16(p0 - h0, p1 - h1);
        }
        l[a] += sum;
        // this mask's previous P V is complete: its P buffers are free and O_a holds it
        if (e > 0 && !__all_sync(0xffffffffu, wait_bar(b.pv_done(a), (uint32_t)(e - 1) & 1u, abort_addr, status))) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (rescale && e > 0) {  // O_a holds the earlier tiles' P V (tile 0's MMA overwrites it); this
                                 // thread rescales its half of the columns
          const uint32_t tO = tmem + lane_off + C::o_col(a) + (uint32_t)(kOCols * half);
#pragma unroll 1
          for (int q = 0; q < kOCols / 32; ++q) {
            uint32_t o[32];
            tmem_ld32(tO + q * 32, o);
            tmem_ld_wait();
            tmem_ld_fence32(o);
#pragma unroll
            for (int y = 0; y < 32; ++y) o[y] = __float_as_uint(__uint_as_float(o[y]) * alpha);
            tmem_st32(tO + q * 32, o);
          }
          tmem_st_wait();
        }
        // this thread's 64 bytes of the row (16-byte units 4 half .. 4 half + 3) in both buffers
        const uint32_t rowb = (uint32_t)lr * 128u, sw = (uint32_t)lr & 7u;
#pragma unroll
        for (uint32_t u = 0; u < 4; ++u) {
          const uint32_t off = rowb + (((4u * (uint32_t)half + u) ^ sw) << 4);
          st_shared_v4(sP + (2 * a) * C::kPBytes + off, hi[4 * u], hi[4 * u + 1], hi[4 * u + 2], hi[4 * u + 3]);
          st_shared_v4(sP + (2 * a + 1) * C::kPBytes + off, lo[4 * u], lo[4 * u + 1], lo[4 * u + 2], lo[4 * u + 3]);
        }
        fence_proxy_async_shared();
        tc_fence_before();
        mbar_arrive(b.p_ready(a));
      }
      if (!ok) break;
    }
    // ---- this chunk's state of the row: O (unnormalised; each thread its half of the columns),
    // running max (log2 units), sum (both threads' halves)
    bool done = ok && ntiles > 0;
#pragma unroll
    for (int a = 0; a < 3; ++a) {
      if (done) xsum[(a * 2 + half) * kRtRows + lr] = l[a];
    }
    if (done) mbar_arrive(b.fin());
    done = done && __all_sync(0xffffffffu, wait_bar(b.fin(), 0, abort_addr, status));
#pragma unroll
    for (int a = 0; a < 3; ++a)
      done = done && __all_sync(0xffffffffu, wait_bar(b.pv_done(a), (uint32_t)(ntiles - 1) & 1u, abort_addr, status));
    if (done) {
      tc_fence_after();
      const bool write = ridx < P.n_rows;
      float* dst = P.part + (((size_t)h * P.n_rows + (write ? ridx : 0)) * P.G + g) * 3 * (D + 2);
#pragma unroll
      for (int a = 0; a < 3; ++a) {
#pragma unroll 1
        for (int q = 0; q < kOCols / 32; ++q) {
          uint32_t o[32];
          tmem_ld32(tmem + lane_off + C::o_col(a) + (uint32_t)(kOCols * half) + q * 32, o);
          tmem_ld_wait();
          tmem_ld_fence32(o);
          if (write) {  // (a row's state is 4-byte aligned only: scalar stores)
#pragma unroll
            for (int y = 0; y < 32; ++y) dst[a * (D + 2) + kOCols * half + q * 32 + y] = __uint_as_float(o[y]);
          }
        }
        if (write && half == 0) {
          dst[a * (D + 2) + D] = m[a];
          dst[a * (D + 2) + D + 1] = xsum[(a * 2) * kRtRows + lr] + xsum[(a * 2 + 1) * kRtRows + lr];
        }
      }
    } else if (ntiles == 0 && ridx < P.n_rows && half == 0) {  // an empty chunk: nothing kept
      float* dst = P.part + (((size_t)h * P.n_rows + ridx) * P.G + g) * 3 * (D + 2);
      for (int a = 0; a < 3; ++a) {
        for (int y = 0; y < D; ++y) dst[a * (D + 2) + y] = 0.f;
        dst[a * (D + 2) + D] = -INFINITY;
        dst[a * (D + 2) + D + 1] = 0.f;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kRtMma) tmem_dealloc(tmem, 512);
}

// One block of three warps per (sampled row, head): warp a combines the chunks' states of mask a
// (dense, spatial, temporal), then warp 0 takes the row's squared errors of the sparse outputs
// against the dense one. Lane g holds chunk g's maximum and sum (at most 32 chunks), so the common
// maximum and the rescaled sum are warp reductions; the chunks' partial outputs are read four
// chunks at a time, their loads in flight together.
__global__ void __launch_bounds__(96) route_merge_kernel(const RouteParams P) {
  __shared__ float o_s[3][128];
  const int ridx = blockIdx.x, h = blockIdx.y, lane = threadIdx.x & 31, a = threadIdx.x >> 5;
  float* w = P.rowerr + ((size_t)h * P.n_rows + ridx) * 3;
  const int r = P.rows[ridx];
  if (r < 0 || r >= P.N) {  // rows outside the sequence contribute nothing (the whole block leaves)
    if (threadIdx.x < 3) w[threadIdx.x] = 0.f;
    return;
  }
  const int D = P.D, W = D + 2, G = P.G;
  const float* base = P.part + ((size_t)h * P.n_rows + ridx) * G * 3 * W;
  const float* mine = base + (lane * 3 + a) * W;  // this lane's chunk, lane < G
  const float mg = lane < G ? mine[D] : -INFINITY;
  const float lg = lane < G ? mine[D + 1] : 0.f;
  const float M = warp_max(mg);
  const float fl = (mg == -INFINITY) ? 0.f : exp2f(mg - M);
  const float L = warp_sum(lg * fl);
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
  for (int g = 0; g < G; ++g) {
    const float f = __shfl_sync(0xffffffffu, fl, g);
    const float* src = base + (g * 3 + a) * W;
#pragma unroll
    for (int x = 0; x < 4; ++x)
      if (lane + 32 * x < D) acc[x] = fmaf(src[lane + 32 * x], f, acc[x]);
  }
  const float inv = L > 0.f ? 1.f / L : 0.f;
#pragma unroll
  for (int x = 0; x < 4; ++x)
    if (lane + 32 * x < D) o_s[a][lane + 32 * x] = acc[x] * inv;
  __syncthreads();
  if (a != 0) return;
  float es = 0.f, et = 0.f, ed = 0.f;
#pragma unroll
  for (int x = 0; x < 4; ++x) {
    if (lane + 32 * x >= D) continue;
    const float od = o_s[0][lane + 32 * x], os = o_s[1][lane + 32 * x], ot = o_s[2][lane + 32 * x];
    es = fmaf(os - od, os - od, es);
    et = fmaf(ot - od, ot - od, et);
    ed = fmaf(od, od, ed);
  }
  es = warp_sum(es);
  et = warp_sum(et);
  ed = warp_sum(ed);
  if (lane == 0) {
    w[0] = es;
    w[1] = et;
    w[2] = ed;
  }
}

// One warp per head: fixed-order sums over the sampled rows (lane j takes rows j, j + 32, ...,
// then a butterfly over the lanes; the order never depends on timing), then the route.
__global__ void route_reduce_kernel(const RouteParams P) {
  const int h = blockIdx.x, lane = threadIdx.x;
  double es = 0.0, et = 0.0, ed = 0.0;
  for (int r = lane; r < P.n_rows; r += 32) {
    const float* w = P.rowerr + ((size_t)h * P.n_rows + r) * 3;
    es += w[0];
    et += w[1];
    ed += w[2];
  }
  es = warp_sum(es);
  et = warp_sum(et);
  ed = warp_sum(ed);
  if (lane != 0) return;
  const double den = ed > 0.0 ? ed : 1.0;
  P.route[h] = (es <= et) ? SVG_ROUTE_SPATIAL : SVG_ROUTE_TEMPORAL;
  if (P.err) {
    P.err[2 * h] = (float)(es / den);
    P.err[2 * h + 1] = (float)(et / den);
  }
}

template <int D>
static cudaError_t launch_tc(const RouteTcParams& T, int nblk_rows, cudaStream_t st) {
  using C = RtCfg<D>;
  auto kern = route_tc_kernel<D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
  if (e != cudaSuccess) return e;
  kern<<<dim3(nblk_rows, T.H, T.G), kRtThreads, C::kSmemBytes, st>>>(T);
  return cudaGetLastError();
}

int launch_route(const void* q, const CUtensorMap* tm_k, const CUtensorMap* tm_v, int heads, int N, int d, float scale,
                 svg_geom geom, svg_mask mask, const int32_t* rows, int n_rows, void* work, uint8_t* route, float* err,
                 int num_sms, cudaStream_t st) {
  RouteParams P;
  memset(&P, 0, sizeof(P));
  P.H = heads;
  P.N = N;
  P.D = d;
  P.sl2 = scale * 1.4426950408889634f;
  P.gs = make_geom(geom, mask, SVG_ROUTE_SPATIAL);
  P.gt = make_geom(geom, mask, SVG_ROUTE_TEMPORAL);
  P.rows = rows;
  P.n_rows = n_rows;
  const int nblk_rows = (n_rows + kRtRows - 1) / kRtRows;
  P.chunk = route_chunk_len(N, route_launch_chunks(N, nblk_rows, heads, num_sms, 1));
  P.G = (N + P.chunk - 1) / P.chunk;  // non-empty chunks, at most route_chunks(N)
  unsigned char* wb = static_cast<unsigned char*>(work);
  P.rowerr = reinterpret_cast<float*>(wb + kRouteStatusBytes);
  P.part = reinterpret_cast<float*>(wb + kRouteStatusBytes + route_rowerr_bytes(heads, n_rows));
  P.route = route;
  P.err = err;
  RouteTcParams T;
  memset(&T, 0, sizeof(T));
  T.tm_k = *tm_k;
  T.tm_v = *tm_v;
  T.q = static_cast<const __nv_bfloat16*>(q);
  T.H = heads;
  T.N = N;
  T.sl2 = P.sl2;
  T.gs = P.gs;
  T.gt = P.gt;
  T.rows = rows;
  T.n_rows = n_rows;
  T.G = P.G;
  T.chunk = P.chunk;
  T.part = P.part;
  T.status = reinterpret_cast<int*>(wb);
  cudaError_t e = cudaMemsetAsync(wb, 0, sizeof(int), st);
  if (e != cudaSuccess) return record_cuda_error("cudaMemsetAsync(route status)", e);
  e = d == 128 ? launch_tc<128>(T, nblk_rows, st) : launch_tc<64>(T, nblk_rows, st);
  if (e != cudaSuccess) return record_cuda_error("launch route_tc_kernel", e);
  route_merge_kernel<<<dim3(n_rows, heads), 96, 0, st>>>(P);
  route_reduce_kernel<<<heads, 32, 0, st>>>(P);
  e = cudaGetLastError();
  return e == cudaSuccess ? SVG_OK : record_cuda_error("launch route kernels", e);
}

}  // namespace svg
