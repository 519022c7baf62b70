// svg_route.cu -- head routing by sampled rows.
//
// Sparse VideoGen profiles heads at inference time and routes each one to the spatial or the
// temporal mask by sampling ("Sparse Attention Patterns": heads are routed dynamically based on
// sampling; summary: SVG profiles heads at inference time). Read here as: attend a few sampled
// query rows of the head under the dense mask and under both sparse masks, and route the head to
// the sparse mask whose outputs are closer to the dense ones (relative squared error over the
// sampled rows; ties go to spatial).
//
// route_partial_kernel: one block = 32 sampled rows of one head x one chunk of the keys. K/V tiles
// of 64 keys are staged in shared memory as bf16; warp w owns rows 4w..4w+3 and keeps, per row and
// mask (dense / spatial / temporal), an online softmax in fp32 on the CUDA cores: scores with keys
// lane and lane + 32 (register-blocked 4 rows x 2 keys), then P V with output dims
// [lane * D/32, (lane + 1) * D/32). The unnormalised state (O, running max, running sum) of each
// chunk is written out; route_merge_kernel combines the chunks of a row and writes
// (|O_s - O_d|^2, |O_t - O_d|^2, |O_d|^2); route_reduce_kernel sums those per head in a fixed
// order (deterministic) and sets the route.
#include <cuda_bf16.h>

#include "svg_common.cuh"

namespace svg {

constexpr int kRouteRows = 32;      // sampled rows per block (4 per warp)
constexpr int kRouteKeys = 64;      // keys per shared-memory tile
constexpr int kRouteThreads = 256;
constexpr int kRouteMaxChunks = 32;
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
// for) whose blocks fill the GPU's 2 x SM block slots best over whole waves -- a last, mostly empty
// wave costs as much as a full one; among equals the larger count (shorter blocks).
inline int route_launch_chunks(int64_t N, int row_blocks, int heads, int num_sms) {
  const int64_t per_chunk = (int64_t)row_blocks * heads;
  const int64_t slots = 2 * (int64_t)(num_sms > 0 ? num_sms : 1);
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

size_t route_rowerr_bytes(int heads, int n_rows) {
  return ((size_t)heads * n_rows * 3 * sizeof(float) + 255) / 256 * 256;
}
size_t route_work_bytes(int heads, int64_t N, int d, int n_rows) {
  return route_rowerr_bytes(heads, n_rows) +
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

template <int D>
struct RouteCfg {
  static constexpr int KP = D + 8;   // padded bf16 K row: 16-byte reads of 8 consecutive lanes hit distinct banks
  static constexpr int DPL = D / 32;
  static constexpr size_t kQ = (size_t)kRouteRows * D * 4;
  static constexpr size_t kP = (size_t)kRouteRows * kRouteKeys * 16;
  static constexpr size_t kK = (size_t)kRouteKeys * KP * 2;
  static constexpr size_t kV = (size_t)kRouteKeys * D * 2;
  static constexpr size_t kBytes = kQ + kP + kK + kV + kRouteRows * 4;
};

__device__ __forceinline__ void bf16x8_to_f32(const uint4 u, float* f) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, off));
  return x;
}
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
  return x;
}

template <int D>
__global__ void __launch_bounds__(kRouteThreads, 2) route_partial_kernel(const RouteParams P) {
  using C = RouteCfg<D>;
  constexpr int DPL = C::DPL, KP = C::KP;
  extern __shared__ __align__(16) unsigned char smem[];
  float* sQ = reinterpret_cast<float*>(smem);                                // [32][D], times sl2
  float4* sP = reinterpret_cast<float4*>(smem + C::kQ);                      // [32][64] {dense, spatial, temporal, -}
  __nv_bfloat16* sK = reinterpret_cast<__nv_bfloat16*>(smem + C::kQ + C::kP);          // [64][KP]
  __nv_bfloat16* sV = reinterpret_cast<__nv_bfloat16*>(smem + C::kQ + C::kP + C::kK);  // [64][D]
  int* sRow = reinterpret_cast<int*>(smem + C::kQ + C::kP + C::kK + C::kV);           // [32]
  const int h = blockIdx.y, g = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int j_begin = g * P.chunk;
  const int j_end = min(P.N, j_begin + P.chunk);
  if (tid < kRouteRows) {
    const int idx = blockIdx.x * kRouteRows + tid;
    int r = idx < P.n_rows ? P.rows[idx] : -1;
    sRow[tid] = (r >= 0 && r < P.N) ? r : -1;  // rows outside the sequence attend with Q = 0, unused
  }
  __syncthreads();
  const size_t hoff = (size_t)h * P.N * D;
  for (int x = tid; x < kRouteRows * D; x += kRouteThreads) {
    const int rr = x / D, c = x - rr * D, r = sRow[rr];
    sQ[x] = r >= 0 ? __bfloat162float(P.q[hoff + (size_t)r * D + c]) * P.sl2 : 0.f;
  }
  const int S = P.gs.S;
  int ti[4], si[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = max(sRow[4 * warp + i], 0);
    ti[i] = r / S;
    si[i] = r - ti[i] * S;
  }
  float m[4][3], l[4][3], o[4][3][DPL];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int a = 0; a < 3; ++a) {
      m[i][a] = -INFINITY;
      l[i][a] = 0.f;
#pragma unroll
      for (int x = 0; x < DPL; ++x) o[i][a][x] = 0.f;
    }

  for (int j0 = j_begin; j0 < j_end; j0 += kRouteKeys) {
    const int nt = min(kRouteKeys, j_end - j0);
    __syncthreads();  // every warp is done with the previous tile
    constexpr int CPR = D / 8;  // 16-byte pieces per row
    for (int c = tid; c < kRouteKeys * CPR; c += kRouteThreads) {
      const int key = c / CPR, part = c - key * CPR;
      uint4 kv = make_uint4(0u, 0u, 0u, 0u), vv = kv;
      if (key < nt) {
        const size_t off = hoff + (size_t)(j0 + key) * D + part * 8;
        kv = __ldg(reinterpret_cast<const uint4*>(P.k + off));
        vv = __ldg(reinterpret_cast<const uint4*>(P.v + off));
      }
      *reinterpret_cast<uint4*>(sK + key * KP + part * 8) = kv;
      *reinterpret_cast<uint4*>(sV + key * D + part * 8) = vv;
    }
    __syncthreads();
    // ---- scores of rows 4w..4w+3 with keys j0 + lane and j0 + lane + 32 (log2 units)
    float sc[4][2];
#pragma unroll
    for (int i = 0; i < 4; ++i) sc[i][0] = sc[i][1] = 0.f;
#pragma unroll 4
    for (int st = 0; st < D / 8; ++st) {
      float fa[8], fb[8];
      bf16x8_to_f32(*reinterpret_cast<const uint4*>(sK + lane * KP + st * 8), fa);
      bf16x8_to_f32(*reinterpret_cast<const uint4*>(sK + (lane + 32) * KP + st * 8), fb);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float4 q0 = *reinterpret_cast<const float4*>(sQ + (4 * warp + i) * D + st * 8);
        const float4 q1 = *reinterpret_cast<const float4*>(sQ + (4 * warp + i) * D + st * 8 + 4);
        const float qq[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
#pragma unroll
        for (int x = 0; x < 8; ++x) {
          sc[i][0] = fmaf(qq[x], fa[x], sc[i][0]);
          sc[i][1] = fmaf(qq[x], fb[x], sc[i][1]);
        }
      }
    }
    // ---- masks and the three online softmaxes per row
    const int ja = j0 + lane, jb = j0 + lane + 32;
    const bool ina = lane < nt, inb = lane + 32 < nt;
    const int tja = ja / S, sja = ja - tja * S, tjb = jb / S, sjb = jb - tjb * S;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const bool keep[3][2] = {
          {ina, inb},
          {ina && (tja < P.gs.F0 || abs(ti[i] - tja) <= P.gs.k), inb && (tjb < P.gs.F0 || abs(ti[i] - tjb) <= P.gs.k)},
          {ina && (tja < P.gt.F0 || abs(si[i] - sja) <= P.gt.b), inb && (tjb < P.gt.F0 || abs(si[i] - sjb) <= P.gt.b)}};
      float p[3][2];
#pragma unroll
      for (int a = 0; a < 3; ++a) {
        const float x0 = keep[a][0] ? sc[i][0] : -INFINITY;
        const float x1 = keep[a][1] ? sc[i][1] : -INFINITY;
        const float mn = fmaxf(m[i][a], warp_max(fmaxf(x0, x1)));
        const float alpha = (mn == -INFINITY) ? 1.f : exp2f(m[i][a] - mn);
        p[a][0] = keep[a][0] ? exp2f(x0 - mn) : 0.f;
        p[a][1] = keep[a][1] ? exp2f(x1 - mn) : 0.f;
        l[i][a] = l[i][a] * alpha + warp_sum(p[a][0] + p[a][1]);
        m[i][a] = mn;
#pragma unroll
        for (int x = 0; x < DPL; ++x) o[i][a][x] *= alpha;
      }
      sP[(4 * warp + i) * kRouteKeys + lane] = make_float4(p[0][0], p[1][0], p[2][0], 0.f);
      sP[(4 * warp + i) * kRouteKeys + lane + 32] = make_float4(p[0][1], p[1][1], p[2][1], 0.f);
    }
    __syncwarp();
    // ---- O += P V over the tile's keys (P = 0 and V = 0 past the end)
#pragma unroll 2
    for (int jj = 0; jj < kRouteKeys; ++jj) {
      float vv[DPL];
      if constexpr (DPL == 4) {
        const uint2 u = *reinterpret_cast<const uint2*>(sV + jj * D + lane * DPL);
        vv[0] = __uint_as_float(u.x << 16);
        vv[1] = __uint_as_float(u.x & 0xffff0000u);
        vv[2] = __uint_as_float(u.y << 16);
        vv[3] = __uint_as_float(u.y & 0xffff0000u);
      } else {
        static_assert(DPL == 2, "head dim 64 or 128");
        const uint32_t u = *reinterpret_cast<const uint32_t*>(sV + jj * D + lane * DPL);
        vv[0] = __uint_as_float(u << 16);
        vv[1] = __uint_as_float(u & 0xffff0000u);
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float4 pp = sP[(4 * warp + i) * kRouteKeys + jj];
#pragma unroll
        for (int x = 0; x < DPL; ++x) {
          o[i][0][x] = fmaf(pp.x, vv[x], o[i][0][x]);
          o[i][1][x] = fmaf(pp.y, vv[x], o[i][1][x]);
          o[i][2][x] = fmaf(pp.z, vv[x], o[i][2][x]);
        }
      }
    }
  }
  // ---- this chunk's state of every row the block holds
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int ridx = blockIdx.x * kRouteRows + 4 * warp + i;
    if (ridx >= P.n_rows) continue;
    float* dst = P.part + (((size_t)h * P.n_rows + ridx) * P.G + g) * 3 * (D + 2);
#pragma unroll
    for (int a = 0; a < 3; ++a) {
#pragma unroll
      for (int x = 0; x < DPL; ++x) dst[a * (D + 2) + lane * DPL + x] = o[i][a][x];
      if (lane == 0) {
        dst[a * (D + 2) + D] = m[i][a];
        dst[a * (D + 2) + D + 1] = l[i][a];
      }
    }
  }
}

// One warp per (sampled row, head): combine the chunks' states of each mask, then the row's
// squared errors of the sparse outputs against the dense one.
__global__ void route_merge_kernel(const RouteParams P) {
  const int ridx = blockIdx.x, h = blockIdx.y, lane = threadIdx.x;
  float* w = P.rowerr + ((size_t)h * P.n_rows + ridx) * 3;
  const int r = P.rows[ridx];
  if (r < 0 || r >= P.N) {  // rows outside the sequence contribute nothing
    if (lane < 3) w[lane] = 0.f;
    return;
  }
  const int D = P.D, W = D + 2;
  const float* base = P.part + ((size_t)h * P.n_rows + ridx) * P.G * 3 * W;
  float out[3][4];  // dims lane + 32 x, x < D / 32
#pragma unroll
  for (int a = 0; a < 3; ++a) {
    float M = -INFINITY;
    for (int g = 0; g < P.G; ++g) M = fmaxf(M, base[(g * 3 + a) * W + D]);
    float L = 0.f, acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int g = 0; g < P.G; ++g) {
      const float* src = base + (g * 3 + a) * W;
      const float mg = src[D];
      const float f = (mg == -INFINITY) ? 0.f : exp2f(mg - M);
      L = fmaf(src[D + 1], f, L);
#pragma unroll
      for (int x = 0; x < 4; ++x)
        if (lane + 32 * x < D) acc[x] = fmaf(src[lane + 32 * x], f, acc[x]);
    }
    const float inv = L > 0.f ? 1.f / L : 0.f;
#pragma unroll
    for (int x = 0; x < 4; ++x) out[a][x] = acc[x] * inv;
  }
  float es = 0.f, et = 0.f, ed = 0.f;
#pragma unroll
  for (int x = 0; x < 4; ++x) {
    if (lane + 32 * x >= D) continue;
    const float od = out[0][x], os = out[1][x], ot = out[2][x];
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

// One thread per head: fixed-order sums over the sampled rows, then the route.
__global__ void route_reduce_kernel(const RouteParams P) {
  const int h = blockIdx.x * blockDim.x + threadIdx.x;
  if (h >= P.H) return;
  double es = 0.0, et = 0.0, ed = 0.0;
  for (int r = 0; r < P.n_rows; ++r) {
    const float* w = P.rowerr + ((size_t)h * P.n_rows + r) * 3;
    es += w[0];
    et += w[1];
    ed += w[2];
  }
  const double den = ed > 0.0 ? ed : 1.0;
  P.route[h] = (es <= et) ? SVG_ROUTE_SPATIAL : SVG_ROUTE_TEMPORAL;
  if (P.err) {
    P.err[2 * h] = (float)(es / den);
    P.err[2 * h + 1] = (float)(et / den);
  }
}

template <int D>
static cudaError_t launch_partial(const RouteParams& P, int nblk_rows, int nchunks, cudaStream_t st) {
  using C = RouteCfg<D>;
  auto kern = route_partial_kernel<D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::kBytes);
  if (e != cudaSuccess) return e;
  kern<<<dim3(nblk_rows, P.H, nchunks), kRouteThreads, C::kBytes, st>>>(P);
  return cudaGetLastError();
}

int launch_route(const void* q, const void* k, const void* v, int heads, int N, int d, float scale, svg_geom geom,
                 svg_mask mask, const int32_t* rows, int n_rows, void* work, uint8_t* route, float* err,
                 int num_sms, cudaStream_t st) {
  RouteParams P;
  P.q = static_cast<const __nv_bfloat16*>(q);
  P.k = static_cast<const __nv_bfloat16*>(k);
  P.v = static_cast<const __nv_bfloat16*>(v);
  P.H = heads;
  P.N = N;
  P.D = d;
  P.sl2 = scale * 1.4426950408889634f;
  P.gs = make_geom(geom, mask, SVG_ROUTE_SPATIAL);
  P.gt = make_geom(geom, mask, SVG_ROUTE_TEMPORAL);
  P.rows = rows;
  P.n_rows = n_rows;
  const int nblk_rows = (n_rows + kRouteRows - 1) / kRouteRows;
  P.chunk = route_chunk_len(N, route_launch_chunks(N, nblk_rows, heads, num_sms));
  P.G = (N + P.chunk - 1) / P.chunk;  // non-empty chunks, at most route_chunks(N)
  P.rowerr = static_cast<float*>(work);
  P.part = reinterpret_cast<float*>(static_cast<unsigned char*>(work) + route_rowerr_bytes(heads, n_rows));
  P.route = route;
  P.err = err;
  cudaError_t e = d == 128 ? launch_partial<128>(P, nblk_rows, P.G, st) : launch_partial<64>(P, nblk_rows, P.G, st);
  if (e != cudaSuccess) return record_cuda_error("launch route_partial_kernel", e);
  route_merge_kernel<<<dim3(n_rows, heads), 32, 0, st>>>(P);
  route_reduce_kernel<<<(heads + 127) / 128, 128, 0, st>>>(P);
  e = cudaGetLastError();
  return e == cudaSuccess ? SVG_OK : record_cuda_error("launch route kernels", e);
}

}  // namespace svg
