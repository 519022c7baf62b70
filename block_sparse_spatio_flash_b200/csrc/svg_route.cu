// svg_route.cu -- head routing by sampled rows.
//
// Sparse VideoGen profiles heads at inference time and routes each one to the spatial or the
// temporal mask by sampling ("Sparse Attention Patterns": heads are routed dynamically based on
// sampling; summary: SVG profiles heads at inference time). Read here as: attend a few sampled
// query rows of the head under the dense mask and under both sparse masks, and route the head to
// the sparse mask whose outputs are closer to the dense ones (relative squared error over the
// sampled rows; ties go to spatial).
//
// route_rows_kernel: one block = 8 sampled rows (one warp per row) of one head, streaming 64-key
// K/V tiles of the head (original token order) through shared memory; per row three online
// softmaxes (dense / spatial / temporal) in fp32 on CUDA cores. Writes per row
// (|O_s - O_d|^2, |O_t - O_d|^2, |O_d|^2). route_reduce_kernel sums them per head in a fixed
// order (deterministic) and sets the route.
#include <cuda_bf16.h>

#include "svg_common.cuh"

namespace svg {

constexpr int kRouteRowsPerBlock = 8;
constexpr int kRouteTile = 64;

struct RouteParams {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  int H, N, D;
  float sl2;             // scale * log2(e)
  MaskGeom gs, gt;       // spatial / temporal masks on original identities (layout unused)
  const int32_t* rows;   // sampled original query indices
  int n_rows;
  float* work;           // [H][n_rows][3]
  uint8_t* route;        // [H]
  float* err;            // [H][2] nullable: relative errors of spatial / temporal
};

__device__ __forceinline__ bool keep_spatial(const MaskGeom& g, int ti, int tj) {
  return tj < g.F0 || abs(ti - tj) <= g.k;
}
__device__ __forceinline__ bool keep_temporal(const MaskGeom& g, int si, int tj, int sj) {
  return tj < g.F0 || abs(si - sj) <= g.b;
}

template <int D>
__global__ void __launch_bounds__(256) route_rows_kernel(const RouteParams P) {
  extern __shared__ float sm[];
  constexpr int KS = D + 1;               // padded K rows: lanes reading different keys hit distinct banks
  constexpr int DPL = D / 32;             // output dims per lane: dim x * 32 + lane
  float* sK = sm;                         // [kRouteTile][KS]
  float* sV = sK + kRouteTile * KS;       // [kRouteTile][D]
  float* sQ = sV + kRouteTile * D;        // [8][D], pre-scaled by sl2
  const int h = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ridx = blockIdx.x * kRouteRowsPerBlock + warp;
  int i = ridx < P.n_rows ? P.rows[ridx] : -1;
  const bool row_ok = i >= 0 && i < P.N;  // rows outside the sequence contribute nothing
  if (!row_ok) i = 0;
  const size_t hoff = (size_t)h * P.N * D;
  for (int x = lane; x < D; x += 32)
    sQ[warp * D + x] = row_ok ? __bfloat162float(P.q[hoff + (size_t)i * D + x]) * P.sl2 : 0.f;
  const int S = P.gs.S;
  const int ti = i / S, si = i - ti * S;
  // per row and mask (0 dense, 1 spatial, 2 temporal): running max (log2 units), sum, outputs
  float m[3] = {-INFINITY, -INFINITY, -INFINITY}, l[3] = {0.f, 0.f, 0.f};
  float o[3][DPL];
#pragma unroll
  for (int a = 0; a < 3; ++a)
#pragma unroll
    for (int x = 0; x < DPL; ++x) o[a][x] = 0.f;

  for (int j0 = 0; j0 < P.N; j0 += kRouteTile) {
    const int nt = min(kRouteTile, P.N - j0);
    __syncthreads();
    for (int x = threadIdx.x; x < nt * D; x += blockDim.x) {
      const int r = x / D, cidx = x - r * D;
      sK[r * KS + cidx] = __bfloat162float(P.k[hoff + (size_t)j0 * D + x]);
      sV[x] = __bfloat162float(P.v[hoff + (size_t)j0 * D + x]);
    }
    __syncthreads();
    // scores of keys j0 + lane and j0 + 32 + lane, and their mask bits
    float s2[2];
    bool ks[2], kt[2], in[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int jj = u * 32 + lane;
      in[u] = jj < nt;
      float acc = 0.f;
      if (in[u]) {
#pragma unroll 8
        for (int x = 0; x < D; ++x) acc = fmaf(sQ[warp * D + x], sK[jj * KS + x], acc);
      }
      s2[u] = in[u] ? acc : -INFINITY;
      const int j = j0 + jj;
      const int tj = j / S, sj = j - tj * S;
      ks[u] = in[u] && keep_spatial(P.gs, ti, tj);
      kt[u] = in[u] && keep_temporal(P.gt, si, tj, sj);
    }
    float p[3][2];
#pragma unroll
    for (int a = 0; a < 3; ++a) {
      const bool k0 = a == 0 ? in[0] : (a == 1 ? ks[0] : kt[0]);
      const bool k1 = a == 0 ? in[1] : (a == 1 ? ks[1] : kt[1]);
      float mx = fmaxf(k0 ? s2[0] : -INFINITY, k1 ? s2[1] : -INFINITY);
      for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      const float mn = fmaxf(m[a], mx);
      if (mn > m[a]) {
        const float alpha = m[a] == -INFINITY ? 0.f : exp2f(m[a] - mn);
        l[a] *= alpha;
#pragma unroll
        for (int x = 0; x < DPL; ++x) o[a][x] *= alpha;
        m[a] = mn;
      }
      p[a][0] = (k0 && m[a] != -INFINITY) ? exp2f(s2[0] - m[a]) : 0.f;
      p[a][1] = (k1 && m[a] != -INFINITY) ? exp2f(s2[1] - m[a]) : 0.f;
      float ls = p[a][0] + p[a][1];
      for (int off = 16; off > 0; off >>= 1) ls += __shfl_xor_sync(0xffffffffu, ls, off);
      l[a] += ls;
    }
    for (int jj = 0; jj < nt; ++jj) {
      const int src = jj & 31;
      float pj[3];
#pragma unroll
      for (int a = 0; a < 3; ++a) pj[a] = __shfl_sync(0xffffffffu, jj < 32 ? p[a][0] : p[a][1], src);
#pragma unroll
      for (int x = 0; x < DPL; ++x) {
        const float vv = sV[jj * D + x * 32 + lane];
#pragma unroll
        for (int a = 0; a < 3; ++a) o[a][x] = fmaf(pj[a], vv, o[a][x]);
      }
    }
  }
  // per-row errors of the sparse outputs against the dense one
  float es = 0.f, et = 0.f, ed = 0.f;
#pragma unroll
  for (int x = 0; x < DPL; ++x) {
    const float od = l[0] > 0.f ? o[0][x] / l[0] : 0.f;
    const float os = l[1] > 0.f ? o[1][x] / l[1] : 0.f;
    const float ot = l[2] > 0.f ? o[2][x] / l[2] : 0.f;
    es += (os - od) * (os - od);
    et += (ot - od) * (ot - od);
    ed += od * od;
  }
  for (int off = 16; off > 0; off >>= 1) {
    es += __shfl_xor_sync(0xffffffffu, es, off);
    et += __shfl_xor_sync(0xffffffffu, et, off);
    ed += __shfl_xor_sync(0xffffffffu, ed, off);
  }
  if (ridx < P.n_rows && lane == 0) {
    float* w = P.work + ((size_t)h * P.n_rows + ridx) * 3;
    w[0] = row_ok ? es : 0.f;
    w[1] = row_ok ? et : 0.f;
    w[2] = row_ok ? ed : 0.f;
  }
}

// One thread per head: fixed-order sums over the sampled rows, then the route.
__global__ void route_reduce_kernel(const RouteParams P) {
  const int h = blockIdx.x * blockDim.x + threadIdx.x;
  if (h >= P.H) return;
  double es = 0.0, et = 0.0, ed = 0.0;
  for (int r = 0; r < P.n_rows; ++r) {
    const float* w = P.work + ((size_t)h * P.n_rows + r) * 3;
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

int launch_route(const void* q, const void* k, const void* v, int heads, int N, int d, float scale, svg_geom geom,
                 svg_mask mask, const int32_t* rows, int n_rows, float* work, uint8_t* route, float* err,
                 cudaStream_t st) {
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
  P.work = work;
  P.route = route;
  P.err = err;
  const size_t smem = (size_t)(kRouteTile * (d + 1) + kRouteTile * d + kRouteRowsPerBlock * d) * sizeof(float);
  auto kern = d == 128 ? route_rows_kernel<128> : route_rows_kernel<64>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return record_cuda_error("cudaFuncSetAttribute(route_rows_kernel)", e);
  dim3 grid((n_rows + kRouteRowsPerBlock - 1) / kRouteRowsPerBlock, heads);
  kern<<<grid, 256, smem, st>>>(P);
  route_reduce_kernel<<<(heads + 127) / 128, 128, 0, st>>>(P);
  e = cudaGetLastError();
  return e == cudaSuccess ? SVG_OK : record_cuda_error("launch route kernels", e);
}

}  // namespace svg
