// svg_permute.cu -- token reordering of [heads, tokens, d] bf16 tensors.
//
// The case study notes that temporal heads need a different token order than spatial heads
// to expose regular sparsity ("Interesting facts"); the benchmark excludes that reordering
// from its timings (summary; "What we still don't know"). Temporal heads are moved from
// frame-major to space-major order (svg.h gives the exact position map); spatial heads are
// copied unchanged. Written as a gather: every output row reads one source row, so stores are
// fully coalesced and every load is a whole 128/256-byte row. Pure HBM traffic: 2 * bytes.
#include <string.h>

#include "svg_common.cuh"

namespace svg {

unsigned int* checks_counter();

struct PermParams {
  const uint4* in;
  uint4* out;
  int heads, N, row_vec;  // row_vec = 16-byte vectors per row (d*2/16)
  int inverse;
  MaskGeom g;             // route field ignored; per-head route from the bit set
  unsigned int* checks;   // failed-check counter of the checked build
  uint32_t route_bits[kMaxHeads / 32];
};

__global__ void __launch_bounds__(512) permute_kernel(const __grid_constant__ PermParams P) {
  // grid.y = head; a block moves (512 / row_vec) rows per step, one 16-byte vector per thread.
  const int h = blockIdx.y;
  const bool temporal = (P.route_bits[h >> 5] >> (h & 31)) & 1u;
  const int rows_per_step = blockDim.x / P.row_vec;
  const int vec = threadIdx.x % P.row_vec;
  const int r_first = blockIdx.x * rows_per_step + threadIdx.x / P.row_vec;
  const int stride = gridDim.x * rows_per_step;
  if (threadIdx.x >= rows_per_step * P.row_vec) return;
  const uint4* in = P.in + (int64_t)h * P.N * P.row_vec + vec;
  uint4* out = P.out + (int64_t)h * P.N * P.row_vec + vec;
  MaskGeom g = P.g;
  g.route = SVG_ROUTE_TEMPORAL;
  constexpr int kUnroll = 4;
  for (int r0 = r_first; r0 < P.N; r0 += stride * kUnroll) {
    uint4 v[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int r = r0 + u * stride;
      if (r < P.N) {
        int src = r;
        if (temporal) {
          if (!P.inverse) {  // output position r holds the token that sits there
            int t, s;
            pos_to_ts(g, r, t, s);
            src = t * g.S + s;
          } else {           // output token r comes from its position
            const int t = r / g.S;
            src = ts_to_pos(g, t, r - t * g.S);
          }
        }
        if (!check_ok(src >= 0 && src < P.N, P.checks)) src = 0;
        v[u] = __ldg(in + (int64_t)src * P.row_vec);
      }
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int r = r0 + u * stride;
      if (r < P.N) out[(int64_t)r * P.row_vec] = v[u];
    }
  }
}

int launch_permute(const void* in, void* out, int heads, int64_t N, int d, const uint8_t* h_route, svg_geom geom,
                   svg_mask mask, int inverse, int num_sms, cudaStream_t st) {
  PermParams P;
  memset(&P, 0, sizeof(P));
  P.in = static_cast<const uint4*>(in);
  P.out = static_cast<uint4*>(out);
  P.heads = heads;
  P.N = (int)N;
  P.row_vec = d * 2 / 16;
  P.inverse = inverse;
  P.g = make_geom(geom, mask, SVG_ROUTE_TEMPORAL);
  P.checks = checks_counter();
  for (int h = 0; h < heads; ++h)
    if (h_route[h] == SVG_ROUTE_TEMPORAL) P.route_bits[h >> 5] |= 1u << (h & 31);
  // about 8 resident blocks per SM across all heads; each block moves >= 4 steps of rows
  const int rows_per_step = 512 / P.row_vec;
  int64_t bx = ((int64_t)num_sms * 8 + heads - 1) / heads;
  const int64_t need = (N + (int64_t)rows_per_step * 4 - 1) / ((int64_t)rows_per_step * 4);
  if (bx > need) bx = need;
  if (bx < 1) bx = 1;
  permute_kernel<<<dim3((unsigned)bx, (unsigned)heads), 512, 0, st>>>(P);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? SVG_OK : record_cuda_error("launch permute_kernel", e);
}

}  // namespace svg
