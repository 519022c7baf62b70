// svg_api.cu -- the extern "C" entry points of libsvgattn (declared in include/svg.h).
//
// Host side only: argument validation, tensor-map encoding, launch configuration. Every
// numeric step runs in the kernels of svg_tilemap.cu, svg_permute.cu and svg_attention.cu.
// Nothing here allocates device memory.
#include <math.h>
#include <mutex>
#include <stdlib.h>
#include <stdio.h>
#include <string.h>

#include "svg_common.cuh"

namespace svg {
int build_tilemap(svg_geom geom, svg_mask mask, svg_tile tile, int route, void* ws, cudaStream_t st);
int launch_permute(const void* in, void* out, int heads, int64_t N, int d, const uint8_t* h_route, svg_geom geom,
                   svg_mask mask, int inverse, int num_sms, cudaStream_t st);
int launch_attention(const AttnParams& P, int d, int bk, int grid, bool p_smem, cudaStream_t st);
size_t route_work_bytes(int heads, int64_t N, int d, int n_rows);
int launch_route(const void* q, const CUtensorMap* tm_k, const CUtensorMap* tm_v, int heads, int N, int d, float scale,
                 svg_geom geom, svg_mask mask, const int32_t* rows, int n_rows, void* work, uint8_t* route, float* err,
                 int num_sms, cudaStream_t st);
}  // namespace svg

using namespace svg;

namespace svg {
int record_cuda_error(const char* what, int cuda_error);
unsigned int* checks_counter();
}

#if SVG_CHECKED
// Failed-check counter of the checked build (see SVG_CHECKED in svg_common.cuh).
static __device__ unsigned int g_checks_failed;
#endif

// Device address of the counter (null in the release build, whose kernels never use it).
unsigned int* svg::checks_counter() {
#if SVG_CHECKED
  void* p = nullptr;
  return cudaGetSymbolAddress(&p, g_checks_failed) == cudaSuccess ? static_cast<unsigned int*>(p) : nullptr;
#else
  return nullptr;
#endif
}

namespace {

constexpr int kMaxDevices = 64;

thread_local char g_last_error[192] = "none";

// Compute capability and SM count of the current device (cached per device).
int device_info(int* num_sms) {
  static std::mutex mu;
  static int sms[kMaxDevices] = {0};
  static int ok[kMaxDevices] = {0};  // 0 unknown, 1 sm_100, -1 other
  int dev = 0;
  cudaError_t ge = cudaGetDevice(&dev);
  if (ge != cudaSuccess) return record_cuda_error("cudaGetDevice", ge);
  if (dev < 0 || dev >= kMaxDevices) return SVG_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(mu);
  if (ok[dev] == 0) {
    int major = 0, minor = 0, n = 0;
    cudaError_t e1 = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    if (e1 == cudaSuccess) e1 = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    if (e1 == cudaSuccess) e1 = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (e1 != cudaSuccess) return record_cuda_error("cudaDeviceGetAttribute", e1);
    ok[dev] = (major == 10 && minor == 0) ? 1 : -1;
    sms[dev] = n;
  }
  if (ok[dev] != 1) return SVG_ERR_UNSUPPORTED;
  if (num_sms) *num_sms = sms[dev];
  return SVG_OK;
}

bool geom_ok(const svg_geom& g) {
  if (g.frames < 1 || g.grid_h < 1 || g.grid_w < 1) return false;
  const int64_t n = (int64_t)g.frames * g.grid_h * g.grid_w;
  return n >= 1 && n <= kMaxTokens;
}

bool mask_ok(const svg_geom& g, const svg_mask& m) {
  return m.frame_window >= 0 && m.spatial_band >= 0 && m.sink_frames >= 0 && m.sink_frames <= g.frames &&
         (m.variant == SVG_MASK_EXACT || m.variant == SVG_MASK_ROUNDED) &&
         (m.layout == SVG_LAYOUT_SINK_PREFIX || m.layout == SVG_LAYOUT_FULL_SPACE_MAJOR);
}

bool tile_ok(const svg_tile& t) {
  return (t.bq == 64 || t.bq == 128 || t.bq == 256 || t.bq == 512) && (t.bk == 64 || t.bk == 128);
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static std::once_flag once;
  static EncodeTiledFn fn = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// [heads, tokens, d] bf16 viewed as a 3-D tensor (d, tokens, heads); box = 64 columns
// (128 bytes, one swizzle atom wide) x box_rows rows x 1 head; rows past the end read 0.
int encode_qkv_map(CUtensorMap* m, const void* base, int heads, int tokens, int d, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return record_cuda_error("cudaGetDriverEntryPoint(cuTensorMapEncodeTiled)", (int)cudaErrorSymbolNotFound);
  cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)tokens, (cuuint64_t)heads};
  cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)tokens * d * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    snprintf(g_last_error, sizeof(g_last_error), "cuTensorMapEncodeTiled: CUresult %d", (int)r);
    return SVG_ERR_CUDA;
  }
  return SVG_OK;
}

// [heads, tokens, d] e4m3 (one byte per element, d = 128): box 128 columns (one 128-byte swizzle
// row) x box_rows rows.
int encode_qk8_map(CUtensorMap* m, const void* base, int heads, int tokens, int d, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return record_cuda_error("cudaGetDriverEntryPoint(cuTensorMapEncodeTiled)", (int)cudaErrorSymbolNotFound);
  cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)tokens, (cuuint64_t)heads};
  cuuint64_t strides[2] = {(cuuint64_t)d, (cuuint64_t)tokens * d};
  cuuint32_t box[3] = {128, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    snprintf(g_last_error, sizeof(g_last_error), "cuTensorMapEncodeTiled (e4m3): CUresult %d", (int)r);
    return SVG_ERR_CUDA;
  }
  return SVG_OK;
}

// [heads * tokens, d] bf16 viewed as rows, box 64 columns x 1 row, 128-byte swizzle: the map
// for 4-row gathers of arbitrary rows.
int encode_rows_map(CUtensorMap* m, const void* base, int heads, int64_t tokens, int d) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return record_cuda_error("cudaGetDriverEntryPoint(cuTensorMapEncodeTiled)", (int)cudaErrorSymbolNotFound);
  cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)tokens * heads};
  cuuint64_t strides[1] = {(cuuint64_t)d * 2};
  cuuint32_t box[2] = {64, 1};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    snprintf(g_last_error, sizeof(g_last_error), "cuTensorMapEncodeTiled (rows): CUresult %d", (int)r);
    return SVG_ERR_CUDA;
  }
  return SVG_OK;
}

// [heads, T, S, d] bf16 (original frame-major order) viewed as a 4-D tensor (d, patch, frame, head);
// box = 64 columns x 1 patch x run_len frames x 1 head: one patch's run of frames, rows S apart in
// memory, lands as run_len consecutive 128-byte rows.
int encode_run_map(CUtensorMap* m, const void* base, int heads, int frames, int patches, int d, int run_len) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return record_cuda_error("cudaGetDriverEntryPoint(cuTensorMapEncodeTiled)", (int)cudaErrorSymbolNotFound);
  cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)patches, (cuuint64_t)frames, (cuuint64_t)heads};
  cuuint64_t strides[3] = {(cuuint64_t)d * 2, (cuuint64_t)patches * d * 2, (cuuint64_t)frames * patches * d * 2};
  cuuint32_t box[4] = {64, 1, (cuuint32_t)run_len, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    snprintf(g_last_error, sizeof(g_last_error), "cuTensorMapEncodeTiled (runs): CUresult %d", (int)r);
    return SVG_ERR_CUDA;
  }
  return SVG_OK;
}

// SVG_KERNEL=ps: the single-SM kernel with P staged in shared memory, so that the next key tile's
// S is computed while the softmax of this one runs.
bool use_p_smem() {
  static const bool ps = [] {
    const char* v = getenv("SVG_KERNEL");
    return v && strcmp(v, "ps") == 0;
  }();
  return ps;
}

int check_qkvo(const void* q, const void* k, const void* v, const void* o, const float* lse, int heads,
               int64_t tokens, int d) {
  if (!q || !k || !v || !o) return SVG_ERR_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || (lse && !aligned(lse, 4)))
    return SVG_ERR_ARG;
  if (heads < 1 || heads > kMaxHeads || tokens < 1 || tokens > kMaxTokens) return SVG_ERR_ARG;
  if (d != 64 && d != 128) return SVG_ERR_UNSUPPORTED;
  return SVG_OK;
}

int run_attention(const void* q, const void* k, const void* v, void* o, float* lse, int heads, int64_t tokens,
                  int d, float scale, const uint8_t* h_route, const void* ws_sp, const void* ws_tm,
                  const svg_geom* geom, const svg_mask* mask, int bq, int bk, int mode, bool dense,
                  void* scratch, size_t scratch_bytes, int32_t* d_status, cudaStream_t st, bool fused = false,
                  bool qk8 = false, bool stall = false, int order = kOrderHeadMajor,
                  unsigned long long* cta_trace = nullptr, int trace_ctas = 0) {
  int rc = check_qkvo(q, k, v, o, lse, heads, tokens, d);
  if (rc) return rc;
  if (!scratch || scratch_bytes < kScratchBytes || !aligned(scratch, 16)) return SVG_ERR_ARG;
  if (d_status && !aligned(d_status, 4)) return SVG_ERR_ARG;
  if (order != kOrderHeadMajor && order != kOrderWork) return SVG_ERR_ARG;
  if (cta_trace && (trace_ctas < 1 || !aligned(cta_trace, 8))) return SVG_ERR_ARG;
  if (bk != 64 && bk != 128) return SVG_ERR_UNSUPPORTED;
  if (qk8 && (d != 128 || fused)) return SVG_ERR_UNSUPPORTED;  // e4m3 QK^T: d = 128, permuted order
  // fused order gathers rows of a [heads * tokens, d] view whose row coordinate is a signed 32-bit
  // TMA coordinate
  if (fused && (int64_t)heads * tokens > (int64_t)INT32_MAX) return SVG_ERR_UNSUPPORTED;
  int num_sms = 0;
  rc = device_info(&num_sms);
  if (rc) return rc;

  static AttnParams P;  // large (tensor maps); built under a lock, copied by value at launch
  static std::mutex mu;
  std::lock_guard<std::mutex> lock(mu);
  memset(&P, 0, sizeof(P));
  const int N = (int)tokens;
  P.H = heads;
  P.N = N;
  P.nk = (N + bk - 1) / bk;
  P.npairs = (N + kPairRows - 1) / kPairRows;
  const int64_t items = (int64_t)heads * P.npairs;
  if (items > 0x7FFFFFFF) return SVG_ERR_ARG;
  P.n_items = (int)items;
  const float sc = scale > 0.f ? scale : 1.0f / sqrtf((float)d);
  P.sl2 = sc * 1.4426950408889634f;
  P.dense = dense ? 1 : 0;
  P.bkm = bk;
  P.naive = mode == SVG_MODE_NAIVE ? 1 : 0;
  P.fused = fused && !dense ? 1 : 0;
  P.qk8 = qk8 ? 1 : 0;
  P.inject_stall = stall ? 1 : 0;  // only svg_test_attention_fwd_stall sets it
  P.o = static_cast<__nv_bfloat16*>(o);
  P.lse = lse;
  P.status = d_status ? d_status : static_cast<int*>(scratch);
  P.checks = checks_counter();
  P.counter = reinterpret_cast<unsigned int*>(static_cast<uint8_t*>(scratch) + 8);
  P.counter64 = reinterpret_cast<unsigned long long*>(static_cast<uint8_t*>(scratch) + kCounter64Off);
  P.cta_trace = cta_trace;
  P.trace_ctas = cta_trace ? trace_ctas : 0;
  if (!dense) {
    if (!h_route || !geom || !mask) return SVG_ERR_ARG;
    if (!geom_ok(*geom) || !mask_ok(*geom, *mask)) return SVG_ERR_ARG;
    const svg_tile t{bq, bk};
    if (!tile_ok(t)) return SVG_ERR_UNSUPPORTED;
    if ((int64_t)geom->frames * geom->grid_h * geom->grid_w != tokens) return SVG_ERR_ARG;
    if (mode != SVG_MODE_SPLIT && mode != SVG_MODE_NAIVE) return SVG_ERR_ARG;
    const TmLayout L = tm_layout(N, bq, bk);
    const void* ws[2] = {ws_sp, ws_tm};
    for (int h = 0; h < heads; ++h) {
      if (h_route[h] > 1) return SVG_ERR_ARG;
      if (h_route[h]) P.route_bits[h >> 5] |= 1u << (h & 31);
      P.uses[h_route[h]] = 1;
      ++P.hc[h_route[h]];
    }
    P.order = order;
    for (int c = 0; c < 2; ++c) {
      P.g[c] = make_geom(*geom, *mask, c);
      if (!P.uses[c]) continue;
      if (!ws[c] || !aligned(ws[c], 256)) return SVG_ERR_WORKSPACE;
      const uint8_t* b = static_cast<const uint8_t*>(ws[c]);
      P.hdr[c] = reinterpret_cast<const TmHeader*>(b);
      P.cls[c] = b + L.cls;
      P.pair_ptr[c] = reinterpret_cast<const uint32_t*>(b + L.pair_ptr);
      P.pair_ent[c] = reinterpret_cast<const uint32_t*>(b + L.pair_ent);
      P.pair_cnt[c] = reinterpret_cast<const uint32_t*>(b + L.pair_cnt);
      P.pair_order[c] = reinterpret_cast<const uint32_t*>(b + L.pair_order);
      P.pair_grp[c] = reinterpret_cast<const uint32_t*>(b + L.pair_grp);
    }
    P.variant = mask->variant;
    P.bq = bq;
    P.exp_T = geom->frames;
    P.exp_H = geom->grid_h;
    P.exp_W = geom->grid_w;
    P.exp_k = mask->frame_window;
    P.exp_b = mask->spatial_band;
    P.exp_F0 = mask->sink_frames;
    P.exp_variant = mask->variant;
    P.exp_layout = mask->layout;
    P.exp_bq = bq;
    P.exp_bk = bk;
  }
  // TMA boxes: Q 128 rows, K and V bk rows.
  if (qk8) {
    if ((rc = encode_qk8_map(&P.tm_q, q, heads, N, d, 128))) return rc;
    if ((rc = encode_qk8_map(&P.tm_k, k, heads, N, d, bk))) return rc;
  } else {
    if ((rc = encode_qkv_map(&P.tm_q, q, heads, N, d, 128))) return rc;
    if ((rc = encode_qkv_map(&P.tm_k, k, heads, N, d, bk))) return rc;
  }
  if ((rc = encode_qkv_map(&P.tm_v, v, heads, N, d, bk))) return rc;
  if (P.fused && P.uses[SVG_ROUTE_TEMPORAL]) {
    if ((rc = encode_rows_map(&P.tm_q2, q, heads, N, d))) return rc;
    if ((rc = encode_rows_map(&P.tm_k2, k, heads, N, d))) return rc;
    if ((rc = encode_rows_map(&P.tm_v2, v, heads, N, d))) return rc;
    // runs of one patch's frames as boxes: frames [F0, T) after the sink prefix, or all T frames
    // in the fully space-major order; runs shorter than 4 rows are gathered instead
    const bool fsm = mask->layout == SVG_LAYOUT_FULL_SPACE_MAJOR;
    const int run = fsm ? geom->frames : geom->frames - mask->sink_frames;
    P.run_div = make_fastdiv(run > 0 ? (uint32_t)run : 1u);
    P.runs = run > 0 ? (N - (fsm ? 0 : mask->sink_frames * geom->grid_h * geom->grid_w)) / run : 0;
    if (run >= 4 && run <= 256) {
      const int S = geom->grid_h * geom->grid_w;
      P.run_len = run;
      P.run_t0 = fsm ? 0 : mask->sink_frames;
      if ((rc = encode_run_map(&P.tm_q4, q, heads, geom->frames, S, d, run))) return rc;
      if ((rc = encode_run_map(&P.tm_k4, k, heads, geom->frames, S, d, run))) return rc;
      if ((rc = encode_run_map(&P.tm_v4, v, heads, geom->frames, S, d, run))) return rc;
    }
  }
  cudaError_t me = cudaMemsetAsync(scratch, 0, kScratchBytes, st);
  if (me == cudaSuccess && d_status) me = cudaMemsetAsync(d_status, 0, sizeof(int32_t), st);
  if (me == cudaSuccess && cta_trace) me = cudaMemsetAsync(cta_trace, 0, 32 * (size_t)trace_ctas, st);
  if (me != cudaSuccess) return record_cuda_error("cudaMemsetAsync(scratch)", me);
  const int grid = (int)(P.n_items < num_sms ? P.n_items : num_sms);
  return launch_attention(P, d, bk, grid, use_p_smem(), st);
}

}  // namespace


// ---------------------------------------------------------------------------------------
// Scratch of svg_attention_fwd_noalloc: a file-scope device array, so that callers that
// cannot allocate need not pass one. In host code `g_noalloc_scratch` only names the
// symbol; its device address comes from cudaGetSymbolAddress on every call, with the
// caller's device current.
static __device__ __align__(256) unsigned char g_noalloc_scratch[SVG_NOALLOC_SCRATCH_BYTES];

namespace {

void* noalloc_scratch(int* rc) {
  // looked up on every call (cheap, no device work), so that the address always belongs to the
  // context that is current now, also after a cudaDeviceReset
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
  if (e != cudaSuccess || !p) {
    *rc = record_cuda_error("cudaGetSymbolAddress", e);
    return nullptr;
  }
  return p;
}

}  // namespace

int svg::record_cuda_error(const char* what, int cuda_error) {
  const cudaError_t e = static_cast<cudaError_t>(cuda_error);
  snprintf(g_last_error, sizeof(g_last_error), "%s: %s (%d)", what, cudaGetErrorString(e), cuda_error);
  return SVG_ERR_CUDA;
}

extern "C" {

const char* svg_last_cuda_error(void) { return g_last_error; }

int svg_checked_build(void) { return SVG_CHECKED ? 1 : 0; }

int svg_checks_failed(uint32_t* h_count, int32_t reset) {
  if (!h_count) return SVG_ERR_ARG;
  *h_count = 0;
#if SVG_CHECKED
  cudaError_t e = cudaDeviceSynchronize();
  if (e == cudaSuccess) e = cudaMemcpyFromSymbol(h_count, g_checks_failed, sizeof(uint32_t));
  if (e == cudaSuccess && reset) {
    const uint32_t z = 0;
    e = cudaMemcpyToSymbol(g_checks_failed, &z, sizeof(uint32_t));
  }
  if (e != cudaSuccess) return record_cuda_error("svg_checks_failed", e);
#else
  (void)reset;
#endif
  return SVG_OK;
}

int svg_version(void) { return 10000; }

const char* svg_error_string(int code) {
  switch (code) {
    case SVG_OK: return "ok";
    case SVG_ERR_ARG: return "invalid argument (pointer, alignment, size, shape or parameter)";
    case SVG_ERR_UNSUPPORTED: return "unsupported: needs a compute capability 10.0 (sm_100a) device, d in {64,128}, "
                                     "bq in {64,128,256,512}, bk in {64,128}";
    case SVG_ERR_CUDA: return "a CUDA runtime or driver call failed";
    case SVG_ERR_TIMEOUT: return "a device pipeline wait exceeded its time limit; the kernel stopped early";
    case SVG_ERR_WORKSPACE: return "tile-map workspace missing, too small, misaligned or built for other parameters";
    default: return "unknown error code";
  }
}

size_t svg_tilemap_bytes(svg_geom geom, svg_tile tile) {
  if (!geom_ok(geom) || !tile_ok(tile)) return 0;
  return (size_t)tm_layout((int64_t)geom.frames * geom.grid_h * geom.grid_w, tile.bq, tile.bk).total;
}

int svg_tilemap_get_layout(svg_geom geom, svg_tile tile, svg_tilemap_layout* out) {
  if (!out || !geom_ok(geom)) return SVG_ERR_ARG;
  if (!tile_ok(tile)) return SVG_ERR_UNSUPPORTED;
  const TmLayout L = tm_layout((int64_t)geom.frames * geom.grid_h * geom.grid_w, tile.bq, tile.bk);
  out->total_bytes = L.total;
  out->cls = L.cls;
  out->cnt = L.cnt;
  out->row_ptr = L.row_ptr;
  out->cols = L.cols;
  out->pair_ptr = L.pair_ptr;
  out->pair_ent = L.pair_ent;
  out->pair_cnt = L.pair_cnt;
  out->pair_order = L.pair_order;
  out->pair_grp = L.pair_grp;
  out->nq = L.nq;
  out->nk = L.nk;
  out->npairs = L.npairs;
  return SVG_OK;
}

int svg_build_tilemap(svg_geom geom, svg_mask mask, svg_tile tile, int32_t route, void* d_ws, size_t ws_bytes,
                      void* stream) {
  if (!geom_ok(geom) || !mask_ok(geom, mask) || (route != SVG_ROUTE_SPATIAL && route != SVG_ROUTE_TEMPORAL))
    return SVG_ERR_ARG;
  if (!tile_ok(tile)) return SVG_ERR_UNSUPPORTED;
  if (!d_ws || !aligned(d_ws, 256)) return SVG_ERR_WORKSPACE;
  if (ws_bytes < svg_tilemap_bytes(geom, tile)) return SVG_ERR_WORKSPACE;
  int rc = device_info(nullptr);
  if (rc) return rc;
  return build_tilemap(geom, mask, tile, route, d_ws, static_cast<cudaStream_t>(stream));
}

int svg_tilemap_summary(const void* d_ws, svg_tilemap_summary_t* h_out, void* stream) {
  if (!d_ws || !h_out || !aligned(d_ws, 256)) return SVG_ERR_ARG;
  TmHeader h;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemcpyAsync(&h, d_ws, sizeof(h), cudaMemcpyDeviceToHost, st);
  if (e != cudaSuccess) return record_cuda_error("cudaMemcpyAsync(summary)", e);
  e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return record_cuda_error("cudaStreamSynchronize(summary)", e);
  if (h.magic != kTmMagic) return SVG_ERR_WORKSPACE;
  h_out->retained_exact = h.retained_exact;
  h_out->retained_map = h.retained_map;
  h_out->n_full = h.n_full;
  h_out->n_boundary = h.n_boundary;
  h_out->n_empty = h.n_empty;
  h_out->visited_area = h.visited_area;
  h_out->pair_entries = h.pair_entries;
  h_out->pair_half_tiles = h.pair_half_tiles;
  return SVG_OK;
}

int svg_permute(const void* d_in, void* d_out, int32_t heads, int64_t tokens, int32_t d, const uint8_t* h_route,
                svg_geom geom, svg_mask mask, int32_t inverse, void* stream) {
  if (!d_in || !d_out || !h_route || !aligned(d_in, 16) || !aligned(d_out, 16)) return SVG_ERR_ARG;
  if (heads < 1 || heads > kMaxHeads || !geom_ok(geom) || !mask_ok(geom, mask)) return SVG_ERR_ARG;
  if ((int64_t)geom.frames * geom.grid_h * geom.grid_w != tokens) return SVG_ERR_ARG;
  if (d != 64 && d != 128) return SVG_ERR_UNSUPPORTED;
  if (inverse != 0 && inverse != 1) return SVG_ERR_ARG;
  const uint8_t* a = static_cast<const uint8_t*>(d_in);
  const uint8_t* b = static_cast<const uint8_t*>(d_out);
  const size_t bytes = (size_t)heads * tokens * d * 2;
  if (a < b + bytes && b < a + bytes) return SVG_ERR_ARG;  // must not overlap
  for (int h = 0; h < heads; ++h)
    if (h_route[h] > 1) return SVG_ERR_ARG;
  int num_sms = 0;
  int rc = device_info(&num_sms);
  if (rc) return rc;
  return launch_permute(d_in, d_out, heads, tokens, d, h_route, geom, mask, inverse, num_sms,
                        static_cast<cudaStream_t>(stream));
}

size_t svg_attention_scratch_bytes(void) { return kScratchBytes; }

int svg_attention_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int32_t heads,
                      int64_t tokens, int32_t d, float scale, const uint8_t* h_route, const void* d_ws_spatial,
                      const void* d_ws_temporal, svg_geom geom, svg_mask mask, svg_tile tile, int32_t mode,
                      void* d_scratch, size_t scratch_bytes, int32_t* d_status, void* stream) {
  return run_attention(q, k, v, o, lse, heads, tokens, d, scale, h_route, d_ws_spatial, d_ws_temporal, &geom, &mask,
                       tile.bq, tile.bk, mode, false, d_scratch, scratch_bytes, d_status,
                       static_cast<cudaStream_t>(stream));
}

int svg_attention_fwd_fused(const void* q, const void* k, const void* v, void* o, float* lse, int32_t heads,
                            int64_t tokens, int32_t d, float scale, const uint8_t* h_route, const void* d_ws_spatial,
                            const void* d_ws_temporal, svg_geom geom, svg_mask mask, svg_tile tile, int32_t mode,
                            void* d_scratch, size_t scratch_bytes, int32_t* d_status, void* stream) {
  return run_attention(q, k, v, o, lse, heads, tokens, d, scale, h_route, d_ws_spatial, d_ws_temporal, &geom, &mask,
                       tile.bq, tile.bk, mode, false, d_scratch, scratch_bytes, d_status,
                       static_cast<cudaStream_t>(stream), true);
}

int svg_attention_fwd_ex(const void* q, const void* k, const void* v, void* o, float* lse, int32_t heads,
                         int64_t tokens, int32_t d, float scale, const uint8_t* h_route, const void* d_ws_spatial,
                         const void* d_ws_temporal, svg_geom geom, svg_mask mask, svg_tile tile, int32_t mode,
                         void* d_scratch, size_t scratch_bytes, int32_t* d_status, const svg_launch_opts* opts,
                         void* stream) {
  if (!opts) return SVG_ERR_ARG;
  return run_attention(q, k, v, o, lse, heads, tokens, d, scale, h_route, d_ws_spatial, d_ws_temporal, &geom, &mask,
                       tile.bq, tile.bk, mode, false, d_scratch, scratch_bytes, d_status,
                       static_cast<cudaStream_t>(stream), false, false, false, opts->order,
                       reinterpret_cast<unsigned long long*>(opts->d_cta_trace), opts->trace_ctas);
}

int svg_test_attention_fwd_stall(const void* q, const void* k, const void* v, void* o, float* lse, int32_t heads,
                                 int64_t tokens, int32_t d, float scale, const uint8_t* h_route,
                                 const void* d_ws_spatial, const void* d_ws_temporal, svg_geom geom, svg_mask mask,
                                 svg_tile tile, int32_t mode, void* d_scratch, size_t scratch_bytes,
                                 int32_t* d_status, void* stream) {
  return run_attention(q, k, v, o, lse, heads, tokens, d, scale, h_route, d_ws_spatial, d_ws_temporal, &geom, &mask,
                       tile.bq, tile.bk, mode, false, d_scratch, scratch_bytes, d_status,
                       static_cast<cudaStream_t>(stream), false, false, true);
}

int svg_attention_fwd_qk8(const void* q8, const void* k8, const void* v, void* o, float* lse, int32_t heads,
                          int64_t tokens, int32_t d, float scale, const uint8_t* h_route, const void* d_ws_spatial,
                          const void* d_ws_temporal, svg_geom geom, svg_mask mask, svg_tile tile, int32_t mode,
                          void* d_scratch, size_t scratch_bytes, int32_t* d_status, void* stream) {
  return run_attention(q8, k8, v, o, lse, heads, tokens, d, scale, h_route, d_ws_spatial, d_ws_temporal, &geom, &mask,
                       tile.bq, tile.bk, mode, false, d_scratch, scratch_bytes, d_status,
                       static_cast<cudaStream_t>(stream), false, true);
}

int svg_dense_attention_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int32_t heads,
                            int64_t tokens, int32_t d, float scale, int32_t bk, void* d_scratch, size_t scratch_bytes,
                            int32_t* d_status, void* stream) {
  return run_attention(q, k, v, o, lse, heads, tokens, d, scale, nullptr, nullptr, nullptr, nullptr, nullptr, 0, bk,
                       SVG_MODE_SPLIT, true, d_scratch, scratch_bytes, d_status, static_cast<cudaStream_t>(stream));
}

int svg_attention_fwd_noalloc(const void* q, const void* k, const void* v, void* o, float* lse, int32_t heads,
                              int64_t tokens, int32_t d, float scale, const uint8_t* h_route,
                              const void* d_ws_spatial, const void* d_ws_temporal, svg_geom geom, svg_mask mask,
                              svg_tile tile, int32_t mode, int32_t* d_status, void* stream) {
  if (svg_attention_scratch_bytes() > SVG_NOALLOC_SCRATCH_BYTES) return SVG_ERR_ARG;
  int rc = check_qkvo(q, k, v, o, lse, heads, tokens, d);  // reject bad arguments before any CUDA call
  if (rc) return rc;
  void* scratch = noalloc_scratch(&rc);
  if (!scratch) return rc;
  return run_attention(q, k, v, o, lse, heads, tokens, d, scale, h_route, d_ws_spatial, d_ws_temporal, &geom, &mask,
                       tile.bq, tile.bk, mode, false, scratch, SVG_NOALLOC_SCRATCH_BYTES, d_status,
                       static_cast<cudaStream_t>(stream));
}

size_t svg_route_work_bytes(int32_t heads, int64_t tokens, int32_t d, int32_t n_rows) {
  if (heads < 1 || n_rows < 1 || tokens < 1 || tokens > INT32_MAX || (d != 64 && d != 128)) return 0;
  return route_work_bytes(heads, tokens, d, n_rows);
}

int svg_route_heads(const void* q, const void* k, const void* v, int32_t heads, int64_t tokens, int32_t d, float scale,
                    svg_geom geom, svg_mask mask, const int32_t* d_rows, int32_t n_rows, void* d_work,
                    size_t work_bytes, uint8_t* d_route, float* d_err, void* stream) {
  if (!q || !k || !v || !d_rows || !d_work || !d_route) return SVG_ERR_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(d_rows, 4) || !aligned(d_work, 256) ||
      (d_err && !aligned(d_err, 4)))
    return SVG_ERR_ARG;
  if (heads < 1 || heads > 65535 || n_rows < 1 || !geom_ok(geom) || !mask_ok(geom, mask)) return SVG_ERR_ARG;
  if ((int64_t)geom.frames * geom.grid_h * geom.grid_w != tokens) return SVG_ERR_ARG;
  if (d != 64 && d != 128) return SVG_ERR_UNSUPPORTED;
  if (work_bytes < svg_route_work_bytes(heads, tokens, d, n_rows)) return SVG_ERR_WORKSPACE;
  int num_sms = 0;
  int rc = device_info(&num_sms);
  if (rc) return rc;
  const float sc = scale > 0.f ? scale : 1.0f / sqrtf((float)d);
  CUtensorMap tmk, tmv;  // K / V tiles of 64 keys for the tensor-core kernel
  if ((rc = encode_qkv_map(&tmk, k, heads, (int)tokens, d, 64))) return rc;
  if ((rc = encode_qkv_map(&tmv, v, heads, (int)tokens, d, 64))) return rc;
  return launch_route(q, &tmk, &tmv, heads, (int)tokens, d, sc, geom, mask, d_rows, n_rows, d_work, d_route, d_err,
                      num_sms, static_cast<cudaStream_t>(stream));
}

// ---------------------------------------------------------------------------------------
// Host-buffer entry point: chunks of heads flow through three library streams (copies in,
// compute, copies out) and three device slots, so the copies of one chunk overlap the
// permutation and attention of the neighbouring chunks. With two slots the copy in of chunk
// c + 2 had to wait for the copy out of chunk c, i.e. for its attention: the copy-in stream,
// the bound of the whole call, stalled every chunk; a third slot lets it run ahead.
namespace {

constexpr int kHostSlots = 3;

struct HostPipe {
  cudaStream_t in, comp, out;
  cudaEvent_t h2d[kHostSlots], done[kHostSlots], d2h[kHostSlots];
  std::mutex call;  // one host-buffer call per device at a time: the streams and events are shared
};

HostPipe* host_pipe(int* rc) {
  static std::mutex mu;
  static HostPipe* pipes[kMaxDevices] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    *rc = SVG_ERR_CUDA;
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(mu);
  if (!pipes[dev]) {
    HostPipe* hp = new HostPipe();
    cudaError_t e = cudaStreamCreateWithFlags(&hp->in, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&hp->comp, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&hp->out, cudaStreamNonBlocking);
    for (int i = 0; i < kHostSlots && e == cudaSuccess; ++i) {
      e = cudaEventCreateWithFlags(&hp->h2d[i], cudaEventDisableTiming);
      if (e == cudaSuccess) e = cudaEventCreateWithFlags(&hp->done[i], cudaEventDisableTiming);
      if (e == cudaSuccess) e = cudaEventCreateWithFlags(&hp->d2h[i], cudaEventDisableTiming);
    }
    if (e != cudaSuccess) {  // the partly built pipe is kept out of use (and leaked) on this path
      *rc = record_cuda_error("host pipe streams / events", e);
      return nullptr;
    }
    pipes[dev] = hp;
  }
  return pipes[dev];
}

size_t chunk_tensor_bytes(int64_t tokens, int d, int chunk_heads) {
  return ((size_t)chunk_heads * tokens * d * 2 + 255) / 256 * 256;
}

// Keeps the first nonzero status of the chunks' attention launches (each launch clears its own).
__global__ void keep_status(const int* launch_status, int* call_status) {
  const int v = *launch_status;
  if (v != 0 && *call_status == 0) *call_status = v;
}

}  // namespace

size_t svg_attention_host_buffer_bytes(int64_t tokens, int32_t d, int32_t chunk_heads) {
  if (tokens < 1 || tokens > kMaxTokens || (d != 64 && d != 128) || chunk_heads < 1 || chunk_heads > kMaxHeads)
    return 0;
  return kHostSlots * 7 * chunk_tensor_bytes(tokens, d, chunk_heads) + kScratchBytes + 256;
}

int svg_attention_fwd_host(const void* h_q, const void* h_k, const void* h_v, void* h_o, int32_t heads,
                           int64_t tokens, int32_t d, float scale, const uint8_t* h_route,
                           const void* d_ws_spatial, const void* d_ws_temporal, svg_geom geom, svg_mask mask,
                           svg_tile tile, int32_t mode, int32_t chunk_heads, void* d_buf, size_t buf_bytes) {
  if (!h_q || !h_k || !h_v || !h_o || !h_route || !d_buf || !aligned(d_buf, 256)) return SVG_ERR_ARG;
  if (heads < 1 || heads > kMaxHeads || chunk_heads < 1) return SVG_ERR_ARG;
  if (!geom_ok(geom) || !mask_ok(geom, mask)) return SVG_ERR_ARG;
  if ((int64_t)geom.frames * geom.grid_h * geom.grid_w != tokens) return SVG_ERR_ARG;
  if (d != 64 && d != 128) return SVG_ERR_UNSUPPORTED;
  if (!tile_ok(tile)) return SVG_ERR_UNSUPPORTED;
  if (mode != SVG_MODE_SPLIT && mode != SVG_MODE_NAIVE) return SVG_ERR_ARG;
  for (int h = 0; h < heads; ++h)
    if (h_route[h] > 1) return SVG_ERR_ARG;
  const int ch = chunk_heads < heads ? chunk_heads : heads;
  if (buf_bytes < svg_attention_host_buffer_bytes(tokens, d, ch)) return SVG_ERR_WORKSPACE;
  int num_sms = 0;
  int rc = device_info(&num_sms);
  if (rc) return rc;
  HostPipe* hp = host_pipe(&rc);
  if (!hp) return rc;
  std::lock_guard<std::mutex> lock(hp->call);

  const size_t ta = chunk_tensor_bytes(tokens, d, ch);
  uint8_t* buf = static_cast<uint8_t*>(d_buf);
  void* scratch = buf + kHostSlots * 7 * ta;
  int* call_status = reinterpret_cast<int*>(buf + kHostSlots * 7 * ta + kScratchBytes);
  const size_t head_bytes = (size_t)tokens * d * 2;
  const int nchunks = (heads + ch - 1) / ch;
  cudaError_t e = cudaSuccess;
  const char* what = "";
#define SVG_HOST_TRY(call, name) \
  do {                           \
    e = (call);                  \
    if (e != cudaSuccess) {      \
      what = name;               \
      goto fail;                 \
    }                            \
  } while (0)
  SVG_HOST_TRY(cudaMemsetAsync(call_status, 0, sizeof(int), hp->comp), "cudaMemsetAsync(status)");
  for (int c = 0; c < nchunks; ++c) {
    const int h0 = c * ch, hn = (heads - h0) < ch ? (heads - h0) : ch;
    const size_t off = (size_t)h0 * head_bytes, bytes = (size_t)hn * head_bytes;
    const int s = c % kHostSlots;
    uint8_t* base = buf + (size_t)s * 7 * ta;
    uint8_t *qo = base, *ko = base + ta, *vo = base + 2 * ta;
    uint8_t *qp = base + 3 * ta, *kp = base + 4 * ta, *vp = base + 5 * ta, *op = base + 6 * ta;
    const uint8_t* routes = h_route + h0;
    bool perm = false;
    for (int h = 0; h < hn; ++h) perm |= routes[h] != 0;
    // copies in: the slot's previous chunk must have left the device (its copy out read qo or op)
    if (c >= kHostSlots) SVG_HOST_TRY(cudaStreamWaitEvent(hp->in, hp->d2h[s], 0), "cudaStreamWaitEvent(in)");
    SVG_HOST_TRY(cudaMemcpyAsync(qo, static_cast<const uint8_t*>(h_q) + off, bytes, cudaMemcpyHostToDevice, hp->in),
                 "cudaMemcpyAsync(q in)");
    SVG_HOST_TRY(cudaMemcpyAsync(ko, static_cast<const uint8_t*>(h_k) + off, bytes, cudaMemcpyHostToDevice, hp->in),
                 "cudaMemcpyAsync(k in)");
    SVG_HOST_TRY(cudaMemcpyAsync(vo, static_cast<const uint8_t*>(h_v) + off, bytes, cudaMemcpyHostToDevice, hp->in),
                 "cudaMemcpyAsync(v in)");
    SVG_HOST_TRY(cudaEventRecord(hp->h2d[s], hp->in), "cudaEventRecord(h2d)");
    // compute: temporal heads to their order, attention, O back to the original order
    SVG_HOST_TRY(cudaStreamWaitEvent(hp->comp, hp->h2d[s], 0), "cudaStreamWaitEvent(comp)");
    if (perm) {
      if ((rc = launch_permute(qo, qp, hn, tokens, d, routes, geom, mask, 0, num_sms, hp->comp)) ||
          (rc = launch_permute(ko, kp, hn, tokens, d, routes, geom, mask, 0, num_sms, hp->comp)) ||
          (rc = launch_permute(vo, vp, hn, tokens, d, routes, geom, mask, 0, num_sms, hp->comp)))
        goto fail_rc;
      rc = run_attention(qp, kp, vp, op, nullptr, hn, tokens, d, scale, routes, d_ws_spatial, d_ws_temporal, &geom,
                         &mask, tile.bq, tile.bk, mode, false, scratch, kScratchBytes, nullptr, hp->comp);
      if (rc) goto fail_rc;
      if ((rc = launch_permute(op, qo, hn, tokens, d, routes, geom, mask, 1, num_sms, hp->comp))) goto fail_rc;
    } else {
      rc = run_attention(qo, ko, vo, op, nullptr, hn, tokens, d, scale, routes, d_ws_spatial, d_ws_temporal, &geom,
                         &mask, tile.bq, tile.bk, mode, false, scratch, kScratchBytes, nullptr, hp->comp);
      if (rc) goto fail_rc;
    }
    keep_status<<<1, 1, 0, hp->comp>>>(static_cast<const int*>(scratch), call_status);
    SVG_HOST_TRY(cudaGetLastError(), "launch keep_status");
    SVG_HOST_TRY(cudaEventRecord(hp->done[s], hp->comp), "cudaEventRecord(done)");
    // copy out
    SVG_HOST_TRY(cudaStreamWaitEvent(hp->out, hp->done[s], 0), "cudaStreamWaitEvent(out)");
    SVG_HOST_TRY(cudaMemcpyAsync(static_cast<uint8_t*>(h_o) + off, perm ? qo : op, bytes, cudaMemcpyDeviceToHost,
                                 hp->out),
                 "cudaMemcpyAsync(o out)");
    SVG_HOST_TRY(cudaEventRecord(hp->d2h[s], hp->out), "cudaEventRecord(d2h)");
  }
#undef SVG_HOST_TRY
  {
    e = cudaStreamSynchronize(hp->out);
    if (e == cudaSuccess) e = cudaStreamSynchronize(hp->comp);
    if (e == cudaSuccess) e = cudaStreamSynchronize(hp->in);
    if (e != cudaSuccess) return record_cuda_error("cudaStreamSynchronize(host pipe)", e);
    int32_t st = 0;
    e = cudaMemcpy(&st, call_status, sizeof(st), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return record_cuda_error("cudaMemcpy(status)", e);
    return st;
  }
fail:
  rc = record_cuda_error(what, e);
fail_rc:
  // let whatever was queued finish before the caller may free or reuse its buffers
  cudaStreamSynchronize(hp->out);
  cudaStreamSynchronize(hp->comp);
  cudaStreamSynchronize(hp->in);
  return rc;
}

int svg_read_status(const void* d_scratch_or_status, int32_t* h_status, void* stream) {
  if (!d_scratch_or_status || !h_status || !aligned(d_scratch_or_status, 4)) return SVG_ERR_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemcpyAsync(h_status, d_scratch_or_status, sizeof(int32_t), cudaMemcpyDeviceToHost, st);
  if (e != cudaSuccess) return record_cuda_error("cudaMemcpyAsync(status)", e);
  e = cudaStreamSynchronize(st);
  return e == cudaSuccess ? SVG_OK : record_cuda_error("cudaStreamSynchronize(status)", e);
}

}  // extern "C"
