// svg_tilemap.cu -- tile classification and execution lists for one route class.
//
// "Efficient Kernel Implementation" (tile-aware masking) of the case study classifies tiles
// as full (only retained pairs) or boundary (both kinds) so that full tiles run without the
// mask; empty tiles are never visited. The tile-aligned variant (summary; "What changed")
// rounds the mask to whole tiles. Here every (q-tile, k-tile) pair is counted exactly from
// the per-row kept-key intervals (svg_common.cuh), which is O(1) per row instead of per
// element, then compacted into:
//   * a CSR list of visited k-tiles per q-tile (the data structure the traversal walks);
//   * per 256-row item (two 128-row halves, the attention kernel's unit of work) an entry
//     list with one flag per half: skip / full / masked / full-but-ragged;
//   * the items in descending order of work for the persistent scheduler, with the bounds of each
//     run of equal work.
#include "svg_common.cuh"

namespace svg {

unsigned int* checks_counter();

// Execution lists of groups of G 128-row blocks (pairs: G = 2, the attention kernel's items).
struct GroupLists {
  uint32_t* ptr;    // [ngroups + 1]
  uint32_t* ent;    // [ngroups * nk]
  uint32_t* cnt;    // [2 * ngroups]: entries in which MMA phase h (block index % 2) is active
  uint32_t* order;  // [ngroups] by descending work
  int ngroups;
  unsigned long long* tot_entries;
  unsigned long long* tot_phase_tiles;
};

struct TmParams {
  MaskGeom g;
  int bq, bk, nq, nk, npairs, variant;
  uint8_t* cls;
  uint32_t* cnt;
  uint32_t* row_ptr;
  uint32_t* cols;
  GroupLists pairs;
  TmHeader* hdr;
  unsigned int* checks;  // failed-check counter of the checked build
};

__device__ __forceinline__ unsigned long long block_sum_u64(unsigned long long v, unsigned long long* red) {
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31, nw = blockDim.x >> 5;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  unsigned long long s = 0;
  if (threadIdx.x == 0)
    for (int i = 0; i < nw; ++i) s += red[i];
  return s;  // valid in thread 0 only
}

// One block per q-tile: rows' kept intervals into shared memory, then every k-tile.
__global__ void __launch_bounds__(256) tm_classify(TmParams P, svg_geom geom, svg_mask mask, svg_tile tile,
                                                   int route) {
  __shared__ int lo_s[512], hi_s[512];
  __shared__ unsigned long long red[8];
  const int qt = blockIdx.x;
  const MaskGeom& g = P.g;
  const int r0 = qt * P.bq, r1 = min(g.N, r0 + P.bq), nrows = r1 - r0;
  for (int r = threadIdx.x; r < nrows; r += blockDim.x) {
    int lo, hi;
    row_interval(g, r0 + r, lo, hi);
    lo_s[r] = lo;
    hi_s[r] = hi;
  }
  if (qt == 0 && threadIdx.x == 0) {
    TmHeader* h = P.hdr;
    h->magic = kTmMagic;
    h->version = 1;
    h->T = geom.frames; h->H = geom.grid_h; h->W = geom.grid_w; h->route = route;
    h->k = mask.frame_window; h->b = mask.spatial_band; h->F0 = mask.sink_frames;
    h->variant = mask.variant; h->layout = mask.layout; h->bq = tile.bq; h->bk = tile.bk;
    h->nq = P.nq; h->nk = P.nk; h->npairs = P.npairs; h->N = g.N;
  }
  __syncthreads();
  unsigned long long kept_tot = 0, map_tot = 0, nfull = 0, nbnd = 0, nemp = 0, varea = 0;
  uint32_t visited = 0;
  for (int kt = threadIdx.x; kt < P.nk; kt += blockDim.x) {
    const int c0 = kt * P.bk, c1 = min(g.N, c0 + P.bk);
    uint32_t kept = 0;
    for (int r = 0; r < nrows; ++r) kept += (uint32_t)row_kept_in(g, lo_s[r], hi_s[r], c0, c1);
    const uint32_t area = (uint32_t)nrows * (uint32_t)(c1 - c0);
    uint8_t c;
    if (P.variant == SVG_MASK_ROUNDED) {
      c = (2ull * kept >= area) ? 1 : 0;
      map_tot += c ? area : 0;
    } else {
      c = kept == 0 ? 0 : (kept == area ? 1 : 2);
      map_tot += kept;
    }
    const size_t idx = (size_t)qt * P.nk + kt;
    P.cls[idx] = c;
    P.cnt[idx] = kept;
    kept_tot += kept;
    nfull += c == 1;
    nbnd += c == 2;
    nemp += c == 0;
    if (c) {
      varea += area;
      ++visited;
    }
  }
  // per-q-tile visited count (row_ptr is scanned in place later)
  unsigned long long s;
  s = block_sum_u64(visited, red);
  if (threadIdx.x == 0) P.row_ptr[qt] = (uint32_t)s;
  s = block_sum_u64(kept_tot, red);
  if (threadIdx.x == 0) atomicAdd(&P.hdr->retained_exact, s);
  s = block_sum_u64(map_tot, red);
  if (threadIdx.x == 0) atomicAdd(&P.hdr->retained_map, s);
  s = block_sum_u64(nfull, red);
  if (threadIdx.x == 0) atomicAdd(&P.hdr->n_full, s);
  s = block_sum_u64(nbnd, red);
  if (threadIdx.x == 0) atomicAdd(&P.hdr->n_boundary, s);
  s = block_sum_u64(nemp, red);
  if (threadIdx.x == 0) atomicAdd(&P.hdr->n_empty, s);
  s = block_sum_u64(varea, red);
  if (threadIdx.x == 0) atomicAdd(&P.hdr->visited_area, s);
}

// Flag of the 128-row block starting at row r0 for k-tile kt, combining the classes of the
// q-tiles it overlaps.
__device__ __forceinline__ uint32_t block_flag(const TmParams& P, int r0, int kt) {
  if (r0 >= P.g.N) return kFlagSkip;
  const int r1 = min(P.g.N, r0 + kHalfRows);
  const int qa = r0 / P.bq, qb = (r1 - 1) / P.bq;
  bool any = false, all_full = true;
  for (int qt = qa; qt <= qb; ++qt) {
    const uint8_t c = P.cls[(size_t)qt * P.nk + kt];
    any |= c != 0;
    all_full &= c == 1;
  }
  if (!any) return kFlagSkip;
  if (!all_full) return kFlagMasked;
  const bool ragged = (kt == P.nk - 1) && (P.g.N % P.bk != 0);
  return ragged ? kFlagBounds : kFlagFull;
}

// Entry of group g for k-tile kt (0xFFFFFFFF when no block of the group visits the tile).
template <int G>
__device__ __forceinline__ uint32_t group_entry(const TmParams& P, int g, int kt, uint32_t* phase_bits) {
  uint32_t e = (uint32_t)kt, ph = 0;
#pragma unroll
  for (int i = 0; i < G; ++i) {
    const uint32_t f = block_flag(P, g * G * kHalfRows + i * kHalfRows, kt);
    e |= f << (32 - 2 * G + 2 * i);
    if (f) ph |= 1u << (i & 1);
  }
  *phase_bits = ph;
  return ph ? e : 0xFFFFFFFFu;
}

// One block per group: number of entries and, per MMA phase, entries where it is active.
template <int G>
__global__ void __launch_bounds__(256) tm_group_count(TmParams P, GroupLists L) {
  __shared__ unsigned long long red[8];
  const int g = blockIdx.x;
  uint32_t ne = 0, n0 = 0, n1 = 0;
  for (int kt = threadIdx.x; kt < P.nk; kt += blockDim.x) {
    uint32_t ph;
    const uint32_t e = group_entry<G>(P, g, kt, &ph);
    ne += e != 0xFFFFFFFFu;
    n0 += ph & 1u;
    n1 += (ph >> 1) & 1u;
  }
  unsigned long long s;
  s = block_sum_u64(ne, red);
  if (threadIdx.x == 0) {
    L.ptr[g] = (uint32_t)s;
    atomicAdd(L.tot_entries, s);
  }
  s = block_sum_u64(n0, red);
  if (threadIdx.x == 0) L.cnt[2 * g] = (uint32_t)s;
  const unsigned long long s0 = s;
  s = block_sum_u64(n1, red);
  if (threadIdx.x == 0) {
    L.cnt[2 * g + 1] = (uint32_t)s;
    atomicAdd(L.tot_phase_tiles, s0 + s);
  }
}

// In-place exclusive scan of counts[0..n) into offsets[0..n] (offsets[n] = total); one block.
__device__ void block_exclusive_scan(uint32_t* a, int n) {
  __shared__ uint32_t part[1024];
  const int t = threadIdx.x, nt = blockDim.x;
  const int per = (n + nt - 1) / nt;
  const int b0 = min(n, t * per), b1 = min(n, b0 + per);
  uint32_t s = 0;
  for (int i = b0; i < b1; ++i) s += a[i];
  part[t] = s;
  __syncthreads();
  if (t == 0) {
    uint32_t run = 0;
    for (int i = 0; i < nt; ++i) {
      const uint32_t v = part[i];
      part[i] = run;
      run += v;
    }
    a[n] = run;  // written before anyone else reads a[n]; a[n] is outside every range
  }
  __syncthreads();
  uint32_t run = part[t];
  for (int i = b0; i < b1; ++i) {
    const uint32_t v = a[i];
    a[i] = run;
    run += v;
  }
}

__global__ void __launch_bounds__(1024) tm_scan(TmParams P) {
  block_exclusive_scan(P.row_ptr, P.nq);
  __syncthreads();
  block_exclusive_scan(P.pairs.ptr, P.pairs.ngroups);
}

// Ordered compaction of one row of flags, 256 threads, chunk by chunk, into out[0, cap).
template <typename F>
__device__ void compact_row(int n, uint32_t* out, uint64_t cap, unsigned int* checks, F&& value_of) {
  __shared__ uint32_t wsum[8];
  __shared__ uint32_t base;
  if (threadIdx.x == 0) base = 0;
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  for (int c0 = 0; c0 < n; c0 += blockDim.x) {
    const int i = c0 + threadIdx.x;
    uint32_t v = 0;
    const bool keep = i < n && (v = value_of(i)) != 0xFFFFFFFFu;
    const uint32_t bal = __ballot_sync(0xffffffffu, keep);
    __syncthreads();
    if (l == 0) wsum[w] = __popc(bal);
    __syncthreads();
    uint32_t off = base;
    for (int j = 0; j < w; ++j) off += wsum[j];
    if (keep) {
      const uint32_t at = off + __popc(bal & ((1u << l) - 1));
      if (check_ok(at < cap, checks)) out[at] = v;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      uint32_t tot = 0;
      for (int j = 0; j < (int)(blockDim.x >> 5); ++j) tot += wsum[j];
      base += tot;
    }
  }
}

__global__ void __launch_bounds__(256) tm_fill_cols(TmParams P) {
  const int qt = blockIdx.x;
  const uint8_t* row = P.cls + (size_t)qt * P.nk;
  const uint32_t b0 = P.row_ptr[qt];
  const uint64_t tiles = (uint64_t)P.nq * P.nk;
  compact_row(P.nk, P.cols + b0, check_ok(b0 <= tiles, P.checks) ? tiles - b0 : 0, P.checks, [&](int kt) -> uint32_t {
    const uint8_t c = row[kt];
    return c ? ((uint32_t)kt | ((uint32_t)c << 30)) : 0xFFFFFFFFu;
  });
}

template <int G>
__global__ void __launch_bounds__(256) tm_fill_groups(TmParams P, GroupLists L) {
  const int g = blockIdx.x;
  const uint32_t b0 = L.ptr[g];
  const uint64_t cap = (uint64_t)L.ngroups * P.nk;
  compact_row(P.nk, L.ent + b0, check_ok(b0 <= cap, P.checks) ? cap - b0 : 0, P.checks, [&](int kt) -> uint32_t {
    uint32_t ph;
    return group_entry<G>(P, g, kt, &ph);
  });
}

// Rank of each group by (work descending, index ascending); work = active (entry, phase)s.
__global__ void tm_sort_groups(GroupLists L) {
  const int p = blockIdx.x * blockDim.x + threadIdx.x;
  if (p >= L.ngroups) return;
  const uint32_t wp = L.cnt[2 * p] + L.cnt[2 * p + 1];
  uint32_t rank = 0;
  for (int q = 0; q < L.ngroups; ++q) {
    const uint32_t wq = L.cnt[2 * q] + L.cnt[2 * q + 1];
    rank += (wq > wp) || (wq == wp && q < p);
  }
  if (rank < (uint32_t)L.ngroups) L.order[rank] = (uint32_t)p;
}

// For each position p of the pair order (descending work, ties by index), the bounds [start, end) of
// the run of positions with the same work as p. The work-ordered scheduler of the attention kernel
// hands out one run at a time for every head of a route class, head by head, so that the items in
// flight at a time share each head's K / V rows.
__global__ void tm_work_runs(GroupLists L, uint32_t* grp) {
  const int p = blockIdx.x * blockDim.x + threadIdx.x;
  if (p >= L.ngroups) return;
  auto work = [&](int i) -> uint32_t {
    const uint32_t g = L.order[i];
    return L.cnt[2 * g] + L.cnt[2 * g + 1];
  };
  const uint32_t w = work(p);
  int lo = 0, hi = p;  // first position of the run: work is non-increasing along the order
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (work(mid) > w) lo = mid + 1; else hi = mid;
  }
  grp[2 * p] = (uint32_t)lo;
  lo = p + 1;
  hi = L.ngroups;  // first position after the run
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (work(mid) < w) hi = mid; else lo = mid + 1;
  }
  grp[2 * p + 1] = (uint32_t)lo;
}

int build_tilemap(svg_geom geom, svg_mask mask, svg_tile tile, int route, void* ws, cudaStream_t st) {
  const MaskGeom g = make_geom(geom, mask, route);
  const TmLayout L = tm_layout(g.N, tile.bq, tile.bk);
  uint8_t* base = static_cast<uint8_t*>(ws);
  auto u32 = [&](uint64_t off) { return reinterpret_cast<uint32_t*>(base + off); };
  TmParams P;
  P.g = g;
  P.bq = tile.bq;
  P.bk = tile.bk;
  P.nq = L.nq;
  P.nk = L.nk;
  P.npairs = L.npairs;
  P.variant = mask.variant;
  P.hdr = reinterpret_cast<TmHeader*>(base);
  P.checks = checks_counter();
  P.cls = base + L.cls;
  P.cnt = u32(L.cnt);
  P.row_ptr = u32(L.row_ptr);
  P.cols = u32(L.cols);
  P.pairs = GroupLists{u32(L.pair_ptr), u32(L.pair_ent), u32(L.pair_cnt), u32(L.pair_order), L.npairs,
                       &P.hdr->pair_entries, &P.hdr->pair_half_tiles};
  cudaError_t e = cudaMemsetAsync(base, 0, 256, st);
  if (e != cudaSuccess) return record_cuda_error("cudaMemsetAsync(tile-map header)", e);
  tm_classify<<<L.nq, 256, 0, st>>>(P, geom, mask, tile, route);
  tm_group_count<2><<<L.npairs, 256, 0, st>>>(P, P.pairs);
  tm_scan<<<1, 1024, 0, st>>>(P);
  tm_fill_cols<<<L.nq, 256, 0, st>>>(P);
  tm_fill_groups<2><<<L.npairs, 256, 0, st>>>(P, P.pairs);
  tm_sort_groups<<<(L.npairs + 127) / 128, 128, 0, st>>>(P.pairs);
  tm_work_runs<<<(L.npairs + 127) / 128, 128, 0, st>>>(P.pairs, u32(L.pair_grp));
  e = cudaGetLastError();
  return e == cudaSuccess ? SVG_OK : record_cuda_error("launch tile-map kernels", e);
}

}  // namespace svg
