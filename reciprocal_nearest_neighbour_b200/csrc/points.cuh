// Exact Euclidean nearest neighbours among 3-D points.
//
// MASt3R implements the NN function of fast reciprocal matching according to
// the dimension of its input, and for 3-D points with K-d trees (MASt3R paper
// text quoted in the staskaer.github.io DUSt3R/MASt3R blog, MASt3R matching
// section; the quoted fast_reciprocal_NNs builds a KDTree per point map when
// it does not run on CUDA).  A K-d tree query returns the point at the
// smallest Euclidean distance; this file computes the same result on the GPU
// with a uniform grid instead of a tree: a counting sort of the points by
// cell, then, per query, a search over Chebyshev shells of cells around the
// query's cell that stops once no unsearched cell can hold a point as close
// as the best one found.  Distances are squared distances in fp32; ties go
// to the lowest index.
//
// Several point sets are handled by one launch sequence: two families
// (image 1 and image 2) of nb sets each, set (f, b) at base[f] + b*bstride[f].
// Their cells and sorted points live in shared arrays, set after set, so one
// global prefix sum orders them all.
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

namespace rnn {

constexpr int kPtsThreads = 256;
constexpr int kPtsChunk = 4096;          // points per block in the bounds and count passes
constexpr int kScanThreads = 1024;
constexpr int kScanPer = 8;              // cells per thread in the prefix-sum passes
constexpr int kScanSeg = kScanThreads * kScanPer;

struct PtsSets {
  const float* base[2];  // family f: [nb][n[f]][3] floats, set b at base[f] + b*bstride[f]
  int64_t bstride[2];
  int n[2];              // points per set (>= 1)
  int cap[2];            // grid cells per set (upper bound)
  int blk[2];            // blocks of kPtsChunk points per set
  int nb;                // sets per family
  int nfam;              // 1 or 2
};

// Grid of one set, chosen on the device from its bounding box.
struct PtsGrid {
  float lo[3], hi[3];    // bounding box of the set's points
  float h, inv_h;        // cell edge and its reciprocal
  float margin;          // allowance for rounding in cell assignment and faces
  int dim[3];
  int64_t cell0;         // first cell of this set in the shared arrays
};

__host__ __device__ __forceinline__ int pts_nsets(const PtsSets& ps) { return ps.nfam * ps.nb; }
__host__ __device__ __forceinline__ int64_t pts_cell0(const PtsSets& ps, int s) {
  return s < ps.nb ? static_cast<int64_t>(s) * ps.cap[0]
                   : static_cast<int64_t>(ps.nb) * ps.cap[0] +
                         static_cast<int64_t>(s - ps.nb) * ps.cap[1];
}
__host__ __device__ __forceinline__ int64_t pts_pt0(const PtsSets& ps, int s) {
  return s < ps.nb ? static_cast<int64_t>(s) * ps.n[0]
                   : static_cast<int64_t>(ps.nb) * ps.n[0] +
                         static_cast<int64_t>(s - ps.nb) * ps.n[1];
}
__host__ __device__ __forceinline__ int pts_blk0(const PtsSets& ps, int s) {
  return s < ps.nb ? s * ps.blk[0] : ps.nb * ps.blk[0] + (s - ps.nb) * ps.blk[1];
}
__host__ __device__ __forceinline__ const float* pts_set_base(const PtsSets& ps, int s) {
  return s < ps.nb ? ps.base[0] + static_cast<int64_t>(s) * ps.bstride[0]
                   : ps.base[1] + static_cast<int64_t>(s - ps.nb) * ps.bstride[1];
}
__host__ __device__ __forceinline__ int pts_set_n(const PtsSets& ps, int s) {
  return s < ps.nb ? ps.n[0] : ps.n[1];
}

// Block j of the bounds and count passes -> (set, chunk).
__device__ __forceinline__ void pts_block(const PtsSets& ps, int j, int* s, int* c) {
  const int f0 = ps.nb * ps.blk[0];
  if (j < f0) {
    *s = j / ps.blk[0];
    *c = j - *s * ps.blk[0];
  } else {
    const int r = j - f0;
    *s = ps.nb + r / ps.blk[1];
    *c = r - (r / ps.blk[1]) * ps.blk[1];
  }
}

// Cell of coordinate x along axis a, clamped into the grid (NaN -> 0).
__device__ __forceinline__ int pts_axis_cell(const PtsGrid& g, int a, float x) {
  const float t = fminf(fmaxf(floorf((x - g.lo[a]) * g.inv_h), 0.f), 1073741824.f);
  return min(static_cast<int>(t), g.dim[a] - 1);
}

// Block-wide min (which = 0) or max (which = 1) of one float per thread.
__device__ __forceinline__ float pts_block_reduce(float v, bool is_max, float* sm) {
  for (int o = 16; o > 0; o >>= 1) {
    const float y = __shfl_xor_sync(0xffffffffu, v, o);
    v = is_max ? fmaxf(v, y) : fminf(v, y);
  }
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  __syncthreads();
  if (lane == 0) sm[warp] = v;
  __syncthreads();
  if (warp == 0) {
    v = lane < static_cast<int>(blockDim.x >> 5) ? sm[lane] : (is_max ? -INFINITY : INFINITY);
    for (int o = 16; o > 0; o >>= 1) {
      const float y = __shfl_xor_sync(0xffffffffu, v, o);
      v = is_max ? fmaxf(v, y) : fminf(v, y);
    }
    if (lane == 0) sm[32] = v;
  }
  __syncthreads();
  return sm[32];
}

// Pass 1: bounding box of each block's points (part[j][6] = min xyz, max
// xyz), and the cell counts cleared for pass 2.
__global__ void pts_bounds_kernel(PtsSets ps, float* part, int32_t* start, int64_t nstart,
                                  int* err) {
  __shared__ float sm[33];
  int s, c;
  pts_block(ps, blockIdx.x, &s, &c);
  const float* P = pts_set_base(ps, s);
  const int n = pts_set_n(ps, s);
  const int i0 = c * kPtsChunk, i1 = min(n, i0 + kPtsChunk);
  float mn[3] = {INFINITY, INFINITY, INFINITY}, mx[3] = {-INFINITY, -INFINITY, -INFINITY};
  for (int i = i0 + threadIdx.x; i < i1; i += blockDim.x) {
#pragma unroll
    for (int a = 0; a < 3; ++a) {
      const float x = __ldg(P + 3 * static_cast<int64_t>(i) + a);
      mn[a] = fminf(mn[a], x);
      mx[a] = fmaxf(mx[a], x);
    }
  }
#pragma unroll
  for (int a = 0; a < 3; ++a) {
    const float lo = pts_block_reduce(mn[a], false, sm);
    const float hi = pts_block_reduce(mx[a], true, sm);
    if (threadIdx.x == 0) {
      part[6 * blockIdx.x + a] = lo;
      part[6 * blockIdx.x + 3 + a] = hi;
    }
  }
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t t = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; t < nstart;
       t += stride)
    start[t] = 0;
  if (err && blockIdx.x == 0 && threadIdx.x == 0) *err = 0;
}

// Grid of set s from its bounding box: cubic cells sized for about two
// points per cell edge on a surface through the box (the points of a point
// map lie on a surface), enlarged until the grid has at most `cap` cells.
// Non-finite boxes give one cell.
__device__ void pts_make_grid(const float lo[3], const float hi[3], int n, int cap,
                              int64_t cell0, PtsGrid* g) {
  bool finite = true;
  double e[3];
  for (int a = 0; a < 3; ++a) {
    finite = finite && isfinite(lo[a]) && isfinite(hi[a]);
    e[a] = static_cast<double>(hi[a]) - static_cast<double>(lo[a]);
  }
  g->cell0 = cell0;
  if (!finite) {
    for (int a = 0; a < 3; ++a) {
      g->lo[a] = 0.f;
      g->hi[a] = 0.f;
      g->dim[a] = 1;
    }
    g->h = 1.f;
    g->inv_h = 0.f;  // every point in cell 0
    g->margin = INFINITY;
    return;
  }
  const double emax = fmax(e[0], fmax(e[1], e[2]));
  const double area = e[0] * e[1] + e[1] * e[2] + e[2] * e[0];
  double h;
  if (area > 0.0) h = sqrt(4.0 * area / n);
  else if (emax > 0.0) h = 2.0 * emax / n;
  else h = 1.0;
  if (emax > 0.0 && h < emax / 1048576.0) h = emax / 1048576.0;
  int dim[3];
  int64_t cells = 0;
  for (int it = 0; it < 200; ++it) {
    cells = 1;
    for (int a = 0; a < 3; ++a) {
      dim[a] = static_cast<int>(floor(e[a] / h)) + 1;
      cells *= dim[a];
    }
    if (cells <= cap) break;
    h *= 1.25;
  }
  if (cells > cap) {  // not reached (h grows by 1.25^200); keeps every cell in range
    h = emax > 0.0 ? 2.0 * emax : 1.0;
    dim[0] = dim[1] = dim[2] = 1;
  }
  const float hf = static_cast<float>(h);
  double mag = h + emax;
  for (int a = 0; a < 3; ++a) {
    g->lo[a] = lo[a];
    g->hi[a] = hi[a];
    g->dim[a] = dim[a];
    mag += fabs(static_cast<double>(lo[a]));
  }
  g->h = hf;
  g->inv_h = 1.f / hf;
  g->margin = static_cast<float>(1e-6 * mag);
}

// Pass 2: the grid of each set (from its blocks' boxes), each point's cell,
// and its rank among the points of that cell.
__global__ void pts_count_kernel(PtsSets ps, const float* part, PtsGrid* grids, int32_t* start,
                                 int32_t* cell, int32_t* rank) {
  __shared__ float sm[33];
  __shared__ PtsGrid sg;
  int s, c;
  pts_block(ps, blockIdx.x, &s, &c);
  const int fam = s < ps.nb ? 0 : 1;
  const int b0 = pts_blk0(ps, s);
  float v[6] = {INFINITY, INFINITY, INFINITY, -INFINITY, -INFINITY, -INFINITY};
  for (int j = threadIdx.x; j < ps.blk[fam]; j += blockDim.x)
#pragma unroll
    for (int a = 0; a < 3; ++a) {
      v[a] = fminf(v[a], part[6 * (b0 + j) + a]);
      v[3 + a] = fmaxf(v[3 + a], part[6 * (b0 + j) + 3 + a]);
    }
  float lo[3], hi[3];
#pragma unroll
  for (int a = 0; a < 3; ++a) {
    lo[a] = pts_block_reduce(v[a], false, sm);
    hi[a] = pts_block_reduce(v[3 + a], true, sm);
  }
  const int n = pts_set_n(ps, s);
  if (threadIdx.x == 0) {
    pts_make_grid(lo, hi, n, ps.cap[fam], pts_cell0(ps, s), &sg);
    if (c == 0) grids[s] = sg;
  }
  __syncthreads();
  const PtsGrid g = sg;
  const float* P = pts_set_base(ps, s);
  const int64_t pt0 = pts_pt0(ps, s);
  const int i0 = c * kPtsChunk, i1 = min(n, i0 + kPtsChunk);
  for (int i = i0 + threadIdx.x; i < i1; i += blockDim.x) {
    const float* p = P + 3 * static_cast<int64_t>(i);
    const int cx = pts_axis_cell(g, 0, __ldg(p));
    const int cy = pts_axis_cell(g, 1, __ldg(p + 1));
    const int cz = pts_axis_cell(g, 2, __ldg(p + 2));
    const int64_t gc = g.cell0 + (static_cast<int64_t>(cz) * g.dim[1] + cy) * g.dim[0] + cx;
    cell[pt0 + i] = static_cast<int32_t>(gc);
    rank[pt0 + i] = atomicAdd(start + gc, 1);
  }
}

// Passes 3 to 5: exclusive prefix sum of the cell counts, in place, over
// segments of kScanSeg cells: each segment's sum, an exclusive prefix sum of
// those sums (one block), then each segment's own prefix sum from its
// offset.  start[ncells] (a zero count) becomes the number of points.
__global__ void pts_scan_sum_kernel(const int32_t* start, int64_t nstart, int32_t* seg) {
  const int64_t base = static_cast<int64_t>(blockIdx.x) * kScanSeg +
                       static_cast<int64_t>(threadIdx.x) * kScanPer;
  int sum = 0;
#pragma unroll
  for (int e = 0; e < kScanPer; ++e)
    if (base + e < nstart) sum += start[base + e];
  int tot;
  (void)block_exclusive_scan(sum, &tot);
  if (threadIdx.x == 0) seg[blockIdx.x] = tot;
}

__global__ void pts_scan_seg_kernel(int32_t* seg, int nseg) {
  int carry = 0;
  for (int j0 = 0; j0 < nseg; j0 += kScanSeg) {
    const int base = j0 + static_cast<int>(threadIdx.x) * kScanPer;
    int v[kScanPer];
    int sum = 0;
#pragma unroll
    for (int e = 0; e < kScanPer; ++e) {
      v[e] = base + e < nseg ? seg[base + e] : 0;
      sum += v[e];
    }
    int tot;
    int run = carry + block_exclusive_scan(sum, &tot);
#pragma unroll
    for (int e = 0; e < kScanPer; ++e) {
      if (base + e < nseg) seg[base + e] = run;
      run += v[e];
    }
    carry += tot;
  }
}

__global__ void pts_scan_apply_kernel(int32_t* start, int64_t nstart, const int32_t* seg) {
  const int off = seg[blockIdx.x];
  const int64_t base = static_cast<int64_t>(blockIdx.x) * kScanSeg +
                       static_cast<int64_t>(threadIdx.x) * kScanPer;
  int v[kScanPer];
  int sum = 0;
#pragma unroll
  for (int e = 0; e < kScanPer; ++e) {
    v[e] = base + e < nstart ? start[base + e] : 0;
    sum += v[e];
  }
  int tot;
  int run = off + block_exclusive_scan(sum, &tot);
#pragma unroll
  for (int e = 0; e < kScanPer; ++e) {
    if (base + e < nstart) start[base + e] = run;
    run += v[e];
  }
}

// Pass 5: every point to its place in the cell order, as (x, y, z, index).
__global__ void pts_scatter_kernel(PtsSets ps, const int32_t* start, const int32_t* cell,
                                   const int32_t* rank, float4* sorted, int64_t npts) {
  const int64_t f0 = static_cast<int64_t>(ps.nb) * ps.n[0];
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t gp = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; gp < npts;
       gp += stride) {
    int s;
    int64_t i;
    if (gp < f0) {
      s = static_cast<int>(gp / ps.n[0]);
      i = gp - static_cast<int64_t>(s) * ps.n[0];
    } else {
      const int64_t r = gp - f0;
      s = ps.nb + static_cast<int>(r / ps.n[1]);
      i = r - (r / ps.n[1]) * ps.n[1];
    }
    const float* p = pts_set_base(ps, s) + 3 * i;
    const int pos = start[cell[gp]] + rank[gp];
    sorted[pos] = make_float4(__ldg(p), __ldg(p + 1), __ldg(p + 2),
                              __int_as_float(static_cast<int>(i)));
  }
}

// Points of cells [c0, c1] of one grid row (a contiguous run of sorted
// points) against the best so far.
__device__ __forceinline__ void pts_scan_cells(const float4* __restrict__ sorted,
                                               const int32_t* __restrict__ start, int64_t c0,
                                               int64_t c1, float qx, float qy, float qz,
                                               float& best, int& bi) {
  const int p1 = __ldg(start + c1 + 1);
  for (int p = __ldg(start + c0); p < p1; ++p) {
    const float4 v = __ldg(sorted + p);
    const float dx = qx - v.x, dy = qy - v.y, dz = qz - v.z;
    const float d2 = fmaf(dz, dz, fmaf(dy, dy, dx * dx));
    const int j = __float_as_int(v.w);
    if (d2 < best || (d2 == best && j < bi)) {
      best = d2;
      bi = j;
    }
  }
}

// Nearest point of a set to q, searched by G lanes together (G a power of
// two; the G lanes of an aligned group pass the same q): Chebyshev shells
// k = 0, 1, ... of cells around q's (clamped) cell.  A shell is (2k+1)^2
// grid rows (dz, dy); rows on a z or y face of the cube are scanned whole
// (one contiguous run of sorted points), the others at their two end cells.
// Rows are dealt round-robin to the lanes, and the group's best is merged
// after each shell.  After shell k every unsearched cell lies beyond one of
// the cube's open faces; a point there is at least the face distance away
// along that axis and at least q's distance to the box along the others.
// The search stops when the best squared distance is below that bound (less
// a rounding allowance), or when no face is open.  Returns the squared
// distance; *idx is the point's index in its set (the same in every lane of
// the group).
template <int G>
__device__ float pts_nearest(const PtsGrid g, const float4* __restrict__ sorted,
                             const int32_t* __restrict__ start, float qx, float qy, float qz,
                             int* idx) {
  const int lane = threadIdx.x & 31;
  const int r = lane & (G - 1);
  const unsigned gmask = G == 32 ? 0xffffffffu : (((1u << G) - 1u) << (lane & ~(G - 1)));
  const float q[3] = {qx, qy, qz};
  int c[3];
  float out2[3];  // squared distance from q to the box along each axis
#pragma unroll
  for (int a = 0; a < 3; ++a) {
    c[a] = pts_axis_cell(g, a, q[a]);
    const float o = fmaxf(fmaxf(g.lo[a] - q[a], q[a] - g.hi[a]), 0.f);
    out2[a] = o * o;
  }
  float best = INFINITY;
  int bi = 0x7fffffff;
  const int64_t plane = static_cast<int64_t>(g.dim[0]) * g.dim[1];
  for (int k = 0;; ++k) {
    // the cube's rows clipped to the grid, numbered row-major over (z, y)
    const int z0 = max(c[2] - k, 0), z1 = min(c[2] + k, g.dim[2] - 1);
    const int y0 = max(c[1] - k, 0), y1 = min(c[1] + k, g.dim[1] - 1);
    const int x0 = max(c[0] - k, 0), x1 = min(c[0] + k, g.dim[0] - 1);
    const int ny = y1 - y0 + 1;
    const int nrows = (z1 - z0 + 1) * ny;
    for (int j = r; j < nrows; j += G) {
      const int zi = j / ny;
      const int z = z0 + zi, y = y0 + (j - zi * ny);
      const int64_t row = g.cell0 + z * plane + static_cast<int64_t>(y) * g.dim[0];
      if (z == c[2] - k || z == c[2] + k || y == c[1] - k || y == c[1] + k) {
        pts_scan_cells(sorted, start, row + x0, row + x1, qx, qy, qz, best, bi);
      } else {
        if (c[0] - k >= 0) pts_scan_cells(sorted, start, row + x0, row + x0, qx, qy, qz, best, bi);
        if (c[0] + k < g.dim[0])
          pts_scan_cells(sorted, start, row + x1, row + x1, qx, qy, qz, best, bi);
      }
    }
#pragma unroll
    for (int o = G / 2; o > 0; o >>= 1) {
      const float ob = __shfl_xor_sync(gmask, best, o);
      const int oi = __shfl_xor_sync(gmask, bi, o);
      if (ob < best || (ob == best && oi < bi)) {
        best = ob;
        bi = oi;
      }
    }
    // lower bound on the squared distance to any unsearched cell
    float lb2 = INFINITY;
    bool open = false;
#pragma unroll
    for (int a = 0; a < 3; ++a) {
      const float rest = out2[0] + out2[1] + out2[2] - out2[a];
      if (c[a] - k > 0) {
        open = true;
        const float f = fmaxf(q[a] - (g.lo[a] + static_cast<float>(c[a] - k) * g.h) - g.margin,
                              0.f);
        lb2 = fminf(lb2, fmaf(f, f, rest));
      }
      if (c[a] + k < g.dim[a] - 1) {
        open = true;
        const float f = fmaxf(g.lo[a] + static_cast<float>(c[a] + k + 1) * g.h - q[a] - g.margin,
                              0.f);
        lb2 = fminf(lb2, fmaf(f, f, rest));
      }
    }
    if (!open || best < lb2 * 0.99999f) break;
  }
  *idx = bi == 0x7fffffff ? 0 : bi;  // no finite distance (non-finite input): index 0
  return best;
}

// Lanes per query (measured on 512x384 point maps): four for the
// reciprocal-set sweeps, sixteen for the FRM half-steps, which have a query
// per active seed only and need the extra parallelism to hide latency.
constexpr int kPtsGroupQuery = 4;
constexpr int kPtsGroup = 16;

// Nearest neighbours of nq query points (Q, [nq][3]) in set `set`: index
// and squared distance, or packed keys (score = the squared distance) for
// the mutual test.  Two query families share one launch (the two sweeps of
// the reciprocal set).  kPtsGroupQuery lanes per query.
struct PtsQuery {
  const float* Q;
  int64_t nq;
  int set;
  int32_t* idx;           // or null
  float* dist2;           // or null
  unsigned long long* keys;  // or null
};

__global__ void pts_query_kernel(PtsQuery q0, PtsQuery q1, int nfam, const PtsGrid* grids,
                                 const float4* sorted, const int32_t* start) {
  const int64_t n = q0.nq + (nfam > 1 ? q1.nq : 0);
  constexpr int G = kPtsGroupQuery;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x / G;
  const bool lead = (threadIdx.x & (G - 1)) == 0;
  for (int64_t t = (blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x) / G; t < n;
       t += stride) {
    const bool first = t < q0.nq;
    const PtsQuery& Qf = first ? q0 : q1;
    const int64_t i = first ? t : t - q0.nq;
    const float* p = Qf.Q + 3 * i;
    int j;
    const float d2 =
        pts_nearest<G>(grids[Qf.set], sorted, start, __ldg(p), __ldg(p + 1), __ldg(p + 2), &j);
    if (lead) {
      if (Qf.idx) Qf.idx[i] = j;
      if (Qf.dist2) Qf.dist2[i] = d2;
      if (Qf.keys) Qf.keys[i] = pack_key(d2, j);
    }
  }
}

// Half-step h of FRM on point maps, kPtsGroup lanes per active seed of
// every pair: the NN of the seed's point (NN2: U of image 1 in the image-2
// grid of its pair; NN1: V of image 2 in the image-1 grid), then frm_apply
// by the group's first lane.  Sets 0..B-1 are the image-1 maps, B..2B-1 the
// image-2 maps.  The list and count buffers rotate as in frm_step_kernel.
__global__ void frm_pts_step_kernel(FrmState st, PtsSets ps, const PtsGrid* grids,
                                    const float4* sorted, const int32_t* start, int h,
                                    int nn2_half, int last_iter) {
  const int32_t* cnt_in = st.cnt[h % 3];
  int32_t* cnt_out = st.cnt[(h + 1) % 3];
  const int32_t* list_in = st.list[h % 2];
  int32_t* list_out = st.list[(h + 1) % 2];
  if (blockIdx.x == 0) {
    int32_t* cnt_next = st.cnt[(h + 2) % 3];
    for (int b = threadIdx.x; b < st.B; b += blockDim.x) cnt_next[b] = 0;
  }
  const int32_t* rows = nn2_half ? st.U : st.V;
  const bool lead = (threadIdx.x & (kPtsGroup - 1)) == 0;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x / kPtsGroup;
  for (int64_t x = (blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x) / kPtsGroup;
       x < static_cast<int64_t>(st.B) * st.k; x += stride) {
    const int b = static_cast<int>(x / st.k);
    const int i = static_cast<int>(x - static_cast<int64_t>(b) * st.k);
    if (i >= cnt_in[b]) continue;
    const int64_t base = static_cast<int64_t>(b) * st.k;
    const int s = list_in[base + i];
    const int64_t r = rows[base + s];
    const float* p = nn2_half ? pts_set_base(ps, b) + 3 * r : pts_set_base(ps, ps.nb + b) + 3 * r;
    int j;
    (void)pts_nearest<kPtsGroup>(grids[nn2_half ? ps.nb + b : b], sorted, start, __ldg(p),
                                 __ldg(p + 1), __ldg(p + 2), &j);
    if (lead) frm_apply(st, b, base, s, j, nn2_half, last_iter, list_out, cnt_out);
  }
}

}  // namespace rnn
