// Coarse-to-fine matching: kernels around the reciprocal-set and FRM passes.
//
// High-resolution images are matched coarsely first; the coarse matches then
// guide the matching of enumerated local crops, and the fine matches are
// mapped back to full resolution (cv-learn.com "MASt3R" note, paragraph
// "Coarse-to-fine matching"; the staskaer.github.io DUSt3R/MASt3R blog
// describes the same step as going back to the full-resolution image and
// matching again block by block).  The pages give no formulas for the crops;
// the rules below are integer ones, so that the device and the oracle agree
// exactly:
//   - crops of image 1: along an axis of length L, ceil(L/c) crops of length
//     c at origins floor(a*(L-c)/(n-1)) (0 when n = 1), row-major;
//   - the full-resolution pixel of coarse pixel (yc, xc) of an Hc x Wc map is
//     (floor((2yc+1)*H/(2Hc)), floor((2xc+1)*W/(2Wc)));
//   - a coarse pair belongs to crop b when its image-1 pixel lies inside it;
//     with at least min_coarse of them the crop is on, and its image-2 crop
//     is centred on the floor of their image-2 pixels' mean, clamped into
//     image 2;
//   - the pairs of every crop pair are mapped back by the crops' origins;
//     where crops overlap, the lowest crop index that outputs an image-1
//     pixel gives its pair; the result is sorted by the image-1 pixel.
// This header is included by rnn.cu (it uses block_exclusive_scan).
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

namespace rnn {

struct C2FGeom {
  int Hc1, Wc1, Hc2, Wc2;  // coarse maps
  int H1, W1, H2, W2;      // full-resolution maps
  int ch, cw;              // crop size (at most both images' sizes)
  int ny, nx;              // crops of image 1 along y and x
  int min_coarse;
};

constexpr int kC2FCropCols = 6;  // y0_1, x0_1, y0_2, x0_2, n_coarse, on

__host__ __device__ __forceinline__ int c2f_origin(int a, int n, int L, int c) {
  return n > 1 ? static_cast<int>(static_cast<int64_t>(a) * (L - c) / (n - 1)) : 0;
}

__host__ __device__ __forceinline__ int c2f_fine(int ic, int nc, int n) {
  return static_cast<int>((2 * static_cast<int64_t>(ic) + 1) * n / (2 * static_cast<int64_t>(nc)));
}

// One block per crop of image 1: its coarse pairs, the image-2 crop, on/off.
__global__ void c2f_place_kernel(C2FGeom g, const int32_t* coarse, const int32_t* coarse_count,
                                 int32_t* crops, int32_t* pair_on) {
  __shared__ unsigned long long acc[3];
  const int b = blockIdx.x;
  const int y0 = c2f_origin(b / g.nx, g.ny, g.H1, g.ch);
  const int x0 = c2f_origin(b % g.nx, g.nx, g.W1, g.cw);
  if (threadIdx.x < 3) acc[threadIdx.x] = 0ull;
  __syncthreads();
  const int n = *coarse_count;
  unsigned long long cnt = 0, sy = 0, sx = 0;
  for (int t = threadIdx.x; t < n; t += blockDim.x) {
    const int i = coarse[2 * t], j = coarse[2 * t + 1];
    const int fy = c2f_fine(i / g.Wc1, g.Hc1, g.H1), fx = c2f_fine(i % g.Wc1, g.Wc1, g.W1);
    if (fy >= y0 && fy < y0 + g.ch && fx >= x0 && fx < x0 + g.cw) {
      ++cnt;
      sy += static_cast<unsigned long long>(c2f_fine(j / g.Wc2, g.Hc2, g.H2));
      sx += static_cast<unsigned long long>(c2f_fine(j % g.Wc2, g.Wc2, g.W2));
    }
  }
  if (cnt) {
    atomicAdd(&acc[0], cnt);
    atomicAdd(&acc[1], sy);
    atomicAdd(&acc[2], sx);
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const long long c = static_cast<long long>(acc[0]);
    const int on = c >= (g.min_coarse > 1 ? g.min_coarse : 1) ? 1 : 0;
    int y2 = 0, x2 = 0;
    if (on) {
      const long long cy = static_cast<long long>(acc[1]) / c;
      const long long cx = static_cast<long long>(acc[2]) / c;
      y2 = static_cast<int>(min(max(cy - g.ch / 2, 0ll), static_cast<long long>(g.H2 - g.ch)));
      x2 = static_cast<int>(min(max(cx - g.cw / 2, 0ll), static_cast<long long>(g.W2 - g.cw)));
    }
    int32_t* row = crops + static_cast<int64_t>(b) * kC2FCropCols;
    row[0] = y0;
    row[1] = x0;
    row[2] = y2;
    row[3] = x2;
    row[4] = static_cast<int32_t>(c);
    row[5] = on;
    pair_on[b] = on;
  }
}

// The windows of the crop pairs that are on, as contiguous [B][ch*cw][dp]
// maps (channels past d zero); also clears the map-back arrays.  One 16-byte
// chunk per item.
__global__ void c2f_gather_kernel(C2FGeom g, const uint16_t* F1, const uint16_t* F2, int d,
                                  int dp, const int32_t* crops, int B, uint16_t* out1,
                                  uint16_t* out2, int32_t* tag, int64_t n1, uint32_t* bm,
                                  int64_t nwords) {
  const int rows = g.ch * g.cw;
  const int cpr = dp / 8, creal = d / 8;
  const int64_t per_img = static_cast<int64_t>(B) * rows * cpr;
  const int64_t total = 2 * per_img + n1 + nwords;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t t = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; t < total;
       t += stride) {
    if (t >= 2 * per_img) {
      const int64_t z = t - 2 * per_img;
      if (z < n1) tag[z] = INT32_MAX;
      else bm[z - n1] = 0u;
      continue;
    }
    const int img = t >= per_img ? 1 : 0;
    const int64_t r0 = img ? t - per_img : t;
    const int b = static_cast<int>(r0 / (static_cast<int64_t>(rows) * cpr));
    const int64_t rc = r0 - static_cast<int64_t>(b) * rows * cpr;
    const int r = static_cast<int>(rc / cpr), c = static_cast<int>(rc - (rc / cpr) * cpr);
    const int32_t* row = crops + static_cast<int64_t>(b) * kC2FCropCols;
    if (!row[5]) continue;
    const int y = (img ? row[2] : row[0]) + r / g.cw;
    const int x = (img ? row[3] : row[1]) + r % g.cw;
    const int W = img ? g.W2 : g.W1;
    const uint16_t* src = (img ? F2 : F1) + (static_cast<int64_t>(y) * W + x) * d;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (c < creal) v = __ldg(reinterpret_cast<const uint4*>(src) + c);
    uint16_t* dst = (img ? out2 : out1) + (static_cast<int64_t>(b) * rows + r) * dp;
    reinterpret_cast<uint4*>(dst)[c] = v;
  }
}

// Map-back pass 0 (first = 1): the lowest crop index of every image-1 pixel
// that some crop outputs; pass 1 (first = 0): that crop writes the pixel's
// partner and marks it in the bitmap.
__global__ void c2f_mapback_kernel(C2FGeom g, int B, const int32_t* crops, const int32_t* lpairs,
                                   int64_t capc, const int32_t* lcount, int32_t* tag,
                                   int32_t* partner, uint32_t* bm, int first) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t t = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
       t < static_cast<int64_t>(B) * capc; t += stride) {
    const int b = static_cast<int>(t / capc);
    const int64_t i = t - static_cast<int64_t>(b) * capc;
    if (i >= lcount[b]) continue;
    const int32_t* row = crops + static_cast<int64_t>(b) * kC2FCropCols;
    const int u = lpairs[2 * t], v = lpairs[2 * t + 1];
    const int gu = (row[0] + u / g.cw) * g.W1 + row[1] + u % g.cw;
    if (first) {
      atomicMin(tag + gu, b);
    } else if (tag[gu] == b) {
      partner[gu] = (row[2] + v / g.cw) * g.W2 + row[3] + v % g.cw;
      atomicOr(bm + (gu >> 5), 1u << (gu & 31));
    }
  }
}

// Bitmap compaction in pixel order: pass 1 counts the marked pixels of each
// block of kEmitWords words, pass 2 writes (pixel, partner) from each block's
// offset.  The status word of the call collects the ones of its parts.
constexpr int kEmitWords = 4096;  // 4 words per thread of 1024

__global__ void c2f_count_kernel(const uint32_t* bm, int64_t nwords, int* block_counts) {
  const int64_t w0 = static_cast<int64_t>(blockIdx.x) * kEmitWords + threadIdx.x * 4;
  int c = 0;
#pragma unroll
  for (int e = 0; e < 4; ++e)
    if (w0 + e < nwords) c += __popc(bm[w0 + e]);
  int tot;
  (void)block_exclusive_scan(c, &tot);
  if (threadIdx.x == 0) block_counts[blockIdx.x] = tot;
}

__global__ void c2f_emit_kernel(const uint32_t* bm, int64_t nwords, const int* block_counts,
                                const int32_t* partner, int32_t* pairs, int32_t* count_out,
                                int* status, const int* err_a, const int* err_b) {
  __shared__ int s_off;
  int part = 0;
  for (int j = threadIdx.x; j < static_cast<int>(blockIdx.x); j += blockDim.x)
    part += block_counts[j];
  int tot;
  (void)block_exclusive_scan(part, &tot);
  if (threadIdx.x == 0) s_off = tot;
  __syncthreads();
  const int off = s_off;
  const int64_t w0 = static_cast<int64_t>(blockIdx.x) * kEmitWords + threadIdx.x * 4;
  uint32_t words[4];
  int c = 0;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    words[e] = w0 + e < nwords ? bm[w0 + e] : 0u;
    c += __popc(words[e]);
  }
  int btot;
  int pos = off + block_exclusive_scan(c, &btot);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    uint32_t bits = words[e];
    while (bits) {
      const int bit = __ffs(bits) - 1;
      bits &= bits - 1;
      const int u = static_cast<int>((w0 + e) * 32 + bit);
      pairs[2 * static_cast<int64_t>(pos)] = u;
      pairs[2 * static_cast<int64_t>(pos) + 1] = partner[u];
      ++pos;
    }
  }
  if (blockIdx.x == gridDim.x - 1 && threadIdx.x == 0) {
    *count_out = off + btot;
    *status = *err_a | *err_b;
  }
}

}  // namespace rnn
