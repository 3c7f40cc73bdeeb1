// C ABI of the reciprocal nearest-neighbour library (declared in include/rnn.h).
//
// Every entry point validates its arguments on the host, builds the TMA
// descriptors of the candidate maps, and enqueues a fixed sequence of kernels
// on the caller's stream.  No allocation, no synchronisation: scratch lives in
// the caller's workspace.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <new>

#include <nvtx3/nvToolsExt.h>

#include "mnn_kernel.cuh"
#include "nn_kernel.cuh"
#include "rnn.h"

namespace rnn {

// ------------------------------------------------------------------ helpers
constexpr size_t kAlign = 256;
constexpr int kSmallThreads = 1024;
constexpr int kMnnChunk = 4096;  // rows per block in the mutual test (4 per thread)
constexpr unsigned long long kWaitLimitNs = 1000000000ull;  // 1 s per bounded wait
constexpr int kMaxGraphIters = 64;  // max_iter of a graph plan
#ifndef RNN_PDL
#define RNN_PDL 1  // programmatic dependent launch along the FRM chain
#endif

static size_t align_up(size_t x) { return (x + kAlign - 1) & ~(kAlign - 1); }

// An NVTX range over one ABI call (visible in Nsight Systems; a no-op
// unless a tool is attached).
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

struct Carve {
  uint8_t* base;
  size_t off = 0;
  explicit Carve(void* b) : base(static_cast<uint8_t*>(b)) {}
  template <class T>
  T* take(size_t count) {
    T* p = reinterpret_cast<T*>(base ? base + off : nullptr);
    off = align_up(off + count * sizeof(T));
    return p;
  }
};

struct DeviceInfo {
  int sms = 0;
  bool sm100 = false;
  bool smem_set = false;
  bool op_smem_set = false;  // one-pass exhaustive-set kernels
};

static std::mutex g_mu;
static DeviceInfo g_dev[64];

static rnn_status device_info(DeviceInfo** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return RNN_ECUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceInfo& di = g_dev[dev];
  if (di.sms == 0) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return RNN_ECUDA;
    di.sm100 = (major == 10 && minor == 0);
    di.sms = sms;
  }
  if (!di.sm100) return RNN_EUNSUPPORTED;
  *out = &di;
  return RNN_OK;
}

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static std::once_flag once;
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// Operand geometry for a channel count d.
struct Geometry {
  int kb, nkb, kpad, block_n, nacc, stages, qbufs;
  size_t smem;
};

static size_t tables_bytes() { return sizeof(SharedTables); }

// Candidate tile width for K <= 64: 128 (four accumulators) or 256 (two).
#ifndef RNN_SMALL_K_BLOCK_N
#define RNN_SMALL_K_BLOCK_N 256
#endif

static Geometry geometry(int d) {
  Geometry g;
  if (d <= 16) {
    g.kb = 16; g.nkb = 1;
  } else if (d <= 32) {
    g.kb = 32; g.nkb = 1;
  } else if (d % 64 == 0) {
    g.kb = 64; g.nkb = d / 64;
  } else if (d % 32 == 0) {
    g.kb = 32; g.nkb = d / 32;
  } else {
    g.kb = 16; g.nkb = (d + 15) / 16;
  }
  g.kpad = g.kb * g.nkb;
  g.block_n = g.kpad <= 64 ? RNN_SMALL_K_BLOCK_N : 128;
  g.nacc = 512 / g.block_n;
  const size_t stage = static_cast<size_t>(g.block_n) * g.kpad * 2;
  const size_t qb = static_cast<size_t>(kBlockM) * g.kpad * 2;
  const size_t fixed = 1024 /*align slack*/ + 16 + kBlockM * 4 + 32 * 4 + tables_bytes();
  const size_t budget = 227 * 1024;
  const size_t bars = (2 * kMaxStages + 4 + kMaxAcc + kMmaWarps) * 8;
  const size_t avail = budget - fixed - bars;
  g.qbufs = (2 * qb + 2 * stage <= avail) ? 2 : 1;
  size_t st = (avail - g.qbufs * qb) / stage;
  if (st > kMaxStages) st = kMaxStages;
  // one barrier per stage also signals the accumulators: each epilogue group
  // waits on the stages of its own tiles only, which needs the stage count
  // to be a multiple of the accumulator count (2 or 4)
  if (g.nacc > 2 && st < 4) g.nacc = 2;
  st -= st % g.nacc;
  g.stages = static_cast<int>(st);
  g.smem = fixed + bars + g.stages * stage + g.qbufs * qb;
  // at least half the SM's shared memory, so that two CTAs never share an SM
  // (each one allocates all 512 tensor-memory columns)
  if (g.smem < 116 * 1024) g.smem = 116 * 1024;
  return g;
}

// The one-pass kernel for the exhaustive set covers one K-block of 16, 32 or
// 64; other shapes take the two-sweep form.  Its copies of the maps carry
// kOpPadRows NaN rows past the last pixel: enough for the last unit
// (bm*128 <= 2048 query rows, 8*256 candidate rows) to read nothing but NaN
// beyond the end.  Under the Euclidean metric the copies carry six more
// columns (op_copy_kernel), so that one score serves both directions.
constexpr int64_t kOpPadRows = 2048;
constexpr int kOpAugCols = 6;
static Geometry onepass_geometry(int d, rnn_metric metric) {
  return geometry(d + (metric == RNN_L2 ? kOpAugCols : 0));
}
static bool onepass_fits(const Geometry& g) {
  return g.nkb == 1 && g.block_n == kOpBlockN && (g.kpad == 16 || g.kpad == 32 || g.kpad == 64);
}

// Depth K of the tensor-core tiles for d channels (d rounded up to the
// K-block layout the geometry picks).
static int padded_depth(int d) { return geometry(d).kpad; }

static uint32_t make_idesc(rnn_dtype dt, int block_n) {
  const uint32_t fmt = dt == RNN_BF16 ? 1u : 0u;
  uint32_t d = 0;
  d |= 1u << 4;                                      // accumulator: f32
  d |= fmt << 7;                                     // A format
  d |= fmt << 10;                                    // B format
  d |= static_cast<uint32_t>(block_n >> 3) << 17;    // N
  d |= static_cast<uint32_t>(kBlockM >> 4) << 24;    // M
  return d;
}

// [nbatch][rows][d] map with batch stride `bstride` elements, boxes of
// `box_rows` rows (candidate tiles: g.block_n; query tiles: 128).
static rnn_status make_map(CUtensorMap* m, const void* base, int d, int64_t rows, int nbatch,
                           int64_t bstride, const Geometry& g, int box_rows = 0) {
  auto fn = encode_fn();
  if (!fn) return RNN_ECUDA;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(rows),
                        static_cast<cuuint64_t>(nbatch)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(bstride) * 2};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(g.kb),
                       static_cast<cuuint32_t>(box_rows > 0 ? box_rows : g.block_n), 1};
  cuuint32_t es[3] = {1, 1, 1};
  const CUtensorMapSwizzle sw = g.kb == 64   ? CU_TENSOR_MAP_SWIZZLE_128B
                                : g.kb == 32 ? CU_TENSOR_MAP_SWIZZLE_64B
                                             : CU_TENSOR_MAP_SWIZZLE_32B;
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT16, 3, const_cast<void*>(base), dims, strides,
                  box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? RNN_OK : RNN_ECUDA;
}

// ------------------------------------------------------------- diagnostics
static std::atomic<uint64_t> g_launches{0};
// failure-detection test hook (rnn_test_stall_loads)
static std::atomic<int> g_stall_loads{0};
static std::atomic<unsigned long long> g_stall_limit_ns{kWaitLimitNs};
static void* const* g_timer_start = nullptr;
static void* const* g_timer_stop = nullptr;
static int g_timer_cap = 0;
static int* g_timer_count = nullptr;

// Recording a graph plan: launches are neither counted nor timed.
static thread_local bool t_capturing = false;

// Per device, a stream of this thread that records the bodies of FRM's
// conditional iteration nodes when an FRM call is captured into a graph by
// its caller.  It is made by a call that is not being captured, so that no
// stream is created inside a capture; until then a captured FRM call records
// every iteration unconditionally (the same results).
static thread_local cudaStream_t t_body[64] = {};

// Check the last launch and count it.
static rnn_status launched() {
  if (cudaGetLastError() != cudaSuccess) return RNN_ECUDA;
  if (!t_capturing) g_launches.fetch_add(1, std::memory_order_relaxed);
  return RNN_OK;
}

// Launch with, when `pdl` is set, programmatic stream serialization: the
// grid may be launched while the previous kernel of the stream finishes, and
// waits for it in pdl_wait before reading its output.
template <typename... KArgs, typename... Args>
static void launch_k(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                     cudaStream_t s, bool pdl, Args&&... args) {
  if (!pdl) {  // the plain launch costs the host less
    kernel<<<grid, block, smem, s>>>(std::forward<Args>(args)...);
    return;
  }
  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  (void)cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Benchmark timer (rnn_set_kernel_timer): events around the fused kernels.
static rnn_status timer_begin(cudaStream_t s, int* slot) {
  *slot = -1;
  if (t_capturing || !g_timer_count || !g_timer_start || !g_timer_stop) return RNN_OK;
  const int k = (*g_timer_count)++;
  if (k >= g_timer_cap) return RNN_OK;
  if (cudaEventRecord(static_cast<cudaEvent_t>(g_timer_start[k]), s) != cudaSuccess)
    return RNN_ECUDA;
  *slot = k;
  return RNN_OK;
}

static rnn_status timer_end(cudaStream_t s, int slot) {
  if (slot >= 0 && cudaEventRecord(static_cast<cudaEvent_t>(g_timer_stop[slot]), s) != cudaSuccess)
    return RNN_ECUDA;
  return RNN_OK;
}

static rnn_status launch_nn(const NNParams& p_in, const CUtensorMap& m0, const CUtensorMap& m1,
                            const CUtensorMap& q0, const CUtensorMap& q1, const Geometry& g,
                            DeviceInfo* di, cudaStream_t s, bool pdl = false) {
  NNParams p = p_in;
  p.kb = g.kb;
  p.nkb = g.nkb;
  p.block_n = g.block_n;
  p.stages = g.stages;
  p.nacc = g.nacc;
  p.qbufs = g.qbufs;
  p.target_units = 8 * di->sms;
  {
    // a unit should hold about 4096 tensor-core cycles of work
    const int tile_cycles = (g.kpad / 16) * (g.block_n / 2);
    p.min_tiles = 4096 / tile_cycles > 2 ? 4096 / tile_cycles : 2;
  }
  p.stall_loads = g_stall_loads.load(std::memory_order_relaxed);
  p.wait_limit_ns = p.stall_loads ? g_stall_limit_ns.load(std::memory_order_relaxed)
                                  : kWaitLimitNs;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!di->smem_set) {
      const int sm = 227 * 1024;
      const auto attr = cudaFuncAttributeMaxDynamicSharedMemorySize;
      if (cudaFuncSetAttribute(nn_argmax_kernel<16, 4, 2>, attr, sm) != cudaSuccess ||
          cudaFuncSetAttribute(nn_argmax_kernel<8, 4, 4>, attr, sm) != cudaSuccess ||
          cudaFuncSetAttribute(nn_argmax_kernel<16, 2, 2, true>, attr, sm) != cudaSuccess ||
          cudaFuncSetAttribute(nn_argmax_kernel<16, 4, 2, false, true>, attr, sm) !=
              cudaSuccess ||
          cudaFuncSetAttribute(nn_argmax_kernel<8, 4, 4, false, true>, attr, sm) != cudaSuccess ||
          cudaFuncSetAttribute(nn_argmax_kernel<16, 2, 2, true, true>, attr, sm) != cudaSuccess)
        return RNN_ECUDA;
      di->smem_set = true;
    }
  }
  int slot = -1;
  {
    const rnn_status tr = timer_begin(s, &slot);
    if (tr != RNN_OK) return tr;
  }
  // Epilogue layout.  Two 256-column accumulators: sixteen warps, all on
  // every tile, each 64 columns of its lane quadrant in one copy, so an
  // accumulator is held for one round trip to tensor memory and the fold
  // follows its release.  Two 128-column accumulators: eight warps, one group
  // per accumulator.  Four: sixteen warps copying 64, one group per
  // accumulator.
  const dim3 grid(di->sms);
  if (g.nacc == 2 && g.block_n == 256) {
    const dim3 block((kEpiWarp0 + 16) * 32);
    if (pdl)
      launch_k(nn_argmax_kernel<16, 2, 2, true, true>, grid, block, g.smem, s, true, p, m0, m1,
               q0, q1);
    else
      launch_k(nn_argmax_kernel<16, 2, 2, true>, grid, block, g.smem, s, false, p, m0, m1, q0,
               q1);
  } else if (g.nacc == 2) {
    const dim3 block((kEpiWarp0 + 8) * 32);
    if (pdl)
      launch_k(nn_argmax_kernel<8, 4, 4, false, true>, grid, block, g.smem, s, true, p, m0, m1,
               q0, q1);
    else
      launch_k(nn_argmax_kernel<8, 4, 4>, grid, block, g.smem, s, false, p, m0, m1, q0, q1);
  } else {
    const dim3 block((kEpiWarp0 + 16) * 32);
    if (pdl)
      launch_k(nn_argmax_kernel<16, 4, 2, false, true>, grid, block, g.smem, s, true, p, m0, m1,
               q0, q1);
    else
      launch_k(nn_argmax_kernel<16, 4, 2>, grid, block, g.smem, s, false, p, m0, m1, q0, q1);
  }
  const rnn_status r = launched();
  return r == RNN_OK ? timer_end(s, slot) : r;
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
static bool aligned256(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 255u) == 0; }

static rnn_status check_desc(const void* p, int d) {
  if (!p) return RNN_EINVAL;
  if (d <= 0) return RNN_EINVAL;
  if (d % 8 != 0 || !aligned16(p)) return RNN_EALIGN;
  if (d > 256) return RNN_EUNSUPPORTED;
  return RNN_OK;
}

static bool valid_dtype(rnn_dtype dt) { return dt == RNN_F16 || dt == RNN_BF16; }
static bool valid_metric(rnn_metric m) { return m == RNN_DOT || m == RNN_L2; }

// -------------------------------------------------------------- small kernels
__global__ void zero_keys_kernel(unsigned long long* a, int64_t na, unsigned long long* b,
                                 int64_t nb, int* err) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < na + nb;
       i += stride) {
    if (i < na) a[i] = 0ull; else b[i - na] = 0ull;
  }
  if (blockIdx.x == 0 && threadIdx.x == 0) *err = 0;
}

// Row forms the fused kernel reads (all [nbatch][rows][kpad], zero beyond
// the written columns):
//   kFormPad    the d channels (d < kpad happens for d = 8, 24, 40, ...: over
//               the caller's d-wide rows every box would zero-fill part of
//               itself and fetch rows straddling L2 sectors, which costs the
//               d = 24 sweep about a fifth of its time);
//   kFormQuery  the channels, then 1, 1, 1 (Euclidean metric, query side);
//   kFormCand   the channels, then c1, c2, c3 with c1 + c2 + c3 = -|x|^2/2
//               (Euclidean metric, candidate side).
// With both augmented forms the tensor cores compute q.x - |x|^2/2 =
// (|q|^2 - |q - x|^2)/2, whose largest value over x is the nearest x.
// |x|^2 is summed in fp32 from exact products and split into three 16-bit
// parts; on k/64 inputs every part and every partial sum is a multiple of
// 2^-13 well inside fp32's range, so the augmented score stays exact.
constexpr int kFormPad = 0, kFormQuery = 1, kFormCand = 2;
constexpr int kAugCols = 3;  // extra columns of the Euclidean forms

__device__ __forceinline__ float bits_to_f(uint16_t h, bool bf16) {
  return bf16 ? __bfloat162float(__ushort_as_bfloat16(h)) : __half2float(__ushort_as_half(h));
}
__device__ __forceinline__ uint16_t f_to_bits(float x, bool bf16) {
  return bf16 ? __bfloat16_as_ushort(__float2bfloat16_rn(x))
              : __half_as_ushort(__float2half_rn(x));
}

// One thread per 16-byte chunk of the output, so that reads and writes are
// coalesced; map b of the batch is grid row blockIdx.y.  d is a multiple of
// 8, so a chunk lies wholly among the channels or wholly past them; the first
// chunk past them holds the augmentation (its thread reads the whole row for
// |x|^2), the rest are zero.  kCpr: chunks per output row when known at
// compile time (the index split is then a multiply and shift), else 0.
template <bool kBf16>
__device__ __forceinline__ uint4 prep_chunk(const uint4* __restrict__ in, int c, int creal,
                                            int form) {
  uint4 v = make_uint4(0, 0, 0, 0);
  if (c < creal) {
    v = __ldg(in + c);
  } else if (c == creal && form != kFormPad) {
    uint16_t aug[kAugCols];
    if (form == kFormQuery) {
      aug[0] = aug[1] = aug[2] = f_to_bits(1.0f, kBf16);
    } else {
      float n2 = 0.f;
      for (int cc = 0; cc < creal; ++cc) {
        const uint4 x = __ldg(in + cc);
        const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float lo = bits_to_f(static_cast<uint16_t>(w[e] & 0xFFFFu), kBf16);
          const float hi = bits_to_f(static_cast<uint16_t>(w[e] >> 16), kBf16);
          n2 = fmaf(lo, lo, n2);
          n2 = fmaf(hi, hi, n2);
        }
      }
      float rest = -0.5f * n2;
#pragma unroll
      for (int e = 0; e < kAugCols; ++e) {
        aug[e] = f_to_bits(rest, kBf16);
        rest -= bits_to_f(aug[e], kBf16);
      }
    }
    v.x = static_cast<uint32_t>(aug[0]) | (static_cast<uint32_t>(aug[1]) << 16);
    v.y = static_cast<uint32_t>(aug[2]);
  }
  return v;
}

// One thread per 16-byte chunk of the output, so that reads and writes are
// coalesced; map b of the batch is grid row blockIdx.y.  d is a multiple of
// 8, so a chunk lies wholly among the channels or wholly past them; the first
// chunk past them holds the augmentation (its thread reads the whole row for
// |x|^2), the rest are zero.  kCpr: chunks per output row when known at
// compile time (the index split is then a multiply and shift), else 0.  Each
// thread handles two chunks a grid stride apart per step, both loads ahead of
// both stores, for twice the reads in flight.
template <bool kBf16, int kCpr>
__global__ void prep_rows_kernel(const uint16_t* __restrict__ src, int64_t bstride,
                                 int64_t rows, int d, uint16_t* __restrict__ dst, int kpad,
                                 int form) {
  const int cpr = kCpr ? kCpr : kpad / 8, creal = d / 8;  // chunks per output / input row
  const int64_t b = blockIdx.y;
  const int64_t total = rows * cpr;  // chunks of map b
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const uint16_t* __restrict__ sb = src + b * bstride;
  uint4* __restrict__ db = reinterpret_cast<uint4*>(dst) + b * total;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += 2 * stride) {
    const int64_t i2 = i + stride;
    const int64_t r = i / cpr, r2 = i2 / cpr;
    const uint4 v = prep_chunk<kBf16>(reinterpret_cast<const uint4*>(sb + r * d),
                                      static_cast<int>(i - r * cpr), creal, form);
    uint4 v2 = make_uint4(0, 0, 0, 0);
    if (i2 < total)
      v2 = prep_chunk<kBf16>(reinterpret_cast<const uint4*>(sb + r2 * d),
                             static_cast<int>(i2 - r2 * cpr), creal, form);
    db[i] = v;
    if (i2 < total) db[i2] = v2;
  }
}

// ------------------------------------------------------------------ locate
// The fused kernel leaves, per query, the largest score and the first column
// c0 of the first 32-column chunk that reaches it.  locate_chunk recomputes
// the scores of that chunk (one candidate per lane, fp32 fused multiply-adds
// over the channels in order) and returns the lowest column that reaches
// their maximum.  On inputs whose products and partial sums are exact in
// fp32 (the quantised k/64 maps) the recomputed scores equal the tensor
// cores' bit for bit, so the result is the exact lowest-index argmax; on
// other inputs the two roundings can differ only between scores within fp32
// rounding of each other.  Warp-collective: all lanes pass the same query.
__device__ __forceinline__ float h2f(uint16_t h, bool bf16) {
  return bf16 ? __bfloat162float(__ushort_as_bfloat16(h)) : __half2float(__ushort_as_half(h));
}

template <bool kBf16>
__device__ __forceinline__ float dot_rows(const uint16_t* a, const uint16_t* b, int d) {
  float acc = 0.f;
  for (int c = 0; c < d; c += 8) {
    const uint4 x = __ldg(reinterpret_cast<const uint4*>(a + c));
    const uint4 y = __ldg(reinterpret_cast<const uint4*>(b + c));
    const uint32_t xs[4] = {x.x, x.y, x.z, x.w}, ys[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      acc = fmaf(h2f(static_cast<uint16_t>(xs[e] & 0xFFFFu), kBf16),
                 h2f(static_cast<uint16_t>(ys[e] & 0xFFFFu), kBf16), acc);
      acc = fmaf(h2f(static_cast<uint16_t>(xs[e] >> 16), kBf16),
                 h2f(static_cast<uint16_t>(ys[e] >> 16), kBf16), acc);
    }
  }
  return acc;
}

template <bool kBf16>
__device__ __forceinline__ int locate_chunk(const uint16_t* q, const uint16_t* X, int n_cand,
                                            int ld, int c0, float* best = nullptr) {
  // a key no candidate reached (only after a fused kernel that gave up on a
  // wait) leaves index -1: locate chunk 0 so that every later index is valid
  if (c0 < 0 || c0 >= n_cand) c0 = 0;
  const int lane = threadIdx.x & 31;
  const int j = c0 + lane;
  float sc = -__int_as_float(0x7f800000);
  if (j < n_cand) sc = dot_rows<kBf16>(q, X + static_cast<int64_t>(j) * ld, ld);
  float m = sc;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  const unsigned hit = __ballot_sync(0xffffffffu, sc == m);
  if (best) *best = m;
  return c0 + __ffs(hit) - 1;
}

// |q|^2 over the first d channels of a row, in fp32 (exact products).
template <bool kBf16>
__device__ __forceinline__ float sqnorm_row(const uint16_t* q, int d) {
  return dot_rows<kBf16>(q, q, d);
}

// Score a caller sees: the dot product, or with the Euclidean forms the
// squared distance |q|^2 - 2 (q.x - |x|^2/2) of the located candidate.
template <bool kBf16>
__device__ __forceinline__ float reported_score(const uint16_t* q, int d, bool l2, float key_s,
                                                float located_s) {
  return l2 ? sqnorm_row<kBf16>(q, d) - 2.f * located_s : key_s;
}

// nn_argmax results: locate every query's index, write index and score.
// Q and X rows are ld elements apart (the caller's rows, or their forms).
template <bool kBf16>
__global__ void locate_unpack_kernel(const unsigned long long* keys, int64_t n, const uint16_t* Q,
                                     const uint16_t* X, int nx, int ld, int d, int l2,
                                     int32_t* idx, float* score) {
  const int64_t w0 = (blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x) >> 5;
  const int64_t nw = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  for (int64_t i = w0; i < n; i += nw) {
    const unsigned long long k = keys[i];
    const uint16_t* q = Q + i * ld;
    float m;
    const int j = locate_chunk<kBf16>(q, X, nx, ld, key_index(k), &m);
    const float sc = reported_score<kBf16>(q, d, l2 != 0, key_score(k), m);
    if ((threadIdx.x & 31) == 0) {
      idx[i] = j;
      if (score) score[i] = sc;
    }
  }
}

// Both sweeps of the reciprocal set: rewrite each packed key with its exact
// index and the reported score (rows of image 1, Q1, against the candidates
// of image 2, X2; then rows of image 2, Q2, against X1).
template <bool kBf16>
__global__ void locate_mnn_kernel(unsigned long long* rowk, int64_t n1, unsigned long long* colk,
                                  int64_t n2, const uint16_t* Q1, const uint16_t* X1,
                                  const uint16_t* Q2, const uint16_t* X2, int ld, int d,
                                  int l2) {
  const int64_t w0 = (blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x) >> 5;
  const int64_t nw = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  for (int64_t i = w0; i < n1 + n2; i += nw) {
    const bool row = i < n1;
    const int64_t r = row ? i : i - n1;
    unsigned long long* kp = row ? rowk + r : colk + r;
    const unsigned long long k = *kp;
    const uint16_t* q = (row ? Q1 : Q2) + r * ld;
    float m;
    const int j = row ? locate_chunk<kBf16>(q, X2, static_cast<int>(n2), ld, key_index(k), &m)
                      : locate_chunk<kBf16>(q, X1, static_cast<int>(n1), ld, key_index(k), &m);
    const float sc = reported_score<kBf16>(q, d, l2 != 0, key_score(k), m);
    if ((threadIdx.x & 31) == 0) *kp = pack_key(sc, j);
  }
}

// Block-wide exclusive scan of one int per thread (blockDim.x <= 1024).
__device__ int block_exclusive_scan(int v, int* total) {
  __shared__ int warp_sums[33];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = (blockDim.x + 31) >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = lane < nw ? warp_sums[lane] : 0;
    int wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += y;
    }
    if (lane < nw) warp_sums[lane] = wi - w;
    if (lane == nw - 1) warp_sums[32] = wi;
  }
  __syncthreads();
  const int r = warp_sums[warp] + incl - v;
  *total = warp_sums[32];
  __syncthreads();
  return r;
}

__device__ __forceinline__ bool is_mutual(const unsigned long long* rowk,
                                          const unsigned long long* colk, int64_t i, int* j) {
  *j = key_index(rowk[i]);
  return key_index(colk[*j]) == static_cast<int>(i);
}

// Pass 1 of the reciprocal test: mutual count per block of kMnnChunk rows,
// and the optional per-pixel outputs.
__global__ void mnn_count_kernel(const unsigned long long* rowk, int64_t n1,
                                 const unsigned long long* colk, int64_t n2, int* block_counts,
                                 int nblocks1,
                                 int32_t* rowarg, float* rowmax, int32_t* colarg,
                                 float* colmax) {
  const int64_t base = static_cast<int64_t>(blockIdx.x) * kMnnChunk;
  int c = 0;
  for (int e = 0; e < kMnnChunk / kSmallThreads; ++e) {
    const int64_t i = base + static_cast<int64_t>(e) * kSmallThreads + threadIdx.x;
    if (i < n1) {
      int j;
      c += is_mutual(rowk, colk, i, &j) ? 1 : 0;
      if (rowarg) rowarg[i] = j;
      if (rowmax) rowmax[i] = key_score(rowk[i]);
    }
    if (i < n2) {
      if (colarg) colarg[i] = key_index(colk[i]);
      if (colmax) colmax[i] = key_score(colk[i]);
    }
  }
  // block total
  int total;
  (void)block_exclusive_scan(c, &total);
  if (threadIdx.x == 0 && static_cast<int>(blockIdx.x) < nblocks1) block_counts[blockIdx.x] = total;
}

// Pass 2: each block finds its offset from the counts of the blocks before
// it and writes its mutual pairs in increasing i.
__global__ void mnn_write_kernel(const unsigned long long* rowk, int64_t n1,
                                 const unsigned long long* colk, const int* block_counts,
                                 int nblocks, int32_t* pairs, int32_t* count_out) {
  __shared__ int s_off;
  int part = 0;
  for (int b = threadIdx.x; b < blockIdx.x; b += blockDim.x) part += block_counts[b];
  int tot;
  (void)block_exclusive_scan(part, &tot);
  if (threadIdx.x == 0) s_off = tot;
  __syncthreads();
  int off = s_off;
  const int64_t base = static_cast<int64_t>(blockIdx.x) * kMnnChunk;
  // rows of this thread: kMnnChunk/kSmallThreads consecutive rows, so that a
  // thread-order scan keeps increasing i
  constexpr int per = kMnnChunk / kSmallThreads;
  int js[per];
  bool ms[per];
  int c = 0;
#pragma unroll
  for (int e = 0; e < per; ++e) {
    const int64_t i = base + static_cast<int64_t>(threadIdx.x) * per + e;
    ms[e] = false;
    if (i < n1) ms[e] = is_mutual(rowk, colk, i, &js[e]);
    c += ms[e] ? 1 : 0;
  }
  int btot;
  int pos = off + block_exclusive_scan(c, &btot);
#pragma unroll
  for (int e = 0; e < per; ++e) {
    if (ms[e]) {
      const int64_t i = base + static_cast<int64_t>(threadIdx.x) * per + e;
      pairs[2 * static_cast<int64_t>(pos)] = static_cast<int32_t>(i);
      pairs[2 * static_cast<int64_t>(pos) + 1] = js[e];
      ++pos;
    }
  }
  if (blockIdx.x == nblocks - 1 && threadIdx.x == 0) *count_out = off + btot;
}

// Mutual test on plain argmax arrays (the reciprocal set assembled from NN
// results computed elsewhere, e.g. on several GPUs): pass 1 counts per block
// of kMnnChunk rows; pass 2 writes the pairs in increasing i.  An index out of
// range is never mutual.
__device__ __forceinline__ bool is_mutual_arg(const int32_t* rowarg, const int32_t* colarg,
                                              int64_t n2, int64_t i, int* j) {
  *j = rowarg[i];
  return *j >= 0 && *j < n2 && colarg[*j] == static_cast<int32_t>(i);
}

__global__ void mutual_count_kernel(const int32_t* rowarg, int64_t n1, const int32_t* colarg,
                                    int64_t n2, int* block_counts) {
  const int64_t base = static_cast<int64_t>(blockIdx.x) * kMnnChunk;
  int c = 0;
  for (int e = 0; e < kMnnChunk / kSmallThreads; ++e) {
    const int64_t i = base + static_cast<int64_t>(e) * kSmallThreads + threadIdx.x;
    int j;
    if (i < n1 && is_mutual_arg(rowarg, colarg, n2, i, &j)) ++c;
  }
  int total;
  (void)block_exclusive_scan(c, &total);
  if (threadIdx.x == 0) block_counts[blockIdx.x] = total;
}

__global__ void mutual_write_kernel(const int32_t* rowarg, int64_t n1, const int32_t* colarg,
                                    int64_t n2, const int* block_counts, int32_t* pairs,
                                    int32_t* count_out) {
  __shared__ int s_off;
  int part = 0;
  for (int b = threadIdx.x; b < static_cast<int>(blockIdx.x); b += blockDim.x)
    part += block_counts[b];
  int tot;
  (void)block_exclusive_scan(part, &tot);
  if (threadIdx.x == 0) s_off = tot;
  __syncthreads();
  const int off = s_off;
  const int64_t base = static_cast<int64_t>(blockIdx.x) * kMnnChunk;
  constexpr int per = kMnnChunk / kSmallThreads;
  int js[per];
  bool ms[per];
  int c = 0;
#pragma unroll
  for (int e = 0; e < per; ++e) {
    const int64_t i = base + static_cast<int64_t>(threadIdx.x) * per + e;
    ms[e] = i < n1 && is_mutual_arg(rowarg, colarg, n2, i, &js[e]);
    c += ms[e] ? 1 : 0;
  }
  int btot;
  int pos = off + block_exclusive_scan(c, &btot);
#pragma unroll
  for (int e = 0; e < per; ++e) {
    if (ms[e]) {
      const int64_t i = base + static_cast<int64_t>(threadIdx.x) * per + e;
      pairs[2 * static_cast<int64_t>(pos)] = static_cast<int32_t>(i);
      pairs[2 * static_cast<int64_t>(pos) + 1] = js[e];
      ++pos;
    }
  }
  if (blockIdx.x == gridDim.x - 1 && threadIdx.x == 0) *count_out = off + btot;
}

// ------------------------------------------- grouped locate (one-pass M)
// The one-pass kernel leaves row keys whose chunk is kOpRowChunk candidates
// of image 2, and column keys whose chunk is 32*bm candidates of image 1.
// The exact lowest index inside a chunk comes from recomputing the chunk's
// scores (fp32 fused multiply-adds over the channels in order, as in
// locate_chunk).  A column chunk is hundreds of rows, so the queries are
// grouped by chunk first: each chunk's candidates are then read once into
// shared memory and serve all of its queries.  Four launches: count per
// chunk, scan, scatter of the query ids, and the resolve over items of at
// most kLocItem queries of one chunk.
constexpr int kLocItem = 64;     // queries per item of the resolve
constexpr int kLocSlices = 4;    // candidate slices per item (one thread each per query)
constexpr int kLocPad = 8;       // ints between counters: one 32-byte sector each, so that
                                 // the atomics on different chunks do not queue on one line

struct LocParams {
  unsigned long long* rowk;  // [n1] row keys, chunks of lr columns (image 2)
  unsigned long long* colk;  // [n2] column keys, chunks of lc rows (image 1)
  int64_t n1, n2;
  int lr, lc;
  int nch_r, nch;            // row chunks; all chunks (row chunks first)
  int* cnt;                  // [nch * kLocPad] queries per chunk (padded stride)
  int* start;                // [nch + 1] first list position of each chunk
  int* items;                // [nch + 1] first item of each chunk
  int* item_chunk;           // [items] the chunk of each item
  int* cursor;               // [nch * kLocPad] fill counters of the scatter (padded stride)
  uint32_t* list;            // [n1 + n2] query ids: image-1 row i, or n1 + image-2 row j
  const uint16_t* X1;        // rows of image 1 and image 2, ld elements apart
  const uint16_t* X2;
  int ld;
  int l2;                    // Euclidean forms: report -2 x the score (the squared distance)
};

__device__ __forceinline__ int loc_chunk(const LocParams& P, int64_t i) {
  if (i < P.n1) {
    int c0 = key_index(P.rowk[i]);
    if (c0 < 0 || c0 >= P.n2) c0 = 0;  // a key no candidate reached (after an abort)
    return c0 / P.lr;
  }
  int c0 = key_index(P.colk[i - P.n1]);
  if (c0 < 0 || c0 >= P.n1) c0 = 0;
  return P.nch_r + c0 / P.lc;
}

__global__ void zero_words_kernel(int* a, int64_t n) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += stride)
    a[i] = 0;
}

// The one-pass kernel's copy of a map: rows of kpad elements, the d channels
// then zeros, and NaN rows from row n to ntot.  One thread per 16-byte chunk
// of the output.
// Copies of the maps for the one-pass kernel: rows of kpad channels (zeros
// past d), then NaN rows up to ntot.  Under the Euclidean metric the first
// chunk past the channels holds, for image 1 (form kOpFormA),
//   1, 1, 1, p0, p1, p2
// and for image 2 (form kOpFormB)
//   p0, p1, p2, 1, 1, 1
// where p0 + p1 + p2 = -|row|^2/2 (the row's own norm, split greedily into
// three 16-bit parts as in prep_chunk).  The tensor cores then compute
//   q.x - |x|^2/2 - |q|^2/2 = -|q - x|^2/2
// for every pair: the largest value of a row is its nearest image-2 pixel and
// the largest of a column its nearest image-1 pixel.  On k/64 inputs every
// part and partial sum is a multiple of 2^-13 far inside fp32's range, so the
// score is exact.
constexpr int kOpFormDot = 0, kOpFormA = 1, kOpFormB = 2;
template <bool kBf16>
__device__ __forceinline__ uint4 op_aug_chunk(const uint4* __restrict__ row, int creal, int form) {
  float n2 = 0.f;
  for (int cc = 0; cc < creal; ++cc) {
    const uint4 x = __ldg(row + cc);
    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float lo = bits_to_f(static_cast<uint16_t>(w[e] & 0xFFFFu), kBf16);
      const float hi = bits_to_f(static_cast<uint16_t>(w[e] >> 16), kBf16);
      n2 = fmaf(lo, lo, n2);
      n2 = fmaf(hi, hi, n2);
    }
  }
  uint16_t part[3];
  float rest = -0.5f * n2;
#pragma unroll
  for (int e = 0; e < 3; ++e) {
    part[e] = f_to_bits(rest, kBf16);
    rest -= bits_to_f(part[e], kBf16);
  }
  const uint32_t one = f_to_bits(1.0f, kBf16);
  uint16_t h[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  for (int e = 0; e < 3; ++e) {
    h[form == kOpFormA ? e : 3 + e] = static_cast<uint16_t>(one);
    h[form == kOpFormA ? 3 + e : e] = part[e];
  }
  return make_uint4(h[0] | (static_cast<uint32_t>(h[1]) << 16),
                    h[2] | (static_cast<uint32_t>(h[3]) << 16),
                    h[4] | (static_cast<uint32_t>(h[5]) << 16),
                    h[6] | (static_cast<uint32_t>(h[7]) << 16));
}

template <bool kBf16>
__global__ void op_copy_kernel(const uint16_t* __restrict__ src, int64_t n, int d,
                               uint16_t* __restrict__ dst, int kpad, int64_t ntot, int form) {
  const int cpr = kpad / 8, creal = d / 8;
  const uint16_t nan16 = kBf16 ? 0x7FC0u : 0x7E00u;
  const uint32_t nan2 = static_cast<uint32_t>(nan16) * 0x10001u;
  const int64_t total = ntot * cpr, stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += stride) {
    const int64_t r = i / cpr;
    const int c = static_cast<int>(i - r * cpr);
    const uint4* row = reinterpret_cast<const uint4*>(src + r * d);
    uint4 v;
    if (r >= n)
      v = make_uint4(nan2, nan2, nan2, nan2);
    else if (c < creal)
      v = __ldg(row + c);
    else if (c == creal && form != kOpFormDot)
      v = op_aug_chunk<kBf16>(row, creal, form);
    else
      v = make_uint4(0u, 0u, 0u, 0u);
    reinterpret_cast<uint4*>(dst)[i] = v;
  }
}

__global__ void loc_count_kernel(LocParams P) {
  const int64_t n = P.n1 + P.n2, stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += stride) {
    atomicAdd(P.cnt + kLocPad * loc_chunk(P, i), 1);
  }
}

// One block: exclusive scans of the counts and of the items per chunk.
__global__ void loc_scan_kernel(LocParams P) {
  const int n = P.nch;
  const int per = (n + static_cast<int>(blockDim.x) - 1) / static_cast<int>(blockDim.x);
  const int b0 = threadIdx.x * per;
  int sc = 0, si = 0;
  for (int k = 0; k < per; ++k) {
    const int c = b0 + k;
    if (c < n) {
      sc += P.cnt[kLocPad * c];
      si += (P.cnt[kLocPad * c] + kLocItem - 1) / kLocItem;
    }
  }
  int tc, ti;
  int oc = block_exclusive_scan(sc, &tc);
  int oi = block_exclusive_scan(si, &ti);
  for (int k = 0; k < per; ++k) {
    const int c = b0 + k;
    if (c < n) {
      const int k = P.cnt[kLocPad * c];
      const int ni = (k + kLocItem - 1) / kLocItem;
      P.start[c] = oc;
      P.items[c] = oi;
      P.cursor[kLocPad * c] = 0;
      for (int j = 0; j < ni; ++j) P.item_chunk[oi + j] = c;
      oc += k;
      oi += ni;
    }
  }
  if (threadIdx.x == 0) {
    P.start[n] = tc;
    P.items[n] = ti;
  }
}

__global__ void loc_scatter_kernel(LocParams P) {
  const int64_t n = P.n1 + P.n2, stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += stride) {
    const int c = loc_chunk(P, i);
    P.list[P.start[c] + atomicAdd(P.cursor + kLocPad * c, 1)] = static_cast<uint32_t>(i);
  }
}

// Items are slices of at most kLocItem queries of one chunk.  The block
// stages the chunk's candidates as fp32 [len][kD] in shared memory; thread t
// takes query t % kLocItem and the candidate slice t / kLocItem, scans it in
// increasing index with a strict '>' (so it keeps the lowest index reaching
// its slice's largest recomputed score), and the slices meet in index order
// in shared memory.  The key keeps the tensor cores' maximum as its score.
template <bool kBf16, int kD>
__global__ void __launch_bounds__(kLocItem* kLocSlices) loc_resolve_kernel(LocParams P) {
  extern __shared__ float cand[];
  __shared__ float s_best[kLocSlices][kLocItem];
  __shared__ int s_idx[kLocSlices][kLocItem];
  const int total = P.items[P.nch];
  const int qt = threadIdx.x % kLocItem, slice = threadIdx.x / kLocItem;
  for (int it = blockIdx.x; it < total; it += gridDim.x) {
    const int c = P.item_chunk[it];
    const bool rows = c < P.nch_r;
    const int L = rows ? P.lr : P.lc;
    const int64_t ncand = rows ? P.n2 : P.n1;
    const int64_t c0 = static_cast<int64_t>(rows ? c : c - P.nch_r) * L;
    const int len = static_cast<int>(ncand - c0 < L ? ncand - c0 : L);
    const uint16_t* X = rows ? P.X2 : P.X1;
    __syncthreads();  // the previous item's readers are done with `cand` and the slices
    constexpr int kChunks = kD / 8;  // 16-byte pieces of a row
    for (int e = threadIdx.x; e < len * kChunks; e += blockDim.x) {
      const int r = e / kChunks, c8 = e - r * kChunks;
      const uint4 w = __ldg(reinterpret_cast<const uint4*>(X + (c0 + r) * P.ld) + c8);
      const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
      float* dst = cand + r * kD + c8 * 8;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        dst[2 * k] = h2f(static_cast<uint16_t>(ws[k] & 0xFFFFu), kBf16);
        dst[2 * k + 1] = h2f(static_cast<uint16_t>(ws[k] >> 16), kBf16);
      }
    }
    __syncthreads();
    const int q0 = P.start[c] + (it - P.items[c]) * kLocItem;
    const int qend = P.start[c] + P.cnt[kLocPad * c];
    const bool live = q0 + qt < qend;
    int64_t qi = 0;
    float best = -__int_as_float(0x7f800000);
    int bk = -1;
    if (live) {
      const uint32_t id = P.list[q0 + qt];
      qi = rows ? static_cast<int64_t>(id) : static_cast<int64_t>(id) - P.n1;
      const uint16_t* qr = (rows ? P.X1 : P.X2) + qi * P.ld;
      float qv[kD];
#pragma unroll
      for (int ch = 0; ch < kD; ch += 8) {
        const uint4 w = __ldg(reinterpret_cast<const uint4*>(qr + ch));
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          qv[ch + 2 * k] = h2f(static_cast<uint16_t>(ws[k] & 0xFFFFu), kBf16);
          qv[ch + 2 * k + 1] = h2f(static_cast<uint16_t>(ws[k] >> 16), kBf16);
        }
      }
      const int per = (len + kLocSlices - 1) / kLocSlices;
      const int k0 = slice * per, k1 = min(len, k0 + per);
      int k = k0;
      // two candidates at a time: independent sums, compared in index order;
      // the rows come from shared memory as 16-byte vectors (one broadcast
      // per four channels)
      for (; k + 2 <= k1; k += 2) {
        const float4* c0v = reinterpret_cast<const float4*>(cand + k * kD);
        const float4* c1v = reinterpret_cast<const float4*>(cand + (k + 1) * kD);
        float a0 = 0.f, a1 = 0.f;
#pragma unroll
        for (int ch = 0; ch < kD; ch += 4) {
          const float4 x0 = c0v[ch / 4], x1 = c1v[ch / 4];
          a0 = fmaf(qv[ch], x0.x, a0);
          a0 = fmaf(qv[ch + 1], x0.y, a0);
          a0 = fmaf(qv[ch + 2], x0.z, a0);
          a0 = fmaf(qv[ch + 3], x0.w, a0);
          a1 = fmaf(qv[ch], x1.x, a1);
          a1 = fmaf(qv[ch + 1], x1.y, a1);
          a1 = fmaf(qv[ch + 2], x1.z, a1);
          a1 = fmaf(qv[ch + 3], x1.w, a1);
        }
        if (a0 > best) { best = a0; bk = k; }
        if (a1 > best) { best = a1; bk = k + 1; }
      }
      for (; k < k1; ++k) {
        const float* cr = cand + k * kD;
        float acc = 0.f;
#pragma unroll
        for (int ch = 0; ch < kD; ++ch) acc = fmaf(qv[ch], cr[ch], acc);
        if (acc > best) { best = acc; bk = k; }
      }
    }
    s_best[slice][qt] = best;
    s_idx[slice][qt] = bk;
    __syncthreads();
    if (slice == 0 && live) {
      // slices in index order: a later slice wins only with a strictly larger score
#pragma unroll
      for (int sl = 1; sl < kLocSlices; ++sl) {
        if (s_idx[sl][qt] >= 0 && s_best[sl][qt] > best) {
          best = s_best[sl][qt];
          bk = s_idx[sl][qt];
        }
      }
      unsigned long long* kp = rows ? P.rowk + qi : P.colk + qi;
      const float sc = key_score(*kp);
      *kp = pack_key(P.l2 ? -2.f * sc : sc, static_cast<int>(c0 + (bk < 0 ? 0 : bk)));
    }
  }
}

// ------------------------------------------------------------------- FRM
// Options of the quoted fast_reciprocal_NNs (staskaer.github.io DUSt3R/MASt3R
// blog, MASt3R matching section) besides the grid stride: given start pixels
// (made unique and ascending), the pixel tolerance rule, the basin output;
// and the metric of its brute-force matcher.
struct FrmState {
  int* err;
  unsigned* done;   // blocks of a step kernel that finished (graph plans: last-block test)
  // Active seeds of half-step h: list[h % 2] (slots, [B][k], in no particular
  // order) and cnt[h % 3] ([B]).  The kernel of half-step h appends the
  // seeds that stay active to list[(h+1) % 2], counting in cnt[(h+1) % 3],
  // and clears cnt[(h+2) % 3] for the half-step after.
  int32_t* cnt[3];
  int32_t* nseeds;  // [B] seeds of each pair: the grid size, or its unique starts
  int32_t* U;       // [B][k]
  int32_t* V;
  int32_t* Uold;
  int32_t* Vold;
  int32_t* list[2];
  int32_t* nq;      // [B][k] queries made per seed
  uint8_t* act;     // [B][k] 1 while active
  unsigned long long* keys;  // [B][k] NN result per list position
  uint32_t* bitmap; // [B][nwords]: the start set, then the output pixels
  int32_t* partner; // [B][N1] image-2 partner of an output pixel
  int32_t* basin;   // [B][N1 + 1] or null (basin mode)
  // row forms (see prep_rows_kernel) read by the query gather and the locate
  // pass: Q* query side, X* candidate side; pair b at base + b*s1 (image 1)
  // or b*s2 (image 2), rows of ld elements
  const uint16_t* Q1;
  const uint16_t* Q2;
  const uint16_t* X1;
  const uint16_t* X2;
  int64_t s1, s2;
  int ld;
  float pixel_tol;  // > 0: converged when the move from U_old is below it
  int starts;       // 1: the seeds were given (output U_old with pixel_tol)
  const int32_t* pair_on;  // [B] or null: grid seeds only for the pairs marked 1
  int32_t* mcounts; // [B][mblocks] output pixels per bitmap block (merge)
  int B, k, N1, N2, nwords, mblocks;
};

// Merge: threads of its kernels, and bitmap words per block of its count and
// emit kernels (one word per thread).
constexpr int kMergeThreads = 256;

// Row-form copies a call needs: none, one padded copy per map (dot metric,
// d short of the K-block layout), or a query and a candidate form per map
// (Euclidean metric).
enum { kCopiesNone = 0, kCopiesPad = 1, kCopiesEuclid = 2 };

static int copies_for(int d, rnn_metric metric) {
  if (metric == RNN_L2) return kCopiesEuclid;
  return padded_depth(d) != d ? kCopiesPad : kCopiesNone;
}

// K of the tensor-core tiles: the channels, plus the Euclidean augmentation.
static int tile_depth(int d, rnn_metric metric) {
  return padded_depth(d + (metric == RNN_L2 ? kAugCols : 0));
}

struct FrmCopies {
  uint16_t *q1, *x1, *q2, *x2;  // null when not needed (x* alias q* with kCopiesPad)
};

// Workspace layout of a batched FRM call; returns the bytes it needs.
static size_t frm_layout(void* ws, int B, int64_t k, int64_t N1, int64_t N2, int d,
                         rnn_metric metric, FrmState* st, FrmCopies* cp) {
  Carve c(ws);
  st->err = c.take<int>(64);
  st->done = c.take<unsigned>(1);
  for (int i = 0; i < 3; ++i) st->cnt[i] = c.take<int32_t>(B);
  st->nseeds = c.take<int32_t>(B);
  const int64_t kk = k > 0 ? k : 1;
  st->U = c.take<int32_t>(B * kk);
  st->V = c.take<int32_t>(B * kk);
  st->Uold = c.take<int32_t>(B * kk);
  st->Vold = c.take<int32_t>(B * kk);
  for (int i = 0; i < 2; ++i) st->list[i] = c.take<int32_t>(B * kk);
  st->nq = c.take<int32_t>(B * kk);
  st->act = c.take<uint8_t>(B * kk);
  st->keys = c.take<unsigned long long>(B * kk);
  const int64_t nwords = (N1 + 31) / 32;
  st->bitmap = c.take<uint32_t>(B * nwords);
  st->partner = c.take<int32_t>(B * N1);
  const int64_t mblocks = (nwords + kMergeThreads - 1) / kMergeThreads;
  st->mcounts = c.take<int32_t>(B * mblocks);
  const int mode = d > 0 ? copies_for(d, metric) : kCopiesNone;  // d = 0: point maps
  cp->q1 = cp->x1 = cp->q2 = cp->x2 = nullptr;
  if (mode != kCopiesNone) {
    const int kpad = tile_depth(d, metric);
    cp->q1 = c.take<uint16_t>(B * N1 * kpad);
    cp->q2 = c.take<uint16_t>(B * N2 * kpad);
    cp->x1 = cp->q1;
    cp->x2 = cp->q2;
    if (mode == kCopiesEuclid) {
      cp->x1 = c.take<uint16_t>(B * N1 * kpad);
      cp->x2 = c.take<uint16_t>(B * N2 * kpad);
    }
  }
  st->B = B;
  st->k = static_cast<int>(k);
  st->N1 = static_cast<int>(N1);
  st->N2 = static_cast<int>(N2);
  st->nwords = static_cast<int>(nwords);
  st->mblocks = static_cast<int>(mblocks);
  st->basin = nullptr;
  st->pair_on = nullptr;
  return c.off;
}

static size_t frm_bytes(int B, int64_t k, int64_t N1, int64_t N2, int d, rnn_metric metric) {
  FrmState st;
  FrmCopies cp;
  return frm_layout(nullptr, B, k, N1, N2, d, metric, &st, &cp);
}

// Per-seed state of slot s holding pixel u (u < 0: an unused slot).
__device__ __forceinline__ void frm_seed_init(const FrmState& st, int64_t t, int s, int32_t u) {
  st.U[t] = u;
  st.Uold[t] = u;
  st.V[t] = -1;
  st.Vold[t] = -1;
  st.list[0][t] = s;
  st.nq[t] = 0;
  st.act[t] = u >= 0 ? 1 : 0;
  st.keys[t] = 0ull;
}

// Grid seeds (stride S), the converged-pixel bitmap, the basin array.
__global__ void frm_init_kernel(FrmState st, int W1, int S) {
  const int x0 = S / 2;
  const int nx = W1 > x0 ? (W1 - x0 + S - 1) / S : 0;
  const int64_t nseed = static_cast<int64_t>(st.B) * st.k;
  const int64_t nbits = static_cast<int64_t>(st.B) * st.nwords;
  const int64_t nbasin = st.basin ? static_cast<int64_t>(st.B) * (st.N1 + 1) : 0;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t t = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
       t < nseed + nbits + nbasin; t += stride) {
    if (t < nseed) {
      const int s = static_cast<int>(t % st.k);
      const int iy = s / nx, ix = s - (s / nx) * nx;
      frm_seed_init(st, t, s, (x0 + iy * S) * W1 + (x0 + ix * S));
    } else if (t < nseed + nbits) {
      st.bitmap[t - nseed] = 0u;
    } else {
      st.basin[t - nseed - nbits] = -1;
    }
  }
  if (blockIdx.x == 0) {
    for (int b = threadIdx.x; b < st.B; b += blockDim.x) {
      const int k = st.pair_on && !st.pair_on[b] ? 0 : st.k;
      st.cnt[0][b] = k;
      st.cnt[1][b] = 0;
      st.nseeds[b] = k;
    }
    if (threadIdx.x == 0) {
      *st.err = 0;
      *st.done = 0u;
    }
  }
}

// Given start pixels, step 1: clear the bitmaps and the basin array.
__global__ void frm_starts_clear_kernel(FrmState st) {
  const int64_t nbits = static_cast<int64_t>(st.B) * st.nwords;
  const int64_t nbasin = st.basin ? static_cast<int64_t>(st.B) * (st.N1 + 1) : 0;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t t = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
       t < nbits + nbasin; t += stride) {
    if (t < nbits) st.bitmap[t] = 0u;
    else st.basin[t - nbits] = -1;
  }
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    *st.err = 0;
    *st.done = 0u;
  }
}

// Step 2: mark every start in its pair's bitmap (starts outside the image
// are ignored), which makes them unique.
__global__ void frm_starts_mark_kernel(FrmState st, const int32_t* init, int64_t n_init) {
  const int64_t n = static_cast<int64_t>(st.B) * n_init;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t t = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; t < n;
       t += stride) {
    const int64_t b = t / n_init;
    const int32_t u = init[t];
    if (u >= 0 && u < st.N1)
      atomicOr(st.bitmap + b * st.nwords + (u >> 5), 1u << (u & 31));
  }
}

// Step 3 (one CTA per pair): the marked pixels in increasing order become
// the seeds; the bitmap is cleared again for the merge.
__global__ void frm_starts_compact_kernel(FrmState st) {
  const int b = blockIdx.x;
  uint32_t* bm = st.bitmap + static_cast<int64_t>(b) * st.nwords;
  const int per = (st.nwords + blockDim.x - 1) / blockDim.x;
  const int w0 = threadIdx.x * per;
  const int w1 = min(st.nwords, w0 + per);
  int c = 0;
  for (int w = w0; w < w1; ++w) c += __popc(bm[w]);
  int tot;
  int pos = block_exclusive_scan(c, &tot);
  const int64_t base = static_cast<int64_t>(b) * st.k;
  for (int w = w0; w < w1; ++w) {
    uint32_t bits = bm[w];
    bm[w] = 0u;
    while (bits) {
      const int bit = __ffs(bits) - 1;
      bits &= bits - 1;
      frm_seed_init(st, base + pos, pos, w * 32 + bit);
      ++pos;
    }
  }
  // unused slots (duplicated or out-of-image starts)
  for (int s = tot + threadIdx.x; s < st.k; s += blockDim.x) frm_seed_init(st, base + s, s, -1);
  if (threadIdx.x == 0) {
    st.cnt[0][b] = tot;
    st.cnt[1][b] = 0;
    st.nseeds[b] = tot;
  }
}

// Result j of a half-step for seed slot s of pair b: store the NN found,
// apply the convergence test, refresh the old copies at the end of an
// iteration, and append the seed to the next list if it stays active.  In
// basin mode the NN2 half-step deactivates no one and the NN1 half-step
// records basin[U_old] = U for every seed it served.  A seed's result does not
// depend on its place in the list, so the order in which the appends land
// changes nothing.
__device__ __forceinline__ void frm_apply(const FrmState& st, int b, int64_t base, int s, int j,
                                          int nn2_half, int last_iter, int32_t* list_out,
                                          int32_t* cnt_out) {
  st.nq[base + s] += 1;
  int still;
  if (nn2_half) {
    st.V[base + s] = j;
    still = st.basin ? 1 : j != st.Vold[base + s];
  } else {
    st.U[base + s] = j;
    if (st.basin) st.basin[static_cast<int64_t>(b) * (st.N1 + 1) + st.Uold[base + s]] = j;
    still = j != st.Uold[base + s];
    if (still && !last_iter) {
      st.Uold[base + s] = j;
      st.Vold[base + s] = st.V[base + s];
    }
  }
  if (still) list_out[base + atomicAdd(cnt_out + b, 1)] = s;
  else st.act[base + s] = 0;
}

// Result of half-step h for every active seed of every pair (one warp per
// seed): the warp resolves the exact index inside the kept chunk (NN2
// queries are rows U of image 1 against image 2, NN1 queries rows V of image
// 2 against image 1, in the row forms the tensor cores read), then lane 0
// applies it (frm_apply).
template <bool kBf16>
__global__ void frm_step_kernel(FrmState st, int h, int nn2_half, int last_iter,
                                cudaGraphConditionalHandle next) {
  pdl_wait();
  pdl_trigger();
  const int32_t* cnt_in = st.cnt[h % 3];
  int32_t* cnt_out = st.cnt[(h + 1) % 3];
  const int32_t* list_in = st.list[h % 2];
  int32_t* list_out = st.list[(h + 1) % 2];
  if (blockIdx.x == 0) {
    int32_t* cnt_next = st.cnt[(h + 2) % 3];
    for (int b = threadIdx.x; b < st.B; b += blockDim.x) cnt_next[b] = 0;
  }
  const int64_t w0 = (blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x) >> 5;
  const int64_t nw = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  const int n_cand = nn2_half ? st.N2 : st.N1;
  const int32_t* rows = nn2_half ? st.U : st.V;
  // The active seeds of all pairs as one range: prefix of the counts over
  // the pairs (one per thread; B <= blockDim.x), so that the warps visit only
  // active seeds and a launch with none ends after the scan.  Above 2^31 slots
  // in all, the warps visit every slot instead.
  __shared__ int s_pref[kSmallThreads + 1];
  const bool compact = static_cast<int64_t>(st.B) * st.k < INT32_MAX;
  int64_t n_items = static_cast<int64_t>(st.B) * st.k;
  if (compact) {
    int total;
    const int c = static_cast<int>(threadIdx.x) < st.B ? cnt_in[threadIdx.x] : 0;
    const int ex = block_exclusive_scan(c, &total);
    if (static_cast<int>(threadIdx.x) < st.B) s_pref[threadIdx.x] = ex;
    if (threadIdx.x == 0) s_pref[st.B] = total;
    __syncthreads();
    n_items = total;
  }
  for (int64_t x = w0; x < n_items; x += nw) {
    int b, i;
    if (compact) {
      // the last pair whose first active seed is at or before x
      int lo = 0, hi = st.B;  // s_pref[lo] <= x < s_pref[hi]
      while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (s_pref[mid] <= x) lo = mid; else hi = mid;
      }
      b = lo;
      i = static_cast<int>(x - s_pref[lo]);
    } else {
      b = static_cast<int>(x / st.k);
      i = static_cast<int>(x - static_cast<int64_t>(b) * st.k);
      if (i >= cnt_in[b]) continue;
    }
    const int64_t base = static_cast<int64_t>(b) * st.k;
    const uint16_t* Dq = nn2_half ? st.Q1 + b * st.s1 : st.Q2 + b * st.s2;
    const uint16_t* Dx = nn2_half ? st.X2 + b * st.s2 : st.X1 + b * st.s1;
    const int s = list_in[base + i];
    const unsigned long long key = st.keys[base + i];
    const int64_t qr = rows[base + s];
    const int j = locate_chunk<kBf16>(Dq + qr * st.ld, Dx, n_cand, st.ld, key_index(key));
    if ((threadIdx.x & 31) == 0) {
      st.keys[base + i] = 0ull;
      frm_apply(st, b, base, s, j, nn2_half, last_iter, list_out, cnt_out);
    }
  }
  if (next) {
    // graph plans: the last block to finish enables the next iteration's
    // conditional node when some seed of some pair is still active
    __shared__ int s_last;
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) s_last = atomicAdd(st.done, 1u) == gridDim.x - 1;
    __syncthreads();
    if (s_last && threadIdx.x == 0) {
      __threadfence();
      int any = 0;
      for (int b = 0; b < st.B; ++b) any |= __ldcg(cnt_out + b) > 0;
      cudaGraphSetConditional(next, any ? 1u : 0u);
      *st.done = 0u;
    }
  }
}

// Unique output pairs of every pair, sorted by the image-1 pixel, in three
// kernels over many blocks (the pairs on grid.y).  A seed is in the output
// when it is no longer active, or, with a pixel tolerance, when its last move
// (U_old -> U) is shorter than the tolerance; the pair is (U, V), or
// (U_old, V) with a tolerance and given starts.  An output pixel determines
// its partner (a mutual pair, or a start's match), so a bitmap over image 1
// de-duplicates and sorts.
//
// Mark: one thread per seed slot marks its output pixel in the bitmap,
// writes the partner, and fills the seed state.
__global__ void frm_mark_kernel(FrmState st, int W1, int32_t* seed_state) {
  pdl_wait();
  pdl_trigger();
  const int b = blockIdx.y;
  const int s = blockIdx.x * blockDim.x + threadIdx.x;
  if (s >= st.k) return;
  const int64_t base = static_cast<int64_t>(b) * st.k;
  const int ns = st.nseeds[b];
  int conv = 0;
  int32_t u = -1, v = -1;
  if (s < ns) {
    u = st.U[base + s];
    v = st.V[base + s];
    int32_t uo = u;
    if (st.pixel_tol > 0.f) {
      const int32_t u0 = st.Uold[base + s];
      // in double, as the distance is written down
      const double dy = static_cast<double>(u0 / W1 - u / W1);
      const double dx = static_cast<double>(u0 % W1 - u % W1);
      conv = sqrt(dy * dy + dx * dx) < static_cast<double>(st.pixel_tol);
      if (st.starts) uo = u0;
    } else {
      conv = st.act[base + s] == 0;
    }
    if (conv) {
      atomicOr(st.bitmap + static_cast<int64_t>(b) * st.nwords + (uo >> 5), 1u << (uo & 31));
      st.partner[static_cast<int64_t>(b) * st.N1 + uo] = v;
    }
  }
  if (seed_state) {
    int32_t* o = seed_state + (base + s) * 4;
    o[0] = u;
    o[1] = v;
    o[2] = s < ns ? st.nq[base + s] : 0;
    o[3] = conv;
  }
}

// Count: output pixels in each block of kMergeThreads bitmap words.
__global__ void frm_count_kernel(FrmState st) {
  pdl_wait();
  pdl_trigger();
  const int b = blockIdx.y;
  const int w = blockIdx.x * kMergeThreads + threadIdx.x;
  const int c = w < st.nwords ? __popc(st.bitmap[static_cast<int64_t>(b) * st.nwords + w]) : 0;
  int tot;
  (void)block_exclusive_scan(c, &tot);
  if (threadIdx.x == 0) st.mcounts[static_cast<int64_t>(b) * st.mblocks + blockIdx.x] = tot;
}

// Emit: each block writes (pixel, partner) for its words from its offset in
// the pair's output; the last block of a pair writes the pair's count.
__global__ void frm_emit_kernel(FrmState st, int32_t* pairs, int64_t cap, int32_t* count_out) {
  pdl_wait();
  const int b = blockIdx.y;
  const int32_t* mc = st.mcounts + static_cast<int64_t>(b) * st.mblocks;
  int part = 0;
  for (int j = threadIdx.x; j < static_cast<int>(blockIdx.x); j += kMergeThreads) part += mc[j];
  int off;
  (void)block_exclusive_scan(part, &off);
  const int w = blockIdx.x * kMergeThreads + threadIdx.x;
  uint32_t bits = w < st.nwords ? st.bitmap[static_cast<int64_t>(b) * st.nwords + w] : 0u;
  int btot;
  int pos = off + block_exclusive_scan(__popc(bits), &btot);
  int32_t* out = pairs + static_cast<int64_t>(b) * cap * 2;
  const int32_t* partner = st.partner + static_cast<int64_t>(b) * st.N1;
  while (bits) {
    const int bit = __ffs(bits) - 1;
    bits &= bits - 1;
    const int u = w * 32 + bit;
    out[2 * static_cast<int64_t>(pos)] = u;
    out[2 * static_cast<int64_t>(pos) + 1] = partner[u];
    ++pos;
  }
  if (blockIdx.x == gridDim.x - 1 && threadIdx.x == 0) count_out[b] = off + btot;
}

}  // namespace rnn

// 3-D point kernels (they use FrmState, frm_apply and block_exclusive_scan)
#include "points.cuh"
// coarse-to-fine kernels (they use block_exclusive_scan)
#include "c2f.cuh"

namespace rnn {

static int grid_for(int64_t n, int sms) {
  int64_t g = (n + kSmallThreads - 1) / kSmallThreads;
  if (g > 4LL * sms) g = 4LL * sms;
  if (g < 1) g = 1;
  return static_cast<int>(g);
}

// The three merge launches (mark, count, emit) of a batched FRM call.
static rnn_status frm_merge(const FrmState& st, int W1, int32_t* pairs, int64_t cap,
                            int32_t* count_out, int32_t* seed_state, cudaStream_t s, bool pdl) {
  const unsigned B = static_cast<unsigned>(st.B);
  const dim3 blk(kMergeThreads);
  launch_k(frm_mark_kernel, dim3((st.k + kMergeThreads - 1) / kMergeThreads, B), blk, 0, s, pdl,
           st, W1, seed_state);
  rnn_status r = launched();
  if (r != RNN_OK) return r;
  launch_k(frm_count_kernel, dim3(st.mblocks, B), blk, 0, s, pdl, st);
  if ((r = launched()) != RNN_OK) return r;
  launch_k(frm_emit_kernel, dim3(st.mblocks, B), blk, 0, s, pdl, st, pairs, cap, count_out);
  return launched();
}

static rnn_status frm_step(const FrmState& st, int h, int nn2_half, int last_iter,
                           rnn_dtype dt, int grid, cudaStream_t s,
                           cudaGraphConditionalHandle next = 0, bool pdl = false) {
  if (dt == RNN_BF16)
    launch_k(frm_step_kernel<true>, dim3(grid), dim3(kSmallThreads), 0, s, pdl, st, h, nn2_half,
             last_iter, next);
  else
    launch_k(frm_step_kernel<false>, dim3(grid), dim3(kSmallThreads), 0, s, pdl, st, h, nn2_half,
             last_iter, next);
  return launched();
}

static int64_t num_seeds(int H, int W, int S) {
  const int o = S / 2;
  const int64_t ny = H > o ? (H - o + S - 1) / S : 0;
  const int64_t nx = W > o ? (W - o + S - 1) / S : 0;
  return ny * nx;
}

// One launch of the row-form preparation over [nbatch][rows][d] maps.
static rnn_status prep_rows(const void* src, int64_t bstride, int64_t rows, int nbatch, int d,
                            uint16_t* dst, int kpad, int form, rnn_dtype dt, DeviceInfo* di,
                            cudaStream_t s) {
  // the same number of threads as one 1-D grid over all maps, split evenly
  const int64_t per = rows * (kpad / 8);
  const int g1 = grid_for(per * nbatch, di->sms);
  const dim3 grid(static_cast<unsigned>(std::max<int64_t>(
                      1, std::min<int64_t>((g1 + nbatch - 1) / nbatch,
                                           (per + kSmallThreads - 1) / kSmallThreads))),
                  static_cast<unsigned>(nbatch));
  const uint16_t* in = static_cast<const uint16_t*>(src);
  auto go = [&](auto kernel) {
    kernel<<<grid, kSmallThreads, 0, s>>>(in, bstride, rows, d, dst, kpad, form);
  };
  const int cpr = kpad / 8;
  if (dt == RNN_BF16) {
    if (cpr == 4) go(prep_rows_kernel<true, 4>);
    else if (cpr == 8) go(prep_rows_kernel<true, 8>);
    else go(prep_rows_kernel<true, 0>);
  } else {
    if (cpr == 4) go(prep_rows_kernel<false, 4>);
    else if (cpr == 8) go(prep_rows_kernel<false, 8>);
    else go(prep_rows_kernel<false, 0>);
  }
  return launched();
}

// Seeds of every pair: the grid of stride S, or the given starts made
// unique and ascending; state, bitmaps and basin array cleared.
static rnn_status frm_seed(const FrmState& st, const int32_t* init, int64_t n_init, int W1,
                           int S, DeviceInfo* di, cudaStream_t s) {
  const int64_t B = st.B, k = st.k;
  const int64_t nbasin = st.basin ? B * (static_cast<int64_t>(st.N1) + 1) : 0;
  rnn_status r;
  if (init) {
    frm_starts_clear_kernel<<<grid_for(B * st.nwords + nbasin, di->sms), kSmallThreads, 0, s>>>(
        st);
    if ((r = launched()) != RNN_OK) return r;
    if (n_init > 0) {
      frm_starts_mark_kernel<<<grid_for(B * n_init, di->sms), kSmallThreads, 0, s>>>(st, init,
                                                                                    n_init);
      if ((r = launched()) != RNN_OK) return r;
    }
    frm_starts_compact_kernel<<<static_cast<int>(B), kSmallThreads, 0, s>>>(st);
  } else {
    frm_init_kernel<<<grid_for(B * k + B * st.nwords + nbasin, di->sms), kSmallThreads, 0, s>>>(
        st, W1, S);
  }
  return launched();
}

// The FRM loop over B pairs with every option; frm entry points call it.
static rnn_status frm_run(int B, const void* D1, int64_t bs1, const void* D2, int64_t bs2, int H1,
                          int W1, int H2, int W2, int d, rnn_dtype dt, rnn_metric metric,
                          const int32_t* init, int64_t n_init, int S, int max_iter,
                          float pixel_tol, int32_t* pairs, int64_t cap, int32_t* count_out,
                          int32_t* seed_state, int32_t* basin, void* ws, size_t ws_bytes,
                          cudaStream_t s, const int32_t* pair_on = nullptr,
                          cudaStream_t body_stream = nullptr) {
  // body_stream non-null: `s` is capturing a graph plan; iterations 2..max_iter
  // go into conditional (if) nodes, each enabled by the previous iteration's
  // last step kernel when a seed is still active, and captured on body_stream.
  // A call that the caller captures into a graph does the same on this
  // thread's body stream, when it has one.
  NvtxRange nvtx_range("rnn_frm_match");
  const bool own_plan = body_stream != nullptr;
  if (B < 1) return RNN_EINVAL;
  if (B > RNN_MAX_BATCH) return RNN_EUNSUPPORTED;
  if (H1 <= 0 || W1 <= 0 || H2 <= 0 || W2 <= 0 || max_iter < 1) return RNN_EINVAL;
  if (!valid_dtype(dt) || !valid_metric(metric)) return RNN_EINVAL;
  if (pair_on && init) return RNN_EINVAL;  // per-pair enable is for grid seeds
  if (init ? n_init < 0 : S < 1) return RNN_EINVAL;
  if (!(pixel_tol >= 0.f) || (pixel_tol > 0.f && !init)) return RNN_EINVAL;
  rnn_status st0 = check_desc(D1, d);
  if (st0 != RNN_OK) return st0;
  st0 = check_desc(D2, d);
  if (st0 != RNN_OK) return st0;
  const int64_t N1 = static_cast<int64_t>(H1) * W1, N2 = static_cast<int64_t>(H2) * W2;
  if (N1 >= INT32_MAX || N2 > INT32_MAX) return RNN_EINVAL;
  if (bs1 < N1 * d || bs2 < N2 * d || bs1 % 8 != 0 || bs2 % 8 != 0) return RNN_EINVAL;
  if (!pairs || !count_out) return RNN_EINVAL;
  const int64_t k = init ? n_init : num_seeds(H1, W1, S);
  if (k > INT32_MAX) return RNN_EINVAL;
  // outputs are mutual pairs (distinct V), except (start, match) pairs under
  // a pixel tolerance, where only the starts are distinct
  const int64_t need = pixel_tol > 0.f ? k : (k < N2 ? k : N2);
  if (cap < need) return RNN_ECAPACITY;
  if (!ws || !aligned256(ws) || ws_bytes < frm_bytes(B, k, N1, N2, d, metric))
    return RNN_EWORKSPACE;
  DeviceInfo* di = nullptr;
  rnn_status r = device_info(&di);
  if (r != RNN_OK) return r;
  bool caller_capture = false;
  if (!body_stream) {
    int dev = 0;
    cudaStreamCaptureStatus cst = cudaStreamCaptureStatusNone;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return RNN_ECUDA;
    if (cudaStreamIsCapturing(s, &cst) != cudaSuccess) {
      cudaGetLastError();
      cst = cudaStreamCaptureStatusNone;
    }
    if (cst == cudaStreamCaptureStatusActive) {
      body_stream = max_iter <= kMaxGraphIters ? t_body[dev] : nullptr;
      caller_capture = true;
    } else if (!t_body[dev] &&
               cudaStreamCreateWithFlags(&t_body[dev], cudaStreamNonBlocking) != cudaSuccess) {
      t_body[dev] = nullptr;  // no body stream: captures record every iteration
      cudaGetLastError();
    }
  }
  // recorded into the caller's graph: the launches are neither counted nor timed
  struct CaptureFlag {
    bool on, prev;
    explicit CaptureFlag(bool o) : on(o), prev(t_capturing) {
      if (on) t_capturing = true;
    }
    ~CaptureFlag() {
      if (on) t_capturing = prev;
    }
  } capture_flag(caller_capture);
  // programmatic dependent launches along the chain of FRM kernels, on a
  // stream or recorded into a graph plan (a caller's capture records plain
  // launches)
  const bool pdl = RNN_PDL && (own_plan || !t_capturing);

  FrmState st;
  FrmCopies cp;
  frm_layout(ws, B, k, N1, N2, d, metric, &st, &cp);
  st.basin = basin;
  st.pixel_tol = pixel_tol;
  st.starts = init ? 1 : 0;
  st.pair_on = pair_on;
  const Geometry g = geometry(d + (metric == RNN_L2 ? kAugCols : 0));
  const int mode = copies_for(d, metric);
  if (k == 0) {
    // no seeds: every count is zero (the basin, if asked for, untouched pixels)
    if (cudaMemsetAsync(count_out, 0, sizeof(int32_t) * B, s) != cudaSuccess) return RNN_ECUDA;
    if (cudaMemsetAsync(st.err, 0, sizeof(int), s) != cudaSuccess) return RNN_ECUDA;
    if (basin && cudaMemsetAsync(basin, 0xFF, sizeof(int32_t) * B * (N1 + 1), s) != cudaSuccess)
      return RNN_ECUDA;
    return RNN_OK;
  }
  if (mode == kCopiesNone) {
    st.Q1 = st.X1 = static_cast<const uint16_t*>(D1);
    st.Q2 = st.X2 = static_cast<const uint16_t*>(D2);
    st.s1 = bs1;
    st.s2 = bs2;
    st.ld = d;
  } else {
    const int qform = mode == kCopiesEuclid ? kFormQuery : kFormPad;
    if ((r = prep_rows(D1, bs1, N1, B, d, cp.q1, g.kpad, qform, dt, di, s)) != RNN_OK) return r;
    if ((r = prep_rows(D2, bs2, N2, B, d, cp.q2, g.kpad, qform, dt, di, s)) != RNN_OK) return r;
    if (mode == kCopiesEuclid) {
      if ((r = prep_rows(D1, bs1, N1, B, d, cp.x1, g.kpad, kFormCand, dt, di, s)) != RNN_OK)
        return r;
      if ((r = prep_rows(D2, bs2, N2, B, d, cp.x2, g.kpad, kFormCand, dt, di, s)) != RNN_OK)
        return r;
    }
    st.Q1 = cp.q1;
    st.Q2 = cp.q2;
    st.X1 = cp.x1;
    st.X2 = cp.x2;
    st.s1 = N1 * g.kpad;
    st.s2 = N2 * g.kpad;
    st.ld = g.kpad;
  }
  CUtensorMap map1, map2;
  if ((r = make_map(&map1, st.X1, st.ld, N1, B, st.s1, g)) != RNN_OK) return r;
  if ((r = make_map(&map2, st.X2, st.ld, N2, B, st.s2, g)) != RNN_OK) return r;

  if ((r = frm_seed(st, init, n_init, W1, S, di, s)) != RNN_OK) return r;
  // the step kernels: one resident wave (two blocks of 1024 a SM) at most
  const int lgrid = std::min(grid_for(static_cast<int64_t>(B) * k * 32, di->sms), 2 * di->sms);

  NNParams p;
  std::memset(&p, 0, sizeof(p));
  p.nfam = 1;
  p.d = st.ld;  // the gather copies whole rows of the forms
  p.idesc = make_idesc(dt, g.block_n);
  p.err = st.err;
  NNFamily& F = p.fam[0];
  F.slot_bstride = k;

  F.nbatch = B;
  F.keys = st.keys;
  F.key_bstride = k;
  // one iteration (two half-steps) on stream q; the NN1 step enables `next`
  auto iteration = [&](int it, cudaStream_t q, cudaGraphConditionalHandle next) -> rnn_status {
    const int h = 2 * (it - 1);
    rnn_status e;
    // half-step 1: V = NN2(U)
    F.q_list = st.list[h % 2];
    F.q_count_dev = st.cnt[h % 3];
    F.q_base = st.Q1;
    F.q_bstride = st.s1;
    F.q_index = st.U;
    F.n_cand = static_cast<int32_t>(N2);
    if ((e = launch_nn(p, map2, map2, map2, map2, g, di, q, pdl)) != RNN_OK) return e;
    if ((e = frm_step(st, h, 1, 0, dt, lgrid, q, 0, pdl)) != RNN_OK) return e;
    // half-step 2: U = NN1(V)
    F.q_list = st.list[(h + 1) % 2];
    F.q_count_dev = st.cnt[(h + 1) % 3];
    F.q_base = st.Q2;
    F.q_bstride = st.s2;
    F.q_index = st.V;
    F.n_cand = static_cast<int32_t>(N1);
    if ((e = launch_nn(p, map1, map1, map1, map1, g, di, q, pdl)) != RNN_OK) return e;
    return frm_step(st, h + 1, 0, it == max_iter ? 1 : 0, dt, lgrid, q, next, pdl);
  };
  if (!body_stream) {
    for (int it = 1; it <= max_iter; ++it)
      if ((r = iteration(it, s, 0)) != RNN_OK) return r;
  } else {
    cudaStreamCaptureStatus cst;
    cudaGraph_t cg = nullptr;
    if (cudaStreamGetCaptureInfo(s, &cst, nullptr, &cg, nullptr, nullptr) != cudaSuccess ||
        cst != cudaStreamCaptureStatusActive || !cg)
      return RNN_ECUDA;
    // condition handles of iterations 2..max_iter (0 unless enabled this launch)
    cudaGraphConditionalHandle hnd[kMaxGraphIters + 1] = {};
    for (int it = 2; it <= max_iter; ++it)
      if (cudaGraphConditionalHandleCreate(&hnd[it], cg, 0, cudaGraphCondAssignDefault) !=
          cudaSuccess)
        return RNN_ECUDA;
    if ((r = iteration(1, s, max_iter > 1 ? hnd[2] : 0)) != RNN_OK) return r;
    for (int it = 2; it <= max_iter; ++it) {
      const cudaGraphNode_t* deps = nullptr;
      size_t ndeps = 0;
      if (cudaStreamGetCaptureInfo(s, &cst, nullptr, nullptr, &deps, &ndeps) != cudaSuccess)
        return RNN_ECUDA;
      // the params union has no default constructor: zeroed storage instead
      alignas(cudaGraphNodeParams) unsigned char cp_raw[sizeof(cudaGraphNodeParams)] = {};
      cudaGraphNodeParams& cp = *reinterpret_cast<cudaGraphNodeParams*>(cp_raw);
      cp.type = cudaGraphNodeTypeConditional;
      cp.conditional.handle = hnd[it];
      cp.conditional.type = cudaGraphCondTypeIf;
      cp.conditional.size = 1;
      cudaGraphNode_t node;
      if (cudaGraphAddNode(&node, cg, deps, ndeps, &cp) != cudaSuccess) return RNN_ECUDA;
      if (cudaStreamUpdateCaptureDependencies(s, &node, 1, cudaStreamSetCaptureDependencies) !=
          cudaSuccess)
        return RNN_ECUDA;
      if (cudaStreamBeginCaptureToGraph(body_stream, cp.conditional.phGraph_out[0], nullptr,
                                        nullptr, 0, cudaStreamCaptureModeThreadLocal) !=
          cudaSuccess)
        return RNN_ECUDA;
      r = iteration(it, body_stream, it < max_iter ? hnd[it + 1] : 0);
      cudaGraph_t body;
      const cudaError_t ce = cudaStreamEndCapture(body_stream, &body);
      if (r != RNN_OK) return r;
      if (ce != cudaSuccess) return RNN_ECUDA;
    }
  }
  return frm_merge(st, W1, pairs, cap, count_out, seed_state, s, pdl);
}

// ------------------------------------------------------------- 3-D points
constexpr int64_t kPtsMaxSet = 1 << 28;  // points per set

struct PtsWs {
  float* part;      // [nblocks][6] block bounding boxes
  PtsGrid* grids;   // [nsets]
  int32_t* start;   // [nstart] cell counts, then the first sorted point of each cell
  int32_t* cell;    // [npts] global cell of each point
  int32_t* rank;    // [npts] its rank in the cell
  int32_t* seg;     // [nseg] segment sums of the prefix sum
  float4* sorted;   // [npts] (x, y, z, index bits) in cell order
  int64_t nstart = 0, npts = 0;
  int nblocks = 0, nseg = 0;
};

// nb sets of n0 points (family 0) and, with nfam = 2, nb sets of n1 points.
static PtsSets pts_sets(const float* b0, int64_t s0, int64_t n0, const float* b1, int64_t s1,
                        int64_t n1, int nb, int nfam) {
  PtsSets ps;
  std::memset(&ps, 0, sizeof(ps));
  ps.nb = nb;
  ps.nfam = nfam;
  const float* base[2] = {b0, b1};
  const int64_t bs[2] = {s0, s1}, n[2] = {n0, n1};
  for (int f = 0; f < nfam; ++f) {
    ps.base[f] = base[f];
    ps.bstride[f] = bs[f];
    ps.n[f] = static_cast<int>(n[f]);
    ps.cap[f] = static_cast<int>(2 * n[f] + 64);
    ps.blk[f] = static_cast<int>((n[f] + kPtsChunk - 1) / kPtsChunk);
  }
  return ps;
}

static size_t pts_layout(Carve& c, const PtsSets& ps, PtsWs* w) {
  int64_t cells = 0, npts = 0, nblocks = 0;
  for (int f = 0; f < ps.nfam; ++f) {
    cells += static_cast<int64_t>(ps.nb) * ps.cap[f];
    npts += static_cast<int64_t>(ps.nb) * ps.n[f];
    nblocks += static_cast<int64_t>(ps.nb) * ps.blk[f];
  }
  w->nstart = cells + 1;
  w->npts = npts;
  w->nblocks = static_cast<int>(nblocks);
  w->nseg = static_cast<int>((w->nstart + kScanSeg - 1) / kScanSeg);
  w->part = c.take<float>(6 * nblocks);
  w->grids = c.take<PtsGrid>(pts_nsets(ps));
  w->start = c.take<int32_t>(w->nstart);
  w->cell = c.take<int32_t>(npts);
  w->rank = c.take<int32_t>(npts);
  w->seg = c.take<int32_t>(w->nseg);
  w->sorted = c.take<float4>(npts);
  return c.off;
}

// Sizes the shared arrays can index (int32 cells and sorted positions).
static bool pts_fits(const PtsSets& ps) {
  PtsWs w;
  Carve c(nullptr);
  pts_layout(c, ps, &w);
  return w.nstart <= INT32_MAX && w.npts <= INT32_MAX;
}

static bool pts_ptr_ok(const float* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

// Grids of every set: bounds, cells and ranks, prefix sum, scatter.
static rnn_status pts_build(const PtsSets& ps, const PtsWs& w, int* err, DeviceInfo* di,
                            cudaStream_t s) {
  rnn_status r;
  pts_bounds_kernel<<<w.nblocks, kPtsThreads, 0, s>>>(ps, w.part, w.start, w.nstart, err);
  if ((r = launched()) != RNN_OK) return r;
  pts_count_kernel<<<w.nblocks, kPtsThreads, 0, s>>>(ps, w.part, w.grids, w.start, w.cell,
                                                     w.rank);
  if ((r = launched()) != RNN_OK) return r;
  pts_scan_sum_kernel<<<w.nseg, kScanThreads, 0, s>>>(w.start, w.nstart, w.seg);
  if ((r = launched()) != RNN_OK) return r;
  pts_scan_seg_kernel<<<1, kScanThreads, 0, s>>>(w.seg, w.nseg);
  if ((r = launched()) != RNN_OK) return r;
  pts_scan_apply_kernel<<<w.nseg, kScanThreads, 0, s>>>(w.start, w.nstart, w.seg);
  if ((r = launched()) != RNN_OK) return r;
  pts_scatter_kernel<<<grid_for(w.npts, di->sms), kSmallThreads, 0, s>>>(ps, w.start, w.cell,
                                                                         w.rank, w.sorted,
                                                                         w.npts);
  return launched();
}

// Blocks of kPtsThreads for `lanes` lanes per query, grid-stride beyond 8
// blocks per SM.
static int pts_query_grid(int64_t n, int sms, int lanes) {
  int64_t g = (n * lanes + kPtsThreads - 1) / kPtsThreads;
  if (g > 8LL * sms) g = 8LL * sms;
  return static_cast<int>(g < 1 ? 1 : g);
}

static size_t pts_frm_layout(void* ws, int B, int64_t k, int64_t N1, int64_t N2, FrmState* st,
                             PtsSets* ps, PtsWs* w) {
  FrmCopies cp;
  const size_t off = frm_layout(ws, B, k, N1, N2, 0, RNN_L2, st, &cp);
  Carve c(ws);
  c.off = off;
  *ps = pts_sets(nullptr, 3 * N1, N1, nullptr, 3 * N2, N2, B, 2);
  return pts_layout(c, *ps, w);
}

// FRM on point maps: as frm_run, with the NN of each half-step found by the
// grid search (frm_pts_step_kernel) instead of the tensor-core kernel.
static rnn_status frm_run_pts(int B, const float* P1, int64_t bs1, const float* P2, int64_t bs2,
                              int H1, int W1, int H2, int W2, const int32_t* init,
                              int64_t n_init, int S, int max_iter, float pixel_tol,
                              int32_t* pairs, int64_t cap, int32_t* count_out,
                              int32_t* seed_state, int32_t* basin, void* ws, size_t ws_bytes,
                              cudaStream_t s) {
  NvtxRange nvtx_range("rnn_pts_frm_match");
  if (B < 1) return RNN_EINVAL;
  if (B > RNN_MAX_BATCH) return RNN_EUNSUPPORTED;
  if (H1 <= 0 || W1 <= 0 || H2 <= 0 || W2 <= 0 || max_iter < 1) return RNN_EINVAL;
  if (init ? n_init < 0 : S < 1) return RNN_EINVAL;
  if (!(pixel_tol >= 0.f) || (pixel_tol > 0.f && !init)) return RNN_EINVAL;
  if (!P1 || !P2) return RNN_EINVAL;
  if (!pts_ptr_ok(P1) || !pts_ptr_ok(P2)) return RNN_EALIGN;
  const int64_t N1 = static_cast<int64_t>(H1) * W1, N2 = static_cast<int64_t>(H2) * W2;
  if (N1 > kPtsMaxSet || N2 > kPtsMaxSet) return RNN_EUNSUPPORTED;
  if (bs1 < 3 * N1 || bs2 < 3 * N2) return RNN_EINVAL;
  if (!pairs || !count_out) return RNN_EINVAL;
  const int64_t k = init ? n_init : num_seeds(H1, W1, S);
  if (k > INT32_MAX) return RNN_EINVAL;
  const int64_t need = pixel_tol > 0.f ? k : (k < N2 ? k : N2);
  if (cap < need) return RNN_ECAPACITY;
  FrmState st;
  PtsSets ps;
  PtsWs w;
  const size_t bytes = pts_frm_layout(nullptr, B, k, N1, N2, &st, &ps, &w);
  if (!pts_fits(ps)) return RNN_EUNSUPPORTED;
  if (!ws || !aligned256(ws) || ws_bytes < bytes) return RNN_EWORKSPACE;
  DeviceInfo* di = nullptr;
  rnn_status r = device_info(&di);
  if (r != RNN_OK) return r;
  pts_frm_layout(ws, B, k, N1, N2, &st, &ps, &w);
  ps.base[0] = P1;
  ps.base[1] = P2;
  ps.bstride[0] = bs1;
  ps.bstride[1] = bs2;
  st.basin = basin;
  st.pixel_tol = pixel_tol;
  st.starts = init ? 1 : 0;
  if (k == 0) {
    if (cudaMemsetAsync(count_out, 0, sizeof(int32_t) * B, s) != cudaSuccess) return RNN_ECUDA;
    if (cudaMemsetAsync(st.err, 0, sizeof(int), s) != cudaSuccess) return RNN_ECUDA;
    if (basin && cudaMemsetAsync(basin, 0xFF, sizeof(int32_t) * B * (N1 + 1), s) != cudaSuccess)
      return RNN_ECUDA;
    return RNN_OK;
  }
  if ((r = frm_seed(st, init, n_init, W1, S, di, s)) != RNN_OK) return r;
  if ((r = pts_build(ps, w, nullptr, di, s)) != RNN_OK) return r;
  const int qg = pts_query_grid(static_cast<int64_t>(B) * k, di->sms, kPtsGroup);
  for (int it = 1; it <= max_iter; ++it) {
    const int h = 2 * (it - 1);
    frm_pts_step_kernel<<<qg, kPtsThreads, 0, s>>>(st, ps, w.grids, w.sorted, w.start, h, 1, 0);
    if ((r = launched()) != RNN_OK) return r;
    frm_pts_step_kernel<<<qg, kPtsThreads, 0, s>>>(st, ps, w.grids, w.sorted, w.start, h + 1, 0,
                                                   it == max_iter ? 1 : 0);
    if ((r = launched()) != RNN_OK) return r;
  }
  return frm_merge(st, W1, pairs, cap, count_out, seed_state, s, false);
}

}  // namespace rnn

// ====================================================================== ABI
using namespace rnn;

extern "C" {

const char* rnn_status_string(rnn_status s) {
  switch (s) {
    case RNN_OK: return "RNN_OK";
    case RNN_EINVAL: return "RNN_EINVAL: invalid argument";
    case RNN_EALIGN: return "RNN_EALIGN: d must be a multiple of 8 and pointers 16-byte aligned";
    case RNN_ECAPACITY: return "RNN_ECAPACITY: output capacity below the guaranteed maximum";
    case RNN_ECUDA: return "RNN_ECUDA: a CUDA call failed";
    case RNN_ETIMEOUT: return "RNN_ETIMEOUT: a kernel's bounded wait ran out";
    case RNN_EUNSUPPORTED: return "RNN_EUNSUPPORTED: unsupported size or device";
    case RNN_EWORKSPACE: return "RNN_EWORKSPACE: workspace missing, too small or misaligned";
  }
  return "unknown rnn_status";
}

int rnn_abi_version(void) { return 7; }

uint64_t rnn_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

void rnn_set_kernel_timer(void* const* start_events, void* const* stop_events, int capacity,
                          int* recorded) {
  std::lock_guard<std::mutex> lk(g_mu);
  const bool on = start_events && stop_events && recorded && capacity > 0;
  g_timer_start = on ? start_events : nullptr;
  g_timer_stop = on ? stop_events : nullptr;
  g_timer_cap = on ? capacity : 0;
  g_timer_count = on ? recorded : nullptr;
}

void rnn_test_stall_loads(int on, uint64_t wait_limit_ns) {
  g_stall_limit_ns.store(on && wait_limit_ns > 0 ? wait_limit_ns : kWaitLimitNs,
                         std::memory_order_relaxed);
  g_stall_loads.store(on ? 1 : 0, std::memory_order_relaxed);
}

rnn_status rnn_workspace_status(const void* workspace, rnn_stream_t stream) {
  if (!workspace) return RNN_EINVAL;
  int err = 0;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(&err, workspace, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return RNN_ECUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return RNN_ECUDA;
  return err ? RNN_ETIMEOUT : RNN_OK;
}

// Workspace of the nearest-neighbour call: error word, packed keys, and with
// the Euclidean metric the query and candidate forms.
static size_t nn_layout(void* ws, int64_t nq, int64_t nx, int d, rnn_metric metric, int** err,
                        unsigned long long** keys, uint16_t** qf, uint16_t** xf) {
  Carve c(ws);
  *err = c.take<int>(64);
  *keys = c.take<unsigned long long>(nq > 0 ? nq : 1);
  *qf = *xf = nullptr;
  if (metric == RNN_L2 && d > 0) {
    const int kpad = tile_depth(d, metric);
    *qf = c.take<uint16_t>((nq > 0 ? nq : 1) * kpad);
    *xf = c.take<uint16_t>((nx > 0 ? nx : 1) * kpad);
  }
  return c.off;
}

size_t rnn_nn_workspace_size_ex(int64_t nq, int64_t nx, int d, rnn_metric metric) {
  int* e;
  unsigned long long* k;
  uint16_t *a, *b;
  return nn_layout(nullptr, nq > 0 ? nq : 0, nx > 0 ? nx : 0, d, metric, &e, &k, &a, &b);
}

size_t rnn_nn_workspace_size(int64_t nq) { return rnn_nn_workspace_size_ex(nq, 0, 0, RNN_DOT); }

rnn_status rnn_nn_argmax_ex(const void* Q, int64_t nq, const void* X, int64_t nx, int d,
                            rnn_dtype dtype, rnn_metric metric, int32_t* idx_out,
                            float* score_out, void* workspace, size_t ws_bytes,
                            rnn_stream_t stream) {
  NvtxRange nvtx_range("rnn_nn_argmax");
  if (nq < 0 || nx < 1 || nq > INT32_MAX || nx > INT32_MAX) return RNN_EINVAL;
  if (!valid_dtype(dtype) || !valid_metric(metric)) return RNN_EINVAL;
  rnn_status r = check_desc(X, d);
  if (r != RNN_OK) return r;
  if (nq > 0) {  // with no queries, Q and idx_out may be null
    if ((r = check_desc(Q, d)) != RNN_OK) return r;
    if (!idx_out) return RNN_EINVAL;
  }
  if (!workspace || !aligned256(workspace) ||
      ws_bytes < rnn_nn_workspace_size_ex(nq, nx, d, metric))
    return RNN_EWORKSPACE;
  DeviceInfo* di = nullptr;
  if ((r = device_info(&di)) != RNN_OK) return r;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int* err;
  unsigned long long* keys;
  uint16_t *qf, *xf;
  nn_layout(workspace, nq, nx, d, metric, &err, &keys, &qf, &xf);
  zero_keys_kernel<<<grid_for(nq, di->sms), kSmallThreads, 0, s>>>(keys, nq, nullptr, 0, err);
  if ((r = launched()) != RNN_OK) return r;
  if (nq == 0) return RNN_OK;
  const bool l2 = metric == RNN_L2;
  const Geometry g = geometry(d + (l2 ? kAugCols : 0));
  const uint16_t* q16 = static_cast<const uint16_t*>(Q);
  const uint16_t* x16 = static_cast<const uint16_t*>(X);
  int ld = d;
  if (l2) {
    if ((r = prep_rows(Q, nq * d, nq, 1, d, qf, g.kpad, kFormQuery, dtype, di, s)) != RNN_OK)
      return r;
    if ((r = prep_rows(X, nx * d, nx, 1, d, xf, g.kpad, kFormCand, dtype, di, s)) != RNN_OK)
      return r;
    q16 = qf;
    x16 = xf;
    ld = g.kpad;
  }
  CUtensorMap mx, mq;
  if ((r = make_map(&mx, x16, ld, nx, 1, nx * ld, g)) != RNN_OK) return r;
  if ((r = make_map(&mq, q16, ld, nq, 1, nq * ld, g, kBlockM)) != RNN_OK) return r;
  NNParams p;
  std::memset(&p, 0, sizeof(p));
  p.nfam = 1;
  p.d = ld;
  p.idesc = make_idesc(dtype, g.block_n);
  p.err = err;
  NNFamily& F = p.fam[0];
  F.q_base = q16;
  F.q_count = static_cast<int32_t>(nq);
  F.n_cand = static_cast<int32_t>(nx);
  F.nbatch = 1;
  F.keys = keys;
  F.q_tma = 1;
  if ((r = launch_nn(p, mx, mx, mq, mq, g, di, s)) != RNN_OK) return r;
  const int lg = grid_for(nq * 32, di->sms);
  if (dtype == RNN_BF16)
    locate_unpack_kernel<true><<<lg, kSmallThreads, 0, s>>>(
        keys, nq, q16, x16, static_cast<int>(nx), ld, d, l2, idx_out, score_out);
  else
    locate_unpack_kernel<false><<<lg, kSmallThreads, 0, s>>>(
        keys, nq, q16, x16, static_cast<int>(nx), ld, d, l2, idx_out, score_out);
  return launched();
}

rnn_status rnn_nn_argmax(const void* Q, int64_t nq, const void* X, int64_t nx, int d,
                         rnn_dtype dtype, int32_t* idx_out, float* score_out, void* workspace,
                         size_t ws_bytes, rnn_stream_t stream) {
  return rnn_nn_argmax_ex(Q, nq, X, nx, d, dtype, RNN_DOT, idx_out, score_out, workspace,
                          ws_bytes, stream);
}

// Workspace of the reciprocal set: error word, packed keys of both sweeps,
// block counts, and the row forms: a zero-padded copy of each map (dot
// metric, d = 8, 24, 40, ...), or a query and a candidate form of each map
// (Euclidean metric).
struct MnnWs {
  int* err;
  unsigned long long *rowk, *colk;
  int* counts;
  uint16_t *q1, *x1, *q2, *x2;
  // grouped locate of the one-pass path (chunks: at most n2/64 row chunks and
  // n1/32 column chunks)
  int64_t nch_max;
  int *loc_cnt, *loc_start, *loc_items, *loc_item_chunk, *loc_cursor;
  uint32_t* loc_list;
};

static size_t mnn_layout(void* ws, int64_t n1, int64_t n2, int d, rnn_metric metric, MnnWs* w) {
  Carve c(ws);
  w->err = c.take<int>(64);
  w->rowk = c.take<unsigned long long>(n1 > 0 ? n1 : 1);
  w->colk = c.take<unsigned long long>(n2 > 0 ? n2 : 1);
  w->counts = c.take<int>((n1 + kMnnChunk - 1) / kMnnChunk + 1);
  w->nch_max = (n2 + kOpRowChunk - 1) / kOpRowChunk + (n1 + 31) / 32;
  w->loc_cnt = c.take<int>(kLocPad * (w->nch_max + 1));
  w->loc_cursor = c.take<int>(kLocPad * (w->nch_max + 1));
  w->loc_start = c.take<int>(w->nch_max + 1);
  w->loc_items = c.take<int>(w->nch_max + 1);
  // items: at most one per chunk beyond the full ones
  w->loc_item_chunk = c.take<int>(w->nch_max + (n1 + n2) / kLocItem + 2);
  w->loc_list = c.take<uint32_t>(n1 + n2 > 0 ? n1 + n2 : 1);
  w->q1 = w->x1 = w->q2 = w->x2 = nullptr;
  const int mode = d > 0 ? copies_for(d, metric) : kCopiesNone;
  if (d > 0 && onepass_fits(onepass_geometry(d, metric))) {
    // one-pass form: padded rows, then kOpPadRows NaN rows
    const int kpad = onepass_geometry(d, metric).kpad;
    w->q1 = w->x1 = c.take<uint16_t>((n1 + kOpPadRows) * kpad);
    w->q2 = w->x2 = c.take<uint16_t>((n2 + kOpPadRows) * kpad);
  } else if (mode != kCopiesNone) {
    const int kpad = tile_depth(d, metric);
    w->q1 = c.take<uint16_t>(n1 * kpad);
    w->q2 = c.take<uint16_t>(n2 * kpad);
    w->x1 = w->q1;
    w->x2 = w->q2;
    if (mode == kCopiesEuclid) {
      w->x1 = c.take<uint16_t>(n1 * kpad);
      w->x2 = c.take<uint16_t>(n2 * kpad);
    }
  }
  return c.off;
}

size_t rnn_mnn_workspace_size_ex(int H1, int W1, int H2, int W2, int d, rnn_metric metric) {
  const int64_t n1 = static_cast<int64_t>(H1 > 0 ? H1 : 0) * (W1 > 0 ? W1 : 0);
  const int64_t n2 = static_cast<int64_t>(H2 > 0 ? H2 : 0) * (W2 > 0 ? W2 : 0);
  MnnWs w;
  return mnn_layout(nullptr, n1, n2, d > 0 ? d : 0, metric, &w);
}

size_t rnn_mnn_workspace_size(int H1, int W1, int H2, int W2, int d) {
  return rnn_mnn_workspace_size_ex(H1, W1, H2, W2, d, RNN_DOT);
}

}  // extern "C"

// ---------------------------------------------------- one-pass exhaustive M
struct OnePassPlan {
  int bm, bn, mblocks, nblocks, nmma;
};

// Unit shape: the largest that shared memory holds (bm query tiles of
// 128 x kpad, bm a power of two and at least 2, so that the tiles of every
// pass alternate between the two accumulators; query tiles past the last row
// read the NaN tail; 8 candidate tiles), halved along the longer side until
// there are at least two units per SM.  Two MMA-issuing warps when
// every shared-memory slot's reuse period is at least 5 tiles (2*bm for a
// candidate slot, bm*bn for a query slot).
static OnePassPlan onepass_plan(int64_t n1, int64_t n2, int kpad, int sms) {
  const int mt = static_cast<int>((n1 + 127) / 128);
  const int nt = static_cast<int>((n2 + kOpBlockN - 1) / kOpBlockN);
  auto blocks = [](int t, int b) { return (t + b - 1) / b; };
  int bm = kpad == 64 ? 8 : kOpMaxBm;
  while (bm > 2 && bm > mt) bm >>= 1;
  int bn = std::min(kOpMaxBn, nt);
  while (static_cast<int64_t>(blocks(mt, bm)) * blocks(nt, bn) < 2LL * sms && (bm > 2 || bn > 1)) {
    if (bn > 1 && (bn >= bm || bm <= 2))
      bn = (bn + 1) / 2;
    else
      bm >>= 1;
  }
  const int nmma = (bm >= 4 && bm * bn >= 8) ? 2 : 1;
  return {bm, bn, blocks(mt, bm), blocks(nt, bn), nmma};
}

template <bool kBf16>
static rnn_status loc_resolve_launch(int d, const LocParams& P, int grid, size_t smem,
                                     cudaStream_t s) {
  switch (d) {
    case 8: loc_resolve_kernel<kBf16, 8><<<grid, kLocItem * kLocSlices, smem, s>>>(P); break;
    case 16: loc_resolve_kernel<kBf16, 16><<<grid, kLocItem * kLocSlices, smem, s>>>(P); break;
    case 24: loc_resolve_kernel<kBf16, 24><<<grid, kLocItem * kLocSlices, smem, s>>>(P); break;
    case 32: loc_resolve_kernel<kBf16, 32><<<grid, kLocItem * kLocSlices, smem, s>>>(P); break;
    case 64: loc_resolve_kernel<kBf16, 64><<<grid, kLocItem * kLocSlices, smem, s>>>(P); break;
    default: return RNN_EUNSUPPORTED;
  }
  return launched();
}

template <bool kBf16>
static cudaError_t loc_resolve_attr(int smem) {
  const auto a = cudaFuncAttributeMaxDynamicSharedMemorySize;
  cudaError_t e = cudaSuccess;
  if (e == cudaSuccess) e = cudaFuncSetAttribute(loc_resolve_kernel<kBf16, 8>, a, smem);
  if (e == cudaSuccess) e = cudaFuncSetAttribute(loc_resolve_kernel<kBf16, 16>, a, smem);
  if (e == cudaSuccess) e = cudaFuncSetAttribute(loc_resolve_kernel<kBf16, 24>, a, smem);
  if (e == cudaSuccess) e = cudaFuncSetAttribute(loc_resolve_kernel<kBf16, 32>, a, smem);
  if (e == cudaSuccess) e = cudaFuncSetAttribute(loc_resolve_kernel<kBf16, 64>, a, smem);
  return e;
}

// Keys of both directions from one pass over the scores, then the grouped
// locate.  X1, X2: the rows the tensor maps read (ld elements apart).
static rnn_status mnn_onepass(const uint16_t* X1, int64_t n1, const uint16_t* X2, int64_t n2,
                              int ld, int d, bool l2, rnn_dtype dtype, const Geometry& g,
                              const MnnWs& w, DeviceInfo* di, cudaStream_t s) {
  constexpr int kLocSmem = 64 * 1024;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!di->op_smem_set) {
      if (cudaFuncSetAttribute(mnn_onepass_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               227 * 1024) != cudaSuccess ||
          loc_resolve_attr<false>(kLocSmem) != cudaSuccess ||
          loc_resolve_attr<true>(kLocSmem) != cudaSuccess)
        return RNN_ECUDA;
      di->op_smem_set = true;
    }
  }
  const OnePassPlan pl = onepass_plan(n1, n2, g.kpad, di->sms);
  CUtensorMap am, bm;
  rnn_status r;
  const int64_t r1 = n1 + kOpPadRows, r2 = n2 + kOpPadRows;  // rows with the NaN tail
  if ((r = make_map(&am, X1, ld, r1, 1, r1 * ld, g, 32)) != RNN_OK) return r;
  if ((r = make_map(&bm, X2, ld, r2, 1, r2 * ld, g, kOpBlockN)) != RNN_OK) return r;
  OnePassParams p;
  std::memset(&p, 0, sizeof(p));
  p.n1 = static_cast<int>(n1);
  p.n2 = static_cast<int>(n2);
  p.kpad = g.kpad;
  p.bm = pl.bm;
  p.bn = pl.bn;
  p.mblocks = pl.mblocks;
  p.nblocks = pl.nblocks;
  p.nmma = pl.nmma;
  p.idesc = make_idesc(dtype, kOpBlockN);
  p.rowk = w.rowk;
  p.colk = w.colk;
  p.err = w.err;
  p.stall_loads = g_stall_loads.load(std::memory_order_relaxed);
  p.wait_limit_ns = p.stall_loads ? g_stall_limit_ns.load(std::memory_order_relaxed)
                                  : kWaitLimitNs;
  const size_t smem = onepass_smem(g.kpad, pl.bm).total + 1024;
  const int units = pl.mblocks * pl.nblocks;
  int slot = -1;
  if ((r = timer_begin(s, &slot)) != RNN_OK) return r;
  mnn_onepass_kernel<<<std::min(units, di->sms), kOpThreads, smem, s>>>(p, am, bm);
  if ((r = launched()) != RNN_OK) return r;
  if ((r = timer_end(s, slot)) != RNN_OK) return r;

  LocParams P;
  P.rowk = w.rowk;
  P.colk = w.colk;
  P.n1 = n1;
  P.n2 = n2;
  P.lr = kOpRowChunk;
  P.lc = 32 * pl.bm;
  P.nch_r = static_cast<int>((n2 + P.lr - 1) / P.lr);
  P.nch = P.nch_r + static_cast<int>((n1 + P.lc - 1) / P.lc);
  P.cnt = w.loc_cnt;
  P.start = w.loc_start;
  P.items = w.loc_items;
  P.item_chunk = w.loc_item_chunk;
  P.cursor = w.loc_cursor;
  P.list = w.loc_list;
  P.X1 = X1;
  P.X2 = X2;
  P.ld = ld;
  P.l2 = l2 ? 1 : 0;
  zero_words_kernel<<<grid_for(kLocPad * P.nch, di->sms), kSmallThreads, 0, s>>>(
      P.cnt, static_cast<int64_t>(kLocPad) * P.nch);
  if ((r = launched()) != RNN_OK) return r;
  loc_count_kernel<<<grid_for(n1 + n2, di->sms), kSmallThreads, 0, s>>>(P);
  if ((r = launched()) != RNN_OK) return r;
  loc_scan_kernel<<<1, kSmallThreads, 0, s>>>(P);
  if ((r = launched()) != RNN_OK) return r;
  loc_scatter_kernel<<<grid_for(n1 + n2, di->sms), kSmallThreads, 0, s>>>(P);
  if ((r = launched()) != RNN_OK) return r;
  const int64_t max_items = P.nch + (n1 + n2) / kLocItem + 1;
  const int rg = static_cast<int>(std::min<int64_t>(max_items, 8LL * di->sms));
  // the Euclidean forms are recomputed over all their channels
  const int kd = l2 ? ld : d;
  const size_t lsm = static_cast<size_t>(std::max(P.lr, P.lc)) * kd * sizeof(float);
  return dtype == RNN_BF16 ? loc_resolve_launch<true>(kd, P, rg, lsm, s)
                           : loc_resolve_launch<false>(kd, P, rg, lsm, s);
}

extern "C" {

rnn_status rnn_mnn_exhaustive_ex(const void* D1, int H1, int W1, const void* D2, int H2, int W2,
                                 int d, rnn_dtype dtype, rnn_metric metric, int32_t* pairs_out,
                                 int64_t cap, int32_t* count_out, int32_t* rowarg_out,
                                 float* rowmax_out, int32_t* colarg_out, float* colmax_out,
                                 void* workspace, size_t ws_bytes, rnn_stream_t stream) {
  NvtxRange nvtx_range("rnn_mnn_exhaustive");
  if (H1 <= 0 || W1 <= 0 || H2 <= 0 || W2 <= 0) return RNN_EINVAL;
  if (!valid_dtype(dtype) || !valid_metric(metric)) return RNN_EINVAL;
  rnn_status r = check_desc(D1, d);
  if (r != RNN_OK) return r;
  if ((r = check_desc(D2, d)) != RNN_OK) return r;
  const int64_t n1 = static_cast<int64_t>(H1) * W1, n2 = static_cast<int64_t>(H2) * W2;
  if (n1 > INT32_MAX || n2 > INT32_MAX) return RNN_EINVAL;
  if (!pairs_out || !count_out) return RNN_EINVAL;
  if (cap < (n1 < n2 ? n1 : n2)) return RNN_ECAPACITY;
  if (!workspace || !aligned256(workspace) ||
      ws_bytes < rnn_mnn_workspace_size_ex(H1, W1, H2, W2, d, metric))
    return RNN_EWORKSPACE;
  DeviceInfo* di = nullptr;
  if ((r = device_info(&di)) != RNN_OK) return r;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  MnnWs w;
  mnn_layout(workspace, n1, n2, d, metric, &w);
  const int nblk1 = static_cast<int>((n1 + kMnnChunk - 1) / kMnnChunk);
  const int nblk2 = static_cast<int>((n2 + kMnnChunk - 1) / kMnnChunk);

  const bool l2 = metric == RNN_L2;
  const Geometry g = geometry(d + (l2 ? kAugCols : 0));
  const Geometry og = onepass_geometry(d, metric);
  const int nb = nblk1 > nblk2 ? nblk1 : nblk2;
  zero_keys_kernel<<<grid_for(n1 + n2, di->sms), kSmallThreads, 0, s>>>(w.rowk, n1, w.colk, n2,
                                                                        w.err);
  if ((r = launched()) != RNN_OK) return r;
  if (onepass_fits(og)) {
    // every score once, reduced by rows and by columns
    const uint16_t* s1 = static_cast<const uint16_t*>(D1);
    const uint16_t* s2 = static_cast<const uint16_t*>(D2);
    const int f1 = l2 ? kOpFormA : kOpFormDot, f2 = l2 ? kOpFormB : kOpFormDot;
    const int g1 = grid_for((n1 + kOpPadRows) * og.kpad / 8, di->sms);
    const int g2 = grid_for((n2 + kOpPadRows) * og.kpad / 8, di->sms);
    if (dtype == RNN_BF16) {
      op_copy_kernel<true><<<g1, kSmallThreads, 0, s>>>(s1, n1, d, w.q1, og.kpad,
                                                        n1 + kOpPadRows, f1);
      if ((r = launched()) != RNN_OK) return r;
      op_copy_kernel<true><<<g2, kSmallThreads, 0, s>>>(s2, n2, d, w.q2, og.kpad,
                                                        n2 + kOpPadRows, f2);
    } else {
      op_copy_kernel<false><<<g1, kSmallThreads, 0, s>>>(s1, n1, d, w.q1, og.kpad,
                                                         n1 + kOpPadRows, f1);
      if ((r = launched()) != RNN_OK) return r;
      op_copy_kernel<false><<<g2, kSmallThreads, 0, s>>>(s2, n2, d, w.q2, og.kpad,
                                                         n2 + kOpPadRows, f2);
    }
    if ((r = launched()) != RNN_OK) return r;
    if ((r = mnn_onepass(w.q1, n1, w.q2, n2, og.kpad, d, l2, dtype, og, w, di, s)) != RNN_OK)
      return r;
    mnn_count_kernel<<<nb, kSmallThreads, 0, s>>>(w.rowk, n1, w.colk, n2, w.counts, nblk1,
                                                  rowarg_out, rowmax_out, colarg_out, colmax_out);
    if ((r = launched()) != RNN_OK) return r;
    mnn_write_kernel<<<nblk1, kSmallThreads, 0, s>>>(w.rowk, n1, w.colk, w.counts, nblk1,
                                                     pairs_out, count_out);
    return launched();
  }
  // tensor maps and locate rows over the row forms, or over the inputs
  const uint16_t* Q1 = static_cast<const uint16_t*>(D1);
  const uint16_t* Q2 = static_cast<const uint16_t*>(D2);
  const uint16_t* X1 = Q1;
  const uint16_t* X2 = Q2;
  int ld = d;
  const int mode = copies_for(d, metric);
  if (mode != kCopiesNone) {
    const int qform = l2 ? kFormQuery : kFormPad;
    if ((r = prep_rows(D1, n1 * d, n1, 1, d, w.q1, g.kpad, qform, dtype, di, s)) != RNN_OK)
      return r;
    if ((r = prep_rows(D2, n2 * d, n2, 1, d, w.q2, g.kpad, qform, dtype, di, s)) != RNN_OK)
      return r;
    if (l2) {
      if ((r = prep_rows(D1, n1 * d, n1, 1, d, w.x1, g.kpad, kFormCand, dtype, di, s)) != RNN_OK)
        return r;
      if ((r = prep_rows(D2, n2 * d, n2, 1, d, w.x2, g.kpad, kFormCand, dtype, di, s)) != RNN_OK)
        return r;
    }
    Q1 = w.q1;
    Q2 = w.q2;
    X1 = w.x1;
    X2 = w.x2;
    ld = g.kpad;
  }
  CUtensorMap m1, m2, q1, q2;
  if ((r = make_map(&m1, X1, ld, n1, 1, n1 * ld, g)) != RNN_OK) return r;
  if ((r = make_map(&m2, X2, ld, n2, 1, n2 * ld, g)) != RNN_OK) return r;
  if ((r = make_map(&q1, Q1, ld, n1, 1, n1 * ld, g, kBlockM)) != RNN_OK) return r;
  if ((r = make_map(&q2, Q2, ld, n2, 1, n2 * ld, g, kBlockM)) != RNN_OK) return r;
  NNParams p;
  std::memset(&p, 0, sizeof(p));
  p.nfam = 2;
  p.d = ld;
  p.idesc = make_idesc(dtype, g.block_n);
  p.err = w.err;
  // sweep 1: rows of D1 against D2 -> NN2; sweep 2: rows of D2 against D1 -> NN1
  p.fam[0].q_base = Q1;
  p.fam[0].q_count = static_cast<int32_t>(n1);
  p.fam[0].n_cand = static_cast<int32_t>(n2);
  p.fam[0].nbatch = 1;
  p.fam[0].keys = w.rowk;
  p.fam[1].q_base = Q2;
  p.fam[1].q_count = static_cast<int32_t>(n2);
  p.fam[1].n_cand = static_cast<int32_t>(n1);
  p.fam[1].nbatch = 1;
  p.fam[1].keys = w.colk;
  p.fam[0].q_tma = 1;
  p.fam[1].q_tma = 1;
  if ((r = launch_nn(p, m2, m1, q1, q2, g, di, s)) != RNN_OK) return r;
  {
    const int lg = grid_for((n1 + n2) * 32, di->sms);
    if (dtype == RNN_BF16)
      locate_mnn_kernel<true><<<lg, kSmallThreads, 0, s>>>(w.rowk, n1, w.colk, n2, Q1, X1, Q2,
                                                           X2, ld, d, l2);
    else
      locate_mnn_kernel<false><<<lg, kSmallThreads, 0, s>>>(w.rowk, n1, w.colk, n2, Q1, X1, Q2,
                                                            X2, ld, d, l2);
    if ((r = launched()) != RNN_OK) return r;
  }
  mnn_count_kernel<<<nb, kSmallThreads, 0, s>>>(w.rowk, n1, w.colk, n2, w.counts, nblk1,
                                                rowarg_out, rowmax_out, colarg_out, colmax_out);
  if ((r = launched()) != RNN_OK) return r;
  mnn_write_kernel<<<nblk1, kSmallThreads, 0, s>>>(w.rowk, n1, w.colk, w.counts, nblk1,
                                                   pairs_out, count_out);
  return launched();
}

rnn_status rnn_mnn_exhaustive(const void* D1, int H1, int W1, const void* D2, int H2, int W2,
                              int d, rnn_dtype dtype, int32_t* pairs_out, int64_t cap,
                              int32_t* count_out, int32_t* rowarg_out, float* rowmax_out,
                              int32_t* colarg_out, float* colmax_out, void* workspace,
                              size_t ws_bytes, rnn_stream_t stream) {
  return rnn_mnn_exhaustive_ex(D1, H1, W1, D2, H2, W2, d, dtype, RNN_DOT, pairs_out, cap,
                               count_out, rowarg_out, rowmax_out, colarg_out, colmax_out,
                               workspace, ws_bytes, stream);
}

int64_t rnn_frm_num_seeds(int H1, int W1, int seed_stride) {
  if (H1 <= 0 || W1 <= 0 || seed_stride < 1) return 0;
  return num_seeds(H1, W1, seed_stride);
}

int64_t rnn_frm_max_pairs(int H1, int W1, int H2, int W2, int seed_stride) {
  const int64_t k = rnn_frm_num_seeds(H1, W1, seed_stride);
  const int64_t n2 = static_cast<int64_t>(H2 > 0 ? H2 : 0) * (W2 > 0 ? W2 : 0);
  return k < n2 ? k : n2;
}

size_t rnn_frm_workspace_size_ex(int B, int H1, int W1, int H2, int W2, int d,
                                 rnn_metric metric, int seed_stride, int64_t n_init) {
  if (B < 1 || H1 <= 0 || W1 <= 0 || H2 <= 0 || W2 <= 0 || d <= 0) return 0;
  if (!valid_metric(metric) || (n_init < 0 && seed_stride < 1)) return 0;
  const int64_t k = n_init >= 0 ? n_init : num_seeds(H1, W1, seed_stride);
  return frm_bytes(B, k, static_cast<int64_t>(H1) * W1, static_cast<int64_t>(H2) * W2, d,
                   metric);
}

size_t rnn_frm_workspace_size(int B, int H1, int W1, int H2, int W2, int d, int seed_stride) {
  return rnn_frm_workspace_size_ex(B, H1, W1, H2, W2, d, RNN_DOT, seed_stride, -1);
}

rnn_status rnn_frm_match(const void* D1, int H1, int W1, const void* D2, int H2, int W2, int d,
                         rnn_dtype dtype, int seed_stride, int max_iter, int32_t* pairs_out,
                         int64_t cap, int32_t* count_out, int32_t* seed_state_out,
                         void* workspace, size_t ws_bytes, rnn_stream_t stream) {
  const int64_t n1 = static_cast<int64_t>(H1) * W1, n2 = static_cast<int64_t>(H2) * W2;
  return frm_run(1, D1, n1 * d, D2, n2 * d, H1, W1, H2, W2, d, dtype, RNN_DOT, nullptr, 0,
                 seed_stride, max_iter, 0.f, pairs_out, cap, count_out, seed_state_out, nullptr,
                 workspace, ws_bytes, reinterpret_cast<cudaStream_t>(stream));
}

rnn_status rnn_frm_match_batched(int B, const void* D1, int64_t d1_batch_stride, const void* D2,
                                 int64_t d2_batch_stride, int H1, int W1, int H2, int W2, int d,
                                 rnn_dtype dtype, int seed_stride, int max_iter,
                                 int32_t* pairs_out, int64_t cap, int32_t* count_out,
                                 int32_t* seed_state_out, void* workspace, size_t ws_bytes,
                                 rnn_stream_t stream) {
  return frm_run(B, D1, d1_batch_stride, D2, d2_batch_stride, H1, W1, H2, W2, d, dtype, RNN_DOT,
                 nullptr, 0, seed_stride, max_iter, 0.f, pairs_out, cap, count_out,
                 seed_state_out, nullptr, workspace, ws_bytes,
                 reinterpret_cast<cudaStream_t>(stream));
}

rnn_status rnn_frm_match_ex(int B, const void* D1, int64_t d1_batch_stride, const void* D2,
                            int64_t d2_batch_stride, int H1, int W1, int H2, int W2, int d,
                            rnn_dtype dtype, rnn_metric metric, const int32_t* init_xy1,
                            int64_t n_init, int seed_stride, int max_iter, float pixel_tol,
                            int32_t* pairs_out, int64_t cap, int32_t* count_out,
                            int32_t* seed_state_out, int32_t* basin_out, void* workspace,
                            size_t ws_bytes, rnn_stream_t stream) {
  return frm_run(B, D1, d1_batch_stride, D2, d2_batch_stride, H1, W1, H2, W2, d, dtype, metric,
                 init_xy1, n_init, seed_stride, max_iter, pixel_tol, pairs_out, cap, count_out,
                 seed_state_out, basin_out, workspace, ws_bytes,
                 reinterpret_cast<cudaStream_t>(stream));
}

// ------------------------------------------------------------ graph plans
struct rnn_frm_graph {
  cudaGraphExec_t exec;
};

rnn_status rnn_frm_graph_create(int B, const void* D1, int64_t d1_batch_stride, const void* D2,
                                int64_t d2_batch_stride, int H1, int W1, int H2, int W2, int d,
                                rnn_dtype dtype, rnn_metric metric, const int32_t* init_xy1,
                                int64_t n_init, int seed_stride, int max_iter, float pixel_tol,
                                int32_t* pairs_out, int64_t cap, int32_t* count_out,
                                int32_t* seed_state_out, int32_t* basin_out, void* workspace,
                                size_t ws_bytes, rnn_frm_graph_t* graph_out) {
  if (!graph_out) return RNN_EINVAL;
  *graph_out = nullptr;
  if (max_iter > kMaxGraphIters) return RNN_EUNSUPPORTED;
  DeviceInfo* di = nullptr;
  rnn_status r = device_info(&di);  // device queries stay outside the capture
  if (r != RNN_OK) return r;
  cudaStream_t s = nullptr, body = nullptr;
  if (cudaStreamCreateWithFlags(&s, cudaStreamNonBlocking) != cudaSuccess) return RNN_ECUDA;
  if (cudaStreamCreateWithFlags(&body, cudaStreamNonBlocking) != cudaSuccess) {
    cudaStreamDestroy(s);
    return RNN_ECUDA;
  }
  cudaGraph_t graph = nullptr;
  cudaGraphExec_t exec = nullptr;
  if (cudaStreamBeginCapture(s, cudaStreamCaptureModeThreadLocal) != cudaSuccess) {
    r = RNN_ECUDA;
  } else {
    t_capturing = true;
    r = frm_run(B, D1, d1_batch_stride, D2, d2_batch_stride, H1, W1, H2, W2, d, dtype, metric,
                init_xy1, n_init, seed_stride, max_iter, pixel_tol, pairs_out, cap, count_out,
                seed_state_out, basin_out, workspace, ws_bytes, s, nullptr, body);
    t_capturing = false;
    const cudaError_t ce = cudaStreamEndCapture(s, &graph);
    if (r == RNN_OK && ce != cudaSuccess) r = RNN_ECUDA;
  }
  if (r == RNN_OK && cudaGraphInstantiate(&exec, graph, 0) != cudaSuccess) r = RNN_ECUDA;
  if (graph) cudaGraphDestroy(graph);
  cudaStreamDestroy(body);
  cudaStreamDestroy(s);
  cudaGetLastError();  // a failed capture leaves its error; the status says it
  if (r != RNN_OK) {
    if (exec) cudaGraphExecDestroy(exec);
    return r;
  }
  rnn_frm_graph* gp = new (std::nothrow) rnn_frm_graph;
  if (!gp) {
    cudaGraphExecDestroy(exec);
    return RNN_ECUDA;
  }
  gp->exec = exec;
  *graph_out = gp;
  return RNN_OK;
}

rnn_status rnn_frm_graph_launch(rnn_frm_graph_t graph, rnn_stream_t stream) {
  if (!graph) return RNN_EINVAL;
  NvtxRange nvtx_range("rnn_frm_graph_launch");
  if (cudaGraphLaunch(graph->exec, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return RNN_ECUDA;
  return RNN_OK;
}

void rnn_frm_graph_destroy(rnn_frm_graph_t graph) {
  if (!graph) return;
  cudaGraphExecDestroy(graph->exec);
  delete graph;
}

// ------------------------------------------------ mutual test of NN arrays
size_t rnn_mnn_mutual_workspace_size(int64_t n1) {
  Carve c(nullptr);
  c.take<int>(64);
  c.take<int>((n1 > 0 ? n1 : 1) / kMnnChunk + 2);
  return c.off;
}

rnn_status rnn_mnn_mutual(const int32_t* rowarg, int64_t n1, const int32_t* colarg, int64_t n2,
                          int32_t* pairs_out, int64_t cap, int32_t* count_out, void* workspace,
                          size_t ws_bytes, rnn_stream_t stream) {
  NvtxRange nvtx_range("rnn_mnn_mutual");
  if (n1 < 1 || n2 < 1 || n1 > INT32_MAX || n2 > INT32_MAX) return RNN_EINVAL;
  if (!rowarg || !colarg || !pairs_out || !count_out) return RNN_EINVAL;
  if (cap < (n1 < n2 ? n1 : n2)) return RNN_ECAPACITY;
  if (!workspace || !aligned256(workspace) || ws_bytes < rnn_mnn_mutual_workspace_size(n1))
    return RNN_EWORKSPACE;
  DeviceInfo* di = nullptr;
  rnn_status r = device_info(&di);
  if (r != RNN_OK) return r;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  Carve c(workspace);
  int* err = c.take<int>(64);
  int* counts = c.take<int>(n1 / kMnnChunk + 2);
  if (cudaMemsetAsync(err, 0, sizeof(int), s) != cudaSuccess) return RNN_ECUDA;
  const int nblk = static_cast<int>((n1 + kMnnChunk - 1) / kMnnChunk);
  mutual_count_kernel<<<nblk, kSmallThreads, 0, s>>>(rowarg, n1, colarg, n2, counts);
  if ((r = launched()) != RNN_OK) return r;
  mutual_write_kernel<<<nblk, kSmallThreads, 0, s>>>(rowarg, n1, colarg, n2, counts, pairs_out,
                                                     count_out);
  return launched();
}

// --------------------------------------------------------- coarse-to-fine
// Crop geometry of a call; false when a size is not positive.
static bool c2f_geom(int Hc1, int Wc1, int Hc2, int Wc2, int H1, int W1, int H2, int W2,
                     int crop_h, int crop_w, int min_coarse, C2FGeom* g) {
  if (Hc1 <= 0 || Wc1 <= 0 || Hc2 <= 0 || Wc2 <= 0 || H1 <= 0 || W1 <= 0 || H2 <= 0 ||
      W2 <= 0 || crop_h <= 0 || crop_w <= 0)
    return false;
  g->Hc1 = Hc1;
  g->Wc1 = Wc1;
  g->Hc2 = Hc2;
  g->Wc2 = Wc2;
  g->H1 = H1;
  g->W1 = W1;
  g->H2 = H2;
  g->W2 = W2;
  g->ch = std::min(crop_h, std::min(H1, H2));
  g->cw = std::min(crop_w, std::min(W1, W2));
  g->ny = (H1 + g->ch - 1) / g->ch;
  g->nx = (W1 + g->cw - 1) / g->cw;
  g->min_coarse = min_coarse;
  return true;
}

struct C2FWs {
  int* status;              // header: OR of the parts' status words
  int32_t* coarse;          // [mc][2] reciprocal pairs of the coarse maps
  int32_t* coarse_count;
  int32_t* crops;           // [B][6] crop table (the caller's, when given)
  int32_t* pair_on;         // [B]
  uint16_t *crop1, *crop2;  // [B][ch*cw][dp] windows
  int32_t* lpairs;          // [B][capc][2] FRM pairs of each crop pair
  int32_t* lcount;          // [B]
  int32_t* tag;             // [N1] lowest crop index outputting each pixel
  int32_t* partner;         // [N1]
  uint32_t* bm;             // [nwords]
  int* bcounts;             // [nblk]
  void* mnn_ws;
  size_t mnn_bytes;
  void* frm_ws;
  size_t frm_bytes;
  int64_t mc, k, capc, rows, n1, nwords;
  int B, dp, nblk;
};

static size_t c2f_layout(void* ws, const C2FGeom& g, int dc, int d, rnn_metric metric, int S,
                         C2FWs* w) {
  Carve c(ws);
  w->B = g.ny * g.nx;
  w->rows = static_cast<int64_t>(g.ch) * g.cw;
  w->k = num_seeds(g.ch, g.cw, S);
  w->capc = std::max<int64_t>(1, std::min(w->k, w->rows));
  w->mc = std::min(static_cast<int64_t>(g.Hc1) * g.Wc1, static_cast<int64_t>(g.Hc2) * g.Wc2);
  w->n1 = static_cast<int64_t>(g.H1) * g.W1;
  w->nwords = (w->n1 + 31) / 32;
  w->nblk = static_cast<int>((w->nwords + kEmitWords - 1) / kEmitWords);
  w->dp = metric == RNN_DOT ? padded_depth(d) : d;
  w->status = c.take<int>(64);
  w->coarse = c.take<int32_t>(2 * w->mc);
  w->coarse_count = c.take<int32_t>(1);
  w->crops = c.take<int32_t>(static_cast<int64_t>(w->B) * kC2FCropCols);
  w->pair_on = c.take<int32_t>(w->B);
  w->crop1 = c.take<uint16_t>(w->B * w->rows * w->dp);
  w->crop2 = c.take<uint16_t>(w->B * w->rows * w->dp);
  w->lpairs = c.take<int32_t>(2 * w->B * w->capc);
  w->lcount = c.take<int32_t>(w->B);
  w->tag = c.take<int32_t>(w->n1);
  w->partner = c.take<int32_t>(w->n1);
  w->bm = c.take<uint32_t>(w->nwords);
  w->bcounts = c.take<int>(w->nblk);
  w->mnn_bytes = rnn_mnn_workspace_size_ex(g.Hc1, g.Wc1, g.Hc2, g.Wc2, dc, metric);
  w->mnn_ws = c.take<uint8_t>(w->mnn_bytes);
  w->frm_bytes = frm_bytes(w->B, w->k, w->rows, w->rows, w->dp, metric);
  w->frm_ws = c.take<uint8_t>(w->frm_bytes);
  return c.off;
}

int rnn_c2f_num_crops(int H1, int W1, int H2, int W2, int crop_h, int crop_w) {
  C2FGeom g;
  if (!c2f_geom(1, 1, 1, 1, H1, W1, H2, W2, crop_h, crop_w, 1, &g)) return 0;
  return g.ny * g.nx;
}

int64_t rnn_c2f_max_pairs(int H1, int W1, int H2, int W2, int crop_h, int crop_w,
                          int seed_stride) {
  C2FGeom g;
  if (seed_stride < 1 || !c2f_geom(1, 1, 1, 1, H1, W1, H2, W2, crop_h, crop_w, 1, &g)) return 0;
  const int64_t rows = static_cast<int64_t>(g.ch) * g.cw;
  const int64_t per = std::min(num_seeds(g.ch, g.cw, seed_stride), rows);
  return std::min(static_cast<int64_t>(H1) * W1, per * g.ny * g.nx);
}

size_t rnn_c2f_workspace_size(int Hc1, int Wc1, int Hc2, int Wc2, int dc, int H1, int W1,
                              int H2, int W2, int d, rnn_metric metric, int crop_h, int crop_w,
                              int seed_stride) {
  C2FGeom g;
  if (!valid_metric(metric) || dc <= 0 || d <= 0 || seed_stride < 1 ||
      !c2f_geom(Hc1, Wc1, Hc2, Wc2, H1, W1, H2, W2, crop_h, crop_w, 1, &g))
    return 0;
  C2FWs w;
  return c2f_layout(nullptr, g, dc, d, metric, seed_stride, &w);
}

rnn_status rnn_c2f_match(const void* C1, int Hc1, int Wc1, const void* C2, int Hc2, int Wc2,
                         int dc, const void* F1, int H1, int W1, const void* F2, int H2, int W2,
                         int d, rnn_dtype dtype, rnn_metric metric, int crop_h, int crop_w,
                         int seed_stride, int max_iter, int min_coarse, int32_t* pairs_out,
                         int64_t cap, int32_t* count_out, int32_t* crops_out, void* workspace,
                         size_t ws_bytes, rnn_stream_t stream) {
  NvtxRange nvtx_range("rnn_c2f_match");
  C2FGeom g;
  if (!c2f_geom(Hc1, Wc1, Hc2, Wc2, H1, W1, H2, W2, crop_h, crop_w, min_coarse, &g))
    return RNN_EINVAL;
  if (!valid_dtype(dtype) || !valid_metric(metric)) return RNN_EINVAL;
  if (seed_stride < 1 || max_iter < 1 || !pairs_out || !count_out) return RNN_EINVAL;
  rnn_status r;
  if ((r = check_desc(C1, dc)) != RNN_OK || (r = check_desc(C2, dc)) != RNN_OK ||
      (r = check_desc(F1, d)) != RNN_OK || (r = check_desc(F2, d)) != RNN_OK)
    return r;
  const int64_t n1 = static_cast<int64_t>(H1) * W1, n2 = static_cast<int64_t>(H2) * W2;
  if (n1 >= INT32_MAX || n2 >= INT32_MAX) return RNN_EINVAL;
  if (g.ny * static_cast<int64_t>(g.nx) > RNN_MAX_BATCH) return RNN_EUNSUPPORTED;
  if (cap < rnn_c2f_max_pairs(H1, W1, H2, W2, crop_h, crop_w, seed_stride))
    return RNN_ECAPACITY;
  if (!workspace || !aligned256(workspace) ||
      ws_bytes < rnn_c2f_workspace_size(Hc1, Wc1, Hc2, Wc2, dc, H1, W1, H2, W2, d, metric,
                                        crop_h, crop_w, seed_stride))
    return RNN_EWORKSPACE;
  DeviceInfo* di = nullptr;
  if ((r = device_info(&di)) != RNN_OK) return r;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  C2FWs w;
  c2f_layout(workspace, g, dc, d, metric, seed_stride, &w);
  if (crops_out) w.crops = crops_out;
  // 1. the reciprocal set of the coarse maps
  if ((r = rnn_mnn_exhaustive_ex(C1, Hc1, Wc1, C2, Hc2, Wc2, dc, dtype, metric, w.coarse, w.mc,
                                 w.coarse_count, nullptr, nullptr, nullptr, nullptr, w.mnn_ws,
                                 w.mnn_bytes, stream)) != RNN_OK)
    return r;
  // 2. crop table; 3. windows of the crop pairs that are on
  c2f_place_kernel<<<w.B, 256, 0, s>>>(g, w.coarse, w.coarse_count, w.crops, w.pair_on);
  if ((r = launched()) != RNN_OK) return r;
  const int64_t items = 2 * static_cast<int64_t>(w.B) * w.rows * (w.dp / 8) + w.n1 + w.nwords;
  c2f_gather_kernel<<<grid_for(items, di->sms), kSmallThreads, 0, s>>>(
      g, static_cast<const uint16_t*>(F1), static_cast<const uint16_t*>(F2), d, w.dp, w.crops,
      w.B, w.crop1, w.crop2, w.tag, w.n1, w.bm, w.nwords);
  if ((r = launched()) != RNN_OK) return r;
  // 4. FRM on every crop pair that is on (grid seeds), in one batched loop
  const int64_t bs = w.rows * w.dp;
  if ((r = frm_run(w.B, w.crop1, bs, w.crop2, bs, g.ch, g.cw, g.ch, g.cw, w.dp, dtype, metric,
                   nullptr, 0, seed_stride, max_iter, 0.f, w.lpairs, w.capc, w.lcount, nullptr,
                   nullptr, w.frm_ws, w.frm_bytes, s, w.pair_on)) != RNN_OK)
    return r;
  // 5. map back, first crop per image-1 pixel, pixel order
  const int mg = grid_for(static_cast<int64_t>(w.B) * w.capc, di->sms);
  c2f_mapback_kernel<<<mg, kSmallThreads, 0, s>>>(g, w.B, w.crops, w.lpairs, w.capc, w.lcount,
                                                  w.tag, w.partner, w.bm, 1);
  if ((r = launched()) != RNN_OK) return r;
  c2f_mapback_kernel<<<mg, kSmallThreads, 0, s>>>(g, w.B, w.crops, w.lpairs, w.capc, w.lcount,
                                                  w.tag, w.partner, w.bm, 0);
  if ((r = launched()) != RNN_OK) return r;
  c2f_count_kernel<<<w.nblk, kSmallThreads, 0, s>>>(w.bm, w.nwords, w.bcounts);
  if ((r = launched()) != RNN_OK) return r;
  c2f_emit_kernel<<<w.nblk, kSmallThreads, 0, s>>>(
      w.bm, w.nwords, w.bcounts, w.partner, pairs_out, count_out, w.status,
      static_cast<const int*>(w.mnn_ws), static_cast<const int*>(w.frm_ws));
  return launched();
}

// ------------------------------------------------------------- 3-D points
static size_t pts_nn_layout(void* ws, int64_t nq, int64_t nx, int** err, PtsSets* ps,
                            PtsWs* w) {
  Carve c(ws);
  *err = c.take<int>(64);
  (void)nq;
  *ps = pts_sets(nullptr, 3 * nx, nx, nullptr, 0, 0, 1, 1);
  return pts_layout(c, *ps, w);
}

size_t rnn_pts_nn_workspace_size(int64_t nq, int64_t nx) {
  int* e;
  PtsSets ps;
  PtsWs w;
  return pts_nn_layout(nullptr, nq > 0 ? nq : 0, nx > 0 ? nx : 1, &e, &ps, &w);
}

rnn_status rnn_pts_nn(const float* Q, int64_t nq, const float* X, int64_t nx, int32_t* idx_out,
                      float* dist2_out, void* workspace, size_t ws_bytes, rnn_stream_t stream) {
  NvtxRange nvtx_range("rnn_pts_nn");
  if (nq < 0 || nx < 1 || nq > INT32_MAX) return RNN_EINVAL;
  if (nx > kPtsMaxSet) return RNN_EUNSUPPORTED;
  if (!X || (nq > 0 && (!Q || !idx_out))) return RNN_EINVAL;
  if (!pts_ptr_ok(X) || (nq > 0 && !pts_ptr_ok(Q))) return RNN_EALIGN;
  if (!workspace || !aligned256(workspace) || ws_bytes < rnn_pts_nn_workspace_size(nq, nx))
    return RNN_EWORKSPACE;
  DeviceInfo* di = nullptr;
  rnn_status r = device_info(&di);
  if (r != RNN_OK) return r;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int* err;
  PtsSets ps;
  PtsWs w;
  pts_nn_layout(workspace, nq, nx, &err, &ps, &w);
  ps.base[0] = X;
  if ((r = pts_build(ps, w, err, di, s)) != RNN_OK) return r;
  if (nq == 0) return RNN_OK;
  PtsQuery q{Q, nq, 0, idx_out, dist2_out, nullptr};
  pts_query_kernel<<<pts_query_grid(nq, di->sms, kPtsGroupQuery), kPtsThreads, 0, s>>>(
      q, q, 1, w.grids, w.sorted, w.start);
  return launched();
}

static size_t pts_mnn_layout(void* ws, int64_t n1, int64_t n2, MnnWs* m, PtsSets* ps, PtsWs* w) {
  Carve c(ws);
  m->err = c.take<int>(64);
  m->rowk = c.take<unsigned long long>(n1 > 0 ? n1 : 1);
  m->colk = c.take<unsigned long long>(n2 > 0 ? n2 : 1);
  m->counts = c.take<int>((n1 + kMnnChunk - 1) / kMnnChunk + 1);
  *ps = pts_sets(nullptr, 3 * n1, n1, nullptr, 3 * n2, n2, 1, 2);
  return pts_layout(c, *ps, w);
}

size_t rnn_pts_mnn_workspace_size(int H1, int W1, int H2, int W2) {
  const int64_t n1 = static_cast<int64_t>(H1 > 0 ? H1 : 1) * (W1 > 0 ? W1 : 1);
  const int64_t n2 = static_cast<int64_t>(H2 > 0 ? H2 : 1) * (W2 > 0 ? W2 : 1);
  MnnWs m;
  PtsSets ps;
  PtsWs w;
  return pts_mnn_layout(nullptr, n1, n2, &m, &ps, &w);
}

rnn_status rnn_pts_mnn(const float* P1, int H1, int W1, const float* P2, int H2, int W2,
                       int32_t* pairs_out, int64_t cap, int32_t* count_out, int32_t* rowarg_out,
                       float* rowd2_out, int32_t* colarg_out, float* cold2_out, void* workspace,
                       size_t ws_bytes, rnn_stream_t stream) {
  NvtxRange nvtx_range("rnn_pts_mnn");
  if (H1 <= 0 || W1 <= 0 || H2 <= 0 || W2 <= 0) return RNN_EINVAL;
  if (!P1 || !P2 || !pairs_out || !count_out) return RNN_EINVAL;
  if (!pts_ptr_ok(P1) || !pts_ptr_ok(P2)) return RNN_EALIGN;
  const int64_t n1 = static_cast<int64_t>(H1) * W1, n2 = static_cast<int64_t>(H2) * W2;
  if (n1 > kPtsMaxSet || n2 > kPtsMaxSet) return RNN_EUNSUPPORTED;
  if (cap < (n1 < n2 ? n1 : n2)) return RNN_ECAPACITY;
  if (!workspace || !aligned256(workspace) ||
      ws_bytes < rnn_pts_mnn_workspace_size(H1, W1, H2, W2))
    return RNN_EWORKSPACE;
  DeviceInfo* di = nullptr;
  rnn_status r = device_info(&di);
  if (r != RNN_OK) return r;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  MnnWs m;
  PtsSets ps;
  PtsWs w;
  pts_mnn_layout(workspace, n1, n2, &m, &ps, &w);
  ps.base[0] = P1;
  ps.base[1] = P2;
  if ((r = pts_build(ps, w, m.err, di, s)) != RNN_OK) return r;
  // sweep 1: points of image 1 in the image-2 grid (set 1) -> NN2; sweep 2
  // the other way -> NN1
  PtsQuery q1{P1, n1, 1, nullptr, nullptr, m.rowk};
  PtsQuery q2{P2, n2, 0, nullptr, nullptr, m.colk};
  pts_query_kernel<<<pts_query_grid(n1 + n2, di->sms, kPtsGroupQuery), kPtsThreads, 0, s>>>(
      q1, q2, 2, w.grids, w.sorted, w.start);
  if ((r = launched()) != RNN_OK) return r;
  const int nblk1 = static_cast<int>((n1 + kMnnChunk - 1) / kMnnChunk);
  const int nblk2 = static_cast<int>((n2 + kMnnChunk - 1) / kMnnChunk);
  const int nb = nblk1 > nblk2 ? nblk1 : nblk2;
  mnn_count_kernel<<<nb, kSmallThreads, 0, s>>>(m.rowk, n1, m.colk, n2, m.counts, nblk1,
                                                rowarg_out, rowd2_out, colarg_out, cold2_out);
  if ((r = launched()) != RNN_OK) return r;
  mnn_write_kernel<<<nblk1, kSmallThreads, 0, s>>>(m.rowk, n1, m.colk, m.counts, nblk1,
                                                   pairs_out, count_out);
  return launched();
}

size_t rnn_pts_frm_workspace_size(int B, int H1, int W1, int H2, int W2, int seed_stride,
                                  int64_t n_init) {
  if (B < 1) B = 1;
  const int64_t N1 = static_cast<int64_t>(H1 > 0 ? H1 : 1) * (W1 > 0 ? W1 : 1);
  const int64_t N2 = static_cast<int64_t>(H2 > 0 ? H2 : 1) * (W2 > 0 ? W2 : 1);
  const int64_t k = n_init >= 0 ? n_init : (seed_stride >= 1 ? num_seeds(H1, W1, seed_stride) : 0);
  FrmState st;
  PtsSets ps;
  PtsWs w;
  return pts_frm_layout(nullptr, B, k, N1, N2, &st, &ps, &w);
}

rnn_status rnn_pts_frm_match(int B, const float* P1, int64_t p1_batch_stride, const float* P2,
                             int64_t p2_batch_stride, int H1, int W1, int H2, int W2,
                             const int32_t* init_xy1, int64_t n_init, int seed_stride,
                             int max_iter, float pixel_tol, int32_t* pairs_out, int64_t cap,
                             int32_t* count_out, int32_t* seed_state_out, int32_t* basin_out,
                             void* workspace, size_t ws_bytes, rnn_stream_t stream) {
  return frm_run_pts(B, P1, p1_batch_stride, P2, p2_batch_stride, H1, W1, H2, W2, init_xy1,
                     n_init, seed_stride, max_iter, pixel_tol, pairs_out, cap, count_out,
                     seed_state_out, basin_out, workspace, ws_bytes,
                     reinterpret_cast<cudaStream_t>(stream));
}

}  // extern "C"

// ============================================== nearest neighbours, no allocation
//
// Some callers cannot allocate device memory: a plugin whose host framework
// owns every device buffer and only lends it the inputs and outputs, or a
// latency-bound serving loop in which cudaMalloc/cudaFree would synchronise
// the device and stall other work.  For them rnn_nn_argmax_noalloc keeps its
// scratch (the packed per-query keys and the status word) in the fixed array
// below instead of a caller workspace.  The array is part of the library's
// device image, so every GPU that loads the library holds it until the
// process exits.
namespace rnn {

static __device__ __align__(256) unsigned char
    g_noalloc_scratch[256 + RNN_NN_NOALLOC_MAX_QUERIES * sizeof(unsigned long long)];

static std::mutex g_noalloc_mu;
static void* g_noalloc_ptr[64];

// Device address of the scratch array on the current device (host code only
// knows the array by a host-side stand-in name).  It is looked up with that
// device current on every call whose stream is not being captured, so that a
// context made anew after cudaDeviceReset gets its own address; a call on a
// capturing stream uses the address the device's last such lookup found
// (none yet: RNN_ECUDA).
static rnn_status noalloc_scratch(cudaStream_t s, void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return RNN_ECUDA;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(s, &cs) != cudaSuccess) return RNN_ECUDA;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (cs == cudaStreamCaptureStatusNone) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
      return RNN_ECUDA;
    g_noalloc_ptr[dev] = p;
  }
  if (!g_noalloc_ptr[dev]) return RNN_ECUDA;
  *out = g_noalloc_ptr[dev];
  return RNN_OK;
}

}  // namespace rnn

extern "C" rnn_status rnn_nn_argmax_noalloc(const void* Q, int64_t nq, const void* X, int64_t nx,
                                            int d, rnn_dtype dtype, int32_t* idx_out,
                                            float* score_out, rnn_stream_t stream) {
  if (nq > RNN_NN_NOALLOC_MAX_QUERIES) return RNN_EUNSUPPORTED;
  if (nq < 0) return RNN_EINVAL;
  void* scratch = nullptr;
  const rnn_status r =
      rnn::noalloc_scratch(reinterpret_cast<cudaStream_t>(stream), &scratch);
  if (r != RNN_OK) return r;
  static_assert(sizeof(rnn::g_noalloc_scratch) >= 256 + RNN_NN_NOALLOC_MAX_QUERIES * 8,
                "scratch array too small");
  return rnn_nn_argmax(Q, nq, X, nx, d, dtype, idx_out, score_out, scratch,
                       sizeof(rnn::g_noalloc_scratch), stream);
}

// The status word of the shared scratch array (the first int, which every
// call clears before its kernels run): RNN_ETIMEOUT when a bounded wait of the
// last call ran out.  One 4-byte copy to the host and a synchronisation of
// `stream`; nothing is allocated.
extern "C" rnn_status rnn_nn_argmax_noalloc_status(rnn_stream_t stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  void* scratch = nullptr;
  rnn_status r = rnn::noalloc_scratch(s, &scratch);
  if (r != RNN_OK) return r;
  int err = 0;
  if (cudaMemcpyAsync(&err, scratch, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return RNN_ECUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return RNN_ECUDA;
  return err ? RNN_ETIMEOUT : RNN_OK;
}
