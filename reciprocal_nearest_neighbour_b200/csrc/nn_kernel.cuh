// Fused similarity + argmax on the 5th-generation tensor cores.
//
// For a tile of 128 query descriptors and a stream of candidate tiles, the
// scores S = Q * X^T are accumulated in fp32 in tensor memory (tcgen05.mma,
// kind::f16) and reduced on the fly to the largest score of each query row
// and the first 32-column chunk that reaches it.  No score ever leaves the
// SM.  This is the NN1/NN2 operator of the reciprocal set and of Fast
// Reciprocal Matching (cv-learn.com "MASt3R" note, paragraph "Fast reciprocal
// matching (FRM)"), on the dot-product reading of "nearest".
//
// Work decomposition.  A launch holds up to two "families" of problems (the
// two sweeps of the exhaustive set, or the pairs of a batched FRM half-step).
// A family has `nbatch` independent problems; problem b has `count_b`
// queries (fixed, or read from device memory) and `n_cand` candidates.  Each
// problem's queries are cut into 128-row m-tiles; each m-tile's candidate
// range is cut into S contiguous splits.  A work unit is one (m-tile, split);
// CTAs take units round-robin.  Partial results meet in one 64-bit key per
// query: the score bits in the upper word (ordered as unsigned integers) and
// the complement of the index in the lower word, merged with atomicMax, so
// the merge gives the largest score and then the lowest index whatever the
// order of arrival.
//
// Warp roles (4 + kEpiWarps warps):
//   warp 0      TMA producer: candidate tiles into a ring of shared-memory stages
//   warps 1-2   MMA issuers, alternating tiles (warp 1 owns tensor memory).
//               Every wait, fence and commit in an issuing thread costs it
//               hundreds of cycles of latency, which one warp would pay
//               serially on every tile; two warps overlap them.
//   warp 3      query tiles: a TMA box when the rows are contiguous, else
//               indexed rows gathered with plain loads into the same swizzle
//   warps 4..   epilogue (8 or 16 warps).  With kOneGroup all of them take
//               every tile, each a column part; otherwise they form groups
//               that each own one accumulator (tiles g, g+nacc, ...), so that
//               one group reduces while another waits.  Warp w reads TMEM
//               lanes 32*(w%4).. and its part of the columns, hands the
//               accumulator back after its last copy of the tile, folds the
//               values 32 at a time into its row's running maximum, and keeps
//               the first 32-column chunk that reached it.
//
// The exact lowest index inside the kept chunk is not resolved here: the
// packed key carries the chunk's first column, and a small pass afterwards
// recomputes that chunk's 32 scores (locate_chunk, in rnn.cu).  Keeping the
// locate out of the loop leaves the epilogue with one maximum per score and
// three instructions per chunk, with no branches and no shared-memory
// traffic.  Whole chunks compare by their maxima with a strict '>' in
// increasing column order, so the kept chunk is the first that holds the row
// maximum and its lowest maximal column is the lowest-index argmax.
#pragma once
#include <cstdint>
#include <cuda.h>
#include "ptx.cuh"

namespace rnn {

constexpr int kBlockM = 128;
constexpr int kMmaWarps = 2;     // warps 1..kMmaWarps issue MMAs
constexpr int kGatherWarp = 3;
constexpr int kEpiWarp0 = 4;
constexpr int kChunk = 32;       // columns folded per maximum; the locate pass resolves within one
constexpr int kMaxBatchTable = 1024;
constexpr int kMaxStages = 16;   // candidate ring depth limit
constexpr int kMaxAcc = 4;       // accumulator buffers in tensor memory (512 columns in all)
constexpr int kUnitTiles = 8;    // fixed cost of a work unit, in tiles (split-count choice)

// Error bits written to the device error word.
constexpr int kErrWaitProducer = 1 << 0;
constexpr int kErrWaitMma = 1 << 1;
constexpr int kErrWaitGather = 1 << 2;
constexpr int kErrWaitEpilogue = 1 << 3;
constexpr int kErrDrain = 1 << 4;

struct NNFamily {
  const uint16_t* q_base;       // query rows (fp16/bf16 bits), problem b at q_base + b*q_bstride
  int64_t q_bstride;            // elements
  const int32_t* q_list;        // optional: query position -> slot
  const int32_t* q_index;       // optional: slot -> query row
  int64_t slot_bstride;         // elements between problems in q_list / q_index
  const int32_t* q_count_dev;   // optional: per-problem query counts in device memory
  int32_t q_count;              // query count when q_count_dev is null
  int32_t n_cand;               // candidates per problem
  int32_t nbatch;               // problems
  unsigned long long* keys;     // per-query packed result, problem b at keys + b*key_bstride
  int64_t key_bstride;
  int32_t q_tma;                // 1: query rows are contiguous, load them with the Q tensor map
};

struct NNParams {
  NNFamily fam[2];
  int nfam;
  int d;            // channels (multiple of 8)
  int kb;           // K-block width in elements: 16, 32 or 64 (32/64/128-byte swizzle)
  int nkb;          // K-blocks; padded depth K = kb * nkb
  int block_n;      // candidates per stage: 256 or 128
  int stages;       // candidate ring depth
  int nacc;         // accumulators of block_n columns: 2 or 4, nacc * block_n <= 512,
                    // stages a multiple of nacc
  int qbufs;        // query tile buffers: 1 or 2
  uint32_t idesc;   // tcgen05 instruction descriptor
  int target_units; // units to aim for when choosing the split count
  int min_tiles;    // fewest candidate tiles per unit (amortises the query-tile load)
  int* err;         // device error word
  unsigned long long wait_limit_ns;
  int stall_loads;  // failure-detection test: the producer loads no candidate tile, so the
                    // MMA warps' bounded wait on it runs out and the kernel reports a timeout
};

// Packed key: larger is better (higher score, then lower index).
__device__ __forceinline__ unsigned long long pack_key(float s, int idx) {
  s = __fadd_rn(s, 0.0f);  // -0 -> +0 so that equal scores pack equally
  const uint32_t b = __float_as_uint(s);
  const uint32_t o = (b & 0x80000000u) ? ~b : (b | 0x80000000u);
  return (static_cast<unsigned long long>(o) << 32) | (0xFFFFFFFFu - static_cast<uint32_t>(idx));
}
__device__ __forceinline__ int key_index(unsigned long long k) {
  return static_cast<int>(0xFFFFFFFFu - static_cast<uint32_t>(k));
}
__device__ __forceinline__ float key_score(unsigned long long k) {
  const uint32_t o = static_cast<uint32_t>(k >> 32);
  const uint32_t b = (o & 0x80000000u) ? (o & 0x7FFFFFFFu) : ~o;
  return __uint_as_float(b);
}

// Shared-memory descriptor of a K-major operand tile stored with the
// 32/64/128-byte swizzle (rows of kb elements, 8-row groups).
__device__ __forceinline__ uint64_t make_sdesc(uint32_t saddr, int kb) {
  const uint32_t row_bytes = static_cast<uint32_t>(kb) * 2u;
  const uint64_t sbo = (8u * row_bytes) >> 4;
  const uint64_t layout = (kb == 64) ? 2u : (kb == 32) ? 4u : 6u;
  uint64_t desc = 0;
  desc |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  desc |= static_cast<uint64_t>(1u) << 16;  // leading byte offset (unused with swizzle)
  desc |= sbo << 32;
  desc |= static_cast<uint64_t>(1u) << 46;  // descriptor version for sm_100
  desc |= layout << 61;
  return desc;
}

// Index of the 16-byte chunk `c` of row `r` after the swizzle of a tile with
// kb-element rows (the same pattern the TMA unit writes).
__device__ __forceinline__ int swz_chunk(int r, int c, int kb) {
  if (kb == 64) return c ^ (r & 7);
  if (kb == 32) return c ^ ((r >> 1) & 3);
  return c ^ ((r >> 2) & 1);
}

struct UnitInfo {
  int f, b, m, t0, t1, nrows;
};

struct SharedTables {
  int mt_prefix[2][kMaxBatchTable + 1];  // per family: m-tile prefix over problems
  int fam_tiles[2];                      // m-tiles per family
  int split[2];                          // splits per m-tile per family
  int fam_units[2];
  int total_units;
  int ntiles[2];                         // candidate tiles per problem
};

__device__ __forceinline__ int family_count(const NNFamily& F, int b) {
  return F.q_count_dev ? F.q_count_dev[b] : F.q_count;
}

__device__ __forceinline__ UnitInfo decode_unit(const NNParams& p, const SharedTables& T, int u) {
  UnitInfo ui;
  int f = 0;
  if (u >= T.fam_units[0]) {
    u -= T.fam_units[0];
    f = 1;
  }
  const NNFamily& F = p.fam[f];
  const int S = T.split[f];
  const int mt = u / S, sp = u - (u / S) * S;
  // problem b: last b with mt_prefix[f][b] <= mt
  int lo = 0, hi = F.nbatch;  // invariant: prefix[lo] <= mt < prefix[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (T.mt_prefix[f][mid] <= mt) lo = mid; else hi = mid;
  }
  ui.f = f;
  ui.b = lo;
  ui.m = mt - T.mt_prefix[f][lo];
  const int cnt = family_count(F, lo);
  ui.nrows = min(kBlockM, cnt - ui.m * kBlockM);
  const int nt = T.ntiles[f];
  ui.t0 = static_cast<int>((static_cast<long long>(sp) * nt) / S);
  ui.t1 = static_cast<int>((static_cast<long long>(sp + 1) * nt) / S);
  return ui;
}

// Exclusive scan of `n` values (n <= kMaxBatchTable) of m-tile counts into
// T.mt_prefix[f][0..n], by all threads of the block (at least 256, at most
// 32 warps).
__device__ void build_prefix(const NNFamily& F, int* prefix, int* scratch_warp) {
  const int n = F.nbatch;
  const int nthreads = blockDim.x, nwarps = nthreads >> 5;
  const int per = (n + nthreads - 1) / nthreads;
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  int vals[4];
  int local = 0;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const int b = t * per + e;
    int v = 0;
    if (e < per && b < n) {
      const int c = family_count(F, b);
      v = (c + kBlockM - 1) / kBlockM;
    }
    vals[e] = v;
    local += v;
  }
  int incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) scratch_warp[warp] = incl;
  __syncthreads();
  if (t == 0) {
    int run = 0;
    for (int w = 0; w < nwarps; ++w) {
      const int x = scratch_warp[w];
      scratch_warp[w] = run;
      run += x;
    }
    scratch_warp[nwarps] = run;
  }
  __syncthreads();
  int run = scratch_warp[warp] + incl - local;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const int b = t * per + e;
    if (e < per && b < n) prefix[b] = run;
    run += vals[e];
  }
  if (t == 0) prefix[n] = scratch_warp[nwarps];
  __syncthreads();
}

// Largest of 32 values with three-input maxima (17 instructions).
__device__ __forceinline__ float max32(const float (&v)[32]) {
  float a[11];
#pragma unroll
  for (int i = 0; i < 10; ++i) a[i] = fmax3(v[3 * i], v[3 * i + 1], v[3 * i + 2]);
  a[10] = fmaxf(v[30], v[31]);
  const float b0 = fmax3(a[0], a[1], a[2]), b1 = fmax3(a[3], a[4], a[5]);
  const float b2 = fmax3(a[6], a[7], a[8]), b3 = fmaxf(a[9], a[10]);
  return fmaxf(fmax3(b0, b1, b2), b3);
}

// kEpiWarps: epilogue warps (8 or 16); kChunks: 32-column chunks of each
// tile read by one of them; kBatch: chunks per copy from tensor memory to
// registers; kOneGroup: all epilogue warps take every tile (each a column
// part of it) instead of one group per accumulator; kPdl: launched as a
// programmatic dependent of the previous kernel (the FRM chain), so it waits
// for that kernel before reading the query counts.  The wait is compiled only
// into that form: a kernel that holds it costs more to launch plainly.
template <int kEpiWarps, int kChunks, int kBatch, bool kOneGroup = false, bool kPdl = false>
__global__ void __launch_bounds__((kEpiWarp0 + kEpiWarps) * 32, 1)
nn_argmax_kernel(const __grid_constant__ NNParams p, const __grid_constant__ CUtensorMap tmap0,
                 const __grid_constant__ CUtensorMap tmap1,
                 const __grid_constant__ CUtensorMap qmap0,
                 const __grid_constant__ CUtensorMap qmap1) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 1024-byte alignment for the swizzled tiles
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const int kpad = p.kb * p.nkb;
  const uint32_t stage_bytes = static_cast<uint32_t>(p.block_n) * kpad * 2;
  const uint32_t kblk_bytes_x = static_cast<uint32_t>(p.block_n) * p.kb * 2;
  const uint32_t q_bytes = static_cast<uint32_t>(kBlockM) * kpad * 2;
  const uint32_t kblk_bytes_q = static_cast<uint32_t>(kBlockM) * p.kb * 2;

  uint8_t* x_tiles = smem;
  uint8_t* q_tiles = x_tiles + static_cast<size_t>(p.stages) * stage_bytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(q_tiles + static_cast<size_t>(p.qbufs) * q_bytes);
  uint64_t* full_bar = bars;
  // done_bar[s]: the MMAs that read stage s have completed.  One commit per
  // tile tells both the producer (the stage may be refilled) and the
  // epilogue (the accumulator of that tile is ready): every tcgen05.commit
  // costs the tensor pipe tens of cycles, and a tile is only a few hundred.
  uint64_t* done_bar = bars + p.stages;
  uint64_t* qfull_bar = bars + 2 * p.stages;
  uint64_t* qempty_bar = qfull_bar + 2;
  uint64_t* tempty_bar = qempty_bar + 2;
  uint64_t* drain_bar = tempty_bar + kMaxAcc;
  uint32_t* misc = reinterpret_cast<uint32_t*>(drain_bar + kMmaWarps);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
  int* qrows = reinterpret_cast<int*>(misc + 4);            // [128]
  int* scan_scratch = qrows + kBlockM;                       // [warps + 1]
  SharedTables* T = reinterpret_cast<SharedTables*>(scan_scratch + 32);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // epilogue warps per group: one group per accumulator, or with kOneGroup a
  // single group taking every tile
  const int epi_per_group = kOneGroup ? kEpiWarps : kEpiWarps / p.nacc;
  // tensor-memory allocation: a power of two of at least 32 columns
  uint32_t ncols = 32;
  while (ncols < static_cast<uint32_t>(p.nacc * p.block_n)) ncols <<= 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < p.stages; ++s) {
      mbar_init(smem_u32(&full_bar[s]), 1);
      mbar_init(smem_u32(&done_bar[s]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&qfull_bar[i]), 1);
      mbar_init(smem_u32(&qempty_bar[i]), kMmaWarps);
    }
    for (int i = 0; i < p.nacc; ++i) mbar_init(smem_u32(&tempty_bar[i]), epi_per_group);
    for (int i = 0; i < kMmaWarps; ++i) mbar_init(smem_u32(&drain_bar[i]), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmap0);
    if (p.nfam > 1) tma_prefetch_desc(&tmap1);
    if (p.fam[0].q_tma) tma_prefetch_desc(&qmap0);
    if (p.nfam > 1 && p.fam[1].q_tma) tma_prefetch_desc(&qmap1);
  }
  // everything below reads the previous kernel's output (query counts, lists)
  if constexpr (kPdl) pdl_wait();
  // unit table
  for (int f = 0; f < 2; ++f) {
    if (f < p.nfam) {
      build_prefix(p.fam[f], T->mt_prefix[f], scan_scratch);
    }
  }
  if (warp == 0) {
    // every lane derives the same sizes; the split counts are then tried
    // one per lane and the lanes agree on the best with a min-reduction
    // (a serial search in one thread costs microseconds of 64-bit division
    // on every launch)
    int fam_tiles[2], ntiles[2], caps[2];
    int tiles_total = 0;
    for (int f = 0; f < 2; ++f) {
      fam_tiles[f] = f < p.nfam ? T->mt_prefix[f][p.fam[f].nbatch] : 0;
      ntiles[f] = f < p.nfam ? (p.fam[f].n_cand + p.block_n - 1) / p.block_n : 1;
      caps[f] = max(1, ntiles[f] / max(1, p.min_tiles));
      tiles_total += fam_tiles[f];
    }
    // split count: enough units for the target, and among the counts from
    // there up to 2x that (units of at least min_tiles tiles) the one whose
    // round-robin deal gives the CTAs the smallest largest share, the
    // smallest such count on a tie.  When the target needs more splits than
    // min_tiles allows (a few query tiles, as in the late FRM half-steps),
    // the counts from half that cap up to it.
    int S0 = tiles_total > 0 ? (p.target_units + tiles_total - 1) / tiles_total : 1;
    if (S0 < 1) S0 = 1;
    int cap = 1;
    for (int f = 0; f < 2; ++f)
      if (f < p.nfam) cap = max(cap, caps[f]);
    const int Smax = max(1, min(2 * S0, cap));
    const int Smin = max(1, min(S0, Smax / 2));
    const unsigned grid = gridDim.x;
    unsigned long long best = ~0ull;  // (share << 24) | count
    for (int c = Smin + lane; c <= Smax; c += 32) {
      unsigned units = 0;
      int biggest = 1;  // tiles of the largest unit
      for (int f = 0; f < 2; ++f) {
        if (fam_tiles[f] == 0) continue;
        const int Sf = min(c, caps[f]);
        units += static_cast<unsigned>(fam_tiles[f]) * static_cast<unsigned>(Sf);
        biggest = max(biggest, (ntiles[f] + Sf - 1) / Sf);
      }
      // each unit also costs about kUnitTiles tiles (query tile, pipeline
      // fill, final merge)
      const unsigned long long share =
          static_cast<unsigned long long>((units + grid - 1) / grid) * (biggest + kUnitTiles);
      const unsigned long long key = (share << 24) | static_cast<unsigned>(c);
      best = key < best ? key : best;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const unsigned long long y = __shfl_xor_sync(0xffffffffu, best, o);
      best = y < best ? y : best;
    }
    if (lane == 0) {
      const int S = best == ~0ull ? Smin : static_cast<int>(best & 0xFFFFFFull);
      int total = 0;
      for (int f = 0; f < 2; ++f) {
        const int Sf = min(S, caps[f]);
        T->fam_tiles[f] = fam_tiles[f];
        T->ntiles[f] = ntiles[f];
        T->split[f] = Sf;
        T->fam_units[f] = fam_tiles[f] * Sf;
        total += T->fam_units[f];
      }
      T->total_units = total;
    }
  }
  __syncthreads();
  const int total_units = T->total_units;
  if (total_units == 0) return;  // no live query (late FRM half-steps): no tensor memory
  if (warp == 1) {
    tmem_alloc(smem_u32(misc), ncols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = misc[0];
  const uint64_t lim = p.wait_limit_ns;

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      long long issued = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < total_units && ok; u += gridDim.x) {
        const UnitInfo ui = decode_unit(p, *T, u);
        const CUtensorMap* map = ui.f == 0 ? &tmap0 : &tmap1;
        for (int t = ui.t0; t < ui.t1; ++t) {
          if (!mbar_wait_sleep(smem_u32(&done_bar[stage]), phase ^ 1u, abort_flag, p.err,
                               kErrWaitProducer, lim)) {
            ok = false;
            break;
          }
          const uint32_t fb = smem_u32(&full_bar[stage]);
          if (!p.stall_loads) {
            mbar_arrive_expect_tx(fb, stage_bytes);
            const uint32_t dst = smem_u32(x_tiles + static_cast<size_t>(stage) * stage_bytes);
            for (int kk = 0; kk < p.nkb; ++kk)
              tma_load_3d(dst + kk * kblk_bytes_x, map, fb, kk * p.kb, t * p.block_n, ui.b);
            ++issued;
          }
          if (++stage == p.stages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        // wait (bounded) for the loads still in flight before the CTA exits
        const long long n = issued < p.stages ? issued : p.stages;
        for (long long q = issued - n; q < issued; ++q) {
          const int s = static_cast<int>(q % p.stages);
          const uint32_t ph = static_cast<uint32_t>((q / p.stages) & 1);
          const uint64_t t0 = globaltimer_ns();
          while (!mbar_try_wait(smem_u32(&full_bar[s]), ph)) {
            if (globaltimer_ns() - t0 > lim) {
              atomicOr(p.err, kErrDrain);
              break;
            }
          }
        }
      }
    }
  } else if (warp <= kMmaWarps) {
    // ------------------------------------------------------ MMA issuers
    // Warp 1 takes the tiles g = 0, 2, 4, ... of this CTA's sequence, warp 2
    // the odd ones (nacc is even, so each warp keeps its own accumulators).
    // The loop runs on warp-uniform values and one elected lane issues.
    const int mw = warp - 1;
    int stage = 0, acc = 0, qb = 0;
    uint32_t phase = 0, acc_phase = 0, qphase = 0;
    bool ok = true, any = false;
    const int ksteps = kpad / 16;
    const int spk = p.kb / 16;                                   // K-steps per K-block
    const uint64_t a_desc0 = make_sdesc(smem_u32(q_tiles), p.kb);
    const uint64_t b_desc0 = make_sdesc(smem_u32(x_tiles), p.kb);
    const uint32_t a_jump = (kblk_bytes_q - (spk - 1) * 32) >> 4;  // to the next K-block
    const uint32_t b_jump = (kblk_bytes_x - (spk - 1) * 32) >> 4;
    const uint32_t q_step = q_bytes >> 4, x_step = stage_bytes >> 4;
    const uint32_t idesc = p.idesc;
    for (int u = blockIdx.x; u < total_units && ok; u += gridDim.x) {
      const UnitInfo ui = decode_unit(p, *T, u);
      ok = __all_sync(0xffffffffu,
                      mbar_wait(smem_u32(&qfull_bar[qb]), qphase, abort_flag, p.err, kErrWaitMma,
                                lim));
      if (!ok) break;
      const uint64_t a_unit = a_desc0 + static_cast<uint64_t>(qb) * q_step;
      for (int t = ui.t0; t < ui.t1; ++t) {
        if ((acc & 1) == mw) {
          ok = __all_sync(0xffffffffu,
                          mbar_wait(smem_u32(&full_bar[stage]), phase, abort_flag, p.err,
                                    kErrWaitMma, lim) &&
                              mbar_wait_sleep(smem_u32(&tempty_bar[acc]), acc_phase ^ 1u,
                                              abort_flag, p.err, kErrWaitMma, lim));
          if (!ok) break;
          tc_fence_after();
          const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * p.block_n);
          uint64_t a = a_unit, b = b_desc0 + static_cast<uint64_t>(stage) * x_step;
          int w = 0;
          for (int k = 0; k < ksteps; ++k) {
            umma_f16_warp(d_tmem, a, b, idesc, k > 0 ? 1u : 0u);
            if (++w == spk) {
              w = 0;
              a += a_jump;
              b += b_jump;
            } else {
              a += 2;
              b += 2;
            }
          }
          umma_commit_warp(smem_u32(&done_bar[stage]));
          __syncwarp();
          any = true;
        }
        if (++stage == p.stages) {
          stage = 0;
          phase ^= 1u;
        }
        if (++acc == p.nacc) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      if (!ok) break;
      // the query tile is free once both warps' MMAs of the unit are done
      umma_commit_warp(smem_u32(&qempty_bar[qb]));
      __syncwarp();
      if (++qb == p.qbufs) {
        qb = 0;
        qphase ^= 1u;
      }
    }
    if (!ok && any) {
      // let every MMA this warp issued finish before tensor memory is released
      umma_commit_warp(smem_u32(&drain_bar[mw]));
      __syncwarp();
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(smem_u32(&drain_bar[mw]), 0)) {
        if (globaltimer_ns() - t0 > lim) {
          if (lane == 0) atomicOr(p.err, kErrDrain);
          break;
        }
      }
    }
  } else if (warp == kGatherWarp) {
    // ---------------------------------------------------- query gather
    int qb = 0;
    uint32_t qphase = 0;
    int q_last = 0;
    uint32_t q_last_phase = 0;
    bool q_any = false;
    const int nch_real = p.d / 8;       // 16-byte chunks holding data
    const int nch_row = kpad / 8;       // chunks per padded row
    const int ch_per_kblk = p.kb / 8;
    for (int u = blockIdx.x; u < total_units; u += gridDim.x) {
      const UnitInfo ui = decode_unit(p, *T, u);
      if (!mbar_wait_sleep(smem_u32(&qempty_bar[qb]), qphase ^ 1u, abort_flag, p.err,
                           kErrWaitGather, lim))
        break;
      const NNFamily& F = p.fam[ui.f];
      if (F.q_tma) {
        // contiguous query rows: one TMA box per K-block, rows past the end are zero
        if (lane == 0) {
          const uint32_t qf = smem_u32(&qfull_bar[qb]);
          mbar_arrive_expect_tx(qf, q_bytes);
          const uint32_t dst = smem_u32(q_tiles + static_cast<size_t>(qb) * q_bytes);
          const CUtensorMap* qm = ui.f == 0 ? &qmap0 : &qmap1;
          for (int kk = 0; kk < p.nkb; ++kk)
            tma_load_3d(dst + kk * kblk_bytes_q, qm, qf, kk * p.kb, ui.m * kBlockM, ui.b);
        }
        __syncwarp();
        q_last = qb;
        q_last_phase = qphase;
        q_any = true;
        if (++qb == p.qbufs) {
          qb = 0;
          qphase ^= 1u;
        }
        continue;
      }
      for (int r = lane; r < kBlockM; r += 32) {
        int row = -1;
        if (r < ui.nrows) {
          int pos = ui.m * kBlockM + r;
          int slot = F.q_list ? __ldg(F.q_list + ui.b * F.slot_bstride + pos) : pos;
          row = F.q_index ? __ldg(F.q_index + ui.b * F.slot_bstride + slot) : slot;
        }
        qrows[r] = row;
      }
      __syncwarp();
      const uint16_t* qsrc = F.q_base + ui.b * F.q_bstride;
      uint8_t* qdst = q_tiles + static_cast<size_t>(qb) * q_bytes;
      const int items = kBlockM * nch_row;
      for (int it0 = 0; it0 < items; it0 += 32 * 8) {
        uint4 v[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int it = it0 + j * 32 + lane;
          v[j] = make_uint4(0, 0, 0, 0);
          if (it < items) {
            const int r = it / nch_row, c = it - (it / nch_row) * nch_row;
            const int row = qrows[r];
            if (row >= 0 && c < nch_real)
              v[j] = __ldg(reinterpret_cast<const uint4*>(qsrc + static_cast<int64_t>(row) * p.d) + c);
          }
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int it = it0 + j * 32 + lane;
          if (it < items) {
            const int r = it / nch_row, c = it - (it / nch_row) * nch_row;
            const int kblk = c / ch_per_kblk, cw = c - kblk * ch_per_kblk;
            uint8_t* dst = qdst + kblk * kblk_bytes_q + r * (p.kb * 2) +
                           swz_chunk(r, cw, p.kb) * 16;
            *reinterpret_cast<uint4*>(dst) = v[j];
          }
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&qfull_bar[qb]));
      if (++qb == p.qbufs) {
        qb = 0;
        qphase ^= 1u;
      }
    }
    if (*abort_flag && q_any && lane == 0) {
      // a query-tile TMA load may still be in flight: wait for it (bounded)
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(smem_u32(&qfull_bar[q_last]), q_last_phase)) {
        if (globaltimer_ns() - t0 > lim) {
          atomicOr(p.err, kErrDrain);
          break;
        }
      }
    }
  } else {
    // --------------------------------------------------------- epilogue
    // Group `grp` reduces the tiles of accumulator grp (one group per
    // accumulator), or with kOneGroup the one group takes every tile; within
    // it, warp w covers TMEM lanes
    // 32*(w%4).. and column part `part` of each tile, kBatch chunks of 32
    // columns per copy to registers.  After the last copy of a tile the
    // accumulator goes back to the MMA warps, before that copy is folded: with
    // one copy per tile (kChunks == kBatch) it is held for one round trip.
    const int ew = warp - kEpiWarp0;
    const int quad = warp & 3;
    const int grp = ew / epi_per_group;
    const int part = (ew - grp * epi_per_group) >> 2;
    const int row = quad * 32 + lane;
    constexpr int cols_part = kChunk * kChunks;
    // with one group per accumulator the group's accumulator column is fixed;
    // with kOneGroup it is added per tile
    const uint32_t lane_base =
        tmem_base + (static_cast<uint32_t>(quad * 32) << 16) +
        static_cast<uint32_t>((kOneGroup ? 0 : grp * p.block_n) + part * cols_part);
    int acc = 0, stage = 0;  // position of tile t in this CTA's tile sequence
    uint32_t phase = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < total_units && ok; u += gridDim.x) {
      const UnitInfo ui = decode_unit(p, *T, u);
      const NNFamily& F = p.fam[ui.f];
      float best = -__int_as_float(0x7f800000);
      int bcol = -1;  // first column of the first chunk that reached `best`
      for (int t = ui.t0; t < ui.t1; ++t) {
        if (kOneGroup || acc == grp) {
          // stages is a multiple of nacc, so done_bar[stage] is only ever
          // used by this group's tiles, and its next phase needs this tile's
          // accumulator back: the parity below cannot be a phase behind
          // every lane polls the same barrier and abort word, so the outcome
          // is the same in all lanes unless the barrier completes during an
          // abort; a warp-wide vote here costs 8 % of the sweep
          if (!mbar_wait_sleep(smem_u32(&done_bar[stage]), phase, abort_flag, p.err,
                               kErrWaitEpilogue, lim)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const int col0 = t * p.block_n + part * cols_part;   // first candidate of this part
          const int valid = F.n_cand - col0;                    // candidates left from col0
#pragma unroll
          for (int h = 0; h < kChunks; h += kBatch) {
            float v[kBatch][kChunk];
#pragma unroll
            for (int c = 0; c < kBatch; ++c)
              tmem_ld32(lane_base + static_cast<uint32_t>((kOneGroup ? acc * p.block_n : 0) +
                                                          kChunk * (h + c)),
                        v[c]);
            tmem_wait_ld_regs(v[0]);
#pragma unroll
            for (int c = 1; c < kBatch; ++c) reg_fence(v[c]);
            if (h + kBatch == kChunks) {
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(smem_u32(&tempty_bar[acc]));
              // keep the reductions below the release
#pragma unroll
              for (int c = 0; c < kBatch; ++c) reg_fence(v[c]);
            }
            if (valid < kChunk * (h + kBatch)) {
              // ragged last tile: columns past the candidates never win
#pragma unroll
              for (int c = 0; c < kBatch; ++c)
#pragma unroll
                for (int k = 0; k < kChunk; ++k)
                  if (kChunk * (h + c) + k >= valid) v[c][k] = -__int_as_float(0x7f800000);
            }
#pragma unroll
            for (int c = 0; c < kBatch; ++c) {
              const float m = max32(v[c]);
              const bool up = m > best;
              best = up ? m : best;
              bcol = up ? col0 + kChunk * (h + c) : bcol;
            }
          }
        }
        if (++stage == p.stages) {
          stage = 0;
          phase ^= 1u;
        }
        if (++acc == p.nacc) acc = 0;
      }
      if (!ok) break;
      if (row < ui.nrows && bcol >= 0) {
        unsigned long long* kp = F.keys + ui.b * F.key_bstride + ui.m * kBlockM + row;
        atomicMax(kp, pack_key(best, bcol));
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, ncols);
  }
}

}  // namespace rnn
