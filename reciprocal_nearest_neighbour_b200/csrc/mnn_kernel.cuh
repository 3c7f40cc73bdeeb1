// One-pass fused kernel for the exhaustive reciprocal set.
//
// M = {(i,j) | j = NN2(D1_i) and i = NN1(D2_j)} (cv-learn.com "MASt3R" note,
// paragraph "Fast reciprocal matching (FRM)") needs the largest score of
// every row AND of every column of S = D1 * D2^T.  The two-sweep form
// (nn_kernel.cuh with both families) computes every score twice on the
// tensor cores.  This kernel computes each 128 x 256 tile of S once
// (tcgen05.mma, fp32 in tensor memory) and reduces it in both directions.
//
// Tensor-memory reads.  Each epilogue warp owns a quadrant q of the 128
// lanes (rows) and a 64-column part p of the tile.  It reads its 32 x 64
// block with two tcgen05.ld.16x128b.x16, which gives every thread 4 rows x 16
// columns (rows g, g+8, g+16, g+24 with g = lane/4; columns 4j + s with
// s = lane%4).  So a thread holds 4 rows of each of its columns, and each
// column needs only a cross-lane step over 8 lanes, each row over 4 lanes.
// (16x256b gives the same shape of ownership but reads tensor memory at
// about half the rate on B200: ~520 against ~270 cycles per 128 x 256 tile
// and SM.)
//
// Loop order.  A work unit is bm m-tiles (image-1 rows) x bn n-tiles (image-2
// rows).  For each n-tile, the m-tiles go by in the inner loop, so every
// thread keeps the running maximum of its 16 columns in registers over the
// whole inner loop (two three-input maxima per column and tile), merges
// them across its 8 lanes once per n-tile and writes them to the global keys
// with atomicMax (one chunk per quadrant, so no meeting between warps).  Row
// partials (one per row and 64-column part, after a two-step shuffle across
// 4 lanes) go to shared memory, where each (m-tile, row, part) slot keeps the
// best over the n-tiles with the first n-tile that reached it; they are
// merged and written once per unit.
//
// Metric.  The kernel takes the largest score of rows and columns of
// whatever the copies of the maps give: the dot product, or under the
// Euclidean metric the copies' extra columns make every score
// -|q - x|^2 / 2, symmetric in the two maps (op_copy_kernel in rnn.cu).
//
// Ragged edges.  The maps are read from copies whose rows past the last
// pixel (up to a whole unit) are NaN, so every score there is NaN, and the
// three-input maximum (like fmaxf) returns the other operands when one is
// NaN: those rows and columns never take part, with no masks in the loop.  A
// part or quadrant wholly past the end reduces to NaN and is skipped when
// written.
//
// Chunks and the exact index.  As in the row-only kernel, the fold keeps the
// maximum and the first chunk reaching it; a locate pass afterwards resolves
// the lowest index inside the chunk.  Row chunks are the 64-column parts.
// For columns, the quadrant is the finest piece a lane-group merge can name,
// so the query tile of m-tile l of m-block mb is gathered as four 32-row
// slices: quadrant q holds rows mb*128*bm + 32*(bm*q + l) + [0, 32).  Then
// quadrant q over the bm m-tiles of the block is the contiguous range
// [mb*128*bm + 32*bm*q, +32*bm): the column chunk.  Chunks compare by their
// maxima with a strict '>' in increasing order, so the kept chunk is the
// first that holds the maximum.
//
// Warp roles (19 warps):
//   warp 0       TMA producer: the bm query tiles of a unit (four 32-row
//                boxes each) once per unit, the candidate tile once per n-tile
//   warps 1-2    MMA issuers, one per accumulator (tile l of an n-pass uses
//                accumulator l % 2).  Each waits for its own accumulator, so
//                the two turnarounds (commit, wake-up, release, re-issue)
//                overlap.  A shared-memory slot is refilled once both warps
//                have committed after its last reader; that is safe while a
//                slot's reuse period is at least 5 tiles (a warp can run at
//                most 4 tiles ahead of the other), so small units use warp 1
//                alone (nmma = 1).
//   warps 3..18  epilogue, quadrant q = warp % 4, part p = (warp - 3) / 4.
//                The epilogue warps beside the MMA warps (q = 1, 2) run about
//                a tile behind the others and their releases gate every next
//                MMA: they poll the accumulator barrier without suspending (a
//                suspended wait wakes up later).  The warps of q = 0, 3 wait
//                ahead of them and suspend.
#pragma once
#include <cstdint>
#include <type_traits>
#include <cuda.h>
#include "nn_kernel.cuh"
#include "ptx.cuh"

namespace rnn {

constexpr int kOpEpiWarp0 = 3;
constexpr int kOpEpiWarps = 16;
constexpr int kOpThreads = (kOpEpiWarp0 + kOpEpiWarps) * 32;  // 608
constexpr int kOpBlockN = 256;
constexpr int kOpMaxBm = 16;      // query tiles a unit holds in shared memory
constexpr int kOpMaxBn = 8;       // candidate tiles per unit (row chunk ids are bytes)
constexpr int kOpRowChunk = 64;   // columns of a row chunk (one epilogue warp's part)

struct OnePassParams {
  int n1, n2;            // image-1 rows (tensor-memory lanes), image-2 rows (columns)
  int kpad;              // K of the tiles: 16, 32 or 64 (one K-block, swizzle 2*kpad bytes)
  int bm, bn;            // m-tiles (an even power of two) and n-tiles of a unit
  int nmma;              // MMA-issuing warps: 2, or 1 for small units
  int mblocks, nblocks;  // units = mblocks * nblocks; unit u -> (u % mblocks, u / mblocks)
  uint32_t idesc;
  unsigned long long* rowk;  // [n1] (score, first column of the row chunk), atomicMax
  unsigned long long* colk;  // [n2] (score, first row of the column chunk), atomicMax
  int* err;
  unsigned long long wait_limit_ns;
  int stall_loads;       // failure-detection test: load nothing, so the MMA warp's wait runs out
};

// Shared-memory layout, offsets from the 1024-byte aligned base.
struct OnePassSmem {
  uint32_t a_off, b_off, rbest_off, rchunk_off, bar_off, misc_off, total;
};

__host__ __device__ inline OnePassSmem onepass_smem(int kpad, int bm) {
  OnePassSmem s;
  const uint32_t a_bytes = 128u * static_cast<uint32_t>(kpad) * 2u;
  const uint32_t b_bytes = 256u * static_cast<uint32_t>(kpad) * 2u;
  s.a_off = 0;
  s.b_off = s.a_off + static_cast<uint32_t>(bm) * a_bytes;
  s.rbest_off = s.b_off + 2u * b_bytes;                             // float [bm][4][128]
  s.rchunk_off = s.rbest_off + static_cast<uint32_t>(bm) * 4u * 128u * 4u;  // u8 [bm][4][128]
  s.bar_off = (s.rchunk_off + static_cast<uint32_t>(bm) * 4u * 128u + 15u) & ~15u;
  // a_full[16], a_empty[16], b_full[2], b_empty[2], acc_full[2], acc_empty[2],
  // rowbar, drain[2]
  s.misc_off = s.bar_off + (2u * kOpMaxBm + 11u) * 8u;
  s.total = s.misc_off + 16u;
  return s;
}

// Row state of one (m-tile, row, part) slot: the best score over the
// n-tiles so far and the first n-tile that reached it.  The first n-tile
// writes the slot whatever it held (also when y is NaN: a part wholly past
// the last image-2 row); a later n-tile n replaces it only with a strictly
// larger y.  Branch-free.
__device__ __forceinline__ void row_state_first(uint32_t slot, uint32_t cslot, float y) {
  asm volatile(
      "st.shared.f32 [%0], %2;\n\t"
      "st.shared.u8 [%1], 0;" ::"r"(slot),
      "r"(cslot), "f"(y)
      : "memory");
}
__device__ __forceinline__ void row_state_update(uint32_t slot, uint32_t cslot, float y, int n) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t.reg .f32 o;\n\t"
      "ld.shared.f32 o, [%0];\n\t"
      "setp.gt.f32 p, %2, o;\n\t"
      "@p st.shared.f32 [%0], %2;\n\t"
      "@p st.shared.u8 [%1], %3;\n\t}" ::"r"(slot),
      "r"(cslot), "f"(y), "r"(n)
      : "memory");
}

// Keep one of two values and send the other to the partner lane `mask`
// away; the lane whose bit is set keeps `hi`.  Returns the larger of the
// kept value and the partner's.
__device__ __forceinline__ float swap_max(float lo, float hi, bool bit, int mask) {
  const float send = bit ? lo : hi;
  const float keep = bit ? hi : lo;
  return fmaxf(keep, __shfl_xor_sync(0xffffffffu, send, mask));
}

__global__ void __launch_bounds__(kOpThreads, 1)
mnn_onepass_kernel(const __grid_constant__ OnePassParams p,
                   const __grid_constant__ CUtensorMap amap,   // image-1 rows, 32-row boxes
                   const __grid_constant__ CUtensorMap bmap) { // image-2 rows, 256-row boxes
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const OnePassSmem L = onepass_smem(p.kpad, p.bm);
  uint8_t* a_tiles = smem + L.a_off;
  uint8_t* b_tiles = smem + L.b_off;
  float* rbest = reinterpret_cast<float*>(smem + L.rbest_off);
  uint8_t* rchunk = smem + L.rchunk_off;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bar_off);
  uint64_t* a_full = bars;
  uint64_t* a_empty = bars + kOpMaxBm;
  uint64_t* b_full = bars + 2 * kOpMaxBm;
  uint64_t* b_empty = b_full + 2;
  uint64_t* acc_full = b_empty + 2;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* rowbar = acc_empty + 2;
  uint64_t* drain_bar = rowbar + 1;  // [2], one per MMA warp
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + L.misc_off);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t a_bytes = 128u * static_cast<uint32_t>(p.kpad) * 2u;
  const uint32_t b_bytes = 256u * static_cast<uint32_t>(p.kpad) * 2u;
  const int units = p.mblocks * p.nblocks;
  const int bm = p.bm, bn = p.bn;

  if (threadIdx.x == 0) {
    for (int l = 0; l < bm; ++l) {
      mbar_init(smem_u32(&a_full[l]), 1);
      mbar_init(smem_u32(&a_empty[l]), p.nmma);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&b_full[i]), 1);
      mbar_init(smem_u32(&b_empty[i]), p.nmma);
      mbar_init(smem_u32(&acc_full[i]), 1);
      mbar_init(smem_u32(&acc_empty[i]), kOpEpiWarps);
    }
    mbar_init(smem_u32(rowbar), kOpEpiWarps);
    mbar_init(smem_u32(&drain_bar[0]), 1);
    mbar_init(smem_u32(&drain_bar[1]), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&amap);
    tma_prefetch_desc(&bmap);
  }
  __syncthreads();
  if (static_cast<int>(blockIdx.x) >= units) return;
  if (warp == 1) {
    tmem_alloc(smem_u32(misc), 512);
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
      int a_it = 0;         // unit iterations: each query slot is loaded once per unit
      long long b_cnt = 0;  // candidate tiles loaded
      // parity of the phase the last load issued into each candidate slot
      // completes (-1: none); query slots 0..a_n-1 were last loaded in unit
      // iteration a_last, the others in a_last - 1
      int b_par0 = -1, b_par1 = -1, a_last = -1, a_n = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < units && ok; u += gridDim.x, ++a_it) {
        const int mb = u % p.mblocks, nb = u / p.mblocks;
        for (int n = 0; n < bn && ok; ++n) {
          const int bs = static_cast<int>(b_cnt & 1);
          const uint32_t use = static_cast<uint32_t>((b_cnt >> 1) & 1);  // phase of this use
          if (!mbar_wait_sleep(smem_u32(&b_empty[bs]), use ^ 1u, abort_flag, p.err,
                               kErrWaitProducer, lim)) {
            ok = false;
            break;
          }
          if (!p.stall_loads) {
            const uint32_t fb = smem_u32(&b_full[bs]);
            mbar_arrive_expect_tx(fb, b_bytes);
            tma_load_3d(smem_u32(b_tiles + bs * b_bytes), &bmap, fb, 0, (nb * bn + n) * kOpBlockN,
                        0);
            if (bs == 0) b_par0 = static_cast<int>(use); else b_par1 = static_cast<int>(use);
          }
          ++b_cnt;
          if (n != 0) continue;
          for (int l = 0; l < bm; ++l) {
            if (!mbar_wait_sleep(smem_u32(&a_empty[l]), static_cast<uint32_t>(a_it & 1) ^ 1u,
                                 abort_flag, p.err, kErrWaitProducer, lim)) {
              ok = false;
              break;
            }
            if (!p.stall_loads) {
              const uint32_t fa = smem_u32(&a_full[l]);
              mbar_arrive_expect_tx(fa, a_bytes);
              const uint32_t dst = smem_u32(a_tiles + l * a_bytes);
              for (int q = 0; q < 4; ++q)
                tma_load_3d(dst + q * (a_bytes / 4), &amap, fa, 0,
                            mb * 128 * bm + 32 * (bm * q + l), 0);
              a_last = a_it;
              a_n = l + 1;
            }
          }
        }
      }
      if (!ok) {
        // wait (bounded) for the loads still in flight before the CTA exits
        const uint64_t t0 = globaltimer_ns();
        for (int i = 0; i < 2 + bm; ++i) {
          const int al = i - 2 < a_n ? a_last : a_last - 1;
          const int par = i == 0 ? b_par0 : i == 1 ? b_par1 : (al < 0 ? -1 : (al & 1));
          if (par < 0) continue;
          const uint32_t bar = smem_u32(i < 2 ? &b_full[i] : &a_full[i - 2]);
          while (!mbar_try_wait(bar, static_cast<uint32_t>(par))) {
            if (globaltimer_ns() - t0 > lim) {
              atomicOr(p.err, kErrDrain);
              break;
            }
          }
        }
      }
    }
  } else if (warp <= 2) {
    // ------------------------------------------------------ MMA issuers
    const int mw = warp - 1;
    long long b_cnt = 0;
    int a_it = 0;
    uint32_t ph = 0;  // phase of this warp's accumulator's next use (bit per accumulator)
    bool ok = mw < p.nmma, any = false;
    const uint64_t a_desc0 = make_sdesc(smem_u32(a_tiles), p.kpad);
    const uint64_t b_desc0 = make_sdesc(smem_u32(b_tiles), p.kpad);
    const uint32_t a_step = a_bytes >> 4, b_step = b_bytes >> 4;
    const int ksteps = p.kpad / 16;
    const uint32_t idesc = p.idesc;
    for (int u = blockIdx.x; u < units && ok; u += gridDim.x, ++a_it) {
      for (int n = 0; n < bn && ok; ++n, ++b_cnt) {
        const int bs = static_cast<int>(b_cnt & 1);
        const uint32_t bpar = static_cast<uint32_t>((b_cnt >> 1) & 1);
        bool b_seen = false;  // this warp has seen the candidate tile of this pass land
        for (int l = 0; l < bm; ++l) {
          const int acc = l & 1;
          if (p.nmma == 1 || acc == mw) {
            const uint32_t aph = (ph >> acc) & 1u;
            // a query slot lands once per unit (this warp's slots are the same
            // in every pass: bm is even when two warps issue), the candidate
            // tile once per pass
            ok = __all_sync(0xffffffffu,
                            (n > 0 || mbar_wait_sleep(smem_u32(&a_full[l]),
                                                      static_cast<uint32_t>(a_it & 1),
                                                      abort_flag, p.err, kErrWaitMma, lim)) &&
                                (b_seen || mbar_wait_sleep(smem_u32(&b_full[bs]), bpar,
                                                           abort_flag, p.err, kErrWaitMma,
                                                           lim)) &&
                                mbar_wait_sleep(smem_u32(&acc_empty[acc]), aph ^ 1u, abort_flag,
                                                p.err, kErrWaitMma, lim));
            if (!ok) break;
            b_seen = true;
            ph ^= 1u << acc;
            tc_fence_after();
            const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * kOpBlockN);
            const uint64_t a = a_desc0 + static_cast<uint64_t>(l) * a_step;
            const uint64_t b = b_desc0 + static_cast<uint64_t>(bs) * b_step;
            for (int k = 0; k < ksteps; ++k)
              umma_f16_warp(d_tmem, a + 2 * k, b + 2 * k, idesc, k > 0 ? 1u : 0u);
            umma_commit_warp(smem_u32(&acc_full[acc]));
            any = true;
          }
          // every MMA warp commits after the last reader of a slot (each
          // commit covers that warp's MMAs so far)
          if (n == bn - 1) umma_commit_warp(smem_u32(&a_empty[l]));
          if (l == bm - 1) umma_commit_warp(smem_u32(&b_empty[bs]));
          __syncwarp();
        }
      }
    }
    if (mw < p.nmma && !ok && any) {
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
  } else {
    // --------------------------------------------------------- epilogue
    const int e = warp - kOpEpiWarp0;
    const int q = warp & 3;        // tensor-memory lane quadrant this warp may read
    const bool spin = q == 1 || q == 2;  // shares its sub-partition with an MMA warp
    const int part = e >> 2;       // 64-column part of the tile
    const int g = lane >> 2, s = lane & 3;
    const bool s0 = (lane & 1) != 0, s1 = (lane & 2) != 0;
    const bool g0 = (lane & 4) != 0, g1 = (lane & 8) != 0, g2 = (lane & 16) != 0;
    const bool lane0 = lane == 0;
    const uint32_t tq = tmem_base + (static_cast<uint32_t>(32 * q) << 16) +
                        static_cast<uint32_t>(64 * part);
    // this lane's row-state slot: row 32q + g + 8s of part `part`, per m-tile l
    const int rslot = part * 128 + 32 * q + g + 8 * s;
    const uint32_t rb_s = smem_u32(rbest) + 4u * rslot, rc_s = smem_u32(rchunk) + rslot;
    const uint32_t full0 = smem_u32(&acc_full[0]), full1 = smem_u32(&acc_full[1]);
    const uint32_t empty0 = smem_u32(&acc_empty[0]), empty1 = smem_u32(&acc_empty[1]);
    const float ninf = -__int_as_float(0x7f800000);
    // phase of the accumulators' next results: tiles alternate between the
    // two (bm is even), so both accumulators' k-th uses share the parity k % 2
    uint32_t ph = 0;
    int rowphase = 0;
    bool ok = true;
    float pm[16];      // running maxima of this thread's 16 columns over its rows

    // One tile (query tile l of the n-pass, candidate tile n) in accumulator
    // kAcc: read the 4 x 16 block (rows g, g+8 into va, rows g+16, g+24 into
    // vb; column 4j + s in registers 2j and 2j + 1), hand the accumulator
    // back, fold it.
    auto tile = [&](auto acc_c, auto first_c, int l, int n) -> bool {
      constexpr int kAcc = decltype(acc_c)::value;
      constexpr bool kFirst = decltype(first_c)::value;  // n == 0
      // the sub-partitions of the two MMA warps (q = 1, 2) set the tile period
      // and poll; the other two wait ahead of them, and suspend so that their
      // polling adds nothing to the barrier traffic
      const uint32_t fb = kAcc ? full1 : full0;
      if (!(spin ? mbar_wait_spin(fb, ph, abort_flag, p.err, kErrWaitEpilogue, lim)
                 : mbar_wait_sleep(fb, ph, abort_flag, p.err, kErrWaitEpilogue, lim)))
        return false;
      if (kAcc) ph ^= 1u;
      tc_fence_after();
      float va[32], vb[32];
      const uint32_t ta = tq + static_cast<uint32_t>(kAcc * kOpBlockN);
      tmem_ld16x128_x16(ta, va);
      tmem_ld16x128_x16(ta + (16u << 16), vb);
      tmem_wait_ld_regs(va);
      reg_fence(vb);
      tc_fence_before();
      __syncwarp();
      if (lane0) mbar_arrive(kAcc ? empty1 : empty0);
      reg_fence(va);
      reg_fence(vb);
      // columns: two three-input maxima per column; rows: one chain per row
      float r0 = fmaxf(va[0], va[2]), r1 = fmaxf(va[1], va[3]);
      float r2 = fmaxf(vb[0], vb[2]), r3 = fmaxf(vb[1], vb[3]);
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        pm[j] = fmax3(pm[j], va[2 * j], va[2 * j + 1]);
        pm[j] = fmax3(pm[j], vb[2 * j], vb[2 * j + 1]);
        if (j >= 2 && (j & 1) == 0) {
          r0 = fmax3(r0, va[2 * j], va[2 * j + 2]);
          r1 = fmax3(r1, va[2 * j + 1], va[2 * j + 3]);
          r2 = fmax3(r2, vb[2 * j], vb[2 * j + 2]);
          r3 = fmax3(r3, vb[2 * j + 1], vb[2 * j + 3]);
        }
      }
      // across the 4 lanes holding the same rows: lane s ends with row g + 8s
      const float x0 = swap_max(r0, r1, s0, 1);  // row (s & 1)
      const float x1 = swap_max(r2, r3, s0, 1);  // row 2 + (s & 1)
      const float y = swap_max(x0, x1, s1, 2);   // row s
      if (kFirst)
        row_state_first(rb_s + 2048u * l, rc_s + 512u * l, y);
      else
        row_state_update(rb_s + 2048u * l, rc_s + 512u * l, y, n);
      return true;
    };
    // one n-pass: tile l uses accumulator l % 2
    auto pass = [&](auto first_c, int n) -> bool {
      for (int l = 0; l < bm; l += 2) {
        if (!tile(std::integral_constant<int, 0>{}, first_c, l, n)) return false;
        if (!tile(std::integral_constant<int, 1>{}, first_c, l + 1, n)) return false;
      }
      return true;
    };

    for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
      const int mb = u % p.mblocks, nb = u / p.mblocks;
      const int row_base = mb * 128 * bm;
      for (int n = 0; n < bn && ok; ++n) {
        const int col0 = (nb * bn + n) * kOpBlockN + 64 * part;  // first column of this part
#pragma unroll
        for (int c = 0; c < 16; ++c) pm[c] = ninf;
        ok = n == 0 ? pass(std::true_type{}, 0) : pass(std::false_type{}, n);
        if (!ok) break;
        // ---- column flush: over the 8 lanes of this quadrant holding the same columns
        float x[8], y4[4], z[2];
#pragma unroll
        for (int i = 0; i < 8; ++i) x[i] = swap_max(pm[i], pm[i + 8], g2, 16);
#pragma unroll
        for (int i = 0; i < 4; ++i) y4[i] = swap_max(x[i], x[i + 4], g1, 8);
#pragma unroll
        for (int i = 0; i < 2; ++i) z[i] = swap_max(y4[i], y4[i + 2], g0, 4);
        // z[h]: column 8g + 4h + s of this part, over the quadrant's 32*bm rows:
        // the chunk (m-block, quadrant).  Each warp merges its own maxima into
        // the global keys (no meeting with the other quadrants' warps); a
        // quadrant wholly past the last image-1 row holds NaN and is skipped.
        {
          const int c = col0 + 8 * g + s;
          const int chunk_row = row_base + 32 * bm * q;
          if (c < p.n2 && z[0] == z[0]) atomicMax(p.colk + c, pack_key(z[0], chunk_row));
          if (c + 4 < p.n2 && z[1] == z[1])
            atomicMax(p.colk + c + 4, pack_key(z[1], chunk_row));
        }
      }
      if (!ok) break;
      // ---- row flush: every epilogue warp has written its slots for this unit
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(rowbar));
      if (!mbar_wait(smem_u32(rowbar), static_cast<uint32_t>(rowphase & 1), abort_flag, p.err,
                     kErrWaitEpilogue, lim)) {
        ok = false;
        break;
      }
      ++rowphase;
      for (int r = e * 32 + lane; r < bm * 128; r += kOpEpiWarps * 32) {
        const int l = r >> 7, rl = r & 127;
        unsigned long long best = 0;
#pragma unroll
        for (int pp = 0; pp < 4; ++pp) {
          const float v = lds_f32(smem_u32(rbest) + 4u * (l * 512 + pp * 128 + rl));
          const int nn = static_cast<int>(lds_u8(smem_u32(rchunk) + l * 512 + pp * 128 + rl));
          // a part wholly past the last image-2 row holds NaN
          const unsigned long long k =
              v == v ? pack_key(v, (nb * bn + nn) * kOpBlockN + 64 * pp) : 0ull;
          best = k > best ? k : best;
        }
        const int grow = row_base + 32 * (bm * (rl >> 5) + l) + (rl & 31);
        if (grow < p.n1) atomicMax(p.rowk + grow, best);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(rowbar));
      if (!mbar_wait(smem_u32(rowbar), static_cast<uint32_t>(rowphase & 1), abort_flag, p.err,
                     kErrWaitEpilogue, lim)) {
        ok = false;
        break;
      }
      ++rowphase;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

}  // namespace rnn
