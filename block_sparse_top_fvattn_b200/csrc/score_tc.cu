// Block scores Sc[i][j] = <Qbar_i, Kbar_j> * scale of the router (video-generation acceleration
// notes, wzjinhao.cn, §5.2: scaled dot products of block means) on the tensor cores, to fp64
// accuracy.
//
// The pool kernel writes each block mean x (fp64, d values) as a power-of-two scale 2^e with
// max|x| < 2^e and five slices of signed 8-bit integers:
//     x = 2^e * (X_0 2^-7 + X_1 2^-15 + X_2 2^-23 + X_3 2^-31 + X_4 2^-39) + (residual <= 2^(e-40)).
// The dot product of two blocks is then a sum over slice pairs (a, b) of integer dot products
// weighted 2^(e_i + f_j - 14 - 8(a + b)). Pairs of one level l = a + b share a weight, so their
// sum is accumulated in one int32 TMEM accumulator (tcgen05.mma kind::i8, exact; every partial
// sum is below 5 * d * 128^2 < 2^24). Levels 0-4 (15 MMA groups) are kept; the dropped ones are
// below 2^-30 * 2^(e_i + f_j) (a splitting of the operands into small-integer slices whose
// products the tensor cores compute exactly, in the manner of the Ozaki scheme for accurate
// matrix products).
//
// Work: the 128 x 32 output tiles of all heads in (head, row tile, column tile) order, split into
// one contiguous range per CTA (one persistent CTA per SM), so a CTA loads the five Q slices of a
// row tile once (80 KB, resident in shared memory; rows of 128 bytes, one 128-byte swizzle
// span) and only reloads them when its range enters the next row tile. Per column tile the five
// K slices stream through a ring of two tiles' slots; one thread issues tcgen05.mma (kind::i8,
// K = 32 per instruction) into one of two accumulator sets (5 levels x 32 columns at 32-column
// TMEM offsets); eight epilogue warps drain the other set meanwhile
// (two per TMEM lane quarter, 16 columns each), combine the levels in fp64, stage the tile in
// shared memory and write the fp64 logit rows coalesced.
#include <cuda.h>
#include <math.h>

#include "common.cuh"
#include "route.cuh"
#include "tc_ptx.cuh"
#include "tmap.cuh"

namespace fv {

namespace {

constexpr int kRowsQ = 128, kColsK = 32;
constexpr int kKSlots = 2 * kScoreSlices;
constexpr int kEpiWarps = 8;
constexpr int kThreads = (kEpiWarps + 2) * 32;          // + producer warp + MMA warp
constexpr int kLevelCols = kScoreSlices * kColsK;       // one accumulator set: 160 TMEM columns
constexpr uint32_t kWaitLimit = 1u << 22;

template <int D>
struct ScLayout {
  static constexpr int kSteps = D / 32;                         // K = 32 bytes per MMA
  static constexpr int kQSlice = kRowsQ * kSliceRow;            // [128 rows x 128 bytes] = 16 KB
  static constexpr int kKSlot = kColsK * kSliceRow;             // one K slice of one column tile: 4 KB
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kScoreSlices * kQSlice;
  static constexpr int kOffStage = kOffK + kKSlots * kKSlot;
  static constexpr int kOffBar = kOffStage + kRowsQ * kColsK * 8;
  static constexpr int kBytes = kOffBar + 256;
};

struct ScBars {
  uint64_t q_full, q_empty;
  uint64_t k_full[kKSlots], k_empty[kKSlots];
  uint64_t acc_full[2], acc_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

// 2^k for the exponent range of the logits (a normal double), exactly.
__device__ __forceinline__ double pow2(int k) { return __longlong_as_double((long long)(1023 + k) << 52); }

__device__ __forceinline__ void epi_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kEpiWarps * 32) : "memory"); }

// A barrier of the epilogue warps that also returns whether every one of their threads passed
// true, so that they take the same branch (leaving the tile loop) together.
__device__ __forceinline__ bool epi_all(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, 1, %2, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v), "n"(kEpiWarps * 32)
      : "memory");
  return r != 0;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    score_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const int32_t* __restrict__ eq, const int32_t* __restrict__ ek, Dims m, double scale, int ld,
                    double* __restrict__ logits, int32_t* __restrict__ status) {
  using L = ScLayout<D>;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  ScBars* bars = reinterpret_cast<ScBars*>(smem + L::kOffBar);
  double* stage = reinterpret_cast<double*>(smem + L::kOffStage);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* abort = &bars->abort;

  // this CTA's contiguous range of tiles in (head, row tile, column tile) order
  const int nrt = (m.nb + kRowsQ - 1) / kRowsQ, nct = (m.nb + kColsK - 1) / kColsK;
  const int64_t T = m.BH * nrt * nct;
  const int64_t t_begin = T * blockIdx.x / gridDim.x, t_end = T * (blockIdx.x + 1) / gridDim.x;
  auto row_tile = [&](int64_t t) { return t / nct; };           // bh * nrt + rt

  if (threadIdx.x == 0) {
    tc::mbar_init(&bars->q_full, 1);
    tc::mbar_init(&bars->q_empty, 1);
    for (int s = 0; s < kKSlots; ++s) {
      tc::mbar_init(&bars->k_full[s], 1);
      tc::mbar_init(&bars->k_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(&bars->acc_full[s], 1);
      tc::mbar_init(&bars->acc_empty[s], kEpiWarps);
    }
    tc::mbar_init(&bars->drain, 1);
    bars->abort = 0;
    tc::fence_mbar_init();
  }
  if (warp == kEpiWarps + 1) {
    tc::tmem_alloc(&bars->tmem_base, 512);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tbase = bars->tmem_base;

  if (warp == kEpiWarps) {
    if (lane == 0) {
      // ---------------------------------------------------------------- loads
      uint32_t kc = 0, qc = 0;
      int64_t cur = -1;
      for (int64_t t = t_begin; t < t_end; ++t) {
        const int64_t rtile = row_tile(t);
        const int64_t bh = rtile / nrt;
        const int i0 = (int)(rtile - bh * nrt) * kRowsQ, j0 = (int)(t - rtile * nct) * kColsK;
        if (rtile != cur) {
          // the previous row tile's MMAs are done with the Q slices before they are replaced
          if (qc > 0 && !tc::mbar_wait(&bars->q_empty, (qc - 1) & 1, abort, kWaitLimit)) {
            atomicCAS(&bars->abort, 0, 1);
            break;
          }
          tc::mbar_expect_tx(&bars->q_full, kScoreSlices * L::kQSlice);
          for (int a = 0; a < kScoreSlices; ++a)
            tc::tma_load_3d(smem + L::kOffQ + a * L::kQSlice, &tmQ, &bars->q_full, 0, i0, (int)(bh * kScoreSlices + a));
          cur = rtile;
          ++qc;
        }
        bool ok = true;
        for (int b = 0; b < kScoreSlices; ++b, ++kc) {
          const int s = kc % kKSlots;
          if (!tc::mbar_wait(&bars->k_empty[s], ((kc / kKSlots) & 1) ^ 1, abort, kWaitLimit)) {
            ok = false;
            break;
          }
          tc::mbar_expect_tx(&bars->k_full[s], L::kKSlot);
          tc::tma_load_3d(smem + L::kOffK + s * L::kKSlot, &tmK, &bars->k_full[s], 0, j0, (int)(bh * kScoreSlices + b));
        }
        if (!ok) {
          atomicCAS(&bars->abort, 0, 2);
          break;
        }
      }
    }
  } else if (warp == kEpiWarps + 1) {
    if (lane == 0) {
      // ---------------------------------------------------------------- MMAs
      // Column tile j (local index) goes to accumulator set j % 2: level a+b += Q_a K_b^T for
      // a + b < 5. With b outermost, b = 0 touches every level first (a = level), so those MMAs
      // (first K32 step) overwrite. The closing commit runs on every path, and the thread waits
      // for it, so no MMA is in flight when TMEM is released.
      constexpr uint32_t idesc = tc::idesc_s8_s32(kRowsQ, kColsK);
      // Shared-memory descriptors are linear in the start address (bits 0-13 hold address >> 4,
      // and every operand lies below 256 KB), so they are made once and offset by constants.
      const uint64_t qdesc0 = tc::smem_desc_sw128(tc::smem_u32(smem + L::kOffQ), 16, 1024);
      const uint64_t kdesc0 = tc::smem_desc_sw128(tc::smem_u32(smem + L::kOffK), 16, 1024);
      uint32_t kc = 0, qc = 0;
      int64_t cur = -1;
      bool ok = true;
      for (int64_t t = t_begin; ok && t < t_end; ++t) {
        const uint32_t j = (uint32_t)(t - t_begin), buf = j & 1;
        const int64_t rtile = row_tile(t);
        if (rtile != cur) {
          if (!tc::mbar_wait(&bars->q_full, qc & 1, abort, kWaitLimit)) { ok = false; break; }
          cur = rtile;
          ++qc;
        }
        if (!tc::mbar_wait(&bars->acc_empty[buf], ((j >> 1) & 1) ^ 1, abort, kWaitLimit)) { ok = false; break; }
        tc::fence_after_sync();
        const uint32_t dbase = tbase + buf * kLevelCols;
#pragma unroll
        for (int b = 0; b < kScoreSlices; ++b, ++kc) {
          const int s = kc % kKSlots;
          if (!tc::mbar_wait(&bars->k_full[s], (kc / kKSlots) & 1, abort, kWaitLimit)) { ok = false; break; }
          tc::fence_after_sync();
          const uint64_t kd = kdesc0 + (uint64_t)((s * L::kKSlot) >> 4);
#pragma unroll
          for (int a = 0; a < kScoreSlices; ++a) {
            if (a + b >= kScoreSlices) continue;
#pragma unroll
            for (int kk = 0; kk < L::kSteps; ++kk)
              tc::mma_i8(dbase + (a + b) * kColsK, qdesc0 + ((a * L::kQSlice + kk * 32) >> 4), kd + ((kk * 32) >> 4),
                         idesc, (b > 0 || kk > 0) ? 1u : 0u);
          }
          tc::mma_commit(&bars->k_empty[s]);
        }
        if (!ok) break;
        tc::mma_commit(&bars->acc_full[buf]);
        if (t + 1 == t_end || row_tile(t + 1) != rtile) tc::mma_commit(&bars->q_empty);
      }
      if (!ok) atomicCAS(&bars->abort, 0, 3);
      tc::mma_commit(&bars->drain);
      tc::mbar_wait(&bars->drain, 0, abort, kWaitLimit);
    }
  } else {
    // ------------------------------------------------------------------ epilogue (warps 0-7)
    const int quarter = warp & 3, half = warp >> 2;
    const int r = quarter * 32 + lane;                           // tile row == TMEM lane
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    int64_t cur = -1;
    int ei = 0;
    for (int64_t t = t_begin; t < t_end; ++t) {
      const uint32_t j = (uint32_t)(t - t_begin), buf = j & 1;
      const int64_t rtile = row_tile(t);
      const int64_t bh = rtile / nrt;
      const int i0 = (int)(rtile - bh * nrt) * kRowsQ, j0 = (int)(t - rtile * nct) * kColsK;
      if (rtile != cur) {
        ei = i0 + r < m.nb ? eq[bh * m.nb + i0 + r] : 0;
        cur = rtile;
      }
      // the 16 column exponents of this warp's half, one per lane 0-15
      const int jl = j0 + half * 16 + (lane & 15);
      const int ej_l = jl < m.nb ? ek[bh * m.nb + jl] : 0;
      const bool ready = tc::mbar_wait(&bars->acc_full[buf], (j >> 1) & 1, abort, kWaitLimit);
      if (!epi_all(ready && !*abort)) break;                      // every epilogue warp leaves together
      tc::fence_after_sync();
      uint32_t acc[kScoreSlices][16];
#pragma unroll
      for (int l = 0; l < kScoreSlices; ++l)
        tc::tmem_ld16(tbase + lane_off + buf * kLevelCols + l * kColsK + half * 16, acc[l]);
      tc::tmem_ld_wait();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&bars->acc_empty[buf]);     // the set can take the next tile
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        // levels combined from the finest: v = A_0 + 2^-8 (A_1 + 2^-8 (A_2 + ...))
        double v = (double)(int32_t)acc[kScoreSlices - 1][e];
#pragma unroll
        for (int l = kScoreSlices - 2; l >= 0; --l) v = fma(v, 0x1p-8, (double)(int32_t)acc[l][e]);
        const int k = ei + __shfl_sync(0xffffffffu, ej_l, e) - 14;
        const int col = half * 16 + e;
        stage[r * kColsK + ((col + r) & (kColsK - 1))] = (v * scale) * pow2(max(-1000, min(1000, k)));
      }
      epi_sync();
      // coalesced rows: 128 rows x 32 doubles, 256 threads, two consecutive doubles each
      const int ncol = min(kColsK, m.nb - j0);
      for (int x = threadIdx.x; x < kRowsQ * kColsK / 2; x += kEpiWarps * 32) {
        const int rr = x / (kColsK / 2), cc = 2 * (x - rr * (kColsK / 2));
        if (i0 + rr < m.nb) {
          double* dst = logits + (bh * m.nb + i0 + rr) * (int64_t)ld + j0 + cc;
          const double v0 = stage[rr * kColsK + ((cc + rr) & (kColsK - 1))];
          const double v1 = stage[rr * kColsK + ((cc + 1 + rr) & (kColsK - 1))];
          if (cc + 1 < ncol) *reinterpret_cast<double2*>(dst) = make_double2(v0, v1);
          else if (cc < ncol) dst[0] = v0;
        }
      }
      epi_sync();
    }
  }

  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  if (warp == kEpiWarps + 1) tc::tmem_dealloc(tbase, 512);
  if (threadIdx.x == 0 && bars->abort) report_error(status, FVATTN_ERR_TIMEOUT, 30 + bars->abort);
}

template <int D>
cudaError_t launch_score_tc_d(const int8_t* qs, const int8_t* ks, const int32_t* eq, const int32_t* ek, const Dims& m,
                              double scale, double* logits, int32_t* status, int nsm, cudaStream_t st) {
  CUtensorMap mq, mk;
  const uint64_t planes = (uint64_t)m.BH * kScoreSlices;
  if (!make_map_i8_3d(&mq, qs, (uint64_t)kSliceRow, (uint64_t)m.nb, planes, kRowsQ) ||
      !make_map_i8_3d(&mk, ks, (uint64_t)kSliceRow, (uint64_t)m.nb, planes, kColsK))
    return cudaErrorInvalidValue;
  const size_t smem = ScLayout<D>::kBytes + 1024;
  cudaError_t e = cudaFuncSetAttribute(score_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int64_t tiles = m.BH * ((m.nb + kRowsQ - 1) / kRowsQ) * ((m.nb + kColsK - 1) / kColsK);
  const int grid = (int)imin<int64_t>(tiles, nsm);
  score_tc_kernel<D><<<grid, kThreads, smem, st>>>(mq, mk, eq, ek, m, scale, means_ld(m.nb), logits, status);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_score_tc(const int8_t* qs, const int8_t* ks, const int32_t* eq, const int32_t* ek, const Dims& m,
                            double scale, double* logits, int32_t* status, int nsm, cudaStream_t st) {
  if (m.d == 128) return launch_score_tc_d<128>(qs, ks, eq, ek, m, scale, logits, status, nsm, st);
  return launch_score_tc_d<64>(qs, ks, eq, ek, m, scale, logits, status, nsm, st);
}

}  // namespace fv
