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
// Work: the 128 x 64 output tiles of all heads in (head, row tile, column tile) order, split into
// one contiguous range per CTA (one persistent CTA per SM), so a CTA loads the five Q slices of a
// row tile once (80 KB, resident in shared memory; rows of 128 bytes, one 128-byte swizzle
// span) and only reloads them when its range enters the next row tile. The five K slices of a
// column tile stream through a ring of three tiles (one barrier per tile); one thread issues
// tcgen05.mma (kind::i8, M = 128, N = 64, K = 32 per instruction) into one accumulator set of
// 5 levels x 64 columns; sixteen epilogue warps (four per TMEM lane quarter, 16 columns each)
// load the set, release it to the next tile's MMAs, combine the levels in fp64 and write each
// thread's 16 consecutive logits of its row (128 bytes) straight to global memory. An MMA of
// N = 64 costs the issuing thread about what one of N = 32 does, so the wider tile halves the
// instructions per logit; two sets of 5 x 64 columns would not fit the 512 TMEM columns, so the
// set is single and the next tile's MMAs wait only for the epilogue's TMEM loads (59.8 against
// 67.8 us per launch at dit for two sets of N = 32).
#include <cuda.h>
#include <math.h>

#include "common.cuh"
#include "route.cuh"
#include "tc_ptx.cuh"
#include "tmap.cuh"

namespace fv {

namespace {

constexpr int kRowsQ = 128, kColsK = 64;
constexpr int kKTiles = 3;                              // K ring: three column tiles of five slices
constexpr int kEpiWarps = 16;
constexpr int kEpiCols = kColsK / (kEpiWarps / 4);      // columns of a tile per epilogue thread
constexpr int kThreads = (kEpiWarps + 2) * 32;          // + producer warp + MMA warp
constexpr int kLevelCols = kScoreSlices * kColsK;       // one accumulator set: 320 TMEM columns
constexpr int kSets = 2 * kLevelCols <= 512 ? 2 : 1;     // accumulator sets that fit in TMEM
constexpr uint32_t kWaitLimit = 1u << 22;

template <int D>
struct ScLayout {
  static constexpr int kSteps = D / 32;                         // K = 32 bytes per MMA
  static constexpr int kQSlice = kRowsQ * kSliceRow;            // [128 rows x 128 bytes] = 16 KB
  static constexpr int kKSlot = kColsK * kSliceRow;             // one K slice of one column tile: 4 KB
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kScoreSlices * kQSlice;
  static constexpr int kKTile = kScoreSlices * kKSlot;         // the five K slices of one column tile
  static constexpr int kOffBar = kOffK + kKTiles * kKTile;
  static constexpr int kBytes = kOffBar + 256;
};

struct ScBars {
  uint64_t q_full, q_empty;
  uint64_t k_full[kKTiles], k_empty[kKTiles];
  uint64_t acc_full[2], acc_empty[2];
  uint64_t drain;
  uint64_t hold;            // completed by nothing: the failure-path check waits on it
  uint32_t tmem_base;
  int abort;
};

// 2^k for the exponent range of the logits (a normal double), exactly.
__device__ __forceinline__ double pow2(int k) { return __longlong_as_double((long long)(1023 + k) << 52); }

// An int32 as a double, exactly, on the fp64 pipe: the bits 0x43300000:(x + 2^31) are the double
// 2^52 + x + 2^31, from which the constant 2^52 + 2^31 is subtracted without rounding.
__device__ __forceinline__ double i32_to_f64(uint32_t x) {
  return __hiloint2double(0x43300000, (int)(x ^ 0x80000000u)) - 4503601774854144.0;
}

// Walks the tiles of a CTA's range in (head, row tile, column tile) order without divisions.
struct TileCursor {
  int64_t bh;
  int rt, ct, nrt, nct;
  __device__ TileCursor(int64_t t, int nrt_, int nct_) : nrt(nrt_), nct(nct_) {
    const int64_t rtile = t / nct;
    ct = (int)(t - rtile * nct);
    bh = rtile / nrt;
    rt = (int)(rtile - bh * nrt);
  }
  __device__ void next() {
    if (++ct == nct) {
      ct = 0;
      if (++rt == nrt) {
        rt = 0;
        ++bh;
      }
    }
  }
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    score_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const int32_t* __restrict__ eq, const int32_t* __restrict__ ek, Dims m, double scale, int ld,
                    double* __restrict__ logits, int32_t* __restrict__ status, uint32_t hold_polls) {
  using L = ScLayout<D>;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  ScBars* bars = reinterpret_cast<ScBars*>(smem + L::kOffBar);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* abort = &bars->abort;

  // this CTA's contiguous range of tiles in (head, row tile, column tile) order
  const int nrt = (m.nb + kRowsQ - 1) / kRowsQ, nct = (m.nb + kColsK - 1) / kColsK;
  const int64_t T = m.BH * nrt * nct;
  const int64_t t_begin = T * blockIdx.x / gridDim.x, t_end = T * (blockIdx.x + 1) / gridDim.x;

  if (threadIdx.x == 0) {
    tc::mbar_init(&bars->q_full, 1);
    tc::mbar_init(&bars->q_empty, 1);
    for (int s = 0; s < kKTiles; ++s) {
      tc::mbar_init(&bars->k_full[s], 1);
      tc::mbar_init(&bars->k_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(&bars->acc_full[s], 1);
      tc::mbar_init(&bars->acc_empty[s], kEpiWarps);
    }
    tc::mbar_init(&bars->drain, 1);
    tc::mbar_init(&bars->hold, 1);
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
      uint32_t qc = 0, kph = 0;
      int s = 0;
      // parities of the last phases this thread armed (-1: none), waited for before it leaves,
      // so that no copy is still writing shared memory when the CTA exits
      int q_par = -1, k_par[kKTiles];
      for (int x = 0; x < kKTiles; ++x) k_par[x] = -1;
      // failure-path check: a bounded wait on a barrier nothing completes, before any copy
      if (hold_polls > 0 && !tc::mbar_wait(&bars->hold, 0, abort, hold_polls)) atomicCAS(&bars->abort, 0, 4);
      TileCursor tcur(t_begin, nrt, nct);
      for (int64_t t = t_begin; t < t_end && !*abort; ++t, tcur.next()) {
        const int64_t bh = tcur.bh;
        const int i0 = tcur.rt * kRowsQ, j0 = tcur.ct * kColsK;
        if (t == t_begin || tcur.ct == 0) {
          // the previous row tile's MMAs are done with the Q slices before they are replaced
          if (qc > 0 && !tc::mbar_wait(&bars->q_empty, (qc - 1) & 1, abort, kWaitLimit)) {
            atomicCAS(&bars->abort, 0, 1);
            break;
          }
          tc::mbar_expect_tx(&bars->q_full, kScoreSlices * L::kQSlice);
          q_par = (int)(qc & 1);
          for (int a = 0; a < kScoreSlices; ++a)
            tc::tma_load_3d(smem + L::kOffQ + a * L::kQSlice, &tmQ, &bars->q_full, 0, i0, (int)(bh * kScoreSlices + a));
          ++qc;
        }
        // the five K slices of the column tile under one barrier
        if (!tc::mbar_wait(&bars->k_empty[s], kph ^ 1, abort, kWaitLimit)) {
          atomicCAS(&bars->abort, 0, 2);
          break;
        }
        tc::mbar_expect_tx(&bars->k_full[s], L::kKTile);
        k_par[s] = (int)kph;
        for (int b = 0; b < kScoreSlices; ++b)
          tc::tma_load_3d(smem + L::kOffK + s * L::kKTile + b * L::kKSlot, &tmK, &bars->k_full[s], 0, j0,
                          (int)(bh * kScoreSlices + b));
        if (++s == kKTiles) {
          s = 0;
          kph ^= 1;
        }
      }
      if (q_par >= 0) tc::mbar_wait_drain(&bars->q_full, (uint32_t)q_par, kWaitLimit);
      for (int x = 0; x < kKTiles; ++x)
        if (k_par[x] >= 0) tc::mbar_wait_drain(&bars->k_full[x], (uint32_t)k_par[x], kWaitLimit);
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
      uint32_t qc = 0, kph = 0;
      int s = 0;
      bool ok = true;
      TileCursor tcur(t_begin, nrt, nct);
      for (int64_t t = t_begin; ok && t < t_end; ++t, tcur.next()) {
        const uint32_t j = (uint32_t)(t - t_begin), buf = j % kSets, use = j / kSets;
        if (t == t_begin || tcur.ct == 0) {
          if (!tc::mbar_wait(&bars->q_full, qc & 1, abort, kWaitLimit)) { ok = false; break; }
          ++qc;
        }
        // Two waits per tile: every mbarrier wait of this thread stalls the MMA stream for a
        // few hundred cycles even when the phase is already complete.
        if (!tc::mbar_wait(&bars->acc_empty[buf], (use & 1) ^ 1, abort, kWaitLimit) ||
            !tc::mbar_wait(&bars->k_full[s], kph, abort, kWaitLimit)) {
          ok = false;
          break;
        }
        tc::fence_after_sync();
        const uint32_t dbase = tbase + buf * kLevelCols;
        const uint64_t kd0 = kdesc0 + (uint64_t)((s * L::kKTile) >> 4);
#pragma unroll
        for (int b = 0; b < kScoreSlices; ++b) {
#pragma unroll
          for (int a = 0; a < kScoreSlices; ++a) {
            if (a + b >= kScoreSlices) continue;
#pragma unroll
            for (int kk = 0; kk < L::kSteps; ++kk)
              tc::mma_i8(dbase + (a + b) * kColsK, qdesc0 + ((a * L::kQSlice + kk * 32) >> 4),
                         kd0 + ((b * L::kKSlot + kk * 32) >> 4), idesc, (b > 0 || kk > 0) ? 1u : 0u);
          }
        }
        tc::mma_commit(&bars->k_empty[s]);
        if (++s == kKTiles) {
          s = 0;
          kph ^= 1;
        }
        tc::mma_commit(&bars->acc_full[buf]);
        if (t + 1 == t_end || tcur.ct + 1 == nct) tc::mma_commit(&bars->q_empty);
      }
      if (!ok) atomicCAS(&bars->abort, 0, 3);
      tc::mma_commit(&bars->drain);
      tc::mbar_wait_drain(&bars->drain, 0, kWaitLimit);
    }
  } else {
    // ------------------------------------------------------------------ epilogue (warps 0-15)
    // A warp leaves on its own when a wait runs out or another role aborted: no barrier joins
    // the epilogue warps inside the loop. The column exponents of the next tile are loaded one
    // tile ahead.
    const int quarter = warp & 3, part = warp >> 2;
    const int r = quarter * 32 + lane;                           // tile row == TMEM lane
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    auto col_exp = [&](const TileCursor& c) -> int {             // exponent of column lane & 7
      const int jl = c.ct * kColsK + part * kEpiCols + (lane & (kEpiCols - 1));
      return jl < m.nb ? ek[c.bh * m.nb + jl] : 0;
    };
    int ei = 0;
    TileCursor tcur(t_begin, nrt, nct), tnext = tcur;
    int ej_next = t_begin < t_end ? col_exp(tcur) : 0;
    for (int64_t t = t_begin; t < t_end; ++t, tcur.next()) {
      const uint32_t j = (uint32_t)(t - t_begin), buf = j % kSets, use = j / kSets;
      const int64_t bh = tcur.bh;
      const int i0 = tcur.rt * kRowsQ, j0 = tcur.ct * kColsK;
      if (t == t_begin || tcur.ct == 0) ei = i0 + r < m.nb ? eq[bh * m.nb + i0 + r] : 0;
      const int ej_l = ej_next;
      tnext.next();
      if (t + 1 < t_end) ej_next = col_exp(tnext);
      const bool ready = tc::mbar_wait(&bars->acc_full[buf], use & 1, abort, kWaitLimit);
      if (!ready || *abort) break;
      tc::fence_after_sync();
      uint32_t acc[kScoreSlices][kEpiCols];
#pragma unroll
      for (int l = 0; l < kScoreSlices; ++l)
#pragma unroll
        for (int c8 = 0; c8 < kEpiCols; c8 += 8)
          tc::tmem_ld8(tbase + lane_off + buf * kLevelCols + l * kColsK + part * kEpiCols + c8,
                       *reinterpret_cast<uint32_t(*)[8]>(&acc[l][c8]));
      tc::tmem_ld_wait();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&bars->acc_empty[buf]);     // the set can take the next tile
      double out[kEpiCols];
#pragma unroll
      for (int e = 0; e < kEpiCols; ++e) {
        // levels combined from the finest: v = A_0 + 2^-8 (A_1 + 2^-8 (A_2 + ...))
        double v = i32_to_f64(acc[kScoreSlices - 1][e]);
#pragma unroll
        for (int l = kScoreSlices - 2; l >= 0; --l) v = fma(v, 0x1p-8, i32_to_f64(acc[l][e]));
        const int k = ei + __shfl_sync(0xffffffffu, ej_l, e) - 14;
        out[e] = (v * scale) * pow2(max(-1000, min(1000, k)));
      }
      // the thread's 8 consecutive logits of row i0 + r (64 bytes, 64-byte aligned)
      if (i0 + r < m.nb) {
        const int c0 = j0 + part * kEpiCols;
        double* dst = logits + (bh * m.nb + i0 + r) * (int64_t)ld + c0;
        if (c0 + kEpiCols <= m.nb) {
#pragma unroll
          for (int e = 0; e < kEpiCols; e += 2) *reinterpret_cast<double2*>(dst + e) = make_double2(out[e], out[e + 1]);
        } else {
#pragma unroll
          for (int e = 0; e < kEpiCols; ++e)
            if (c0 + e < m.nb) dst[e] = out[e];
        }
      }
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
                              double scale, double* logits, int32_t* status, int nsm, cudaStream_t st,
                              uint32_t hold_polls) {
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
  score_tc_kernel<D><<<grid, kThreads, smem, st>>>(mq, mk, eq, ek, m, scale, means_ld(m.nb), logits, status,
                                                   hold_polls);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_score_tc(const int8_t* qs, const int8_t* ks, const int32_t* eq, const int32_t* ek, const Dims& m,
                            double scale, double* logits, int32_t* status, int nsm, cudaStream_t st,
                            uint32_t hold_polls) {
  if (m.d == 128) return launch_score_tc_d<128>(qs, ks, eq, ek, m, scale, logits, status, nsm, st, hold_polls);
  return launch_score_tc_d<64>(qs, ks, eq, ek, m, scale, logits, status, nsm, st, hold_polls);
}

}  // namespace fv
