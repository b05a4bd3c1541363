// Block scores Sc[i][j] = <Qbar_i, Kbar_j> * scale of the router (video-generation acceleration
// notes, wzjinhao.cn, §5.2: scaled dot products of block means) on the tensor cores, to fp64
// accuracy.
//
// The pool kernel writes each block mean x (fp64, d values) as a power-of-two scale 2^e with
// max|x| < 2^e and five slices of integers in [-128, 128] (exact in bf16):
//     x = 2^e * (X_0 2^-7 + X_1 2^-15 + X_2 2^-23 + X_3 2^-31 + X_4 2^-39) + (residual < 2^(e-46)).
// The dot product of two blocks is then a sum over slice pairs (a, b) of integer dot products
// weighted 2^(e_i + f_j - 14 - 8(a + b)). Pairs of one level l = a + b share a weight, so their
// sum is accumulated in one fp32 TMEM accumulator; every partial sum is an integer below
// 5 * d * 128^2 < 2^24 and therefore exact. Levels 0-4 (15 MMA groups) are kept; the dropped
// ones are below 2^-30 * 2^(e_i + f_j) (a splitting of the operands into small-integer slices
// whose products the tensor cores compute exactly, in the manner of the Ozaki scheme for
// accurate matrix products).
//
// One CTA per 128 x 32 tile of one head's score matrix, two CTAs per SM (5 levels x 32 columns
// at 32-column offsets of a 256-column TMEM allocation): the five K slices stay in shared memory,
// the Q slices stream in 64-dim chunks through four slots; one thread issues tcgen05.mma
// (kind::f16, bf16 -> fp32); then every thread takes one row, combines its levels in fp64 into
// the staging area (the K slices' space) and the CTA writes the fp64 logits row by row,
// coalesced.
#include <cuda.h>
#include <math.h>

#include "common.cuh"
#include "route.cuh"
#include "tc_ptx.cuh"
#include "tmap.cuh"

namespace fv {

namespace {

constexpr int kRowsQ = 128, kColsK = 32;
constexpr int kQSlots = 4;
constexpr uint32_t kWaitLimit = 1u << 22;

template <int D>
struct ScLayout {
  static constexpr int kChunks = D / 64;
  static constexpr int kQChunk = kRowsQ * 128;                  // [128 rows x 64 dims] bf16 = 16 KB
  static constexpr int kKChunk = kColsK * 128;                  // [32 rows x 64 dims] bf16 = 4 KB
  static constexpr int kKSlice = kChunks * kKChunk;
  static constexpr int kOffK = 0;                               // five K slices, later the staging
  static constexpr int kKBytes = kScoreSlices * kKSlice;
  static constexpr int kStage = kRowsQ * kColsK * 8;            // fp64 tile
  static constexpr int kKRegion = ((kKBytes > kStage ? kKBytes : kStage) + 1023) & ~1023;
  static constexpr int kOffQ = kKRegion;                        // Q chunk slots
  static constexpr int kOffE = kOffQ + kQSlots * kQChunk;       // column exponents
  static constexpr int kOffBar = kOffE + kColsK * 4;
  static constexpr int kBytes = kOffBar + 128;
};

struct ScBars {
  uint64_t k_full, q_full[kQSlots], q_empty[kQSlots], done;
  uint32_t tmem_base;
  int abort;
};

// 2^k for the exponent range of the logits (a normal double), exactly.
__device__ __forceinline__ double pow2(int k) { return __longlong_as_double((long long)(1023 + k) << 52); }

template <int D>
__global__ void __launch_bounds__(128, 2)
    score_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const int32_t* __restrict__ eq, const int32_t* __restrict__ ek, Dims m, double scale, int ld,
                    double* __restrict__ logits, int32_t* __restrict__ status) {
  using L = ScLayout<D>;
  constexpr int NQ = kScoreSlices * L::kChunks;                 // Q chunks streamed: (slice, chunk)
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  ScBars* bars = reinterpret_cast<ScBars*>(smem + L::kOffBar);
  int32_t* sE = reinterpret_cast<int32_t*>(smem + L::kOffE);
  double* stage = reinterpret_cast<double*>(smem + L::kOffK);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int j0 = blockIdx.x * kColsK, i0 = blockIdx.y * kRowsQ;
  const int64_t bh = blockIdx.z;
  volatile int* abort = &bars->abort;

  if (threadIdx.x == 0) {
    tc::mbar_init(&bars->k_full, 1);
    for (int s = 0; s < kQSlots; ++s) {
      tc::mbar_init(&bars->q_full[s], 1);
      tc::mbar_init(&bars->q_empty[s], 1);
    }
    tc::mbar_init(&bars->done, 1);
    bars->abort = 0;
    tc::fence_mbar_init();
  }
  if (warp == 1) {
    tc::tmem_alloc(&bars->tmem_base, 256);
    tc::tmem_relinquish();
  }
  if (threadIdx.x < kColsK) {
    const int j = j0 + threadIdx.x;
    sE[threadIdx.x] = j < m.nb ? ek[bh * m.nb + j] : 0;
  }
  const int r = warp * 32 + lane, i = i0 + r;
  const int ei = i < m.nb ? eq[bh * m.nb + i] : 0;      // this thread's row exponent, read early
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tbase = bars->tmem_base;

  if (warp == 0 && lane == 0) {
    // ---- loads: the five K slices once; Q (slice a, 64-dim chunk c) through the slots
    tc::mbar_expect_tx(&bars->k_full, L::kKBytes);
    for (int b = 0; b < kScoreSlices; ++b)
      for (int c = 0; c < L::kChunks; ++c)
        tc::tma_load_3d(smem + L::kOffK + b * L::kKSlice + c * L::kKChunk, &tmK, &bars->k_full, c * 64, j0,
                        (int)(bh * kScoreSlices + b));
    for (int n = 0; n < NQ; ++n) {
      const int s = n % kQSlots, a = n / L::kChunks, c = n % L::kChunks;
      if (n >= kQSlots && !tc::mbar_wait(&bars->q_empty[s], (n / kQSlots - 1) & 1, abort, kWaitLimit)) {
        atomicCAS(&bars->abort, 0, 1);
        break;
      }
      tc::mbar_expect_tx(&bars->q_full[s], L::kQChunk);
      for (int h = 0; h < 2; ++h)
        tc::tma_load_3d(smem + L::kOffQ + s * L::kQChunk + h * 64 * 128, &tmQ, &bars->q_full[s], c * 64,
                        i0 + h * 64, (int)(bh * kScoreSlices + a));
    }
  } else if (warp == 1 && lane == 0) {
    // ---- MMAs: level a+b += Q_a K_b^T for a + b < 5, chunk by chunk of the head dimension; the
    // first MMA into each level (a = 0, first chunk, first K16 step) overwrites it. The closing
    // commit runs on every path, so the teardown can wait for whatever was issued.
    constexpr uint32_t idesc = tc::idesc_bf16_f32(kRowsQ, kColsK, 0, 0);
    const uint32_t kaddr = tc::smem_u32(smem + L::kOffK), qaddr = tc::smem_u32(smem + L::kOffQ);
    bool ok = tc::mbar_wait(&bars->k_full, 0, abort, kWaitLimit);
    for (int n = 0; ok && n < NQ; ++n) {
      const int s = n % kQSlots, a = n / L::kChunks, c = n % L::kChunks;
      if (!tc::mbar_wait(&bars->q_full[s], (n / kQSlots) & 1, abort, kWaitLimit)) {
        ok = false;
        break;
      }
      tc::fence_after_sync();
      for (int b = 0; a + b < kScoreSlices; ++b) {
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t ad = tc::smem_desc_sw128(qaddr + s * L::kQChunk + kk * 32, 16, 1024);
          const uint64_t bd = tc::smem_desc_sw128(kaddr + b * L::kKSlice + c * L::kKChunk + kk * 32, 16, 1024);
          tc::mma_f16(tbase + (a + b) * kColsK, ad, bd, idesc, (a > 0 || c > 0 || kk > 0) ? 1u : 0u);
        }
      }
      tc::mma_commit(&bars->q_empty[s]);
    }
    if (!ok) atomicCAS(&bars->abort, 0, 2);
    tc::mma_commit(&bars->done);
  }
  __syncwarp();

  // ---- epilogue: one row per thread (TMEM lane) into the staging tile, then coalesced rows
  const bool done = __all_sync(0xffffffffu, tc::mbar_wait(&bars->done, 0, abort, kWaitLimit));
  tc::fence_after_sync();
  const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
  if (done && !*abort) {
#pragma unroll 1
    for (int cc = 0; cc < kColsK / 16; ++cc) {
      uint32_t acc[kScoreSlices][16];
#pragma unroll
      for (int l = 0; l < kScoreSlices; ++l) tc::tmem_ld16(tbase + lane_off + l * kColsK + cc * 16, acc[l]);
      tc::tmem_ld_wait();
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const int jj = cc * 16 + e;
        // levels combined from the finest: v = A_0 + 2^-8 (A_1 + 2^-8 (A_2 + ...))
        double v = (double)__uint_as_float(acc[kScoreSlices - 1][e]);
#pragma unroll
        for (int l = kScoreSlices - 2; l >= 0; --l) v = fma(v, 0x1p-8, (double)__uint_as_float(acc[l][e]));
        const int k = ei + sE[jj] - 14;
        stage[r * kColsK + ((jj + r) % kColsK)] = (v * scale) * pow2(max(-1000, min(1000, k)));
      }
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  if (done && !*abort) {
    const int ncol = min(kColsK, m.nb - j0);
    for (int x = threadIdx.x; x < kRowsQ * kColsK; x += blockDim.x) {
      const int rr = x / kColsK, jj = x - rr * kColsK;
      if (i0 + rr < m.nb && jj < ncol)
        logits[(bh * m.nb + i0 + rr) * (int64_t)ld + j0 + jj] = stage[rr * kColsK + ((jj + rr) % kColsK)];
    }
  }
  if (warp == 1) tc::tmem_dealloc(tbase, 256);
  if (threadIdx.x == 0 && bars->abort) report_error(status, FVATTN_ERR_TIMEOUT, 30 + bars->abort);
}

template <int D>
cudaError_t launch_score_tc_d(const __nv_bfloat16* qs, const __nv_bfloat16* ks, const int32_t* eq,
                              const int32_t* ek, const Dims& m, double scale, double* logits, int32_t* status,
                              cudaStream_t st) {
  if (m.BH > 65535) return cudaErrorInvalidValue;
  CUtensorMap mq, mk;
  const uint64_t planes = (uint64_t)m.BH * kScoreSlices;
  if (!make_map_bf16_3d(&mq, qs, (uint64_t)D, (uint64_t)m.nb, planes, 64) ||
      !make_map_bf16_3d(&mk, ks, (uint64_t)D, (uint64_t)m.nb, planes, kColsK))
    return cudaErrorInvalidValue;
  const size_t smem = ScLayout<D>::kBytes + 1024;
  cudaError_t e = cudaFuncSetAttribute(score_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((m.nb + kColsK - 1) / kColsK, (m.nb + kRowsQ - 1) / kRowsQ, (unsigned)m.BH);
  score_tc_kernel<D><<<grid, 128, smem, st>>>(mq, mk, eq, ek, m, scale, means_ld(m.nb), logits, status);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_score_tc(const __nv_bfloat16* qs, const __nv_bfloat16* ks, const int32_t* eq, const int32_t* ek,
                            const Dims& m, double scale, double* logits, int32_t* status, cudaStream_t st) {
  if (m.d == 128) return launch_score_tc_d<128>(qs, ks, eq, ek, m, scale, logits, status, st);
  return launch_score_tc_d<64>(qs, ks, eq, ek, m, scale, logits, status, st);
}

}  // namespace fv
