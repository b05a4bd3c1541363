// Router kernels: block pooling (and the block means' integer slices for the tensor-core score
// GEMM of score_tc.cu), row softmax, Top-p / top-k cut, slack-aware tile augmentation,
// frame-level top-k, forced blocks, CSR rows, per-head loads, tile costs, the longest-first
// order and the token-exact frame codes.
//
// Method: FVAttn blog summary ("腾讯+中山大学新作：视频生成提速2.11×，靠的是RLB和SASA"), section
// "AI视频生成的阿喀琉斯之踵" (Top-p: smallest descending-importance prefix reaching p) and
// section "RLB…" (per-head load = selected block count, heaviest first); video-generation
// acceleration notes (wzjinhao.cn) §5.2 (block means, score = mean(Q)·mean(K)/sqrt(d), local
// band); vLLM-Omni Sol-Attn article §2.1/§2.2 (frame top-k, neighbour and first frames).
#include <math.h>

#include "common.cuh"
#include "route.cuh"
#include "route_dev.cuh"

namespace fv {

// ------------------------------------------------------------------ K1: block pooling
//
// One warp streams one 64-token block of one tensor. Lane l reads the 16-byte vector
// c = l mod CPR of rows r0 + RPI*it (r0 = l / CPR); a batch of 16 loads is issued before any
// is used, so every lane keeps 256 bytes in flight and no barrier is needed. Four rows are
// summed in AccT (fp32 for bf16 input: exact unless the values' exponents are 16+ apart;
// fp64 for fp32 input), the partial sums in fp64 in a fixed order, and the row groups of a
// column are folded with shuffles. The next block's first batch is loaded before the current
// block's epilogue. OUT selects what is written: means [row][d]; the means as signed 8-bit integer
// slices with power-of-two exponents (the operands of the score GEMM); or fp64 sums of the
// tokens before / after the block's first frame boundary, [row][d].

enum PoolOut { kMeans = 0, kSliced = 1, kFrameSums = 2 };

template <typename T, int D, int OUT>
__global__ void __launch_bounds__(128) pool_kernel(const T* __restrict__ Q, const T* __restrict__ K,
                                                   int ntensors, Dims m, int b0, int nbr, int frame_len,
                                                   double* __restrict__ qo, double* __restrict__ ko,
                                                   double* __restrict__ qhi, double* __restrict__ khi,
                                                   SliceOut so) {
  using AccT = typename Acc<T>::type;
  constexpr int VEC = Acc<T>::kVec;
  constexpr int CPR = D / VEC;         // 16-byte vectors per row
  constexpr int RPI = 32 / CPR;        // rows per warp-wide load
  constexpr int NIT = kBlock / RPI;    // loads per lane per block
  constexpr int BATCH = NIT < 16 ? NIT : 16;
  constexpr bool FRAME = OUT == kFrameSums;
  const int lane = threadIdx.x & 31;
  const int c = lane % CPR, r0 = lane / CPR;
  // units: (tensor, head, block) over the blocks [b0, b0 + nbr) of every head
  const int64_t per = m.BH * nbr;
  const int64_t units = per * ntensors;
  const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
  // Software-pipelined over units: the first batch of the next unit is loaded before the current
  // unit's reduction and epilogue, so the epilogue overlaps memory latency.
  auto src_of = [&](int64_t uu) -> const T* {
    const bool k_ = uu >= per;
    const int64_t row_ = k_ ? uu - per : uu;
    const int64_t bh_ = row_ / nbr;
    const int64_t t0_ = (b0 + (row_ - bh_ * nbr)) * kBlock;
    return (k_ ? K : Q) + (bh_ * m.S + t0_) * D + c * VEC;
  };
  auto nvalid_of = [&](int64_t uu) -> int {
    const int64_t row_ = uu >= per ? uu - per : uu;
    return (int)imin<int64_t>(kBlock, m.S - (b0 + row_ % nbr) * kBlock);
  };
  uint4 v[BATCH];
  int64_t u = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (u < units) {
    const T* X0 = src_of(u);
    const int nv0 = nvalid_of(u);
#pragma unroll
    for (int it = 0; it < BATCH; ++it) {
      const int r = r0 + it * RPI;
      v[it] = r < nv0 ? __ldg(reinterpret_cast<const uint4*>(X0 + (int64_t)r * D)) : make_uint4(0, 0, 0, 0);
    }
  }
  for (; u < units; u += nwarps) {
    const bool isK = u >= per;
    const int64_t unit = isK ? u - per : u;      // bh * nbr + (blk - b0)
    const int64_t bh = unit / nbr;
    const int blk = b0 + (int)(unit - bh * nbr);
    const int64_t row = bh * m.nb + blk;
    const int64_t t0 = (int64_t)blk * kBlock;
    const int nvalid = (int)imin<int64_t>(kBlock, m.S - t0);
    const T* X = (isK ? K : Q) + (bh * m.S + t0) * D + c * VEC;
    int boundary = kBlock;
    if (FRAME) boundary = (int)imin<int64_t>(kBlock, (t0 / frame_len + 1) * frame_len - t0);
    double lo[VEC], hi[VEC];
#pragma unroll
    for (int e = 0; e < VEC; ++e) lo[e] = hi[e] = 0.0;
#pragma unroll
    for (int b0 = 0; b0 < NIT; b0 += BATCH) {
      // v holds batch b0 of this unit (loaded by the previous iteration or the prologue)
#pragma unroll
      for (int g = 0; g < BATCH; g += 4) {
        AccT sl[VEC], sh[VEC];
#pragma unroll
        for (int e = 0; e < VEC; ++e) sl[e] = sh[e] = 0;
#pragma unroll
        for (int it = g; it < g + 4; ++it) {
          AccT x[VEC];
          unpack(v[it], x, (const T*)nullptr);
          const bool in_lo = !FRAME || (r0 + (b0 + it) * RPI) < boundary;
#pragma unroll
          for (int e = 0; e < VEC; ++e) {
            if (in_lo) sl[e] += x[e];
            else sh[e] += x[e];
          }
        }
#pragma unroll
        for (int e = 0; e < VEC; ++e) {
          lo[e] += (double)sl[e];
          if (FRAME) hi[e] += (double)sh[e];
        }
      }
      // next batch: the rest of this unit, else the first batch of the next unit
      const bool more = b0 + BATCH < NIT;
      const int64_t un = u + nwarps;
      if (more || un < units) {
        const T* Xn = more ? X : src_of(un);
        const int nvn = more ? nvalid : nvalid_of(un);
        const int base = more ? b0 + BATCH : 0;
#pragma unroll
        for (int it = 0; it < BATCH; ++it) {
          const int r = r0 + (base + it) * RPI;
          v[it] = r < nvn ? __ldg(reinterpret_cast<const uint4*>(Xn + (int64_t)r * D)) : make_uint4(0, 0, 0, 0);
        }
      }
    }
#pragma unroll
    for (int off = CPR; off < 32; off <<= 1)
#pragma unroll
      for (int e = 0; e < VEC; ++e) {
        lo[e] += __shfl_xor_sync(0xffffffffu, lo[e], off);
        if (FRAME) hi[e] += __shfl_xor_sync(0xffffffffu, hi[e], off);
      }
    if (OUT == kSliced) {
      slice_mean<D, VEC>(lo, nvalid, r0, c,
                         (isK ? so.ks : so.qs) + ((bh * kScoreSlices) * m.nb + blk) * (int64_t)kSliceRow,
                         (int64_t)m.nb * kSliceRow, (isK ? so.ek : so.eq) + row);
    } else if (r0 == 0) {
      double* o = isK ? ko : qo;
      if (OUT == kMeans) {
#pragma unroll
        for (int e = 0; e < VEC; ++e) o[row * D + c * VEC + e] = lo[e] / (double)nvalid;
      } else {
        double* oh = isK ? khi : qhi;
#pragma unroll
        for (int e = 0; e < VEC; ++e) {
          o[row * D + c * VEC + e] = lo[e];
          oh[row * D + c * VEC + e] = hi[e];
        }
      }
    }
  }
}

size_t logits_elems(const Dims& m) { return (size_t)m.BH * m.nb * means_ld(m.nb); }

size_t select_smem_bytes(const Dims& m) {
  return (size_t)SEL_WARPS * m.nw * 4 + 16 + (size_t)SEL_WARPS * m.nw * 32 * 8;
}

// Rows of more than 40 * 32 blocks: one warp per query block, the row's logits staged in shared
// memory for the Top-p cut; forced blocks, bitmask row and count; warps 2w and 2w+1 hold the two
// rows of a 128-row tile and write its cost (no top-k and no slack augmentation at this size:
// the host rejects both).
__global__ void __launch_bounds__(SEL_WARPS * 32) select_smem_kernel(const double* __restrict__ logits, Dims m,
                                                                   double p, ForceCfg fc, uint32_t* __restrict__ bits,
                                                                   int32_t* __restrict__ counts,
                                                                   int32_t* __restrict__ tile_cost) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int nbp = m.nw * 32;
  uint32_t* sW = reinterpret_cast<uint32_t*>(smem_raw);                          // [warp][nw]
  double* sE = reinterpret_cast<double*>(smem_raw + (((size_t)SEL_WARPS * m.nw * 4 + 15) & ~(size_t)15));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t bh = blockIdx.y;
  const int i = blockIdx.x * SEL_WARPS + warp;
  const int ld = means_ld(m.nb);
  uint32_t* w = sW + warp * m.nw;
  if (i < m.nb) {
    const double* src = logits + (bh * m.nb + i) * (int64_t)ld;
    double* E = sE + (size_t)warp * nbp;
    for (int j = lane; j < m.nb; j += 32) E[j] = src[j];
    __syncwarp();
    topp_select(E, m.nb, p, w, lane);
    const int64_t grow = bh * m.nb + i;
    finalize_row(w, i, m, fc, lane, bits + grow * m.nw, counts + grow);
  } else {
    for (int q = lane; q < m.nw; q += 32) w[q] = 0;
  }
  __syncthreads();
  if (warp < SEL_WARPS / 2) {
    const int t = blockIdx.x * (SEL_WARPS / 2) + warp;
    if (2 * t < m.nb) {
      const uint32_t* wa = sW + (2 * warp) * m.nw;
      const uint32_t* wb = wa + m.nw;
      int c = 0;
      for (int q = lane; q < m.nw; q += 32) c += __popc(wa[q] | wb[q]);
      c = warp_sum(c);
      if (lane == 0) tile_cost[bh * m.nt + t] = c;
    }
  }
}

// Rows of at most 32 NE blocks: one warp per 128-row tile (query blocks 2t and 2t+1 of one
// head): the cut of both rows in registers, forced blocks, bitmask rows and counts, the tile's
// cost, then (sasa.coef > 0) each row augmented from the other's slack. A warp needs no other
// warp's rows, so the CTA has no barrier and a tile's rows never wait for a slower row of
// another tile. The kernel is bound by the latency of each warp's rows, so it runs with more
// CTAs per SM than its registers alone would allow: rows of up to 512 blocks at 10 (48
// registers and a 40-byte spill: 20 % faster than 8 CTAs at 64 registers; 12 CTAs at 40
// registers spill ten times as much and lose), rows of up to 1280 blocks at 5 (96 registers and
// an 80-byte spill: a third faster than 2 CTAs at 181 registers).
template <int NE>
__global__ void __launch_bounds__(SEL_WARPS * 32, NE == 16 ? 10 : 5)
    select_tile_kernel(const double* __restrict__ logits, Dims m, double p, int kblocks, ForceCfg fc, SasaCfg sasa,
                       uint32_t* __restrict__ bits, int32_t* __restrict__ counts, int32_t* __restrict__ tile_cost) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint32_t* sw = reinterpret_cast<uint32_t*>(smem_raw) + (size_t)warp * 4 * m.nw;   // rows 2t, 2t+1, wc, wo
  const int64_t bh = blockIdx.y;
  const int t = blockIdx.x * SEL_WARPS + warp;
  if (t >= m.nt) return;
  const int ld = means_ld(m.nb);
  uint32_t* w[2] = {sw, sw + m.nw};
  for (int rr = 0; rr < 2; ++rr) {
    const int i = 2 * t + rr;
    if (i >= m.nb) {
      for (int q = lane; q < m.nw; q += 32) w[rr][q] = 0u;
      __syncwarp();
      continue;
    }
    const double* src = logits + (bh * m.nb + i) * (int64_t)ld;
    if (kblocks > 0) topk_select_reg<NE>(src, m.nb, kblocks, w[rr], lane);
    else topp_select_reg<NE>(src, m.nb, p, w[rr], lane);
    const int64_t grow = bh * m.nb + i;
    finalize_row(w[rr], i, m, fc, lane, bits + grow * m.nw, counts + grow);
  }
  int c = 0;
  for (int q = lane; q < m.nw; q += 32) c += __popc(w[0][q] | w[1][q]);
  c = warp_sum(c);
  if (lane == 0) tile_cost[bh * m.nt + t] = c;
  if (sasa.coef > 0.f && 2 * t + 1 < m.nb) {
    uint32_t* wc = sw + 2 * m.nw;
    uint32_t* wo = sw + 3 * m.nw;
    for (int rr = 0; rr < 2; ++rr) {
      const int64_t grow = bh * m.nb + 2 * t + rr;
      sasa_row<NE>(logits + grow * (int64_t)ld, m, sasa, w[rr], w[rr ^ 1], wc, wo, lane, bits + grow * m.nw,
                   counts + grow);
      __syncwarp();
    }
  }
}

static cudaError_t launch_select_smem(const double* logits, const Dims& m, double p, const ForceCfg& fc,
                                      uint32_t* bits, int32_t* counts, int32_t* tile_cost, cudaStream_t st) {
  const size_t smem = select_smem_bytes(m);
  cudaError_t e = cudaFuncSetAttribute(select_smem_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 g((m.nb + SEL_WARPS - 1) / SEL_WARPS, (unsigned)m.BH);
  select_smem_kernel<<<g, SEL_WARPS * 32, smem, st>>>(logits, m, p, fc, bits, counts, tile_cost);
  return cudaGetLastError();
}

template <int NE>
static cudaError_t launch_select_tile_t(const double* logits, const Dims& m, double p, int kblocks, const ForceCfg& fc,
                                        const SasaCfg& sasa, uint32_t* bits, int32_t* counts, int32_t* tile_cost,
                                        cudaStream_t st) {
  const size_t smem = (size_t)SEL_WARPS * 4 * m.nw * 4;
  cudaError_t e =
      cudaFuncSetAttribute(select_tile_kernel<NE>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 g((m.nt + SEL_WARPS - 1) / SEL_WARPS, (unsigned)m.BH);
  select_tile_kernel<NE><<<g, SEL_WARPS * 32, smem, st>>>(logits, m, p, kblocks, fc, sasa, bits, counts, tile_cost);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ frame mode

// Frame means from the per-block segment sums: frame f gathers the "lo" sums of the blocks
// that start inside f and the "hi" sums of the block that starts in f-1 and straddles into f
// (frames are at least one block long, so a block touches at most two frames).
template <int D>
__global__ void __launch_bounds__(D) frame_means_kernel(const double* __restrict__ qlo, const double* __restrict__ qhi,
                                                        const double* __restrict__ klo, const double* __restrict__ khi,
                                                        Dims m, int frame_len, double* __restrict__ qf,
                                                        double* __restrict__ kf) {
  const int f = blockIdx.x;
  const int64_t bh = blockIdx.y;
  const bool isK = blockIdx.z != 0;
  const double* lo = isK ? klo : qlo;
  const double* hi = isK ? khi : qhi;
  const int64_t t0 = (int64_t)f * frame_len, t1 = min(m.S, t0 + frame_len);
  const int b0 = (int)(t0 / kBlock), b1 = (int)((t1 - 1) / kBlock);
  double s = 0.0;
  for (int b = b0; b <= b1; ++b) {
    const int64_t fb = ((int64_t)b * kBlock) / frame_len;
    const double* src = (fb == f) ? lo : hi;
    s += src[(bh * m.nb + b) * D + threadIdx.x];
  }
  (isK ? kf : qf)[(bh * m.F + f) * D + threadIdx.x] = s / (double)(t1 - t0);
}

size_t frame_smem_bytes(const Dims& m) {
  const int fwords = (m.F + 31) / 32;
  return (size_t)m.F * m.F * 8 + (size_t)m.F * fwords * 4 + (size_t)NWARP * 2 * m.nw * 4;
}

// One CTA per head: frame scores s(f,g) = <qf_f, kf_g> * scale in fp64; per query frame the
// top-k key frames (ties to the lower frame); per query block the union over the frames it
// touches, expanded to the key blocks that hold tokens of a kept frame; then forced blocks.
template <int D>
__global__ void __launch_bounds__(256) frame_select_kernel(const double* __restrict__ qf, const double* __restrict__ kf,
                                                           Dims m, int frame_len, int topk, double scale,
                                                           ForceCfg fc, uint32_t* __restrict__ bits,
                                                           int32_t* __restrict__ counts,
                                                           int32_t* __restrict__ tile_cost,
                                                           uint32_t* __restrict__ fsel) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int F = m.F, fwords = (F + 31) / 32;
  double* sS = reinterpret_cast<double*>(smem_raw);                     // [F][F]
  uint32_t* sCh = reinterpret_cast<uint32_t*>(sS + (size_t)F * F);      // [F][fwords]
  uint32_t* sW = sCh + (size_t)F * fwords;                              // [NWARP][2][nw]
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t bh = blockIdx.x;

  for (int x = tid; x < F * F; x += blockDim.x) {
    const int f = x / F, g = x - f * F;
    const double* a = qf + (bh * F + f) * D;
    const double* b = kf + (bh * F + g) * D;
    double s = 0.0;
#pragma unroll 8
    for (int k = 0; k < D; ++k) s = fma(a[k], b[k], s);
    sS[x] = s * scale;
  }
  for (int x = tid; x < F * fwords; x += blockDim.x) sCh[x] = 0;
  __syncthreads();

  const int k = min(topk, F);
  for (int f = warp; f < F; f += NWARP) {
    for (int r = 0; r < k; ++r) {
      double best = -INFINITY;
      int bi = 0x7fffffff;
      for (int g = lane; g < F; g += 32) {
        const bool taken = (sCh[f * fwords + (g >> 5)] >> (g & 31)) & 1u;
        const double v = sS[f * F + g];
        if (!taken && (v > best || (v == best && g < bi))) { best = v; bi = g; }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const double ov = __shfl_xor_sync(0xffffffffu, best, o);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
        if (ov > best || (ov == best && oi < bi)) { best = ov; bi = oi; }
      }
      if (lane == 0) sCh[f * fwords + (bi >> 5)] |= 1u << (bi & 31);
      __syncwarp();
    }
  }
  __syncthreads();
  for (int x = tid; x < F * fwords; x += blockDim.x) fsel[bh * F * fwords + x] = sCh[x];

  uint32_t* w0 = sW + warp * 2 * m.nw;
  for (int t = warp; t < m.nt; t += NWARP) {
#pragma unroll 1
    for (int rr = 0; rr < 2; ++rr) {
      const int i = 2 * t + rr;
      uint32_t* w = w0 + rr * m.nw;
      if (i >= m.nb) {
        for (int q = lane; q < m.nw; q += 32) w[q] = 0;
        __syncwarp();
        continue;
      }
      const int64_t ti0 = (int64_t)i * kBlock, ti1 = min(m.S, ti0 + kBlock) - 1;
      const int f0 = (int)(ti0 / frame_len), f1 = (int)(ti1 / frame_len);
      for (int q = lane; q < m.nw; q += 32) {
        uint32_t x = 0;
        for (int g = 0; g < F; ++g) {
          const uint32_t kept = ((sCh[f0 * fwords + (g >> 5)] | sCh[f1 * fwords + (g >> 5)]) >> (g & 31)) & 1u;
          if (kept) {
            const int a = (int)(((int64_t)g * frame_len) / kBlock);
            const int b = (int)((min(m.S, (int64_t)(g + 1) * frame_len) - 1) / kBlock);
            x |= range_bits(a, b, q);
          }
        }
        w[q] = x;
      }
      __syncwarp();
      const int64_t grow = bh * m.nb + i;
      finalize_row(w, i, m, fc, lane, bits + grow * m.nw, counts + grow);
    }
    if (2 * t < m.nb) {
      int c = 0;
      for (int q = lane; q < m.nw; q += 32) c += __popc(w0[q] | w0[m.nw + q]);
      c = warp_sum(c);
      if (lane == 0) tile_cost[bh * m.nt + t] = c;
    }
    __syncwarp();
  }
}

// ------------------------------------------------------------------ K3: schedule

size_t schedule_smem_bytes(const Dims& m, int* groups) {
  const size_t nb1 = (size_t)m.nb + 1;
  int g = 32;
  while (g > 1 && (size_t)(g + 1) * nb1 * 4 > 200 * 1024) g >>= 1;
  *groups = g;
  return (size_t)(g + 1) * nb1 * 4;
}

// One CTA: CSR row offsets (exclusive scan of the row counts), nnz, per-head loads, and the
// tile order: a stable counting sort of tile costs, largest first, ties by ascending tile id.
// Tiles are split into `groups` contiguous segments with one histogram each, so the sort
// stays stable while the segments are placed in parallel.
__global__ void __launch_bounds__(1024) schedule_kernel(const int32_t* __restrict__ counts,
                                                        const int32_t* __restrict__ tile_cost, Dims m,
                                                        int groups, int32_t* __restrict__ row_ptr,
                                                        int64_t* __restrict__ head_load,
                                                        int64_t* __restrict__ nnz_out,
                                                        int32_t* __restrict__ tile_order, int64_t capacity,
                                                        int32_t* __restrict__ status) {
  extern __shared__ __align__(16) int32_t shs[];
  __shared__ int64_t wsum[32];
  __shared__ int32_t wtot[32];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // ---- row offsets: an exclusive scan of the counts in coalesced 4096-row slices, each
  // thread taking 4 consecutive rows, carried from slice to slice.
  const int64_t N = m.BH * m.nb;
  int64_t carry = 0;
  for (int64_t b0 = 0; b0 < N; b0 += 4096) {
    const int64_t r = b0 + 4 * (int64_t)tid;
    int c[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) c[e] = (r + e < N) ? counts[r + e] : 0;
    const int64_t s = (int64_t)c[0] + c[1] + c[2] + c[3];
    const int64_t incl = warp_incl_scan(s, lane);
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      const int64_t v = wsum[lane];
      const int64_t vi = warp_incl_scan(v, lane);
      wsum[lane] = vi;                                  // inclusive over warps
    }
    __syncthreads();
    int64_t base = carry + (warp ? wsum[warp - 1] : 0) + incl - s;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if (r + e < N) row_ptr[r + e] = (int32_t)base;
      base += c[e];
    }
    carry += wsum[31];
    __syncthreads();
  }
  if (tid == 0) {
    row_ptr[N] = (int32_t)carry;
    *nnz_out = carry;
    if (carry > capacity) report_error(status, FVATTN_ERR_CAPACITY, 1);
    status[3] = (int32_t)(m.BH * m.nt);     // the attention takes every tile of the order
  }
  __syncthreads();
  for (int64_t bh = tid; bh < m.BH; bh += 1024)
    head_load[bh] = (int64_t)row_ptr[(bh + 1) * m.nb] - (int64_t)row_ptr[bh * m.nb];

  // ---- tile order
  const int nb1 = m.nb + 1;
  int32_t* hist = shs;                    // [groups][nb1]: counts, then running offsets
  int32_t* tot = shs + (size_t)groups * nb1;
  for (int x = tid; x < groups * nb1; x += 1024) hist[x] = 0;
  __syncthreads();
  const int64_t NT = m.BH * m.nt;
  const int64_t seg = (NT + groups - 1) / groups;
  if (warp < groups) {
    const int64_t s0 = min(NT, warp * seg), s1 = min(NT, s0 + seg);
    for (int64_t t = s0 + lane; t < s1; t += 32) atomicAdd(&hist[warp * nb1 + tile_cost[t]], 1);
  }
  __syncthreads();
  for (int c = tid; c < nb1; c += 1024) {
    int run = 0;
    for (int g = 0; g < groups; ++g) {
      const int h = hist[g * nb1 + c];
      hist[g * nb1 + c] = run;
      run += h;
    }
    tot[c] = run;
  }
  __syncthreads();
  // base[c] = number of tiles with cost > c: a suffix scan of tot, in chunks per thread.
  {
    const int chunk = (nb1 + 1023) / 1024;
    const int c0 = min(nb1, tid * chunk), c1 = min(nb1, c0 + chunk);
    int ls = 0;
    for (int c = c0; c < c1; ++c) ls += tot[c];
    const int li = warp_incl_scan(ls, lane);
    if (lane == 31) wtot[warp] = li;
    __syncthreads();
    if (warp == 0) {
      const int v = wtot[lane];
      const int vi = warp_incl_scan(v, lane);
      wtot[lane] = vi;   // inclusive over warps
    }
    __syncthreads();
    const int total = wtot[31];
    // tiles with cost >= c0 (all buckets from this thread's chunk upward):
    const int before_incl = (warp ? wtot[warp - 1] : 0) + li;   // sum of buckets [0, c1)
    int above = total - before_incl;                             // sum of buckets [c1, nb1)
    for (int c = c1 - 1; c >= c0; --c) {
      const int tc = tot[c];
      for (int g = 0; g < groups; ++g) hist[g * nb1 + c] += above;
      above += tc;
    }
  }
  __syncthreads();
  if (warp < groups) {
    const int64_t s0 = min(NT, warp * seg), s1 = min(NT, s0 + seg);
    for (int64_t t0 = s0; t0 < s1; t0 += 32) {
      const int64_t t = t0 + lane;
      const bool v = t < s1;
      const int c = v ? tile_cost[t] : -1 - lane;
      const uint32_t peers = __match_any_sync(0xffffffffu, c);
      const uint32_t lower = peers & lanemask_lt();
      int pos = 0;
      if (v) pos = hist[warp * nb1 + c] + __popc(lower);
      __syncwarp();
      if (v) {
        tile_order[pos] = (int32_t)t;
        if (lower == 0) hist[warp * nb1 + c] += __popc(peers);
      }
      __syncwarp();
    }
  }
}

// ------------------------------------------------------------------ token-exact frame codes

// One warp per CSR row: the code of every entry (fvattn_csr.col_code). Token-exact frame mode
// (fsel != null): a query token of frame f may attend the key tokens of the frames kept for f
// (its top-k frames, the frames within +-frame_window, frame 0 when forced); the entry's
// blocks span at most two frames each, so the code holds allow[a][b] for the query block's
// frame a and the key block's frame b and the two in-block boundaries. Block-level forced
// entries (diagonal, band) and every entry outside that mode allow the whole key block.
__global__ void __launch_bounds__(256) code_kernel(const int32_t* __restrict__ row_ptr,
                                                   const int32_t* __restrict__ col_idx, Dims m,
                                                   const uint32_t* __restrict__ fsel, int frame_len, ForceCfg fc,
                                                   int32_t* __restrict__ col_code, int64_t capacity) {
  const int lane = threadIdx.x & 31;
  const int64_t N = m.BH * m.nb;
  const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
  const int fwords = (m.F + 31) / 32;
  for (int64_t row = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); row < N; row += nwarps) {
    const int64_t e0 = row_ptr[row], e1 = imin<int64_t>(row_ptr[row + 1], capacity);
    if (fsel == nullptr) {
      for (int64_t e = e0 + lane; e < e1; e += 32) col_code[e] = kCodeAll;
      continue;
    }
    const int64_t bh = row / m.nb;
    const int i = (int)(row - bh * m.nb);
    const int64_t fl = frame_len;
    const int64_t ti = (int64_t)i * kBlock;
    const int qf0 = (int)(ti / fl), qf1 = (int)((min(m.S, ti + kBlock) - 1) / fl);
    const int qrow = qf1 != qf0 ? (int)(qf1 * fl - ti) : kBlock;
    const uint32_t* G = fsel + bh * m.F * fwords;
    auto kept = [&](int f, int g) -> bool {
      if (fc.frame_window >= 0 && g >= f - fc.frame_window && g <= f + fc.frame_window) return true;
      if (fc.force_first && g == 0) return true;
      return (G[f * fwords + (g >> 5)] >> (g & 31)) & 1u;
    };
    for (int64_t e = e0 + lane; e < e1; e += 32) {
      const int j = col_idx[e];
      const bool forced = (fc.force_diag && j == i) || (fc.local_window > 0 && abs(i - j) <= fc.local_window);
      const int64_t tj = (int64_t)j * kBlock;
      const int kf0 = (int)(tj / fl), kf1 = (int)((min(m.S, tj + kBlock) - 1) / fl);
      const int kcol = kf1 != kf0 ? (int)(kf1 * fl - tj) : kBlock;
      int allow = 0xF;
      if (!forced)
        allow = (kept(qf0, kf0) ? 1 : 0) | (kept(qf0, kf1) ? 2 : 0) | (kept(qf1, kf0) ? 4 : 0) | (kept(qf1, kf1) ? 8 : 0);
      col_code[e] = allow | (kcol << 8) | (qrow << 16);
    }
  }
}

// ------------------------------------------------------------------ K4: CSR columns

__global__ void __launch_bounds__(256) csr_kernel(const uint32_t* __restrict__ bits,
                                                  const int32_t* __restrict__ row_ptr, Dims m,
                                                  int32_t* __restrict__ col_idx, int64_t capacity) {
  const int lane = threadIdx.x & 31;
  const int64_t N = m.BH * m.nb;
  const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t row = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); row < N; row += nwarps) {
    if ((int64_t)row_ptr[row + 1] > capacity) continue;     // reported by the schedule kernel
    const uint32_t* w = bits + row * m.nw;
    int64_t pos = row_ptr[row];
    // Lane l holds word q0 + l; the non-zero words are then expanded one at a time by the whole
    // warp, lane b writing block 32q + b when its bit is set, so that each word's entries go
    // out as one coalesced store in ascending order.
    for (int q0 = 0; q0 < m.nw; q0 += 32) {
      const uint32_t xl = q0 + lane < m.nw ? w[q0 + lane] : 0u;
      uint32_t nz = __ballot_sync(0xffffffffu, xl != 0u);
      while (nz) {
        const int k = __ffs(nz) - 1;
        nz &= nz - 1;
        const uint32_t x = __shfl_sync(0xffffffffu, xl, k);
        if ((x >> lane) & 1u) col_idx[pos + __popc(x & lanemask_lt())] = (q0 + k) * 32 + lane;
        pos += __popc(x);
      }
    }
  }
}

// ------------------------------------------------------------------ launchers

template <typename T, int D>
static cudaError_t launch_pool_td(const void* Q, const void* K, int ntensors, const Dims& m, int b0, int b1, int out,
                                  int frame_len, double* qo, double* ko, double* qhi, double* khi, const SliceOut& so,
                                  int nsm, cudaStream_t st) {
  const int nbr = b1 - b0;
  if (nbr <= 0) return cudaSuccess;
  const int64_t units = m.BH * nbr * ntensors;
  const int grid = (int)imin<int64_t>((units + 3) / 4, (int64_t)nsm * 16);
  const T* q = static_cast<const T*>(Q);
  const T* k = static_cast<const T*>(K);
  if (out == kSliced)
    pool_kernel<T, D, kSliced><<<grid, 128, 0, st>>>(q, k, ntensors, m, b0, nbr, 0, nullptr, nullptr, nullptr, nullptr,
                                                      so);
  else if (out == kFrameSums)
    pool_kernel<T, D, kFrameSums><<<grid, 128, 0, st>>>(q, k, ntensors, m, b0, nbr, frame_len, qo, ko, qhi, khi, so);
  else
    pool_kernel<T, D, kMeans><<<grid, 128, 0, st>>>(q, k, ntensors, m, b0, nbr, 0, qo, ko, nullptr, nullptr, so);
  return cudaGetLastError();
}

// out: 0 = means [row][d], 1 = score slices and exponents, 2 = frame segment sums; blocks
// [b0, b1) of every head.
cudaError_t launch_pool(const void* Q, const void* K, int ntensors, int dtype, const Dims& m, int b0, int b1, int out,
                        int frame_len, double* qo, double* ko, double* qhi, double* khi, const SliceOut& so, int nsm,
                        cudaStream_t st) {
  if (dtype == FVATTN_BF16) {
    if (m.d == 128)
      return launch_pool_td<__nv_bfloat16, 128>(Q, K, ntensors, m, b0, b1, out, frame_len, qo, ko, qhi, khi, so, nsm,
                                                st);
    return launch_pool_td<__nv_bfloat16, 64>(Q, K, ntensors, m, b0, b1, out, frame_len, qo, ko, qhi, khi, so, nsm, st);
  }
  if (m.d == 128)
    return launch_pool_td<float, 128>(Q, K, ntensors, m, b0, b1, out, frame_len, qo, ko, qhi, khi, so, nsm, st);
  return launch_pool_td<float, 64>(Q, K, ntensors, m, b0, b1, out, frame_len, qo, ko, qhi, khi, so, nsm, st);
}


cudaError_t launch_topp(const SliceOut& so, double* logits, const Dims& m, double p, int kblocks, double scale,
                        const ForceCfg& fc, const SasaCfg& sasa, uint32_t* bits, int32_t* counts, int32_t* tile_cost,
                        int32_t* status, int nsm, cudaStream_t st) {
  cudaError_t e = launch_score_tc(so.qs, so.ks, so.eq, so.ek, m, scale, logits, status, nsm, st);
  if (e != cudaSuccess) return e;
  if (m.nb <= 32 * 16) return launch_select_tile_t<16>(logits, m, p, kblocks, fc, sasa, bits, counts, tile_cost, st);
  if (m.nb <= 32 * 40) return launch_select_tile_t<40>(logits, m, p, kblocks, fc, sasa, bits, counts, tile_cost, st);
  return launch_select_smem(logits, m, p, fc, bits, counts, tile_cost, st);
}

cudaError_t launch_frame(const double* qlo, const double* qhi, const double* klo, const double* khi,
                         double* qf, double* kf, const Dims& m, int frame_len, int topk, double scale,
                         const ForceCfg& fc, uint32_t* bits, int32_t* counts, int32_t* tile_cost,
                         uint32_t* fsel, cudaStream_t st) {
  dim3 g1((unsigned)m.F, (unsigned)m.BH, 2);
  const size_t smem = frame_smem_bytes(m);
  cudaError_t e;
  if (m.d == 128) {
    frame_means_kernel<128><<<g1, 128, 0, st>>>(qlo, qhi, klo, khi, m, frame_len, qf, kf);
    e = cudaFuncSetAttribute(frame_select_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    frame_select_kernel<128><<<(unsigned)m.BH, 256, smem, st>>>(qf, kf, m, frame_len, topk, scale, fc, bits, counts,
                                                                tile_cost, fsel);
  } else {
    frame_means_kernel<64><<<g1, 64, 0, st>>>(qlo, qhi, klo, khi, m, frame_len, qf, kf);
    e = cudaFuncSetAttribute(frame_select_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    frame_select_kernel<64><<<(unsigned)m.BH, 256, smem, st>>>(qf, kf, m, frame_len, topk, scale, fc, bits, counts,
                                                               tile_cost, fsel);
  }
  return cudaGetLastError();
}

cudaError_t launch_schedule(const int32_t* counts, const int32_t* tile_cost, const Dims& m, int32_t* row_ptr,
                            int64_t* head_load, int64_t* nnz, int32_t* tile_order, int64_t capacity,
                            int32_t* status, cudaStream_t st) {
  int groups = 32;
  const size_t smem = schedule_smem_bytes(m, &groups);
  cudaError_t e = cudaFuncSetAttribute(schedule_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  schedule_kernel<<<1, 1024, smem, st>>>(counts, tile_cost, m, groups, row_ptr, head_load, nnz, tile_order,
                                         capacity, status);
  return cudaGetLastError();
}

cudaError_t launch_codes(const int32_t* row_ptr, const int32_t* col_idx, const Dims& m, const uint32_t* fsel,
                         int frame_len, const ForceCfg& fc, int32_t* col_code, int64_t capacity, int nsm,
                         cudaStream_t st) {
  const int64_t rows = m.BH * m.nb;
  const int grid = (int)imin<int64_t>((rows + 7) / 8, (int64_t)nsm * 8);
  code_kernel<<<grid, 256, 0, st>>>(row_ptr, col_idx, m, fsel, frame_len, fc, col_code, capacity);
  return cudaGetLastError();
}

cudaError_t launch_csr(const uint32_t* bits, const int32_t* row_ptr, const Dims& m, int32_t* col_idx,
                       int64_t capacity, int nsm, cudaStream_t st) {
  const int64_t rows = m.BH * m.nb;
  const int grid = (int)imin<int64_t>((rows + 7) / 8, (int64_t)nsm * 8);
  csr_kernel<<<grid, 256, 0, st>>>(bits, row_ptr, m, col_idx, capacity);
  return cudaGetLastError();
}

}  // namespace fv
