// Block-sparse attention for fp32 inputs on the CUDA cores, in fp32.
//
// Exact softmax attention of each query token over the tokens of the key blocks that the
// router kept for its query block (FVAttn blog summary, section "AI视频生成的阿喀琉斯之踵";
// the masked attention of the wzjinhao.cn notes §5.2). One CTA per query block of the tiles
// in the router's tile order (the first control[3] entries: every tile, or the tiles of the
// heads kept by fvattn_select_heads); four threads share one query row, each owning d/4
// output columns; keys are visited in ascending block order with an online (running max /
// running sum) softmax.
#include <math.h>

#include "common.cuh"
#include "route.cuh"

namespace fv {

template <int D>
__global__ void __launch_bounds__(256) attn_f32_kernel(const float* __restrict__ Q, const float* __restrict__ K,
                                                       const float* __restrict__ V, Dims m, float scale,
                                                       const int32_t* __restrict__ row_ptr,
                                                       const int32_t* __restrict__ col_idx, int64_t col_cap,
                                                       const int32_t* __restrict__ col_code,
                                                       const int32_t* __restrict__ tile_order,
                                                       int32_t* __restrict__ control,
                                                       float* __restrict__ O, float* __restrict__ lse) {
  constexpr int DQ = D / 4;
  constexpr int KCH = D == 128 ? 32 : 64;     // keys staged per step (shared memory <= 48 KB)
  __shared__ float sK[KCH][D + 1];
  __shared__ float sV[KCH][D];
  const int tid = threadIdx.x;
  const int r = tid >> 2, part = tid & 3;
  const int64_t ntiles = m.BH * m.nt;
  const int64_t k = blockIdx.x;
  if (k >= imin<int64_t>(ntiles, control[3])) return;
  const int tile = tile_order[k];
  if (tile < 0 || tile >= ntiles) return;
  const int64_t bh = tile / m.nt;
  const int i = 2 * (int)(tile - bh * m.nt) + (int)blockIdx.y;
  if (i >= m.nb) return;
  const int64_t t = (int64_t)i * kBlock + r;
  const bool valid_row = t < m.S;
  const int64_t base = bh * m.S * D;

  float q[DQ], o[DQ];
#pragma unroll
  for (int c = 0; c < DQ; ++c) {
    q[c] = valid_row ? Q[base + t * D + part * DQ + c] * scale : 0.f;
    o[c] = 0.f;
  }
  float mx = -INFINITY, l = 0.f;
  const int64_t row = bh * m.nb + i;
#ifdef FVATTN_DEBUG
  if (const int bad = debug_row_check(row_ptr, col_idx, col_cap, row, m.nb)) {   // uniform over the CTA
    if (tid == 0) report_error(control, FVATTN_ERR_INVALID, bad);
    return;
  }
#endif
  const int e0 = row_ptr[row], e1 = row_ptr[row + 1];
  for (int e = e0; e < e1; ++e) {
    const int j = col_idx[e];
    // token-exact frame mode: which side of the key block this row may see (col_code)
    const int code = col_code != nullptr ? col_code[e] : kCodeAll;
    const int side = r >= ((code >> 16) & 0xFF) ? 1 : 0;
    const bool keep0 = (code >> (2 * side)) & 1, keep1 = (code >> (2 * side + 1)) & 1;
    const int kcol = (code >> 8) & 0xFF;
    const int64_t k0 = (int64_t)j * kBlock;
    const int nk_blk = (int)imin<int64_t>(kBlock, m.S - k0);
    for (int c0 = 0; c0 < nk_blk; c0 += KCH) {
    const int nk = min(KCH, nk_blk - c0);
    __syncthreads();
    for (int x = tid; x < KCH * D; x += 256) {
      const int u = x / D, c = x - u * D;
      const bool ok = u < nk;
      sK[u][c] = ok ? K[base + (k0 + c0 + u) * D + c] : 0.f;
      sV[u][c] = ok ? V[base + (k0 + c0 + u) * D + c] : 0.f;
    }
    __syncthreads();
    for (int u = 0; u < nk; ++u) {
      float s = 0.f;
#pragma unroll
      for (int c = 0; c < DQ; ++c) s = fmaf(q[c], sK[u][part * DQ + c], s);
      s += __shfl_xor_sync(0xffffffffu, s, 1);
      s += __shfl_xor_sync(0xffffffffu, s, 2);
      if (c0 + u < kcol ? keep0 : keep1) {
        const float mn = fmaxf(mx, s);
        const float a = expf(mx - mn);
        const float pu = expf(s - mn);
        l = l * a + pu;
#pragma unroll
        for (int c = 0; c < DQ; ++c) o[c] = fmaf(pu, sV[u][part * DQ + c], o[c] * a);
        mx = mn;
      }
    }
    }
  }
  if (valid_row) {
    const float inv = 1.f / l;
#pragma unroll
    for (int c = 0; c < DQ; ++c) O[base + t * D + part * DQ + c] = o[c] * inv;
    if (lse && part == 0) lse[bh * m.S + t] = mx + logf(l);
  }
}

cudaError_t launch_attn_f32(const float* Q, const float* K, const float* V, const Dims& m, float scale,
                            const int32_t* row_ptr, const int32_t* col_idx, int64_t col_cap, const int32_t* col_code,
                            const int32_t* tile_order, int32_t* control, float* O, float* lse, cudaStream_t st) {
  const int64_t ntiles = m.BH * m.nt;
  if (ntiles > 0x7fffffff) return cudaErrorInvalidValue;
  dim3 grid((unsigned)ntiles, 2);
  if (m.d == 128)
    attn_f32_kernel<128><<<grid, 256, 0, st>>>(Q, K, V, m, scale, row_ptr, col_idx, col_cap, col_code, tile_order,
                                               control, O, lse);
  else
    attn_f32_kernel<64><<<grid, 256, 0, st>>>(Q, K, V, m, scale, row_ptr, col_idx, col_cap, col_code, tile_order,
                                              control, O, lse);
  return cudaGetLastError();
}

}  // namespace fv
