// Shared definitions of the fvattn CUDA sources (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "fvattn.h"

namespace fv {

template <typename T>
__host__ __device__ __forceinline__ T imin(T a, T b) { return a < b ? a : b; }
template <typename T>
__host__ __device__ __forceinline__ T imax(T a, T b) { return a < b ? b : a; }

constexpr int kBlock = 64;          // tokens per block (query and key)
constexpr int kTileRows = 128;      // query rows per attention tile = two query blocks

// Sizes derived from a validated fvattn_shape.
struct Dims {
  int64_t BH;     // B * H
  int64_t S;      // tokens
  int d;          // head dim
  int nb;         // blocks per head, ceil(S / 64)
  int nw;         // 32-bit words of one selection bitmask row, ceil(nb / 32)
  int nt;         // 128-row tiles per head, ceil(nb / 2)
  int F;          // frames per head (frame mode), else 0
};

inline Dims make_dims(const fvattn_shape& s, int frame_len) {
  Dims m;
  m.BH = s.B * s.H;
  m.S = s.S;
  m.d = (int)s.d;
  m.nb = (int)((s.S + kBlock - 1) / kBlock);
  m.nw = (m.nb + 31) / 32;
  m.nt = (m.nb + 1) / 2;
  m.F = frame_len > 0 ? (int)((s.S + frame_len - 1) / frame_len) : 0;
  return m;
}

// The first device error wins; later ones are dropped.
__device__ __forceinline__ void report_error(int32_t* status, int code, int detail) {
  if (atomicCAS(status, 0, code) == 0) status[1] = detail;
}

#ifdef FVATTN_DEBUG
// Debug build (-DFVATTN_DEBUG) only: checks the CSR list of one row before a kernel reads it.
// Returns 0, or the failed check: kDbgOffsets (row offsets decreasing, negative or beyond the
// column array's capacity), kDbgColumn (a key block outside [0, nb)), kDbgOrder (the list not
// strictly ascending). Kernels report it as FVATTN_ERR_INVALID with the check in status[1]
// and skip the row; nothing outside the arrays is read.
constexpr int kDbgOffsets = 101, kDbgColumn = 102, kDbgOrder = 103;
__device__ inline int debug_row_check(const int32_t* row_ptr, const int32_t* col_idx, int64_t col_cap, int64_t row,
                                      int nb) {
  const int64_t a = row_ptr[row], b = row_ptr[row + 1];
  if (a < 0 || b < a || b > col_cap) return kDbgOffsets;
  int prev = -1;
  for (int64_t e = a; e < b; ++e) {
    const int j = col_idx[e];
    if (j < 0 || j >= nb) return kDbgColumn;
    if (j <= prev) return kDbgOrder;
    prev = j;
  }
  return 0;
}
#endif

__device__ __forceinline__ uint32_t lanemask_lt() {
  uint32_t m;
  asm volatile("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// Bits of [a, b] (inclusive block indices) that fall in word w.
__device__ __forceinline__ uint32_t range_bits(int a, int b, int w) {
  int lo = max(a, w * 32), hi = min(b, w * 32 + 31);
  if (lo > hi) return 0u;
  int n = hi - lo + 1;
  uint32_t m = (n == 32) ? 0xffffffffu : ((1u << n) - 1u);
  return m << (lo - w * 32);
}

}  // namespace fv
