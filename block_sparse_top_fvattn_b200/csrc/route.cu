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

namespace fv {

// ------------------------------------------------------------------ warp helpers

template <typename T>
__device__ __forceinline__ T warp_sum(T v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ double warp_max(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmax(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

template <typename T>
__device__ __forceinline__ T warp_incl_scan(T v, int lane) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    T u = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += u;
  }
  return v;
}

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

template <typename T> struct Acc;
template <> struct Acc<__nv_bfloat16> { using type = float; static constexpr int kVec = 8; };
template <> struct Acc<float> { using type = double; static constexpr int kVec = 4; };

__device__ __forceinline__ void unpack(const uint4& v, float (&o)[8], const __nv_bfloat16*) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    float2 f = __bfloat1622float2(h[q]);
    o[2 * q] = f.x;
    o[2 * q + 1] = f.y;
  }
}
__device__ __forceinline__ void unpack(const uint4& v, double (&o)[4], const float*) {
  o[0] = __uint_as_float(v.x);
  o[1] = __uint_as_float(v.y);
  o[2] = __uint_as_float(v.z);
  o[3] = __uint_as_float(v.w);
}

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
      // The mean as a power-of-two scale 2^ex and kScoreSlices signed 8-bit digits: with
      // N = rint(x 2^(39-ex)), N = X_0 2^32 + X_1 2^24 + X_2 2^16 + X_3 2^8 + X_4, i.e.
      // x ~ 2^ex sum_a X_a 2^(-7-8a). X_4..X_1 are the balanced base-256 digits (in [-128, 127],
      // taken from the bottom), X_0 the rest. ex is the smallest power of two above max|x|,
      // raised by one when max|N| > 127 * 2^32, so that X_0 stays in [-128, 127] too.
      double r[VEC], mx = 0.0;
#pragma unroll
      for (int e = 0; e < VEC; ++e) {
        r[e] = lo[e] / (double)nvalid;
        mx = fmax(mx, fabs(r[e]));
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) mx = fmax(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      // ex = floor(log2(mx)) + 1 from the exponent field; means below 2^-900 count as 0
      int ex = max(-900, mx > 0.0 ? (int)((__double_as_longlong(mx) >> 52) & 0x7ff) - 1022 : 0);
      if (__double2ll_rn(mx * __longlong_as_double((int64_t)(1023 + 39 - ex) << 52)) > (127ll << 32)) ++ex;
      if (r0 == 0) {
        int8_t* dst = (isK ? so.ks : so.qs) + ((bh * kScoreSlices) * m.nb + blk) * (int64_t)kSliceRow + c * VEC;
        const double sc = __longlong_as_double((int64_t)(1023 + 39 - ex) << 52);   // 2^(39-ex)
        long long n[VEC];
#pragma unroll
        for (int e = 0; e < VEC; ++e) n[e] = __double2ll_rn(r[e] * sc);
#pragma unroll
        for (int a = kScoreSlices - 1; a >= 0; --a) {          // digits from the bottom
          uint32_t word[VEC / 4];
#pragma unroll
          for (int w = 0; w < VEC / 4; ++w) {
            word[w] = 0;
#pragma unroll
            for (int b = 0; b < 4; ++b) {
              long long& x = n[4 * w + b];
              const long long dgt = a > 0 ? ((x + 128) & 255) - 128 : x;
              x = (x - dgt) >> 8;
              word[w] |= ((uint32_t)dgt & 0xffu) << (8 * b);
            }
          }
          int8_t* d = dst + (int64_t)a * m.nb * kSliceRow;
          if (VEC == 8) *reinterpret_cast<uint2*>(d) = make_uint2(word[0], word[VEC / 4 - 1]);
          else *reinterpret_cast<uint32_t*>(d) = word[0];
          if (D < kSliceRow) {                                    // zero upper half (d = 64)
            if (VEC == 8) *reinterpret_cast<uint2*>(d + D) = make_uint2(0u, 0u);
            else *reinterpret_cast<uint32_t*>(d + D) = 0u;
          }
        }
        if (c == 0) (isK ? so.ek : so.eq)[row] = ex;
      }
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

// ------------------------------------------------------------------ forced blocks

// Up to four inclusive block ranges that every row of query block i keeps: the diagonal,
// the band |i-j| <= w, the frames within +-fw of the block's frames, frame 0. An empty
// range has a > b.
__device__ __forceinline__ void forced_ranges(int i, const Dims& m, const ForceCfg& fc, int (&a)[4],
                                              int (&b)[4]) {
#pragma unroll
  for (int r = 0; r < 4; ++r) { a[r] = 1; b[r] = 0; }
  if (fc.force_diag) { a[0] = i; b[0] = i; }
  if (fc.local_window > 0) {
    a[1] = max(0, i - fc.local_window);
    b[1] = min(m.nb - 1, i + fc.local_window);
  }
  if (fc.frame_len > 0) {
    const int64_t fl = fc.frame_len;
    if (fc.frame_window >= 0) {
      const int64_t t0 = (int64_t)i * kBlock, t1 = min(m.S, t0 + kBlock) - 1;
      const int64_t f0 = imax<int64_t>(0, t0 / fl - fc.frame_window);
      const int64_t f1 = imin<int64_t>(m.F - 1, t1 / fl + fc.frame_window);
      a[2] = (int)(f0 * fl / kBlock);
      b[2] = (int)((min(m.S, (f1 + 1) * fl) - 1) / kBlock);
    }
    if (fc.force_first) { a[3] = 0; b[3] = (int)((min(m.S, fl) - 1) / kBlock); }
  }
}

// OR the forced ranges into the row's bitmask (shared memory), store it and its count.
__device__ __forceinline__ int finalize_row(uint32_t* w, int i, const Dims& m, const ForceCfg& fc, int lane,
                                            uint32_t* __restrict__ gbits, int32_t* __restrict__ gcount) {
  int a[4], b[4];
  forced_ranges(i, m, fc, a, b);
  int cnt = 0;
  for (int q = lane; q < m.nw; q += 32) {
    uint32_t x = w[q];
#pragma unroll
    for (int r = 0; r < 4; ++r) x |= range_bits(a[r], b[r], q);
    x &= range_bits(0, m.nb - 1, q);
    w[q] = x;
    gbits[q] = x;
    cnt += __popc(x);
  }
  cnt = warp_sum(cnt);
  if (lane == 0) *gcount = cnt;
  __syncwarp();
  return cnt;
}

// ------------------------------------------------------------------ K2: Top-p

constexpr int NWARP = 8;
constexpr int kExtract = 16;   // max-extraction steps before the bisection fallback

// Order key of a probability weight: the bits of its fp32 rounding (non-negative floats order
// like their bit patterns).
__device__ __forceinline__ uint32_t wkey(double e) { return __float_as_uint(__double2float_rn(e)); }

__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Top-p cut of one row held in shared memory (one warp). On entry E[0..n) are fp64 logits;
// they are replaced by the weights e_j = 2^((s_j - max) log2 e), computed with the SFU on the
// fp64 difference (relative error < 3e-7), and the cut compares masses with p * sum(e), so no
// division is needed. The kept set is the descending prefix (ties: lower index first) of
// minimal length whose mass reaches p. It is found by extracting maxima (REDUX on the fp32
// order key, lowest index on ties) until the mass reaches p, which ends within a few steps
// for peaked rows; flat rows fall back to a bisection over the 32-bit key space for the
// largest key T with mass{key >= T} >= p, keeping every key > T and, in ascending index, as
// many keys == T as the mass needs. All sums are fp64 in a fixed order: the result is
// deterministic. Writes the row's bitmask words w[0..nw).
__device__ void topp_select(double* E, int n, double p, uint32_t* w, int lane) {
  const int nw = (n + 31) / 32;
  if (p >= 1.0) {
    for (int q = lane; q < nw; q += 32) w[q] = range_bits(0, n - 1, q);
    __syncwarp();
    return;
  }
  double mx = -INFINITY;
  for (int j = lane; j < n; j += 32) mx = fmax(mx, E[j]);
  mx = warp_max(mx);
  double z = 0.0;
  for (int j = lane; j < n; j += 32) {
    float ef;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(ef) : "f"((float)((E[j] - mx) * 1.4426950408889634)));
    E[j] = (double)ef;
    z += (double)ef;
  }
  z = warp_sum_d(z);
  const double P = p * z;
  __syncwarp();

  // Max extraction. Each lane keeps the best (key, slot) of its unselected elements. The
  // selected elements are marked in the row's bitmask words themselves (element lane + 32 e is
  // bit `lane` of w[e]), so rows of any length are covered; only the lane that owns an element
  // ever sets its bit.
  for (int q = lane; q < nw; q += 32) w[q] = 0u;
  __syncwarp();
  uint32_t bkey = 0;
  int bslot = -1;
  auto rescan = [&]() {
    bkey = 0;
    bslot = -1;
    for (int e = 0; e < nw; ++e) {
      const int j = lane + 32 * e;
      if (j < n && !((w[e] >> lane) & 1u)) {
        const uint32_t k = wkey(E[j]);
        if (bslot < 0 || k > bkey) { bkey = k; bslot = e; }
      }
    }
  };
  rescan();
  double acc = 0.0;
  bool done = false;
  for (int it = 0; it < kExtract && !done; ++it) {
    const uint32_t gk = __reduce_max_sync(0xffffffffu, bslot >= 0 ? bkey : 0u);
    const uint32_t cand = (bslot >= 0 && bkey == gk) ? (uint32_t)(lane + 32 * bslot) : 0xffffffffu;
    const uint32_t gj = __reduce_min_sync(0xffffffffu, cand);
    if (gj == 0xffffffffu) break;
    acc += E[gj];
    if ((int)(gj & 31) == lane) {
      atomicOr(&w[gj >> 5], 1u << lane);
      rescan();
    }
    __syncwarp();
    done = acc >= P;
  }
  if (done) return;                          // w holds exactly the extracted elements
  // Bisection: largest T with mass{key >= T} >= P. M(0) = z >= P; keys are below 2^31.
  uint32_t lo = 0, hi = 0x7f800001u;
  while (hi - lo > 1) {
    const uint32_t mid = lo + ((hi - lo) >> 1);
    double s = 0.0;
    for (int j = lane; j < n; j += 32)
      if (wkey(E[j]) >= mid) s += E[j];
    s = warp_sum_d(s);
    if (s >= P) lo = mid;
    else hi = mid;
  }
  const uint32_t T = lo;
  double above = 0.0;
  for (int j = lane; j < n; j += 32)
    if (wkey(E[j]) > T) above += E[j];
  above = warp_sum_d(above);
  for (int e = 0; e < nw; ++e) {
    const int j = lane + 32 * e;
    const uint32_t k = j < n ? wkey(E[j]) : 0u;
    uint32_t word = __ballot_sync(0xffffffffu, j < n && k > T);
    uint32_t ties = __ballot_sync(0xffffffffu, j < n && k == T);
    while (ties != 0u && above < P) {           // ties at the cut, lowest index first
      const int b = __ffs(ties) - 1;
      ties &= ties - 1;
      above += E[32 * e + b];
      word |= 1u << b;
    }
    if (lane == 0) w[e] = word;
  }
  __syncwarp();
}

size_t logits_elems(const Dims& m) { return (size_t)m.BH * m.nb * means_ld(m.nb); }

constexpr int SEL_WARPS = 4;

// Pairwise (fixed-order) sum of the lane's masked weights, as fp64: at most log2(NE) + 1
// roundings of fp32 relative error each.
template <int NE>
__device__ __forceinline__ double lane_sum(const float (&e)[NE], const uint32_t (&k)[NE], uint32_t lo_key,
                                           bool strict) {
  float t[NE];
#pragma unroll
  for (int i = 0; i < NE; ++i) t[i] = (strict ? k[i] > lo_key : k[i] >= lo_key) ? e[i] : 0.f;
#pragma unroll
  for (int w = 1; w < NE; w <<= 1)
#pragma unroll
    for (int i = 0; i + w < NE; i += 2 * w) t[i] += t[i + w];
  return (double)t[0];
}

// The Top-p cut of one row with its weights in registers (NE per lane, element j = lane + 32 i),
// the same rule as topp_select: weights e_j = 2^((s_j - max) log2 e) from the SFU on fp64
// logit differences, masses compared with p * sum(e). Both ways below find the cut key T (the
// fp32 key = the weight's bits) and the mass above it; the row then keeps every key > T and, in
// ascending index, as many keys == T as the mass needs. Peaked rows peel key values from the
// top (REDUX max over the lanes' largest remaining keys, all copies of a value at once) until
// the mass reaches p; rows with more than kExtract weights above 1/64, or not done after
// kExtract values, take a bisection over the 32-bit key space. Lane sums are pairwise in fp32
// and folded across the warp in fp64 in a fixed order (deterministic).
template <int NE>
__device__ void topp_select_reg(const double* __restrict__ src, int n, double p, uint32_t* w, int lane) {
  const int nw = (n + 31) / 32;
  if (p >= 1.0) {
    for (int q = lane; q < nw; q += 32) w[q] = range_bits(0, n - 1, q);
    __syncwarp();
    return;
  }
  double s[NE];                              // the row's logits, loaded once
#pragma unroll
  for (int i = 0; i < NE; ++i) {
    const int j = lane + 32 * i;
    s[i] = j < n ? __ldg(src + j) : -INFINITY;
  }
  double mx = -INFINITY;
#pragma unroll
  for (int i = 0; i < NE; ++i) mx = fmax(mx, s[i]);
  mx = warp_max(mx);
  float e[NE];
  uint32_t k[NE];
  int big = 0;
#pragma unroll
  for (int i = 0; i < NE; ++i) {
    const int j = lane + 32 * i;
    float v = 0.f;
    if (j < n) asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(v) : "f"((float)((s[i] - mx) * 1.4426950408889634)));
    e[i] = v;
    k[i] = __float_as_uint(v);
    big += v > 0.015625f;
  }
  const double z = warp_sum_d(lane_sum(e, k, 0u, false));
  const double P = p * z;
  big = warp_sum(big);

  // T: the key of the cut; above: the mass of the keys > T.
  uint32_t T = 0;
  double above = 0.0;
  bool done = false;
  if (big <= kExtract) {
    // Peel the largest remaining key value, with all its copies, until the mass reaches P. Each
    // lane keeps a copy of its keys with the peeled ones zeroed and their maximum.
    uint32_t kx[NE];
    uint32_t lmax = 0;
#pragma unroll
    for (int i = 0; i < NE; ++i) {
      kx[i] = k[i];
      lmax = max(lmax, k[i]);
    }
    double acc = 0.0;
    for (int it = 0; it < kExtract; ++it) {
      const uint32_t gk = __reduce_max_sync(0xffffffffu, lmax);
      if (gk == 0u) break;                       // only zero weights left
      int cnt = 0;
      if (lmax == gk) {
        uint32_t nm = 0;
#pragma unroll
        for (int i = 0; i < NE; ++i) {
          const bool eq = kx[i] == gk;
          cnt += eq;
          kx[i] = eq ? 0u : kx[i];
          nm = max(nm, kx[i]);
        }
        lmax = nm;
      }
      cnt = __reduce_add_sync(0xffffffffu, cnt);
      above = acc;
      acc += (double)cnt * (double)__uint_as_float(gk);
      if (acc >= P) {
        T = gk;
        done = true;
        break;
      }
    }
  }
  if (!done) {
    // Bisection: largest T with mass{key >= T} >= P. Weights are at most 1, so keys <= 0x3f800000.
    uint32_t lo = 0, hi = 0x3f800001u;
    while (hi - lo > 1) {
      const uint32_t mid = lo + ((hi - lo) >> 1);
      const double sm = warp_sum_d(lane_sum(e, k, mid, false));
      if (sm >= P) lo = mid;
      else hi = mid;
    }
    T = lo;
    above = warp_sum_d(lane_sum(e, k, T, true));
  }
  const double tval = (double)__uint_as_float(T);
#pragma unroll
  for (int i = 0; i < NE; ++i) {
    const bool valid = lane + 32 * i < n;
    uint32_t word = __ballot_sync(0xffffffffu, valid && k[i] > T);
    uint32_t ties = __ballot_sync(0xffffffffu, valid && k[i] == T);
    while (ties != 0u && above < P) {           // ties at the cut, lowest index first
      const int b = __ffs(ties) - 1;
      ties &= ties - 1;
      above += tval;
      word |= 1u << b;
    }
    if (lane == 0 && i < nw) w[i] = word;
  }
  __syncwarp();
}

// The kk highest scores of one row (the notes' teaching variant, §5.2: scores.topk), ties to
// the lower block index. The order key of a block is its fp32 score relative to the row
// maximum (s_j - max <= 0) mapped to an unsigned integer that orders like the float; the cut
// is the largest key T with count{key >= T} >= kk, found by bisection, then every key > T and,
// in ascending index, as many keys == T as are needed for kk.
// With `cand` (ceil(n/32) words, shared memory) only the blocks whose bit is set take part, and
// w receives the chosen candidates only; kk must not exceed their number.
template <int NE>
__device__ void topk_select_reg(const double* __restrict__ src, int n, int kk, uint32_t* w, int lane,
                                const uint32_t* cand = nullptr) {
  const int nw = (n + 31) / 32;
  int ncand = n;
  if (cand != nullptr) {
    ncand = 0;
    for (int q = lane; q < nw; q += 32) ncand += __popc(cand[q]);
    ncand = warp_sum(ncand);
  }
  if (kk >= ncand) {
    for (int q = lane; q < nw; q += 32) w[q] = cand != nullptr ? cand[q] : range_bits(0, n - 1, q);
    __syncwarp();
    return;
  }
  double s[NE];
  bool in[NE];
#pragma unroll
  for (int i = 0; i < NE; ++i) {
    const int j = lane + 32 * i;
    s[i] = j < n ? __ldg(src + j) : -INFINITY;
    in[i] = j < n && (cand == nullptr || ((cand[i] >> lane) & 1u));
  }
  double mx = -INFINITY;
#pragma unroll
  for (int i = 0; i < NE; ++i) mx = fmax(mx, s[i]);
  mx = warp_max(mx);
  uint32_t k[NE];
#pragma unroll
  for (int i = 0; i < NE; ++i) {
    const uint32_t b = __float_as_uint((float)(s[i] - mx));
    k[i] = in[i] ? ((b & 0x80000000u) ? ~b : (b | 0x80000000u)) : 0u;
  }
  auto count_ge = [&](uint32_t t, bool strict) {
    int c = 0;
#pragma unroll
    for (int i = 0; i < NE; ++i) c += in[i] && (strict ? k[i] > t : k[i] >= t);
    return warp_sum(c);
  };
  // Bracket: count{key >= min} = every candidate >= kk, count{key >= max + 1} = 0 < kk. The search
  // stops early once exactly kk keys are >= mid: that set is the answer (every key above the
  // final cut plus all its ties).
  uint32_t kmin = 0xffffffffu, kmax = 0u;
#pragma unroll
  for (int i = 0; i < NE; ++i)
    if (in[i]) {
      kmin = min(kmin, k[i]);
      kmax = max(kmax, k[i]);
    }
  uint32_t lo = __reduce_min_sync(0xffffffffu, kmin);
  uint64_t hi = (uint64_t)__reduce_max_sync(0xffffffffu, kmax) + 1;
  while (hi - lo > 1) {
    const uint32_t mid = (uint32_t)(lo + ((hi - lo) >> 1));
    const int c = count_ge(mid, false);
    if (c >= kk) lo = mid;
    else hi = mid;
    if (c == kk) break;
  }
  const uint32_t T = lo;
  int have = count_ge(T, true);
#pragma unroll
  for (int i = 0; i < NE; ++i) {
    uint32_t word = __ballot_sync(0xffffffffu, in[i] && k[i] > T);
    uint32_t ties = __ballot_sync(0xffffffffu, in[i] && k[i] == T);
    while (ties != 0u && have < kk) {
      const int b = __ffs(ties) - 1;
      ties &= ties - 1;
      ++have;
      word |= 1u << b;
    }
    if (lane == 0 && i < nw) w[i] = word;
  }
  __syncwarp();
}

template <int NE>
size_t select_smem_bytes_t(const Dims& m) {
  return NE > 0 ? (size_t)3 * SEL_WARPS * m.nw * 4
                : (size_t)SEL_WARPS * m.nw * 32 * 8 + (size_t)SEL_WARPS * m.nw * 4;
}

// Slack-aware augmentation of one row (FVAttn summary, section "SASA", applied to the 128-row
// tile): the row and its partner i^1 (same tile, the neighbouring warp) step through the union
// of their key blocks together; the row's slack is the union blocks it did not select, and
// when the slack reaches the trigger it gains the floor(coef * slack) best of them in its own
// routing order (the same fp32 order key as the top-k cut, ties to the lower block). Reads the
// pre-augmentation rows in shared memory, writes the row's bitmask and count to global memory.
template <int NE>
__device__ void sasa_row(const double* __restrict__ src, const Dims& m, const SasaCfg& sasa, const uint32_t* ws,
                         const uint32_t* wp, uint32_t* wc, uint32_t* wo, int lane, uint32_t* __restrict__ gbits,
                         int32_t* __restrict__ gcount) {
  int slack = 0, own = 0;
  for (int q = lane; q < m.nw; q += 32) {
    const uint32_t c = wp[q] & ~ws[q];
    wc[q] = c;
    slack += __popc(c);
    own += __popc(ws[q]);
  }
  slack = warp_sum(slack);
  own = warp_sum(own);
  __syncwarp();
  if (slack <= 0 || slack < sasa.trigger) return;
  const int kk = (int)floor((double)sasa.coef * (double)slack);
  if (kk <= 0) return;
  topk_select_reg<NE>(src, m.nb, kk, wo, lane, wc);
  for (int q = lane; q < m.nw; q += 32) gbits[q] = ws[q] | wo[q];
  if (lane == 0) *gcount = own + kk;
}

// One warp per query block: the Top-p cut of its fp64 logit row (in registers when the row
// has at most 32 NE blocks, else through shared memory), forced blocks, bitmask row and count;
// warps 2w and 2w+1 hold the two rows of a 128-row tile and write its cost, then (register
// path, sasa.coef > 0) augment each other's slack.
template <int NE>
__global__ void __launch_bounds__(SEL_WARPS * 32) select_kernel(const double* __restrict__ logits, Dims m, double p,
                                                     int kblocks, ForceCfg fc, SasaCfg sasa,
                                                     uint32_t* __restrict__ bits, int32_t* __restrict__ counts,
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
    if (NE > 0) {
      if (kblocks > 0) topk_select_reg<(NE > 0 ? NE : 1)>(src, m.nb, kblocks, w, lane);
      else topp_select_reg<(NE > 0 ? NE : 1)>(src, m.nb, p, w, lane);
    } else {
      double* E = sE + (size_t)warp * nbp;
      for (int j = lane; j < m.nb; j += 32) E[j] = src[j];
      __syncwarp();
      topp_select(E, m.nb, p, w, lane);
    }
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
  if constexpr (NE > 0) {
    if (sasa.coef > 0.f && i < m.nb && (i ^ 1) < m.nb) {
      // the rows of this CTA's tiles are final in sW; augmentation writes only wc/wo and global
      uint32_t* wc = sW + (size_t)SEL_WARPS * m.nw + (size_t)warp * m.nw;
      uint32_t* wo = sW + (size_t)2 * SEL_WARPS * m.nw + (size_t)warp * m.nw;
      const int64_t grow = bh * m.nb + i;
      sasa_row<NE>(logits + grow * (int64_t)ld, m, sasa, w, sW + (warp ^ 1) * m.nw, wc, wo, lane,
                   bits + grow * m.nw, counts + grow);
    }
  }
}

template <int NE>
static cudaError_t launch_select_t(const double* logits, const Dims& m, double p, int kblocks, const ForceCfg& fc,
                                   const SasaCfg& sasa, uint32_t* bits, int32_t* counts, int32_t* tile_cost,
                                   cudaStream_t st) {
  const size_t smem = select_smem_bytes_t<NE>(m) + 16;
  cudaError_t e = cudaFuncSetAttribute(select_kernel<NE>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 g((m.nb + SEL_WARPS - 1) / SEL_WARPS, (unsigned)m.BH);
  select_kernel<NE><<<g, SEL_WARPS * 32, smem, st>>>(logits, m, p, kblocks, fc, sasa, bits, counts, tile_cost);
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
    int64_t base = row_ptr[row];
    for (int q0 = 0; q0 < m.nw; q0 += 32) {
      const int q = q0 + lane;
      uint32_t x = q < m.nw ? w[q] : 0u;
      const int c = __popc(x);
      const int incl = warp_incl_scan(c, lane);
      int64_t pos = base + incl - c;
      while (x) {
        const int b = __ffs(x) - 1;
        x &= x - 1;
        col_idx[pos++] = q * 32 + b;
      }
      base += __shfl_sync(0xffffffffu, incl, 31);
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
  if (m.nb <= 32 * 16) return launch_select_t<16>(logits, m, p, kblocks, fc, sasa, bits, counts, tile_cost, st);
  if (m.nb <= 32 * 40) return launch_select_t<40>(logits, m, p, kblocks, fc, sasa, bits, counts, tile_cost, st);
  return launch_select_t<0>(logits, m, p, 0, fc, SasaCfg{0.f, 0}, bits, counts, tile_cost, st);
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
