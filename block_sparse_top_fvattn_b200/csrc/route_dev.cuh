// Device helpers of the router kernels (route.cu): warp
// reductions, bf16 / fp32 unpacking, forced blocks, the Top-p and top-k cuts of one row and the
// slack-aware augmentation of a row.
//
// Method: FVAttn blog summary ("腾讯+中山大学新作：视频生成提速2.11×，靠的是RLB和SASA"), section
// "AI视频生成的阿喀琉斯之踵" (Top-p: smallest descending-importance prefix reaching p) and
// section "SASA" (slack filled with the best unselected blocks); video-generation acceleration
// notes (wzjinhao.cn) §5.2 (fixed top-k, local band); vLLM-Omni Sol-Attn article §2.2 (frames
// kept around the query's frames and the first frame).
#pragma once

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

// The block mean lo[e] * (1 / nvalid) of the lane's VEC columns (c * VEC ...), as a power-of-two scale
// 2^ex and kScoreSlices signed 8-bit digits: with N = rint(x 2^(39-ex)),
// N = X_0 2^32 + X_1 2^24 + X_2 2^16 + X_3 2^8 + X_4, i.e. x ~ 2^ex sum_a X_a 2^(-7-8a).
// X_4..X_1 are the balanced base-256 digits (in [-128, 127], taken from the bottom), X_0 the
// rest. ex is the smallest power of two above max|x| over the block's d columns, raised by one
// when max|N| > 127 * 2^32, so that X_0 stays in [-128, 127] too. Called by the whole warp (the
// maximum is folded over all lanes); lanes with r0 == 0 write their columns of the kScoreSlices
// rows at dst + a * plane (rows of kSliceRow bytes, upper half zeroed for d = 64) and lane 0 the
// exponent.
template <int D, int VEC>
__device__ __forceinline__ void slice_mean(const double (&lo)[VEC], int nvalid, int r0, int c, int8_t* dst,
                                           int64_t plane, int32_t* eout) {
  // one division per lane: the mean is lo * (1 / nvalid) (exact for a full block of 64 tokens)
  const double inv = 1.0 / (double)nvalid;
  double r[VEC], mx = 0.0;
#pragma unroll
  for (int e = 0; e < VEC; ++e) {
    r[e] = lo[e] * inv;
    mx = fmax(mx, fabs(r[e]));
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) mx = fmax(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  // ex = floor(log2(mx)) + 1 from the exponent field; means below 2^-900 count as 0
  int ex = max(-900, mx > 0.0 ? (int)((__double_as_longlong(mx) >> 52) & 0x7ff) - 1022 : 0);
  if (__double2ll_rn(mx * __longlong_as_double((int64_t)(1023 + 39 - ex) << 52)) > (127ll << 32)) ++ex;
  if (r0 == 0) {
    int8_t* base = dst + c * VEC;
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
      int8_t* d = base + (int64_t)a * plane;
      if (VEC == 8) *reinterpret_cast<uint2*>(d) = make_uint2(word[0], word[VEC / 4 - 1]);
      else *reinterpret_cast<uint32_t*>(d) = word[0];
      if (D < kSliceRow) {                                    // zero upper half (d = 64)
        if (VEC == 8) *reinterpret_cast<uint2*>(d + D) = make_uint2(0u, 0u);
        else *reinterpret_cast<uint32_t*>(d + D) = 0u;
      }
    }
    if (c == 0) *eout = ex;
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
__device__ inline void topp_select(double* E, int n, double p, uint32_t* w, int lane) {
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

// lane_sum(e, k, lo_key, false) and, in `cnt`, the number of the lane's keys >= lo_key.
template <int NE>
__device__ __forceinline__ double lane_sum_count(const float (&e)[NE], const uint32_t (&k)[NE], uint32_t lo_key,
                                                 int& cnt) {
  int c = 0;
#pragma unroll
  for (int i = 0; i < NE; ++i) c += k[i] >= lo_key;
  cnt = c;
  return lane_sum(e, k, lo_key, false);
}

// The Top-p cut of one row with its weights in registers (NE per lane, element j = lane + 32 i),
// the same rule as topp_select: weights e_j = 2^((s_j - max) log2 e) from the SFU on fp64
// logit differences, masses compared with p * sum(e). Both ways below find the cut key T (the
// fp32 key = the weight's bits) and the mass above it; the row then keeps every key > T and, in
// ascending index, as many keys == T as the mass needs. Peaked rows peel key values from the
// top (REDUX max over the lanes' largest remaining keys, all copies of a value at once) until
// the mass reaches p; rows with more than kExtract weights above 1/64, or not done after
// kExtract values, take a bisection over the 32-bit key space, which stops as soon as a single
// key is left in its bracket (the cut is always one of the row's keys, so that key is the one
// the full bisection would reach). Lane sums are pairwise in fp32 and folded across the warp in
// fp64 in a fixed order (deterministic).
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
    s[i] = j < n ? __ldcg(src + j) : -INFINITY;
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
    // Bisection: largest T with mass{key >= T} >= P. Weights are at most 1, so keys <= 0x3f800000;
    // the bracket starts at the smallest key of the row (its mass is the whole row's). cl / ch
    // count the keys >= lo / >= hi (elements past n have key 0); [lo, hi) always holds a key.
    uint32_t kmin = 0xffffffffu;
#pragma unroll
    for (int i = 0; i < NE; ++i)
      if (lane + 32 * i < n) kmin = min(kmin, k[i]);
    uint32_t lo = __reduce_min_sync(0xffffffffu, kmin), hi = 0x3f800001u;
    int cl = lo > 0u ? n : 32 * NE, ch = 0;
    while (hi - lo > 1 && cl - ch > 1) {
      const uint32_t mid = lo + ((hi - lo) >> 1);
      int c;
      const double sm = warp_sum_d(lane_sum_count(e, k, mid, c));
      c = __reduce_add_sync(0xffffffffu, c);
      if (sm >= P) {
        lo = mid;
        cl = c;
      } else {
        hi = mid;
        ch = c;
      }
    }
    if (cl - ch == 1) {
      // one key in [lo, hi): mass{key >= it} = mass{key >= lo} >= P, every larger key is >= hi
      uint32_t km = 0u;
#pragma unroll
      for (int i = 0; i < NE; ++i) km = max(km, k[i] < hi ? k[i] : 0u);
      T = __reduce_max_sync(0xffffffffu, km);
    } else {
      T = lo;
    }
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
    s[i] = j < n ? __ldcg(src + j) : -INFINITY;
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

}  // namespace fv
