// Block-sparse flash attention on the B200 tensor cores (tcgen05, TMEM, TMA), bf16 inputs,
// fp32 accumulation.
//
// What it computes (FVAttn blog summary, section "AI视频生成的阿喀琉斯之踵"; the masked
// attention of the wzjinhao.cn notes §5.2): for every query token, exact softmax attention
// over the tokens (< S) of the key blocks that the router kept for its query block.
//
// How: a persistent CTA per SM takes 128-row query tiles (query blocks 2t and 2t+1 of one
// head) in the router's longest-first order. A tile walks the ascending union of its two
// block lists; for each key block j:
//   S = Q K_j^T          tcgen05.mma M=128 N=64 K=d, A and B K-major from shared memory,
//                        fp32 accumulator in TMEM (double-buffered)
//   P = exp2(S*c - m)    one thread per row reads its TMEM lane, masks the half-tile whose
//                        list lacks j and the keys >= S, keeps a running max m that is only
//                        raised (with a rescale of O in TMEM) when it grows by more than
//                        2^8, and writes P as bf16 pairs over its S buffer in TMEM
//   O += P V_j           tcgen05.mma M=128 N=d K=64, A = P read from TMEM, V MN-major, O
//                        accumulated in TMEM
// Warp roles: warp 0 issues TMA loads (lane 0: Q once per tile and K_j, lane 1: V_j, each into
// its own 2-stage ring, so a K stage is reloaded as soon as its S MMA is done),
// warp 1 allocates TMEM and issues the MMAs, warps 2-5 do softmax and the epilogue.
// Every mbarrier wait of the MMA-issuing thread stalls its MMA stream for a few hundred cycles
// even when the phase is already complete (measured), so that thread waits only twice per step:
// once for K_j (whose barrier also publishes the step record) and once for P_j together with
// V_j (one barrier); coincident events share one barrier and one commit.
// Every mbarrier wait is bounded; a wait that runs out sets an abort flag and every role
// unwinds: the loaders wait (bounded) for the copies they issued, the MMA thread for its MMAs,
// TMEM is freed and FVATTN_ERR_TIMEOUT is written to the device status word. With hold_polls > 0
// (failure-path check only) the scheduler first waits on a barrier that nothing completes.
#include <cuda.h>
#include <math.h>

#include "common.cuh"
#include "route.cuh"
#include "tc_ptx.cuh"
#include "tmap.cuh"

namespace fv {

namespace {

constexpr int NS = 2;                        // K/V pipeline stages (two CTAs share an SM)
static_assert(NS == 2, "the stage of a step doubles as its S / P buffer index");
constexpr uint32_t kWaitLimit = 1u << 22;    // polls of a bounded wait (seconds, not minutes)
constexpr float kRescaleLog2 = 8.0f;         // raise the running max only when it grows by > 2^8

template <int D>
struct TcLayout {
  static constexpr int kQChunk = kTileRows * 128;     // [128 rows x 64 dims] bf16 = 16 KB
  static constexpr int kQBytes = (D / 64) * kQChunk;
  static constexpr int kKVChunk = kBlock * 128;       // [64 rows x 64 dims] bf16 = 8 KB
  static constexpr int kKBytes = (D / 64) * kKVChunk; // one K_j (or V_j) block
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kQBytes;               // NS stages of K
  static constexpr int kOffV = kOffK + NS * kKBytes;  // NS stages of V
  static constexpr int kOffBar = kOffV + NS * kKBytes;
  static constexpr int kBytes = kOffBar + 512;
  // TMEM: S double buffer at columns 0 and 64 (P, bf16, overwrites the first 32 columns of its
  // S buffer), O at column 128.
  static constexpr uint32_t kTmemCols = 256;
  static constexpr uint32_t kColO = 128;
};

constexpr int NI = 8;        // step records in flight

struct TcBars {
  uint64_t q_full, q_empty;
  uint64_t k_full[NS];
  // With NS == 2 the K/V stage and the S buffer of a step have the same index b = step & 1, so
  // one barrier serves each pair of events that happen together:
  //   s_full[b]:  S of the step done (softmax may read it; its K stage may be refilled)
  //   p_full[b]:  P written by the four softmax warps AND V landed (the V loader's
  //               arrive.expect_tx is the fifth arrival)
  //   pv_done[b]: P.V done (O is stable; the V stage may be refilled)
  uint64_t s_full[2], p_full[2], pv_done[2];
  uint64_t o_full, o_empty;
  uint64_t sched_full[2], sched_empty[2];
  uint64_t info_full[NI];
  uint64_t hold;              // completed by nothing: the failure-path check waits on it
  uint64_t drain;             // MMA drain: every MMA of the CTA has completed
  int p_arrived[4];           // per softmax warp: the last step whose P it published
  int v_armed;                // the last step whose V load was issued
  int sched_tile[2];
  int step_info[NI];          // key block j | membership mask << 28 | last step of tile << 30
  int step_code[NI];          // token mask of the step: allow bits of block 2t (0-3) and 2t+1 (4-7),
                              // key-frame boundary column (8-15), query-frame boundary rows (16-23,
                              // 24-31); see fvattn_csr.col_code
  uint32_t tmem_base;
  int abort;
};

// Ascending union of the key-block lists of query blocks 2t and 2t+1 of one head, with a
// 2-bit membership mask (bit 0: block 2t keeps j, bit 1: block 2t+1 keeps j).
struct PairMerge {
  const int32_t* ci;
  int a, ae, b, be;
  __device__ PairMerge(const int32_t* row_ptr, const int32_t* col_idx, int64_t bh, int t, int nb) {
    ci = col_idx;
    const int64_t r0 = bh * nb + 2 * t;
    a = row_ptr[r0];
    ae = row_ptr[r0 + 1];
    if (2 * t + 1 < nb) {
      b = ae;
      be = row_ptr[r0 + 2];
    } else {
      b = be = 0;
    }
  }
  __device__ __forceinline__ bool more() const { return a < ae || b < be; }
  // ea / eb: the entry of j in the two lists (-1 where the list lacks j).
  __device__ __forceinline__ bool next(int& j, int& mask, int& ea, int& eb) {
    if (a >= ae && b >= be) return false;
    const int ja = a < ae ? ci[a] : 0x7fffffff;
    const int jb = b < be ? ci[b] : 0x7fffffff;
    j = min(ja, jb);
    mask = (ja == j ? 1 : 0) | (jb == j ? 2 : 0);
    ea = ja == j ? a : -1;
    eb = jb == j ? b : -1;
    a += (ja == j);
    b += (jb == j);
    return true;
  }
};

__device__ __forceinline__ void fail(TcBars* bars, int code) {
  atomicCAS(&bars->abort, 0, code);
}

// A bounded wait taken by a whole warp with one outcome for all lanes.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, const volatile int* abort) {
  const bool ok = tc::mbar_wait(bar, parity, abort, kWaitLimit);
  return __all_sync(0xffffffffu, ok);
}

// 2^x by the SFU's ex2.approx instruction (flush-to-zero; 2^-inf = 0).
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Packed pairs of fp32 (one 64-bit register): two FMAs / adds per instruction.
__device__ __forceinline__ uint64_t f2(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void f2_split(uint64_t v, float& a, float& b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
}
__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t fadd2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

__device__ __forceinline__ float max3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

template <int D>
__global__ void __launch_bounds__(192, 2)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, Dims m, float scale_log2,
                   const int32_t* __restrict__ row_ptr, const int32_t* __restrict__ col_idx, int64_t col_cap,
                   const int32_t* __restrict__ col_code, const int32_t* __restrict__ tile_order,
                   int32_t* __restrict__ control, __nv_bfloat16* __restrict__ O, float* __restrict__ lse,
                   uint64_t* __restrict__ stamps, uint32_t hold_polls) {
  using L = TcLayout<D>;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  TcBars* bars = reinterpret_cast<TcBars*>(smem + L::kOffBar);
  unsigned char* sQ = smem + L::kOffQ;
  unsigned char* sK = smem + L::kOffK;
  unsigned char* sV = smem + L::kOffV;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t ntiles = m.BH * m.nt;
  volatile int* abort = &bars->abort;

  if (threadIdx.x == 0) {
    tc::mbar_init(&bars->q_full, 1);
    tc::mbar_init(&bars->q_empty, 1);
    for (int s = 0; s < NS; ++s) {
      tc::mbar_init(&bars->k_full[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(&bars->s_full[s], 1);
      tc::mbar_init(&bars->p_full[s], 5);
      tc::mbar_init(&bars->pv_done[s], 1);
      tc::mbar_init(&bars->sched_full[s], 1);
      tc::mbar_init(&bars->sched_empty[s], 6);    // V loader, MMA thread, four softmax warps
    }
    for (int s = 0; s < NI; ++s) tc::mbar_init(&bars->info_full[s], 1);
    tc::mbar_init(&bars->o_full, 1);
    tc::mbar_init(&bars->o_empty, 4);
    tc::mbar_init(&bars->hold, 1);
    tc::mbar_init(&bars->drain, 1);
    for (int w = 0; w < 4; ++w) bars->p_arrived[w] = -1;
    bars->v_armed = -1;
    bars->abort = 0;
    tc::fence_mbar_init();
  }
  if (warp == 1) {
    tc::tmem_alloc(&bars->tmem_base, L::kTmemCols);
    tc::tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tc::prefetch_tmap(&tmQ);
    tc::prefetch_tmap(&tmK);
    tc::prefetch_tmap(&tmV);
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tbase = bars->tmem_base;
  if (stamps != nullptr && threadIdx.x == 0) {
    uint64_t t_begin;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t_begin));
    stamps[3 * blockIdx.x + 1] = t_begin;
  }

  if (warp == 0) {
    if (lane == 0) {
      // ---------------------------------------------------------- scheduler, Q and K loader
      // Takes the next tile of the longest-first order from the global ticket, publishes it,
      // loads its Q tile, and for every key block of the tile's list publishes a step record
      // and loads K_j. A K stage is refilled as soon as the S MMA that read it is done.
      // The record ring is deep enough that a record is never overwritten before every
      // reader has taken it: record g+NI is written only after S_{g+NI-3} was issued, which
      // follows P_{g+NI-5} of the softmax warps.
      // Entries of the order to process: every tile, or those of the heads kept by
      // fvattn_select_heads (control[3]).
      const int64_t count = imin<int64_t>(ntiles, imax<int64_t>(0, *reinterpret_cast<volatile int32_t*>(&control[3])));
      uint32_t g = 0;
      // parities of the last phases this thread armed (-1: none), waited for before it leaves,
      // so that no copy is still writing shared memory when the CTA exits
      int q_par = -1, k_par[NS] = {-1, -1};
      // failure-path check: a bounded wait on a barrier nothing completes, before any copy
      if (hold_polls > 0 && !tc::mbar_wait(&bars->hold, 0, abort, hold_polls)) fail(bars, 20);
      for (uint32_t n = 0; !*abort; ++n) {
        const int s = n & 1;
        if (!tc::mbar_wait(&bars->sched_empty[s], ((n >> 1) & 1) ^ 1, abort, kWaitLimit)) { fail(bars, 1); break; }
        const int k = atomicAdd(&control[2], 1);
        int tile = -1;
        if (k < count) {
          tile = tile_order[k];
          if (tile < 0 || tile >= ntiles) { fail(bars, 11); tile = -1; }
#ifdef FVATTN_DEBUG
          // debug build: both block lists of the tile are checked before any role reads them
          if (tile >= 0) {
            const int64_t tb = tile / m.nt;
            const int tt = (int)(tile - tb * m.nt);
            int bad = debug_row_check(row_ptr, col_idx, col_cap, tb * m.nb + 2 * tt, m.nb);
            if (!bad && 2 * tt + 1 < m.nb) bad = debug_row_check(row_ptr, col_idx, col_cap, tb * m.nb + 2 * tt + 1, m.nb);
            if (bad) { fail(bars, bad); tile = -1; }
          }
#endif
        }
        bars->sched_tile[s] = tile;
        tc::mbar_arrive(&bars->sched_full[s]);
        if (tile < 0) break;
        const int64_t bh = tile / m.nt;
        const int t = (int)(tile - bh * m.nt);
        if (!tc::mbar_wait(&bars->q_empty, (n & 1) ^ 1, abort, kWaitLimit)) { fail(bars, 2); break; }
        tc::mbar_expect_tx(&bars->q_full, L::kQBytes);
        q_par = n & 1;
        for (int c = 0; c < D / 64; ++c)
          for (int h = 0; h < 2; ++h)
            tc::tma_load_3d(sQ + c * L::kQChunk + h * L::kKVChunk, &tmQ, &bars->q_full, c * 64,
                            t * kTileRows + h * kBlock, (int)bh);
        PairMerge mg(row_ptr, col_idx, bh, t, m.nb);
        int j, mask, ea, eb;
        bool ok = true;
        while (mg.next(j, mask, ea, eb)) {
          bars->step_info[g % NI] = j | (mask << 28) | (mg.more() ? 0 : (1 << 30));
          int code = 0xFF | (kBlock << 8) | (kBlock << 16) | (kBlock << 24);
          if (col_code != nullptr) {
            const int ca = ea >= 0 ? col_code[ea] : kCodeAll;
            const int cb = eb >= 0 ? col_code[eb] : kCodeAll;
            code = (ca & 0xF) | ((cb & 0xF) << 4) | ((((ea >= 0 ? ca : cb) >> 8) & 0xFF) << 8) |
                   (((ca >> 16) & 0xFF) << 16) | (((cb >> 16) & 0xFF) << 24);
          }
          bars->step_code[g % NI] = code;
          tc::mbar_arrive(&bars->info_full[g % NI]);
          const int st = g % NS;
          if (!tc::mbar_wait(&bars->s_full[st], ((g / NS) & 1) ^ 1, abort, kWaitLimit)) { fail(bars, 3); ok = false; break; }
          tc::mbar_expect_tx(&bars->k_full[st], L::kKBytes);
          k_par[st] = (g / NS) & 1;
          for (int c = 0; c < D / 64; ++c)
            tc::tma_load_3d(sK + st * L::kKBytes + c * L::kKVChunk, &tmK, &bars->k_full[st], c * 64, j * kBlock, (int)bh);
          ++g;
        }
        if (!ok) break;
      }
      if (q_par >= 0) tc::mbar_wait_drain(&bars->q_full, (uint32_t)q_par, kWaitLimit);
      for (int st = 0; st < NS; ++st)
        if (k_par[st] >= 0) tc::mbar_wait_drain(&bars->k_full[st], (uint32_t)k_par[st], kWaitLimit);
    } else if (lane == 1) {
      // ---------------------------------------------------------- V loader
      // Loads V_j for the same steps; a V stage is refilled once the P.V that read it is done.
      uint32_t g = 0;
      for (uint32_t n = 0;; ++n) {
        const int s = n & 1;
        if (!tc::mbar_wait(&bars->sched_full[s], (n >> 1) & 1, abort, kWaitLimit)) { fail(bars, 15); break; }
        const int tile = bars->sched_tile[s];
        tc::mbar_arrive(&bars->sched_empty[s]);
        if (tile < 0) break;
        const int64_t bh = tile / m.nt;
        const int t = (int)(tile - bh * m.nt);
        PairMerge mg(row_ptr, col_idx, bh, t, m.nb);
        int j, mask, ea, eb;
        bool ok = true;
        while (mg.next(j, mask, ea, eb)) {
          const int st = g % NS;
          if (!tc::mbar_wait(&bars->pv_done[st], ((g / NS) & 1) ^ 1, abort, kWaitLimit)) { fail(bars, 16); ok = false; break; }
          tc::mbar_expect_tx(&bars->p_full[st], L::kKBytes);
          for (int c = 0; c < D / 64; ++c)
            tc::tma_load_3d(sV + st * L::kKBytes + c * L::kKVChunk, &tmV, &bars->p_full[st], c * 64, j * kBlock, (int)bh);
          *reinterpret_cast<volatile int*>(&bars->v_armed) = (int)g;
          ++g;
        }
        if (!ok) break;
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // Issue order per tile: S_0, [S_1, PV_0], [S_2, PV_1], ..., PV_last. MMAs of one thread run
    // in issue order, so S_{i+2} (same TMEM buffer as S_i / P_i) always follows PV_i.
    if (lane == 0) {
      constexpr uint32_t idS = tc::idesc_bf16_f32(kTileRows, kBlock, 0, 0);
      constexpr uint32_t idO = tc::idesc_bf16_f32(kTileRows, D, 0, 1);
      const uint32_t qaddr = tc::smem_u32(sQ), kaddr0 = tc::smem_u32(sK), vaddr0 = tc::smem_u32(sV);
      uint32_t g = 0, n = 0;
      bool ok = true;
      // O += P_gs V_gs for step gs; `first` = first step of the tile (overwrites O).
      auto pv = [&](uint32_t gs, bool first) -> bool {
        const int pb = gs & 1, st = gs % NS;
        if (!tc::mbar_wait(&bars->p_full[pb], (gs >> 1) & 1, abort, kWaitLimit)) return false;
        if (first && !tc::mbar_wait(&bars->o_empty, (n & 1) ^ 1, abort, kWaitLimit)) return false;
        tc::fence_after_sync();
        const uint32_t vaddr = vaddr0 + st * L::kKBytes;
#pragma unroll
        for (int kk = 0; kk < kBlock / 16; ++kk) {
          const uint64_t b = tc::smem_desc_sw128(vaddr + kk * 16 * 128, L::kKVChunk, 1024);
          tc::mma_f16_tmem_a(tbase + L::kColO, tbase + pb * kBlock + kk * 8, b, idO, (first && kk == 0) ? 0u : 1u);
        }
        tc::mma_commit(&bars->pv_done[pb]);
        return true;
      };
      for (;; ++n) {
        const int s = n & 1;
        if (!tc::mbar_wait(&bars->sched_full[s], (n >> 1) & 1, abort, kWaitLimit)) { fail(bars, 4); ok = false; break; }
        const int tile = bars->sched_tile[s];
        tc::mbar_arrive(&bars->sched_empty[s]);
        if (tile < 0) break;
        if (!tc::mbar_wait(&bars->q_full, n & 1, abort, kWaitLimit)) { fail(bars, 5); ok = false; break; }
        int i = 0;
        for (bool last = false; !last;) {
          const uint32_t gi = g + i;
          const int st = gi % NS, sb = gi & 1;
          // The loader writes the step record before its arrive.expect_tx on k_full (a release),
          // so the record is visible once k_full completes; this thread does not wait on
          // info_full (every mbarrier wait here stalls the MMA stream).
          if (!tc::mbar_wait(&bars->k_full[st], (gi / NS) & 1, abort, kWaitLimit)) {
            fail(bars, 6);
            ok = false;
            break;
          }
          last = (bars->step_info[gi % NI] >> 30) & 1;
          tc::fence_after_sync();
          const uint32_t kaddr = kaddr0 + st * L::kKBytes;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const int c = kk >> 2, off = (kk & 3) * 32;
            const uint64_t a = tc::smem_desc_sw128(qaddr + c * L::kQChunk + off, 16, 1024);
            const uint64_t b = tc::smem_desc_sw128(kaddr + c * L::kKVChunk + off, 16, 1024);
            tc::mma_f16(tbase + sb * kBlock, a, b, idS, kk > 0 ? 1u : 0u);
          }
          tc::mma_commit(&bars->s_full[sb]);        // also frees K stage st (== sb)
          if (i > 0 && !pv(gi - 1, i == 1)) { fail(bars, 7); ok = false; break; }
          ++i;
        }
        if (!ok) break;
        tc::mma_commit(&bars->q_empty);          // every S of this tile issued: Q may be replaced
        if (i > 0 && !pv(g + i - 1, i == 1)) { fail(bars, 8); ok = false; break; }
        tc::mma_commit(&bars->o_full);
        g += i;
      }
      // Drain, on every path: every MMA issued so far has completed before TMEM is released.
      tc::mma_commit(&bars->drain);
      tc::mbar_wait_drain(&bars->drain, 0, kWaitLimit);
    }
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    const int q = warp & 3;                  // TMEM lane quarter this warp may access
    const int r = q * 32 + lane;             // tile row == TMEM lane
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    const int half_bit = (r < kBlock) ? 1 : 2;   // rows 0-63: query block 2t, 64-127: 2t+1
    const uint64_t scale2 = f2(scale_log2, scale_log2);
    uint32_t g = 0;
    for (uint32_t n = 0;; ++n) {
      const int s = n & 1;
      if (!warp_wait(&bars->sched_full[s], (n >> 1) & 1, abort)) { fail(bars, 9); break; }
      const int tile = bars->sched_tile[s];
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&bars->sched_empty[s]);
      if (tile < 0) break;
      const int64_t bh = tile / m.nt;
      const int t = (int)(tile - bh * m.nt);
      float mrow = -INFINITY;
      uint64_t lsum = f2(0.f, 0.f);
      int i = 0;
      bool ok = true;
      for (bool last = false; !last;) {
        const uint32_t gi = g + i;
        const int sb = gi & 1;
        const uint32_t sp = tbase + lane_off + sb * kBlock;     // S_i, then P_i, of this row
        // The step record published by the loader names the key block and its row halves.
        if (!warp_wait(&bars->info_full[gi % NI], (gi / NI) & 1, abort)) { fail(bars, 14); ok = false; break; }
        const int info = bars->step_info[gi % NI];
        const int code = bars->step_code[gi % NI];
        const int j = info & 0x0fffffff, mask = (info >> 28) & 3;
        last = (info >> 30) & 1;
        if (!warp_wait(&bars->s_full[sb], (gi >> 1) & 1, abort)) { fail(bars, 10); ok = false; break; }
        tc::fence_after_sync();
        uint32_t packed[32];
        const bool sel = (mask & half_bit) != 0;               // uniform across the warp
        if (sel) {
          uint32_t sraw[64];
          {
            uint32_t (&lo)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sraw[0]);
            uint32_t (&hi)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sraw[32]);
            tc::tmem_ld32(sp, lo);
            tc::tmem_ld32(sp + 32, hi);
            tc::tmem_ld_wait();
          }
          const int nk = (int)imin<int64_t>(kBlock, m.S - (int64_t)j * kBlock);
          if (nk < kBlock) {                                   // ragged last block: keys >= S
#pragma unroll
            for (int c = 0; c < 64; ++c)
              if (c >= nk) sraw[c] = __float_as_uint(-INFINITY);
          }
          // Token-exact frame mode: the keys of a frame not kept for this row's frame.
          const int hsel = half_bit - 1;                       // 0: block 2t, 1: block 2t+1
          const int allow = (code >> (4 * hsel)) & 0xF;        // uniform across the warp
          if (allow != 0xF) {
            const int side = (r & (kBlock - 1)) >= ((code >> (16 + 8 * hsel)) & 0xFF) ? 1 : 0;
            const int kcol = (code >> 8) & 0xFF;
            const uint64_t low = kcol >= 64 ? ~0ull : ((1ull << kcol) - 1ull);   // columns of the first frame
            const uint64_t keep = (((allow >> (2 * side)) & 1) ? low : 0ull) | (((allow >> (2 * side + 1)) & 1) ? ~low : 0ull);
            const uint32_t klo = (uint32_t)keep, khi = (uint32_t)(keep >> 32);
#pragma unroll
            for (int c = 0; c < 32; ++c) {
              if (!((klo >> c) & 1u)) sraw[c] = __float_as_uint(-INFINITY);
              if (!((khi >> c) & 1u)) sraw[32 + c] = __float_as_uint(-INFINITY);
            }
          }
          float m21[21];
#pragma unroll
          for (int c = 0; c < 21; ++c)
            m21[c] = max3(__uint_as_float(sraw[3 * c]), __uint_as_float(sraw[3 * c + 1]), __uint_as_float(sraw[3 * c + 2]));
          float m7[7];
#pragma unroll
          for (int c = 0; c < 7; ++c) m7[c] = max3(m21[3 * c], m21[3 * c + 1], m21[3 * c + 2]);
          const float mx = max3(max3(m7[0], m7[1], m7[2]), max3(m7[3], m7[4], m7[5]),
                                max3(m7[6], __uint_as_float(sraw[63]), m7[6])) * scale_log2;
          // Raise the running max only when it grows by more than 2^8 (or on the row's first
          // kept block); rows whose O already holds earlier blocks then scale O in TMEM.
          const bool raise = mrow == -INFINITY || mx > mrow + kRescaleLog2;
          const bool scale_o = raise && i > 0 && mrow != -INFINITY;
          if (__any_sync(0xffffffffu, scale_o)) {
            // tcgen05.ld/st are warp-collective: the whole warp takes part, each lane with its
            // own factor (1 for rows that keep their max).
            const uint32_t gp = gi - 1;
            if (!warp_wait(&bars->pv_done[gp & 1], (gp >> 1) & 1, abort)) { fail(bars, 12); ok = false; break; }
            tc::fence_after_sync();
            const float alpha = scale_o ? ex2(mrow - mx) : 1.f;
#pragma unroll 1
            for (int cc = 0; cc < D / 32; ++cc) {
              uint32_t o[32];
              tc::tmem_ld32(tbase + lane_off + L::kColO + cc * 32, o);
              tc::tmem_ld_wait();
#pragma unroll
              for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
              tc::tmem_st32(tbase + lane_off + L::kColO + cc * 32, o);
            }
            tc::tmem_st_wait();
            float l0, l1;
            f2_split(lsum, l0, l1);
            lsum = f2(l0 * alpha, l1 * alpha);
          }
          if (raise) mrow = mx;
          // A row whose keys of every step so far are masked keeps mrow = -inf; its weights
          // are exp2(-inf) = 0 against an offset of 0.
          const float nm = mrow == -INFINITY ? 0.f : -mrow;
          const uint64_t negm = f2(nm, nm);
          uint64_t acc[4] = {f2(0.f, 0.f), f2(0.f, 0.f), f2(0.f, 0.f), f2(0.f, 0.f)};
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            const uint64_t x2 = ffma2(f2(__uint_as_float(sraw[2 * c]), __uint_as_float(sraw[2 * c + 1])), scale2, negm);
            float p0, p1;
            float x0, x1;
            f2_split(x2, x0, x1);
            p0 = ex2(x0);
            p1 = ex2(x1);
            acc[c & 3] = fadd2(acc[c & 3], f2(p0, p1));
            packed[c] = pack_bf16(p0, p1);
          }
          lsum = fadd2(lsum, fadd2(fadd2(acc[0], acc[1]), fadd2(acc[2], acc[3])));
        } else {
#pragma unroll
          for (int c = 0; c < 32; ++c) packed[c] = 0u;
        }
        // P_i (bf16 pairs) over the first 32 columns of its S buffer; S_i is already in registers.
        tc::tmem_st32(sp, packed);
        tc::tmem_st_wait();
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) {
          tc::mbar_arrive(&bars->p_full[sb]);
          *reinterpret_cast<volatile int*>(&bars->p_arrived[q]) = (int)gi;
        }
        ++i;
      }
      if (__any_sync(0xffffffffu, !ok || *abort)) break;
      // ---------------------------------------------------------- epilogue
      if (!warp_wait(&bars->o_full, n & 1, abort)) { fail(bars, 13); break; }
      tc::fence_after_sync();
      float l0, l1;
      f2_split(lsum, l0, l1);
      const float lrow = l0 + l1;
      const int64_t trow = (int64_t)t * kTileRows + r;
      const bool valid = trow < m.S;
      const float inv = 1.f / lrow;
      __nv_bfloat16* orow = O + (bh * m.S + trow) * D;
#pragma unroll 1
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t o[32];
        tc::tmem_ld32(tbase + lane_off + L::kColO + cc * 32, o);
        tc::tmem_ld_wait();
        if (valid) {
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4) {
            uint4 w;
            w.x = pack_bf16(__uint_as_float(o[8 * v4 + 0]) * inv, __uint_as_float(o[8 * v4 + 1]) * inv);
            w.y = pack_bf16(__uint_as_float(o[8 * v4 + 2]) * inv, __uint_as_float(o[8 * v4 + 3]) * inv);
            w.z = pack_bf16(__uint_as_float(o[8 * v4 + 4]) * inv, __uint_as_float(o[8 * v4 + 5]) * inv);
            w.w = pack_bf16(__uint_as_float(o[8 * v4 + 6]) * inv, __uint_as_float(o[8 * v4 + 7]) * inv);
            *reinterpret_cast<uint4*>(orow + cc * 32 + v4 * 8) = w;
          }
        }
      }
      if (valid && lse != nullptr) lse[bh * m.S + trow] = (mrow + log2f(lrow)) * 0.69314718055994531f;
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&bars->o_empty);
      g += i;
    }
  }

  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  if (warp == 1) tc::tmem_dealloc(tbase, L::kTmemCols);
  if (threadIdx.x == 0 && bars->abort) {
    // Every role has stopped. A V copy completes the P barrier of its step only together with
    // the four softmax arrivals; after an abort some of them may never have come, so the missing
    // ones are made here and the copies of the (at most two) V stages in use are waited for.
    const int va = bars->v_armed;
    for (int gg = va - 1; gg <= va; ++gg) {
      if (gg < 0) continue;
      uint64_t* pb = &bars->p_full[gg & 1];
      const uint32_t par = ((uint32_t)gg >> 1) & 1;
      if (tc::mbar_try_wait(pb, par)) continue;
      for (int w = 0; w < 4; ++w)
        if (bars->p_arrived[w] < gg) tc::mbar_arrive(pb);
      tc::mbar_wait_drain(pb, par, kWaitLimit);
    }
    // a tile index out of range (11) or a failed list check of the debug build (>= 100) is a
    // bad argument; every other code is a wait that ran out
    const int ab = bars->abort;
    report_error(control, (ab == 11 || ab >= 100) ? FVATTN_ERR_INVALID : FVATTN_ERR_TIMEOUT, ab);
  }
  if (stamps != nullptr && threadIdx.x == 0) {
    // this CTA's SM and its busy interval (ns), for the SM busy-time imbalance
    uint64_t t_end;
    uint32_t smid;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t_end));
    asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
    stamps[3 * blockIdx.x] = smid;
    stamps[3 * blockIdx.x + 2] = t_end;
  }
}

// [BH, S, d] bf16 viewed as a 3-D tensor (d innermost); 64 x 64 boxes with the 128-byte
// swizzle; rows past S read as zeros and never reach the next head.
bool make_map(CUtensorMap* map, const void* base, const Dims& m) {
  return make_map_bf16_3d(map, base, (uint64_t)m.d, (uint64_t)m.S, (uint64_t)m.BH, (uint32_t)kBlock);
}

template <int D>
cudaError_t launch_tc_d(const void* Q, const void* K, const void* V, const Dims& m, float scale,
                        const int32_t* row_ptr, const int32_t* col_idx, int64_t col_cap, const int32_t* col_code,
                        const int32_t* tile_order, int32_t* control, void* O, float* lse, uint64_t* stamps,
                        uint32_t hold_polls, int nsm, cudaStream_t st) {
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, Q, m) || !make_map(&mk, K, m) || !make_map(&mv, V, m)) return cudaErrorInvalidValue;
  const size_t smem = TcLayout<D>::kBytes + 1024;
  cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int grid = attn_tc_grid(m, nsm);
  attn_tc_kernel<D><<<grid, 192, smem, st>>>(mq, mk, mv, m, scale * 1.4426950408889634f, row_ptr, col_idx,
                                             col_cap, col_code, tile_order, control,
                                             static_cast<__nv_bfloat16*>(O), lse, stamps, hold_polls);
  return cudaGetLastError();
}

}  // namespace

int attn_tc_grid(const Dims& m, int nsm) { return (int)imin<int64_t>(m.BH * m.nt, (int64_t)nsm * 2); }

cudaError_t launch_attn_tc(const void* Q, const void* K, const void* V, const Dims& m, float scale,
                           const int32_t* row_ptr, const int32_t* col_idx, int64_t col_cap, const int32_t* col_code,
                           const int32_t* tile_order, int32_t* control, void* O, float* lse, uint64_t* stamps,
                           uint32_t hold_polls, int nsm, cudaStream_t st) {
  if (m.d == 128)
    return launch_tc_d<128>(Q, K, V, m, scale, row_ptr, col_idx, col_cap, col_code, tile_order, control, O, lse,
                            stamps, hold_polls, nsm, st);
  return launch_tc_d<64>(Q, K, V, m, scale, row_ptr, col_idx, col_cap, col_code, tile_order, control, O, lse, stamps,
                         hold_polls, nsm, st);
}

}  // namespace fv
