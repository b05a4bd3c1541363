// Launchers of the router kernels (route.cu).
#pragma once

#include "common.cuh"

namespace fv {

// Forced-block settings of fvattn_route_cfg, as the kernels use them.
struct ForceCfg {
  int force_diag, local_window, frame_len, frame_window, force_first;
};

// Code of an entry whose key block is attended whole (all four allow bits, no boundaries).
constexpr int32_t kCodeAll = 0xF | (64 << 8) | (64 << 16);

// Row stride of the fp64 block-score matrix: nb rounded up to 32.
__host__ __device__ __forceinline__ int means_ld(int nb) { return (nb + 31) & ~31; }
size_t logits_elems(const Dims& m);      // doubles of the fp64 block-score matrix
size_t frame_smem_bytes(const Dims& m);
size_t schedule_smem_bytes(const Dims& m, int* groups);

// Block means as exact 8-bit integer slices for the tensor-core score GEMM (score_tc.cu): per
// block a power-of-two exponent and kScoreSlices int8 planes, [BH][kScoreSlices][nb][kSliceRow]
// (rows of 128 bytes; for d = 64 the upper half of a row is zero).
constexpr int kScoreSlices = 5;
constexpr int kSliceRow = 128;
struct SliceOut {
  int8_t* qs;
  int8_t* ks;
  int32_t* eq;
  int32_t* ek;
};
cudaError_t launch_score_tc(const int8_t* qs, const int8_t* ks, const int32_t* eq, const int32_t* ek, const Dims& m,
                            double scale, double* logits, int32_t* status, int nsm, cudaStream_t st,
                            uint32_t hold_polls = 0);

// out: 0 = means [row][d] (qo, ko), 1 = score slices and exponents (so), 2 = frame segment sums;
// the blocks [b0, b1) of every head (outputs at their full-layout rows).
cudaError_t launch_pool(const void* Q, const void* K, int ntensors, int dtype, const Dims& m, int b0, int b1, int out,
                        int frame_len, double* qo, double* ko, double* qhi, double* khi, const SliceOut& so, int nsm,
                        cudaStream_t st);
// Slack-aware augmentation of 128-row tiles (fvattn_route_cfg.sasa_coef / sasa_trigger).
struct SasaCfg {
  float coef;
  int trigger;
};

// Scores (tensor cores, from the slices), then the per-row cut. kblocks > 0: keep the kblocks
// highest scores per row instead of the Top-p cut.
cudaError_t launch_topp(const SliceOut& so, double* logits, const Dims& m, double p, int kblocks, double scale,
                        const ForceCfg& fc, const SasaCfg& sasa, uint32_t* bits, int32_t* counts, int32_t* tile_cost,
                        int32_t* status, int nsm, cudaStream_t st);
// fsel: per head, the top-k key frames of every query frame ([BH][F][ceil(F/32)] bits).
cudaError_t launch_frame(const double* qlo, const double* qhi, const double* klo, const double* khi,
                         double* qf, double* kf, const Dims& m, int frame_len, int topk, double scale,
                         const ForceCfg& fc, uint32_t* bits, int32_t* counts, int32_t* tile_cost,
                         uint32_t* fsel, cudaStream_t st);
// Per-entry token-mask codes (fvattn_csr.col_code): token-exact frame codes from fsel, or
// "allow all" when fsel is null.
cudaError_t launch_codes(const int32_t* row_ptr, const int32_t* col_idx, const Dims& m, const uint32_t* fsel,
                         int frame_len, const ForceCfg& fc, int32_t* col_code, int64_t capacity, int nsm,
                         cudaStream_t st);
cudaError_t launch_schedule(const int32_t* counts, const int32_t* tile_cost, const Dims& m, int32_t* row_ptr,
                            int64_t* head_load, int64_t* nnz, int32_t* tile_order, int64_t capacity,
                            int32_t* status, cudaStream_t st);
cudaError_t launch_csr(const uint32_t* bits, const int32_t* row_ptr, const Dims& m, int32_t* col_idx,
                       int64_t capacity, int nsm, cudaStream_t st);

// Compacts the tile order to the tiles of heads with active[bh] != 0 (balance.cu).
cudaError_t launch_select_heads(int32_t* tile_order, const Dims& m, const uint8_t* active, int32_t* control,
                                cudaStream_t st);

// Attention (attn_f32.cu, attn_tc.cu).
// col_code may be null (every entry allows its whole key block).
// col_cap: the capacity of col_idx (read only by the debug build's list checks).
cudaError_t launch_attn_f32(const float* Q, const float* K, const float* V, const Dims& m, float scale,
                            const int32_t* row_ptr, const int32_t* col_idx, int64_t col_cap, const int32_t* col_code,
                            const int32_t* tile_order, int32_t* control, float* O, float* lse, cudaStream_t st);
// stamps: null, or 3 words per CTA of the launch (attn_tc_grid): the SM id and the CTA's busy
// interval [start, end) in ns of %globaltimer. hold_polls: 0, or (failure-path check) the poll
// limit of a first wait on a barrier that nothing completes, so that the kernel times out.
int attn_tc_grid(const Dims& m, int nsm);
cudaError_t launch_attn_tc(const void* Q, const void* K, const void* V, const Dims& m, float scale,
                           const int32_t* row_ptr, const int32_t* col_idx, int64_t col_cap, const int32_t* col_code,
                           const int32_t* tile_order, int32_t* control, void* O, float* lse, uint64_t* stamps,
                           uint32_t hold_polls, int nsm, cudaStream_t st);

}  // namespace fv
