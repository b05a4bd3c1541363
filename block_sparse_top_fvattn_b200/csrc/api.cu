// Host side of the C ABI declared in include/fvattn.h: argument validation, workspace
// layout, and the launch sequence of the router and the attention kernels.
#include <math.h>
#include <string.h>

#include "common.cuh"
#include "route.cuh"

using namespace fv;

namespace {

constexpr int kVersion = (1 << 16) | 3;

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// The CUDA error behind the last FVATTN_ERR_CUDA this thread got (fvattn_last_cuda_error).
thread_local int g_last_cuda_error = 0;

// FVATTN_OK, or FVATTN_ERR_CUDA with the CUDA error recorded for this thread.
int cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return FVATTN_OK;
  g_last_cuda_error = (int)e;
  return FVATTN_ERR_CUDA;
}

int validate_shape(const fvattn_shape* s) {
  if (s == nullptr) return FVATTN_ERR_INVALID;
  if (s->B < 1 || s->H < 1 || s->S < 1 || s->d < 1) return FVATTN_ERR_INVALID;
  if (s->dtype != FVATTN_BF16 && s->dtype != FVATTN_F32) return FVATTN_ERR_INVALID;
  if (!(s->scale >= 0.f) && !(s->scale <= 0.f)) return FVATTN_ERR_INVALID;   // NaN
  if (isinf(s->scale)) return FVATTN_ERR_INVALID;
  if (s->block != kBlock) return FVATTN_ERR_UNSUPPORTED;
  if (s->d != 64 && s->d != 128) return FVATTN_ERR_UNSUPPORTED;
  if (s->S > (int64_t)1 << 30 || s->B * s->H > 65535) return FVATTN_ERR_UNSUPPORTED;
  const int64_t nb = (s->S + kBlock - 1) / kBlock;
  // CSR offsets are int32: the densest selection must fit.
  if (s->B * s->H * nb * nb >= ((int64_t)1 << 31)) return FVATTN_ERR_UNSUPPORTED;
  return FVATTN_OK;
}

int validate_cfg(const fvattn_shape* s, const fvattn_route_cfg* c) {
  if (c == nullptr) return FVATTN_ERR_INVALID;
  if (c->mode != FVATTN_MODE_TOPP && c->mode != FVATTN_MODE_FRAME_TOPK && c->mode != FVATTN_MODE_TOPK_BLOCKS)
    return FVATTN_ERR_INVALID;
  if (c->mode == FVATTN_MODE_TOPK_BLOCKS) {
    if (c->topk_blocks < 1) return FVATTN_ERR_INVALID;
    if ((s->S + kBlock - 1) / kBlock > 1280) return FVATTN_ERR_UNSUPPORTED;
  }
  if (!(c->p > 0.f) || isinf(c->p)) return FVATTN_ERR_INVALID;        // rejects p <= 0 and NaN
  if (c->local_window < 0 || c->frame_len < 0 || c->frame_window < -1) return FVATTN_ERR_INVALID;
  if (c->force_diag != 0 && c->force_diag != 1) return FVATTN_ERR_INVALID;
  if (c->force_first_frame != 0 && c->force_first_frame != 1) return FVATTN_ERR_INVALID;
  if ((c->frame_window >= 0 || c->force_first_frame) && c->frame_len == 0) return FVATTN_ERR_INVALID;
  if (!(c->sasa_coef >= 0.f && c->sasa_coef <= 1.f) || c->sasa_trigger < 0) return FVATTN_ERR_INVALID;
  if (c->frame_exact != 0 && c->frame_exact != 1) return FVATTN_ERR_INVALID;
  if (c->frame_exact && c->mode != FVATTN_MODE_FRAME_TOPK) return FVATTN_ERR_INVALID;
  if (c->sasa_coef > 0.f) {
    if (c->mode == FVATTN_MODE_FRAME_TOPK) return FVATTN_ERR_UNSUPPORTED;
    if ((s->S + kBlock - 1) / kBlock > 1280) return FVATTN_ERR_UNSUPPORTED;
  }
  if (c->mode == FVATTN_MODE_FRAME_TOPK) {
    if (c->frame_len < kBlock || c->topk_frames < 1) return FVATTN_ERR_INVALID;
    const int64_t F = (s->S + c->frame_len - 1) / c->frame_len;
    if (F > 128) return FVATTN_ERR_UNSUPPORTED;
  }
  return FVATTN_OK;
}

struct WsLayout {
  size_t qlo, klo, qhi, khi, qf, kf, fsel, qs, ks, eq, ek, logits, bits, counts, total;
};

size_t take(size_t& off, size_t bytes) {
  const size_t o = off;
  off += (bytes + 255) & ~(size_t)255;
  return o;
}

WsLayout ws_layout(const Dims& m, int mode) {
  WsLayout L{};
  size_t off = 0;
  const bool scored = mode == FVATTN_MODE_TOPP || mode == FVATTN_MODE_TOPK_BLOCKS;
  const size_t means = (size_t)m.BH * m.nb * m.d * sizeof(double);
  if (scored) {
    const size_t slices = (size_t)m.BH * kScoreSlices * m.nb * kSliceRow;
    L.qs = take(off, slices);
    L.ks = take(off, slices);
    L.eq = take(off, (size_t)m.BH * m.nb * sizeof(int32_t));
    L.ek = take(off, (size_t)m.BH * m.nb * sizeof(int32_t));
  } else {
    L.qlo = take(off, means);
    L.klo = take(off, means);
  }
  if (mode == FVATTN_MODE_FRAME_TOPK) {
    L.qhi = take(off, means);
    L.khi = take(off, means);
    const size_t fm = (size_t)m.BH * m.F * m.d * sizeof(double);
    L.qf = take(off, fm);
    L.kf = take(off, fm);
    L.fsel = take(off, (size_t)m.BH * m.F * ((m.F + 31) / 32) * sizeof(uint32_t));
  }
  if (scored) L.logits = take(off, logits_elems(m) * sizeof(double));
  L.bits = take(off, (size_t)m.BH * m.nb * m.nw * sizeof(uint32_t));
  L.counts = take(off, (size_t)m.BH * m.nb * sizeof(int32_t));
  L.total = off;
  return L;
}

int num_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return n;
}

double softmax_scale(const fvattn_shape* s) {
  return s->scale > 0.f ? (double)s->scale : 1.0 / sqrt((double)s->d);
}

}  // namespace

extern "C" {

int fvattn_version(void) { return kVersion; }

int fvattn_last_cuda_error(void) { return g_last_cuda_error; }

const char* fvattn_cuda_error_name(int code) { return cudaGetErrorName((cudaError_t)code); }

const char* fvattn_status_string(int status) {
  switch (status) {
    case FVATTN_OK: return "ok";
    case FVATTN_ERR_INVALID: return "invalid argument";
    case FVATTN_ERR_UNSUPPORTED: return "unsupported shape or configuration";
    case FVATTN_ERR_CAPACITY: return "buffer too small";
    case FVATTN_ERR_CUDA: return "CUDA error";
    case FVATTN_ERR_TIMEOUT: return "device wait timed out";
    default: return "unknown status";
  }
}

int64_t fvattn_csr_max_nnz(const fvattn_shape* shape) {
  const int st = validate_shape(shape);
  if (st != FVATTN_OK) return st;
  const int64_t nb = (shape->S + kBlock - 1) / kBlock;
  return shape->B * shape->H * nb * nb;
}

int64_t fvattn_num_tiles(const fvattn_shape* shape) {
  const int st = validate_shape(shape);
  if (st != FVATTN_OK) return st;
  const int64_t nb = (shape->S + kBlock - 1) / kBlock;
  return shape->B * shape->H * ((nb + 1) / 2);
}

size_t fvattn_route_workspace_bytes(const fvattn_shape* shape, const fvattn_route_cfg* cfg) {
  if (validate_shape(shape) != FVATTN_OK || validate_cfg(shape, cfg) != FVATTN_OK) return 0;
  const Dims m = make_dims(*shape, cfg->frame_len);
  return ws_layout(m, cfg->mode).total;
}

}  // extern "C"

namespace {

// Step 1 of the router for the blocks [b0, b1) of every head, into the workspace.
cudaError_t route_pool(const void* Q, const void* K, const fvattn_shape* shape, const fvattn_route_cfg* cfg,
                       const Dims& m, const WsLayout& L, unsigned char* ws, int b0, int b1, int nsm, cudaStream_t s) {
  if (cfg->mode == FVATTN_MODE_TOPP || cfg->mode == FVATTN_MODE_TOPK_BLOCKS) {
    const SliceOut so{reinterpret_cast<int8_t*>(ws + L.qs), reinterpret_cast<int8_t*>(ws + L.ks),
                      reinterpret_cast<int32_t*>(ws + L.eq), reinterpret_cast<int32_t*>(ws + L.ek)};
    return launch_pool(Q, K, 2, shape->dtype, m, b0, b1, 1, 0, nullptr, nullptr, nullptr, nullptr, so, nsm, s);
  }
  return launch_pool(Q, K, 2, shape->dtype, m, b0, b1, 2, cfg->frame_len, reinterpret_cast<double*>(ws + L.qlo),
                     reinterpret_cast<double*>(ws + L.klo), reinterpret_cast<double*>(ws + L.qhi),
                     reinterpret_cast<double*>(ws + L.khi), SliceOut{}, nsm, s);
}

// Steps 2 and 3 of the router from a workspace whose every block has been pooled.
cudaError_t route_finish(const fvattn_shape* shape, const fvattn_route_cfg* cfg, const fvattn_csr* out, const Dims& m,
                         const WsLayout& L, unsigned char* ws, int nsm, cudaStream_t s) {
  uint32_t* bits = reinterpret_cast<uint32_t*>(ws + L.bits);
  int32_t* counts = reinterpret_cast<int32_t*>(ws + L.counts);
  const double scale = softmax_scale(shape);
  ForceCfg fc{cfg->force_diag, cfg->local_window, cfg->frame_len, cfg->frame_window, cfg->force_first_frame};
  cudaError_t e = cudaMemsetAsync(out->status, 0, 4 * sizeof(int32_t), s);
  if (e != cudaSuccess) return e;
  if (cfg->mode == FVATTN_MODE_TOPP || cfg->mode == FVATTN_MODE_TOPK_BLOCKS) {
    const int kblocks = cfg->mode == FVATTN_MODE_TOPK_BLOCKS ? cfg->topk_blocks : 0;
    const SliceOut so{reinterpret_cast<int8_t*>(ws + L.qs), reinterpret_cast<int8_t*>(ws + L.ks),
                      reinterpret_cast<int32_t*>(ws + L.eq), reinterpret_cast<int32_t*>(ws + L.ek)};
    e = launch_topp(so, reinterpret_cast<double*>(ws + L.logits), m, cfg->p >= 1.f ? 1.0 : (double)cfg->p, kblocks,
                    scale, fc, SasaCfg{cfg->sasa_coef, cfg->sasa_trigger}, bits, counts, out->tile_cost, out->status,
                    nsm, s);
  } else {
    e = launch_frame(reinterpret_cast<double*>(ws + L.qlo), reinterpret_cast<double*>(ws + L.qhi),
                     reinterpret_cast<double*>(ws + L.klo), reinterpret_cast<double*>(ws + L.khi),
                     reinterpret_cast<double*>(ws + L.qf), reinterpret_cast<double*>(ws + L.kf), m, cfg->frame_len,
                     cfg->topk_frames, scale, fc, bits, counts, out->tile_cost,
                     reinterpret_cast<uint32_t*>(ws + L.fsel), s);
  }
  if (e == cudaSuccess)
    e = launch_schedule(counts, out->tile_cost, m, out->row_ptr, out->head_load, out->nnz, out->tile_order,
                        out->col_capacity, out->status, s);
  if (e == cudaSuccess) e = launch_csr(bits, out->row_ptr, m, out->col_idx, out->col_capacity, nsm, s);
  if (e == cudaSuccess && out->col_code != nullptr)
    e = launch_codes(out->row_ptr, out->col_idx, m, cfg->frame_exact ? reinterpret_cast<const uint32_t*>(ws + L.fsel)
                                                                     : nullptr,
                     cfg->frame_len, fc, out->col_code, out->col_capacity, nsm, s);
  return e;
}

int check_route_inputs(const fvattn_shape* shape, const fvattn_route_cfg* cfg, void* workspace,
                       size_t workspace_bytes) {
  int st = validate_shape(shape);
  if (st != FVATTN_OK) return st;
  st = validate_cfg(shape, cfg);
  if (st != FVATTN_OK) return st;
  if (workspace == nullptr || !aligned(workspace, 256)) return FVATTN_ERR_INVALID;
  const Dims m = make_dims(*shape, cfg->frame_len);
  if (workspace_bytes < ws_layout(m, cfg->mode).total) return FVATTN_ERR_CAPACITY;
  return FVATTN_OK;
}

int check_csr_out(const fvattn_shape* shape, const fvattn_route_cfg* cfg, const fvattn_csr* out) {
  if (out == nullptr || !out->row_ptr || !out->col_idx || !out->head_load || !out->tile_cost || !out->tile_order ||
      !out->nnz || !out->status)
    return FVATTN_ERR_INVALID;
  if (cfg->frame_exact && out->col_code == nullptr) return FVATTN_ERR_INVALID;
  const Dims m = make_dims(*shape, cfg->frame_len);
  if (out->col_capacity < m.BH * m.nb * m.nb) return FVATTN_ERR_CAPACITY;
  return FVATTN_OK;
}

}  // namespace

extern "C" {

int fvattn_route(const void* Q, const void* K, const fvattn_shape* shape, const fvattn_route_cfg* cfg,
                 const fvattn_csr* out, void* workspace, size_t workspace_bytes, fvattn_stream_t stream) {
  int st = check_route_inputs(shape, cfg, workspace, workspace_bytes);
  if (st != FVATTN_OK) return st;
  if (Q == nullptr || K == nullptr || !aligned(Q, 16) || !aligned(K, 16)) return FVATTN_ERR_INVALID;
  st = check_csr_out(shape, cfg, out);
  if (st != FVATTN_OK) return st;
  const Dims m = make_dims(*shape, cfg->frame_len);
  const WsLayout L = ws_layout(m, cfg->mode);
  const int nsm = num_sms();
  if (nsm <= 0) return FVATTN_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  cudaError_t e = route_pool(Q, K, shape, cfg, m, L, ws, 0, m.nb, nsm, s);
  if (e == cudaSuccess) e = route_finish(shape, cfg, out, m, L, ws, nsm, s);
  return cuda_status(e);
}

int fvattn_route_pool(const void* Q, const void* K, const fvattn_shape* shape, const fvattn_route_cfg* cfg,
                      int64_t block_begin, int64_t block_end, void* workspace, size_t workspace_bytes,
                      fvattn_stream_t stream) {
  int st = check_route_inputs(shape, cfg, workspace, workspace_bytes);
  if (st != FVATTN_OK) return st;
  if (Q == nullptr || K == nullptr || !aligned(Q, 16) || !aligned(K, 16)) return FVATTN_ERR_INVALID;
  const Dims m = make_dims(*shape, cfg->frame_len);
  if (block_begin < 0 || block_end > m.nb || block_begin >= block_end) return FVATTN_ERR_INVALID;
  const int nsm = num_sms();
  if (nsm <= 0) return FVATTN_ERR_CUDA;
  cudaError_t e = route_pool(Q, K, shape, cfg, m, ws_layout(m, cfg->mode), static_cast<unsigned char*>(workspace),
                             (int)block_begin, (int)block_end, nsm, reinterpret_cast<cudaStream_t>(stream));
  return cuda_status(e);
}

int fvattn_route_finish(const fvattn_shape* shape, const fvattn_route_cfg* cfg, const fvattn_csr* out,
                        void* workspace, size_t workspace_bytes, fvattn_stream_t stream) {
  int st = check_route_inputs(shape, cfg, workspace, workspace_bytes);
  if (st != FVATTN_OK) return st;
  st = check_csr_out(shape, cfg, out);
  if (st != FVATTN_OK) return st;
  const Dims m = make_dims(*shape, cfg->frame_len);
  const int nsm = num_sms();
  if (nsm <= 0) return FVATTN_ERR_CUDA;
  cudaError_t e = route_finish(shape, cfg, out, m, ws_layout(m, cfg->mode), static_cast<unsigned char*>(workspace),
                               nsm, reinterpret_cast<cudaStream_t>(stream));
  return cuda_status(e);
}

}  // extern "C"

namespace {

int sparse_attn(const void* Q, const void* K, const void* V, const fvattn_shape* shape, const fvattn_csr* csr,
                void* O, float* lse, uint64_t* stamps, fvattn_stream_t stream, uint32_t hold_polls = 0) {
  int st = validate_shape(shape);
  if (st != FVATTN_OK) return st;
  if (!Q || !K || !V || !O || !csr || !csr->row_ptr || !csr->col_idx || !csr->tile_order || !csr->status)
    return FVATTN_ERR_INVALID;
  if (!aligned(Q, 16) || !aligned(K, 16) || !aligned(V, 16) || !aligned(O, 16) || (lse && !aligned(lse, 4)))
    return FVATTN_ERR_INVALID;
  const Dims m = make_dims(*shape, 0);
  const float scale = (float)softmax_scale(shape);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (shape->dtype == FVATTN_F32) {
    e = launch_attn_f32(static_cast<const float*>(Q), static_cast<const float*>(K), static_cast<const float*>(V), m,
                        scale, csr->row_ptr, csr->col_idx, csr->col_capacity, csr->col_code, csr->tile_order,
                        csr->status, static_cast<float*>(O), lse, s);
  } else {
    const int nsm = num_sms();
    if (nsm <= 0) return FVATTN_ERR_CUDA;
    if (const cudaError_t me = cudaMemsetAsync(csr->status + 2, 0, sizeof(int32_t), s)) return cuda_status(me);
    e = launch_attn_tc(Q, K, V, m, scale, csr->row_ptr, csr->col_idx, csr->col_capacity, csr->col_code,
                       csr->tile_order, csr->status, O, lse, stamps, hold_polls, nsm, s);
  }
  return cuda_status(e);
}

}  // namespace

extern "C" {

int fvattn_sparse_attn(const void* Q, const void* K, const void* V, const fvattn_shape* shape,
                       const fvattn_csr* csr, void* O, float* lse, fvattn_stream_t stream) {
  return sparse_attn(Q, K, V, shape, csr, O, lse, nullptr, stream);
}

int64_t fvattn_attn_stamp_words(const fvattn_shape* shape) {
  if (validate_shape(shape) != FVATTN_OK || shape->dtype != FVATTN_BF16) return 0;
  const int nsm = num_sms();
  if (nsm <= 0) return 0;
  return 3 * (int64_t)attn_tc_grid(make_dims(*shape, 0), nsm);
}

int fvattn_sparse_attn_stamped(const void* Q, const void* K, const void* V, const fvattn_shape* shape,
                               const fvattn_csr* csr, void* O, float* lse, uint64_t* stamps, int64_t stamp_words,
                               fvattn_stream_t stream) {
  const int st = validate_shape(shape);
  if (st != FVATTN_OK) return st;
  if (shape->dtype != FVATTN_BF16) return FVATTN_ERR_UNSUPPORTED;
  if (stamps == nullptr || !aligned(stamps, 8)) return FVATTN_ERR_INVALID;
  const int64_t need = fvattn_attn_stamp_words(shape);
  if (need <= 0) return FVATTN_ERR_CUDA;
  if (stamp_words < need) return FVATTN_ERR_CAPACITY;
  return sparse_attn(Q, K, V, shape, csr, O, lse, stamps, stream);
}

int fvattn_select_heads(const fvattn_shape* shape, const fvattn_csr* csr, const uint8_t* active,
                        fvattn_stream_t stream) {
  const int st = validate_shape(shape);
  if (st != FVATTN_OK) return st;
  if (!csr || !csr->tile_order || !csr->status || !active) return FVATTN_ERR_INVALID;
  const Dims m = make_dims(*shape, 0);
  if (m.BH * m.nt > 0x7fffffff) return FVATTN_ERR_UNSUPPORTED;
  cudaError_t e = launch_select_heads(csr->tile_order, m, active, csr->status, reinterpret_cast<cudaStream_t>(stream));
  return cuda_status(e);
}

int fvattn_block_means(const void* X, const fvattn_shape* shape, double* out, fvattn_stream_t stream) {
  const int st = validate_shape(shape);
  if (st != FVATTN_OK) return st;
  if (!X || !out || !aligned(X, 16) || !aligned(out, 8)) return FVATTN_ERR_INVALID;
  const Dims m = make_dims(*shape, 0);
  const int nsm = num_sms();
  if (nsm <= 0) return FVATTN_ERR_CUDA;
  cudaError_t e = launch_pool(X, nullptr, 1, shape->dtype, m, 0, m.nb, 0, 0, out, nullptr, nullptr, nullptr, SliceOut{}, nsm,
                              reinterpret_cast<cudaStream_t>(stream));
  return cuda_status(e);
}

size_t fvattn_block_scores_workspace_bytes(const fvattn_shape* shape) {
  if (validate_shape(shape) != FVATTN_OK) return 0;
  return ws_layout(make_dims(*shape, 0), FVATTN_MODE_TOPP).logits;   // the slices and exponents
}

int64_t fvattn_block_scores_ld(const fvattn_shape* shape) {
  if (validate_shape(shape) != FVATTN_OK) return 0;
  return means_ld(make_dims(*shape, 0).nb);
}

int fvattn_block_scores(const void* Q, const void* K, const fvattn_shape* shape, double* scores, void* workspace,
                        size_t workspace_bytes, int32_t* status, fvattn_stream_t stream) {
  const int st = validate_shape(shape);
  if (st != FVATTN_OK) return st;
  if (!Q || !K || !scores || !workspace || !status) return FVATTN_ERR_INVALID;
  if (!aligned(Q, 16) || !aligned(K, 16) || !aligned(scores, 16) || !aligned(workspace, 256) || !aligned(status, 4))
    return FVATTN_ERR_INVALID;
  const Dims m = make_dims(*shape, 0);
  const WsLayout L = ws_layout(m, FVATTN_MODE_TOPP);
  if (workspace_bytes < L.logits) return FVATTN_ERR_CAPACITY;
  const int nsm = num_sms();
  if (nsm <= 0) return FVATTN_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  const SliceOut so{reinterpret_cast<int8_t*>(ws + L.qs), reinterpret_cast<int8_t*>(ws + L.ks),
                    reinterpret_cast<int32_t*>(ws + L.eq), reinterpret_cast<int32_t*>(ws + L.ek)};
  if (const cudaError_t me = cudaMemsetAsync(status, 0, 4 * sizeof(int32_t), s)) return cuda_status(me);
  cudaError_t e = launch_pool(Q, K, 2, shape->dtype, m, 0, m.nb, 1, 0, nullptr, nullptr, nullptr, nullptr, so, nsm, s);
  if (e == cudaSuccess) e = launch_score_tc(so.qs, so.ks, so.eq, so.ek, m, softmax_scale(shape), scores, status, nsm, s);
  return cuda_status(e);
}

int fvattn_sparse_attn_timeout_check(const void* Q, const void* K, const void* V, const fvattn_shape* shape,
                                     const fvattn_csr* csr, void* O, uint32_t polls, fvattn_stream_t stream) {
  const int st = validate_shape(shape);
  if (st != FVATTN_OK) return st;
  if (shape->dtype != FVATTN_BF16) return FVATTN_ERR_UNSUPPORTED;
  if (polls == 0) return FVATTN_ERR_INVALID;
  return sparse_attn(Q, K, V, shape, csr, O, nullptr, nullptr, stream, polls);
}

int fvattn_block_scores_timeout_check(const void* Q, const void* K, const fvattn_shape* shape, double* scores,
                                      void* workspace, size_t workspace_bytes, int32_t* status, uint32_t polls,
                                      fvattn_stream_t stream) {
  const int st = validate_shape(shape);
  if (st != FVATTN_OK) return st;
  if (!Q || !K || !scores || !workspace || !status || polls == 0) return FVATTN_ERR_INVALID;
  if (!aligned(Q, 16) || !aligned(K, 16) || !aligned(scores, 16) || !aligned(workspace, 256) || !aligned(status, 4))
    return FVATTN_ERR_INVALID;
  const Dims m = make_dims(*shape, 0);
  const WsLayout L = ws_layout(m, FVATTN_MODE_TOPP);
  if (workspace_bytes < L.logits) return FVATTN_ERR_CAPACITY;
  const int nsm = num_sms();
  if (nsm <= 0) return FVATTN_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  const SliceOut so{reinterpret_cast<int8_t*>(ws + L.qs), reinterpret_cast<int8_t*>(ws + L.ks),
                    reinterpret_cast<int32_t*>(ws + L.eq), reinterpret_cast<int32_t*>(ws + L.ek)};
  if (const cudaError_t me = cudaMemsetAsync(status, 0, 4 * sizeof(int32_t), s)) return cuda_status(me);
  cudaError_t e = launch_pool(Q, K, 2, shape->dtype, m, 0, m.nb, 1, 0, nullptr, nullptr, nullptr, nullptr, so, nsm, s);
  if (e == cudaSuccess)
    e = launch_score_tc(so.qs, so.ks, so.eq, so.ek, m, softmax_scale(shape), scores, status, nsm, s, polls);
  return cuda_status(e);
}

int fvattn_read_status(const fvattn_csr* csr, fvattn_stream_t stream) {
  if (csr == nullptr || csr->status == nullptr) return FVATTN_ERR_INVALID;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (const cudaError_t se = cudaStreamSynchronize(s)) return cuda_status(se);
  int32_t v = 0;
  if (const cudaError_t ce = cudaMemcpy(&v, csr->status, sizeof(v), cudaMemcpyDeviceToHost)) return cuda_status(ce);
  return v;
}

}  // extern "C"
