/*
 * fvattn.h -- C ABI of libfvattn.so: Top-p block routing and block-sparse attention for
 * video-DiT self-attention on NVIDIA B200 (sm_100a).
 *
 * The method (FVAttn blog summary "腾讯+中山大学新作：视频生成提速2.11×，靠的是RLB和SASA",
 * section "AI视频生成的阿喀琉斯之踵"): split the key/value sequence into fixed blocks, score
 * every key block for each query block, keep the smallest set of blocks, in descending
 * importance, whose cumulative importance reaches p, and run exact softmax attention over
 * the kept blocks only. Block scores are the scaled dot products of block-mean vectors
 * (video-generation acceleration notes, wzjinhao.cn, §5.2 "块稀疏注意力的教学实现").
 *
 * Conventions for every entry point:
 *  - Tensors Q, K, V, O are dense row-major [B, H, S, d] device arrays (the notes' [B,H,L,D]
 *    layout, §5.2), element type given by fvattn_shape.dtype, base 16-byte aligned.
 *  - The caller owns and allocates every buffer. The library never allocates or frees
 *    memory and never synchronises, except fvattn_read_status. All work is enqueued on the
 *    caller's stream, in order; the calls can be captured into a CUDA graph by the caller.
 *  - Argument errors are detected on the host, before any launch, and returned as a negative
 *    fvattn_status; nothing is enqueued then. A failed launch returns FVATTN_ERR_CUDA.
 *    Errors found on the device (capacity exceeded, a bounded wait that ran out) are written
 *    to the device status word (fvattn_csr.status[0]) and read with fvattn_read_status.
 *  - Not thread-safe for concurrent calls that share output or workspace buffers.
 */
#ifndef FVATTN_H
#define FVATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; NULL is the legacy default stream. */
struct CUstream_st;
typedef struct CUstream_st* fvattn_stream_t;

typedef enum {
  FVATTN_OK = 0,
  FVATTN_ERR_INVALID = -1,      /* bad argument: null pointer, size, range, alignment      */
  FVATTN_ERR_UNSUPPORTED = -2,  /* valid but not implemented (block != 64, d not 64/128)   */
  FVATTN_ERR_CAPACITY = -3,     /* an output or workspace buffer is too small              */
  FVATTN_ERR_CUDA = -4,         /* a CUDA runtime call or launch failed                    */
  FVATTN_ERR_TIMEOUT = -5       /* a bounded device-side wait ran out (device status only) */
} fvattn_status;

typedef enum { FVATTN_BF16 = 0, FVATTN_F32 = 1 } fvattn_dtype;

typedef enum {
  FVATTN_MODE_TOPP = 0,        /* FVAttn Top-p over key blocks                             */
  FVATTN_MODE_FRAME_TOPK = 1,  /* Sol-Attn frame-level top-k (vLLM-Omni article §2.1-§2.2) */
  FVATTN_MODE_TOPK_BLOCKS = 2  /* a fixed number of key blocks per query block (the notes'
                                  teaching variant, §5.2: scores.topk(topk_blocks))        */
} fvattn_mode;

/* Problem shape. block must be 64; d must be 64 or 128; scale <= 0 means 1/sqrt(d). */
typedef struct {
  int64_t B, H, S, d;
  int32_t block;
  int32_t dtype;     /* fvattn_dtype */
  float scale;
} fvattn_shape;

/*
 * Routing configuration.
 *  mode              fvattn_mode.
 *  p                 Top-p threshold in (0, 1]; p >= 1 keeps every key block (dense).
 *  force_diag        1: key block i is always kept for query block i.
 *  local_window      w > 0 keeps the band |i - j| <= w (notes §5.2, "邻近块保底"); 0: none.
 *  frame_len         tokens per latent frame; 0: no frame structure. Frame mode needs >= 64.
 *  topk_frames       frame mode: frames kept per query frame by score (>= 1).
 *  frame_window      fw >= 0 keeps the frames within +-fw of the query block's frames
 *                    (Sol-Attn §2.2, neighbouring frames); -1 disables.
 *  force_first_frame 1: the blocks of frame 0 are always kept (Sol-Attn §5.2).
 *  topk_blocks       FVATTN_MODE_TOPK_BLOCKS: key blocks kept per query block by score
 *                    (>= 1; ties go to the lower block index); at most 1280 blocks per row.
 *  sasa_coef         slack-aware sparse augmentation (FVAttn summary, section "SASA"), in
 *                    [0, 1]; 0 disables it. Top-p and top-k modes, at most 1280 blocks per
 *                    row. The two query blocks 2t, 2t+1 of a 128-row attention tile step
 *                    through the union of their key blocks together; a row's slack s is the
 *                    number of union blocks it did not select. A row with s >= sasa_trigger
 *                    also keeps the floor(sasa_coef * s) of those blocks that rank highest in
 *                    its routing order (ties to the lower block index); the product is formed
 *                    exactly from the float value. Both rows are augmented from their sets
 *                    before augmentation, so the union (the tile's cost) does not change.
 *  sasa_trigger      smallest slack, in key blocks, at which a row is augmented (>= 0).
 *  frame_exact       frame mode only, 0 or 1. 1: token-exact attention (Sol-Attn's semantics,
 *                    vLLM-Omni article §2.1-§2.2): a query token of frame f attends exactly the
 *                    key tokens of the frames kept for f (its top-k frames, the frames within
 *                    +-frame_window of f, frame 0 when force_first_frame), plus the whole of
 *                    its block-level forced blocks (diagonal, band). The CSR rows are the same
 *                    as with 0; each entry also gets a code in fvattn_csr.col_code, which must
 *                    then be non-NULL. With 0 a kept key block is attended whole.
 * Forced blocks are added after the cut (a union); they do not count toward p or k.
 */
typedef struct {
  int32_t mode;
  float p;
  int32_t force_diag;
  int32_t local_window;
  int32_t frame_len;
  int32_t topk_frames;
  int32_t frame_window;
  int32_t force_first_frame;
  int32_t topk_blocks;
  float sasa_coef;
  int32_t sasa_trigger;
  int32_t frame_exact;
} fvattn_route_cfg;

/*
 * Router output, all device buffers owned by the caller. With nb = ceil(S/64), BH = B*H,
 * ntiles = BH * ceil(nb/2) (a tile is 128 query rows: query blocks 2t and 2t+1 of one head):
 *  row_ptr    int32 [BH*nb + 1]   CSR row offsets; row = bh*nb + i.
 *  col_idx    int32 [col_capacity] selected key blocks of each row, ascending.
 *  col_capacity                   must be >= fvattn_csr_max_nnz(shape).
 *  head_load  int64 [BH]          selected (query block, key block) pairs per head: the unit
 *                                 of the FVAttn runtime load balancer (blog section "RLB").
 *  tile_cost  int32 [ntiles]      distinct key blocks a 128-row tile visits (union of its
 *                                 two rows).
 *  tile_order int32 [ntiles]      tile ids (bh*ceil(nb/2) + t) by cost, largest first, ties
 *                                 by ascending id: the longest-processing-time order in which
 *                                 the attention kernel's persistent CTAs take tiles.
 *  nnz        int64 [1]           total selected pairs (= row_ptr[BH*nb]).
 *  status     int32 [4]           control block: [0] device status (fvattn_status), [1] error
 *                                 detail, [2] tile ticket of the attention scheduler, [3] number
 *                                 of tile_order entries the attention processes (ntiles after
 *                                 fvattn_route; fewer after fvattn_select_heads).
 *  col_code   int32 [col_capacity] or NULL: per-entry token mask of the key block, written by
 *                                 fvattn_route when non-NULL and applied by fvattn_sparse_attn.
 *                                 Bits 0-3: allow[a][b] at bit 2a+b, a = the query block's
 *                                 first (0) or second (1) frame, b the same for the key block
 *                                 (a 64-token block spans at most two frames of >= 64 tokens);
 *                                 bits 8-15: first column of the key block's second frame, bits
 *                                 16-23: first row of the query block's second frame (64 when the
 *                                 block lies in one frame). Outside token-exact frame mode every
 *                                 entry allows all (0x40400F).
 */
typedef struct {
  int32_t* row_ptr;
  int32_t* col_idx;
  int64_t col_capacity;
  int64_t* head_load;
  int32_t* tile_cost;
  int32_t* tile_order;
  int64_t* nnz;
  int32_t* status;
  int32_t* col_code;
} fvattn_csr;

/* Library version, (major << 16) | minor. */
int fvattn_version(void);

/* The cudaError_t code behind the most recent FVATTN_ERR_CUDA returned to the calling thread
 * (0 if none), and the CUDA runtime's name for a code ("cudaErrorInvalidValue", ...). Host only;
 * the name works without a GPU. */
int fvattn_last_cuda_error(void);
const char* fvattn_cuda_error_name(int code);

/* Static text for a status code. Never NULL. */
const char* fvattn_status_string(int status);

/* BH * nb * nb: the largest possible nnz, hence the col_idx capacity to allocate.
 * Returns a negative fvattn_status for an invalid shape. Host only, no CUDA call. */
int64_t fvattn_csr_max_nnz(const fvattn_shape* shape);

/* BH * ceil(nb/2): entries of tile_cost and tile_order. Negative status if invalid. */
int64_t fvattn_num_tiles(const fvattn_shape* shape);

/* Workspace bytes fvattn_route needs for this shape and configuration (block means in
 * fp64, the fp64 block-score matrix in Top-p mode, per-row selection bitmasks and counts).
 * 0 on invalid arguments. Host only. */
size_t fvattn_route_workspace_bytes(const fvattn_shape* shape, const fvattn_route_cfg* cfg);

/*
 * fvattn_route -- the router (FVAttn Top-p, or Sol-Attn frame top-k), all on the device:
 *   1. block means of Q and K over the valid tokens of each 64-token block (notes §5.2),
 *      accumulated exactly enough to be held in fp64;
 *   2. Top-p: scores Sc[i][j] = <Qbar_i, Kbar_j> * scale in fp64, softmax over j, and the
 *      smallest descending-probability prefix whose mass is >= p (ties: lower j first);
 *      fixed top-k: the same scores, the k highest per row (ties: lower j first);
 *      frame mode: frame means, frame scores, top-k frames per query frame, expanded to the
 *      key blocks that hold tokens of a kept frame;
 *   3. union with the forced blocks of cfg; with sasa_coef > 0, slack-aware augmentation of
 *      each 128-row tile; CSR rows (ascending), per-head loads, tile costs and the
 *      longest-first tile order.
 * Q, K: device [B,H,S,d]; out: caller buffers as above; workspace: device, at least
 * fvattn_route_workspace_bytes(shape, cfg) bytes, 256-byte aligned, contents need not be
 * initialised. Returns FVATTN_OK once everything is enqueued on `stream`.
 */
int fvattn_route(const void* Q, const void* K, const fvattn_shape* shape,
                 const fvattn_route_cfg* cfg, const fvattn_csr* out,
                 void* workspace, size_t workspace_bytes, fvattn_stream_t stream);

/*
 * fvattn_route in two stages, so that step 1 can run on parts of the sequence as they arrive
 * (sequence parallelism: the slices of a head come from different ranks):
 *   fvattn_route_pool   -- step 1 (block means: score slices in Top-p / top-k modes, segment
 *                          sums in frame mode) for the blocks [block_begin, block_end) of every
 *                          head, into the workspace; reads only those blocks' tokens of Q and K.
 *                          0 <= block_begin < block_end <= nb, else FVATTN_ERR_INVALID.
 *   fvattn_route_finish -- steps 2 and 3 from a workspace in which every block of every head has
 *                          been pooled (by one or more fvattn_route_pool calls on the same
 *                          shape, cfg and workspace, ordered before it on `stream` or joined to
 *                          it by the caller); writes `out` as fvattn_route does.
 * fvattn_route(Q, K, ...) equals fvattn_route_pool over [0, nb) followed by
 * fvattn_route_finish, bit for bit. Arguments, workspace size and errors as for fvattn_route.
 */
int fvattn_route_pool(const void* Q, const void* K, const fvattn_shape* shape,
                      const fvattn_route_cfg* cfg, int64_t block_begin, int64_t block_end,
                      void* workspace, size_t workspace_bytes, fvattn_stream_t stream);
int fvattn_route_finish(const fvattn_shape* shape, const fvattn_route_cfg* cfg,
                        const fvattn_csr* out, void* workspace, size_t workspace_bytes,
                        fvattn_stream_t stream);

/*
 * fvattn_sparse_attn -- exact softmax attention over the selected key blocks:
 *   O[t] = sum_u softmax_u(Q[t].K[u] * scale) V[u],  u over the tokens (< S) of the key
 *   blocks listed in the CSR row of t's query block.
 * csr: the output of fvattn_route on the same shape (row_ptr, col_idx, tile_order, status
 * are read; status[2] is reset and used as the work ticket). O: device [B,H,S,d], same
 * dtype as Q. lse: optional device float [B,H,S] receiving the natural-log softmax
 * normaliser of each row (NULL to skip). bf16 runs on the tensor cores (tcgen05, fp32
 * accumulation); f32 runs on the CUDA cores in fp32.
 * The CSR is trusted: this library reads the lists the router wrote. Its checked build
 * (libfvattn_debug.so, the same sources compiled with -DFVATTN_DEBUG) checks every row's list
 * before reading it and, on a failure, skips the row's tile and writes FVATTN_ERR_INVALID to
 * status[0] and the check to status[1]: 101 row offsets decreasing or beyond col_capacity,
 * 102 a key block outside [0, nb), 103 a list not strictly ascending. A tile index outside the
 * grid in tile_order is reported as FVATTN_ERR_INVALID (status[1] = 11) by both builds.
 */
int fvattn_sparse_attn(const void* Q, const void* K, const void* V, const fvattn_shape* shape,
                       const fvattn_csr* csr, void* O, float* lse, fvattn_stream_t stream);

/*
 * fvattn_sparse_attn_stamped -- fvattn_sparse_attn (bf16 only) that also records, for every CTA
 * of the persistent attention grid, the SM it ran on and its busy interval: stamps[3c] = SM id,
 * stamps[3c+1] = start, stamps[3c+2] = end (ns of the GPU's global timer). The busy-time
 * imbalance of the SMs (max / mean of max(end) - min(start) over each SM's CTAs) shows how well
 * the tile order balances the work (the single-GPU analogue of the FVAttn summary's RLB
 * imbalance factor). stamps: device uint64, at least fvattn_attn_stamp_words(shape) words
 * (3 per CTA; the grid depends on the current device's SM count, so that call needs a GPU and
 * returns 0 without one or for fp32). Errors as fvattn_sparse_attn, plus FVATTN_ERR_CAPACITY
 * when stamp_words is too small.
 */
int64_t fvattn_attn_stamp_words(const fvattn_shape* shape);
int fvattn_sparse_attn_stamped(const void* Q, const void* K, const void* V, const fvattn_shape* shape,
                               const fvattn_csr* csr, void* O, float* lse, uint64_t* stamps,
                               int64_t stamp_words, fvattn_stream_t stream);

/*
 * fvattn_block_means -- step 1 of fvattn_route on its own: means of X [B,H,S,d] over the
 * valid tokens of each 64-token block, written as fp64 [B,H,nb,d] to `out` (device).
 */
int fvattn_block_means(const void* X, const fvattn_shape* shape, double* out,
                       fvattn_stream_t stream);

/*
 * fvattn_block_scores -- the scores of step 2 of fvattn_route (Top-p and top-k modes) on
 * their own: scores[bh*nb + i][j] = <Qbar_i, Kbar_j> * scale (FVAttn summary: the importance
 * of key block j for query block i; notes §5.2: scaled dot products of block means), Qbar and
 * Kbar the block means of step 1. The means are split into a power-of-two scale 2^e and five
 * signed 8-bit integer slices, multiplied exactly on the tensor cores and combined in fp64;
 * the terms left out are below 2^-30 * 2^(e_i + e_j).
 * Q, K: device [B,H,S,d] as for fvattn_route, 16-byte aligned. scores: device fp64
 * [B*H*nb][ld], ld = fvattn_block_scores_ld(shape) (nb rounded up to a multiple of 32),
 * 16-byte aligned; columns >= nb are not written. workspace: device, 256-byte aligned, at least
 * fvattn_block_scores_workspace_bytes(shape) bytes. status: device int32[4], zeroed on
 * `stream` before the kernels; a kernel that times out writes FVATTN_ERR_TIMEOUT to status[0].
 * Returns FVATTN_OK once everything is enqueued on `stream`; the caller owns every buffer.
 */
size_t fvattn_block_scores_workspace_bytes(const fvattn_shape* shape);
int64_t fvattn_block_scores_ld(const fvattn_shape* shape);
int fvattn_block_scores(const void* Q, const void* K, const fvattn_shape* shape, double* scores,
                        void* workspace, size_t workspace_bytes, int32_t* status,
                        fvattn_stream_t stream);

/*
 * Failure-path checks of the bounded device waits; the pages have no counterpart. Every wait
 * of the tensor-core kernels on a barrier is bounded: when one runs out, the kernel stops
 * issuing work, waits (bounded) for the copies and MMAs it has in flight, frees its tensor
 * memory, writes FVATTN_ERR_TIMEOUT to the status word and returns, so that the context and
 * the stream stay usable. These two calls make that path run on purpose: they launch the
 * kernels of fvattn_sparse_attn (bf16) and of fvattn_block_scores with one extra wait at the
 * start of every CTA on a barrier that nothing completes, bounded by `polls` (>= 1) polls and
 * taken before any copy or MMA is issued. The wait runs out, the kernel returns without
 * writing O (resp. scores), and FVATTN_ERR_TIMEOUT is left in csr->status[0] (resp.
 * status[0]); read it with fvattn_read_status. Arguments otherwise as for the calls they
 * mirror. Returns FVATTN_ERR_INVALID for polls == 0.
 */
int fvattn_sparse_attn_timeout_check(const void* Q, const void* K, const void* V, const fvattn_shape* shape,
                                     const fvattn_csr* csr, void* O, uint32_t polls, fvattn_stream_t stream);
int fvattn_block_scores_timeout_check(const void* Q, const void* K, const fvattn_shape* shape, double* scores,
                                      void* workspace, size_t workspace_bytes, int32_t* status, uint32_t polls,
                                      fvattn_stream_t stream);

/* Synchronises `stream`, then returns the device status word status[0] (FVATTN_OK or a
 * negative fvattn_status written by a kernel). FVATTN_ERR_CUDA if the copy fails. */
int fvattn_read_status(const fvattn_csr* csr, fvattn_stream_t stream);

/*
 * fvattn_rlb_plan -- runtime load balancing of heads across ranks (FVAttn blog summary,
 * section "RLB"), on the host; makes no CUDA call. With the per-head loads of every rank
 * gathered (each rank's fvattn_csr.head_load: selected block pairs per head), it repeatedly
 * takes the most loaded rank as the sender and the least loaded as the receiver and moves the
 * sender's heaviest head whose move keeps the receiver's load below the sender's, until
 * max / mean of the rank loads is <= target_imbalance, the sender has sent
 * max_moves_per_rank heads, or no head of the sender qualifies. Ties go to the lower rank or
 * head index; a head moves at most once. The plan is a pure function of its inputs, so every
 * rank computes the same one.
 *  loads         host int64 [ranks * heads_per_rank]: load of local head h of rank r at
 *                r * heads_per_rank + h (0 <= load <= 2^40).
 *  moves         host int32 [3 * moves_capacity]: (sender rank, sender's local head, receiver
 *                rank) of each move, in plan order; moves_capacity must be at least
 *                ranks * min(max_moves_per_rank, heads_per_rank).
 *  n_moves       host out: number of moves written.
 *  rank_loads    host int64 [ranks] out (may be NULL): the loads after the moves.
 * Returns FVATTN_OK, FVATTN_ERR_INVALID (null pointer, ranks or heads_per_rank < 1, a load
 * out of range, target_imbalance < 1 or not finite, max_moves_per_rank < 0) or
 * FVATTN_ERR_CAPACITY (moves_capacity too small); nothing is written on error.
 */
int fvattn_rlb_plan(const int64_t* loads, int32_t ranks, int32_t heads_per_rank, double target_imbalance,
                    int32_t max_moves_per_rank, int32_t* moves, int64_t moves_capacity, int32_t* n_moves,
                    int64_t* rank_loads);

/*
 * fvattn_select_heads -- restricts the following fvattn_sparse_attn calls on `csr` to the
 * heads bh with active[bh] != 0 (active: device uint8 [B*H]): compacts csr->tile_order in
 * place, keeping the longest-first order of the kept tiles, and sets csr->status[3] to their
 * number. Output rows of the other heads are left untouched. The next fvattn_route on `csr`
 * selects every head again. Under runtime load balancing a rank skips the heads it sends to
 * other ranks this way. One single-CTA kernel on `stream`; an entry of tile_order that is out
 * of range is dropped and reported as FVATTN_ERR_INVALID in the device status.
 */
int fvattn_select_heads(const fvattn_shape* shape, const fvattn_csr* csr, const uint8_t* active,
                        fvattn_stream_t stream);

/*
 * fvattn_route_static_scratch -- fvattn_route without a caller workspace. The pages have no
 * counterpart of this call; it exists for callers that cannot allocate device memory: hosts
 * that own all device memory through their own fixed pool, or plugin interfaces that pass a
 * library only its input and output pointers, leave no way to obtain a workspace.
 *
 * The router's scratch is a static device array of FVATTN_STATIC_SCRATCH_BYTES that every
 * GPU loading the library holds until the process exits; nothing is allocated or freed.
 * Sizes whose fvattn_route_workspace_bytes exceeds it return FVATTN_ERR_CAPACITY (8 MiB
 * covers, e.g., B*H = 12 heads at S = 8192, d = 128 in Top-p mode). The first call on each
 * device looks up the array's device address (cudaGetSymbolAddress, device current); make
 * that first call before any stream capture. The cached address assumes the device is not
 * reset: after cudaDeviceReset the array may be reloaded elsewhere, so a process that resets a
 * device must not call this entry point on it again. All calls share the one array: calls that
 * overlap on the GPU (other streams, other threads) race and must be serialised by the
 * caller. Q, K, shape, cfg, out and stream are as for fvattn_route.
 */
#define FVATTN_STATIC_SCRATCH_BYTES (8u << 20)
int fvattn_route_static_scratch(const void* Q, const void* K, const fvattn_shape* shape,
                                const fvattn_route_cfg* cfg, const fvattn_csr* out,
                                fvattn_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* FVATTN_H */
