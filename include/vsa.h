/*
 * vsa.h - C ABI of libvsa: VSA-style block-sparse video attention, forward
 * pass, for NVIDIA B200 (sm_100a).
 *
 * The method (sources are web pages, cited by title and section):
 *  - A packed sequence [conditioning prefix | generated video] is split into
 *    64-token tiles: conditioning segments (text, reference image, reference
 *    audio) into segment-pure runs, the video latent grid into 4x4x4 cubes.
 *    ("Ref2VA VSA : noeud d'attention sparse pour le Ref2VA H3", section
 *    "Le correctif d'attention a deux niveaux"; "ComfyUI-Ref2VA-VSA",
 *    "Technical Architecture" and "The Solution: Ref2VAVSAGatePatch".)
 *  - A coarse branch mean-pools Q/K/V per tile, scores query tiles against
 *    video key tiles and selects, per query tile, the video key tiles to attend
 *    exactly (fixed keep fraction or per-head adaptive threshold).
 *    ("BSAI FastH3 Native VSA (recipe)", "The mechanism, briefly" and "The
 *    inputs that matter"; "ComfyUI Agrega Nodo Central de Atencion Dispersa y
 *    Compilador Comfy", section "Atencion dispersa por bloques", Sol-Attn,
 *    top-k and VSA bullets.)
 *  - A fine branch attends each query tile exactly to every conditioning key
 *    token plus its selected video tiles; the output is o_fine + g * o_coarse.
 *
 * Conventions for every call:
 *  - The caller owns all device memory. The library never allocates device
 *    memory, never synchronises a stream (except vsa_sparse_attn_status, which
 *    exists to do exactly that) and enqueues all GPU work on the given stream.
 *  - Tensors are bf16 with head_dim 128, addressed by element strides for the
 *    batch, sequence and head dimensions; the head_dim is contiguous.
 *  - Errors are returned, never raised or aborted. VSA_ERR_UNSUPPORTED means
 *    "this library does not run this case; the caller should run dense
 *    attention" (the pages' rule that every ambiguous case runs dense, "BSAI
 *    FastH3 Native VSA (recipe)", "The mechanism, briefly").
 *  - On an error no GPU work has been enqueued, except where VSA_ERR_CUDA
 *    reports a failed launch.
 */
#ifndef VSA_H_
#define VSA_H_

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

#define VSA_TILE 64
#define VSA_HEAD_DIM 128
#define VSA_MAX_SEGMENTS 64
#define VSA_MAX_EXTRA_TOKENS 64

typedef enum {
  VSA_OK = 0,
  VSA_ERR_INVALID_ARG = 1,          /* malformed argument: null pointer, bad size, bad descriptor */
  VSA_ERR_UNSUPPORTED = 2,          /* valid request this library does not run: caller runs dense */
  VSA_ERR_WORKSPACE_TOO_SMALL = 3,  /* workspace_bytes below the size query's answer */
  VSA_ERR_CUDA = 4,                 /* a CUDA runtime call or launch failed */
  VSA_ERR_TIMEOUT = 5,              /* a kernel gave up waiting (reported by vsa_sparse_attn_status) */
  VSA_ERR_NOT_UPLOADED = 6          /* the layout has no device tables (see vsa_layout_upload) */
} vsa_status;

/* Segment kinds of the packed sequence. Every kind except VIDEO is
 * conditioning: never pruned as keys. */
typedef enum {
  VSA_SEG_TEXT = 0,
  VSA_SEG_REF_IMAGE = 1,
  VSA_SEG_REF_AUDIO = 2,
  VSA_SEG_OTHER_COND = 3,
  VSA_SEG_VIDEO = 4
} vsa_seg_kind;

/* One segment of the packed-sequence descriptor: tokens [start, start+length).
 * For VSA_SEG_VIDEO, grid_t * grid_h * grid_w == length and the tokens are the
 * latent grid in raster order (t slowest, w fastest); other kinds ignore the
 * grid fields. */
typedef struct {
  int32_t kind;
  int32_t grid_t, grid_h, grid_w;
  int64_t start;
  int64_t length;
} vsa_segment;

typedef enum { VSA_SELECT_TOPK = 0, VSA_SELECT_ADAPTIVE = 1 } vsa_select_mode;

/* sink_conditioning ("BSAI FastH3 Native VSA (recipe)", "The inputs that
 * matter"): EXACT_KV = every query attends every conditioning key exactly;
 * EXACT_KV_AND_ROWS = in addition, conditioning query rows attend the whole
 * sequence densely (and get no coarse term); OFF = nothing is protected (the
 * pages' cheapest mode; reading): every tile, conditioning or video, is a
 * candidate key tile, scored, selected and summarised like a video tile, and
 * a query attends exactly only the tokens of its selected tiles.
 * Candidate key tiles: the video tiles (ordinal c = tile id - n_cond_tiles)
 * under EXACT_KV and EXACT_KV_AND_ROWS, every tile (ordinal c = tile id) under
 * OFF; Nc below is their number. */
typedef enum { VSA_SINK_EXACT_KV = 0, VSA_SINK_EXACT_KV_AND_ROWS = 1, VSA_SINK_OFF = 2 } vsa_sink_mode;

typedef enum { VSA_OUT_F32 = 0, VSA_OUT_BF16 = 1 } vsa_out_dtype;

/* Compressed (coarse) branch summaries of the candidate key tiles.
 * MEAN: mean-pooled K and V ("Spark-H3: atencion dispersa por bloques ...",
 * "Que cambia Spark-Attn": mean-pooled key/value summary).
 * REWEIGHT: Spark-Reweight (same section; reading): per (batch, head) the
 * anchor a is the mean query of the video tokens; each candidate tile is
 * summarised by the anchor's softmax weights over its tokens,
 * K~ = sum w_i k_i, V~ = sum w_i v_i with w = softmax_i(scale <a, k_i>), plus
 * the log-mass bias b = log(mean_i exp(scale <a, k_i>)) - scale <a, K~>; the
 * branch is o_coarse = softmax_c(scale <Qbar, K~_c> + b_c) V~_c. The
 * selection always uses the mean-pooled scores. */
typedef enum { VSA_COARSE_MEAN = 0, VSA_COARSE_REWEIGHT = 1 } vsa_coarse_mode;

/* Selection parameters.
 *  mode  : VSA_SELECT_TOPK keeps k = max(1, ceil(keep * Nc)) candidate key
 *          tiles per query tile (Nc = number of candidate tiles, see
 *          vsa_sink_mode; the product is taken in double with a relative guard
 *          of 2^-20); ties go to the lower tile.
 *          VSA_SELECT_ADAPTIVE keeps the candidate key tiles whose score is
 *          >= mean + tau * std of that (batch, head)'s whole score matrix
 *          (population std), and at least the row's argmax.
 *  keep  : (0, 1], used by TOPK.
 *  tau   : >= 0, used by ADAPTIVE.
 *  sink  : vsa_sink_mode.
 *  scale : softmax scale of both branches; <= 0 selects 1/sqrt(128).
 *  coarse: vsa_coarse_mode.
 *  extra_tokens: 0, or E in [1, VSA_MAX_EXTRA_TOKENS]: the E best individual
 *          tokens outside a query tile's selected tiles join its exact key set
 *          (see vsa_extra_tokens_select). */
typedef struct {
  int32_t mode;
  float keep;
  float tau;
  int32_t sink;
  float scale;
  int32_t coarse;
  int32_t extra_tokens;
} vsa_params;

typedef struct vsa_layout vsa_layout;   /* opaque; owns its host tables */

typedef struct {
  int64_t seq_len;
  int32_t n_cond_tiles;      /* conditioning tiles: tile ids [0, n_cond_tiles) */
  int32_t n_video_tiles;     /* video tiles: tile ids [n_cond_tiles, n_tiles) */
  int32_t n_tiles;
  int32_t grid_t, grid_h, grid_w;
  int64_t video_start;       /* first token of the video segment */
  size_t device_bytes;       /* bytes vsa_layout_upload needs */
} vsa_layout_info;

/* ------------------------------------------------------------------------ */
/* Geometry map (token -> tile permutation)                                  */
/* ------------------------------------------------------------------------ */

/* vsa_layout_build: builds the geometry map of a packed sequence on the host
 * ("Le correctif d'attention a deux niveaux", item 1: segment-pure tiles; 4x4x4
 * video cubes, "ComfyUI-Ref2VA-VSA", "Technical Architecture").
 *
 *  segs, n_segs : descriptor, segments in sequence order covering
 *                 [0, seq_len) contiguously, 1 <= n_segs <= VSA_MAX_SEGMENTS,
 *                 exactly one VSA_SEG_VIDEO segment. Conditioning segments may
 *                 come before or after the video.
 *  dev_buf      : optional device buffer of at least info.device_bytes bytes;
 *                 when non-NULL the device tables are uploaded into it on
 *                 `stream` (as vsa_layout_upload does). NULL builds the host
 *                 tables only.
 *  out          : receives the handle; free it with vsa_layout_free. The
 *                 caller keeps dev_buf alive while the handle is used.
 * Tile ids: conditioning tiles first (64-token runs of each conditioning
 * segment in descriptor order, the last run of a segment possibly partial),
 * then the video cubes in raster order over (t/4, h/4, w/4); slots of a cube
 * are raster order over (t, h, w), slots outside the grid are padding.
 * Errors: INVALID_ARG for a malformed descriptor; UNSUPPORTED when there is
 * no video segment, more than one, or seq_len >= 2^31 tokens. */
vsa_status vsa_layout_build(const vsa_segment* segs, int32_t n_segs, int64_t seq_len,
                            void* dev_buf, size_t dev_bytes, cudaStream_t stream,
                            vsa_layout** out);

/* Copies the device tables into dev_buf (>= info.device_bytes, 256-byte
 * aligned) with cudaMemcpyAsync on `stream`, and records dev_buf in the
 * handle. The source is pageable host memory: the call returns once the host
 * tables are staged, so the handle may be freed right after; it is a set-up
 * step and must not be issued while `stream` is being captured. */
vsa_status vsa_layout_upload(vsa_layout* layout, void* dev_buf, size_t dev_bytes,
                             cudaStream_t stream);

vsa_status vsa_layout_query(const vsa_layout* layout, vsa_layout_info* info);

/* Host copies of the tables, any pointer may be NULL:
 *  perm       int32 [n_tiles * 64] : token of (tile, slot), -1 for padding
 *  inv        int32 [seq_len]      : tile * 64 + slot of each token
 *  tile_count int32 [n_tiles]      : valid tokens of each tile
 *  tile_kind  int32 [n_tiles]      : vsa_seg_kind of each tile */
vsa_status vsa_layout_copy_tables(const vsa_layout* layout, int32_t* perm, int32_t* inv,
                                  int32_t* tile_count, int32_t* tile_kind);

void vsa_layout_free(vsa_layout* layout);

/* ------------------------------------------------------------------------ */
/* Coarse branch + selection                                                 */
/* ------------------------------------------------------------------------ */

/* kmax: the row length of the index list (k for TOPK, Nc for ADAPTIVE; Nc =
 * number of candidate key tiles of the sink mode). */
vsa_status vsa_select_kmax(const vsa_layout* layout, const vsa_params* params, int32_t* kmax);

vsa_status vsa_coarse_select_workspace_size(const vsa_layout* layout, int32_t B, int32_t H,
                                            const vsa_params* params, size_t* bytes);

/* vsa_coarse_select: the coarse branch and the block selection
 * ("BSAI FastH3 Native VSA (recipe)", "The mechanism, briefly": scores the
 * blocks and keeps the top slice; "ComfyUI Agrega Nodo Central ...", VSA
 * bullet: coarse compression branch; Sol-Attn bullet: adaptive threshold).
 *
 *  q, k, v        : bf16 [B, S, H, 128] at element strides (stride_b,
 *                   stride_s, stride_h); 16-byte aligned, strides multiples
 *                   of 8.
 *  idx            : int32 [B, H, n_tiles, kmax] out: per query tile the
 *                   selected candidate key tiles as candidate ordinals in
 *                   [0, Nc) (see vsa_sink_mode), ascending; entries past cnt
 *                   are left unspecified.
 *  cnt            : int32 [B, H, n_tiles] out: list lengths.
 *  o_coarse       : float [B, H, n_tiles, 128] out, with COARSE_MEAN:
 *                   sum_c softmax_c(s[qt, c]) * mean(V of candidate tile c),
 *                   s[qt, c] = scale * <mean Q of tile qt, mean K of tile c>
 *                   (the scores the selection uses); with COARSE_REWEIGHT the
 *                   Spark-Reweight form of vsa_coarse_mode.
 *  workspace      : device scratch of vsa_coarse_select_workspace_size bytes,
 *                   256-byte aligned. Bytes [0, 256) hold the call's status
 *                   word and the count of failed calls (see
 *                   vsa_coarse_select_workspace_init); from byte 256,
 *                   3*B*H*n_tiles*128 floats hold the pooled means
 *                   [3 (q,k,v), B, H, n_tiles, 128] after the call.
 * All query tiles are processed, conditioning tiles included (under
 * EXACT_KV_AND_ROWS their lists are ignored by vsa_sparse_attn_fwd).
 * Pooling is fp32. With COARSE_MEAN the scores and the coarse softmax run on
 * the tensor cores with each fp32 mean split into two bf16 terms (three
 * products, fp32 accumulation: fp32-class error), the score matrix stays on
 * chip, and the kernels wait on their own copies and MMAs with bounded waits
 * (VSA_ERR_TIMEOUT in vsa_coarse_select_status when one runs out; the lists
 * are then incomplete, but every consumer in this library clamps list
 * lengths and entries, so nothing reads out of bounds). With COARSE_REWEIGHT
 * they are fp32 FMA. Adaptive mean/std accumulate in fp64. At most 65535
 * candidate tiles with COARSE_MEAN (VSA_ERR_UNSUPPORTED beyond). */
vsa_status vsa_coarse_select(const vsa_layout* layout, const vsa_params* params,
                             int32_t B, int32_t H,
                             const void* q, const void* k, const void* v,
                             int64_t stride_b, int64_t stride_s, int64_t stride_h,
                             int32_t* idx, int32_t* cnt, float* o_coarse,
                             void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* vsa_coarse_select_noalloc: vsa_coarse_select without a workspace argument.
 * The web pages describe no such call; it exists for callers that cannot give
 * this library scratch memory: a host framework that plans every device
 * allocation in advance and allows none outside its plan, or a caller that
 * cannot afford the synchronisation and latency of cudaMalloc inside a step.
 *
 * Same arguments, outputs and results as vsa_coarse_select, minus workspace.
 * The scratch (status words, pooled means, split chunks, marks; the score
 * matrix with COARSE_REWEIGHT) is a fixed 32 MiB buffer inside the library's
 * device image, held by every GPU that loads the library until the process
 * exits. Shapes whose scratch exceeds 32 MiB (vsa_coarse_select_workspace_size
 * of the same shape; the 17k-token, 24-head workload fits, the 1344x768
 * shapes do not) are refused with VSA_ERR_UNSUPPORTED and a message in
 * vsa_last_error_detail. The first call on a device looks up the buffer's
 * device address (once per device, with that device current); make that
 * first call before any stream capture, and do not call it after a
 * cudaDeviceReset of that device (the cached address belongs to the old
 * context). Every call on a device shares the one buffer and leaves its
 * contents behind; each call writes every scratch byte it later reads, so
 * nothing needs clearing, but calls that overlap on the GPU (different
 * streams, or concurrent host threads) race on the buffer. Allocates no
 * memory of any kind. */
vsa_status vsa_coarse_select_noalloc(const vsa_layout* layout, const vsa_params* params,
                                     int32_t B, int32_t H,
                                     const void* q, const void* k, const void* v,
                                     int64_t stride_b, int64_t stride_s, int64_t stride_h,
                                     int32_t* idx, int32_t* cnt, float* o_coarse,
                                     cudaStream_t stream);

/* Zeroes the selection workspace's header, including the count of failed
 * calls that vsa_coarse_select_failed_calls reports. Call once after
 * allocating a workspace. No counterpart on the pages. */
vsa_status vsa_coarse_select_workspace_init(void* workspace, cudaStream_t stream);

/* Synchronises `stream` and reads the status word the most recent
 * vsa_coarse_select on `workspace` left: VSA_OK or VSA_ERR_TIMEOUT (a bounded
 * wait ran out; the lists and o_coarse are incomplete). No counterpart on
 * the pages. */
vsa_status vsa_coarse_select_status(const void* workspace, cudaStream_t stream);

/* Synchronises `stream` and reads how many vsa_coarse_select calls on
 * `workspace` recorded an error since vsa_coarse_select_workspace_init. */
vsa_status vsa_coarse_select_failed_calls(const void* workspace, cudaStream_t stream, uint32_t* count);

/* vsa_coarse_select_status for the built-in buffer of
 * vsa_coarse_select_noalloc on the current device. */
vsa_status vsa_coarse_select_noalloc_status(cudaStream_t stream);

/* ------------------------------------------------------------------------ */
/* extra_tokens                                                              */
/* ------------------------------------------------------------------------ */

vsa_status vsa_extra_tokens_workspace_size(const vsa_layout* layout, int32_t B, int32_t H,
                                           const vsa_params* params, size_t* bytes);

/* vsa_extra_tokens_select: the extra key tokens of every query tile
 * ("ComfyUI Agrega Nodo Central de Atencion Dispersa y Compilador Comfy",
 * section "Atencion dispersa por bloques": extra_tokens adds the best-scoring
 * tokens beyond the selected blocks, to stay closer to dense attention).
 * Reading: for a query tile qt attended sparsely (every tile except dense
 * conditioning rows under EXACT_KV_AND_ROWS), the candidate tokens are the
 * valid tokens of the candidate key tiles qt did not select; token i scores
 * scale * <mean Q of tile qt, k_i>; the E = params->extra_tokens highest, ties
 * to the lower token index, are chosen (fewer when fewer candidates exist).
 *
 *  q, k, strides  : as vsa_coarse_select (v is not read).
 *  idx, cnt, kmax : the lists of vsa_coarse_select with the same params.
 *  extra_idx      : int32 [B, H, n_tiles, E] out: token indices, unordered;
 *                   entries past extra_cnt unspecified.
 *  extra_cnt      : int32 [B, H, n_tiles] out: number of tokens chosen (0 for
 *                   dense conditioning rows).
 *  workspace      : vsa_extra_tokens_workspace_size bytes, 256-byte aligned;
 *                   its first word is the status that vsa_extra_tokens_status
 *                   reads (a kernel wait that ran out).
 * Scores: fp32 accumulation of the exact bf16 keys against the fp32 pooled
 * query split into two bf16 terms (tensor cores; the query to a relative
 * 2^-17), so the chosen set matches an fp64 evaluation except where two
 * scores tie within about fp32 rounding.
 * Errors: INVALID_ARG when params->extra_tokens is 0 (nothing to choose);
 * UNSUPPORTED when a bitmap of the candidate tiles, two top-E lists and one
 * 32 KB key stage per 128 query tiles exceed 227 KB of shared memory (more
 * than about 10k candidate tiles at E = 16, 4.2k at E = 64). */
vsa_status vsa_extra_tokens_select(const vsa_layout* layout, const vsa_params* params,
                                   int32_t B, int32_t H, const void* q, const void* k,
                                   int64_t stride_b, int64_t stride_s, int64_t stride_h,
                                   const int32_t* idx, const int32_t* cnt, int32_t kmax,
                                   int32_t* extra_idx, int32_t* extra_cnt,
                                   void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* Synchronises `stream` and reads the status word a previous
 * vsa_extra_tokens_select left in `workspace`: VSA_OK or VSA_ERR_TIMEOUT. No
 * counterpart on the pages (error reporting of this library). */
vsa_status vsa_extra_tokens_status(const void* workspace, cudaStream_t stream);

/* ------------------------------------------------------------------------ */
/* Fine branch + gate combine                                                */
/* ------------------------------------------------------------------------ */

vsa_status vsa_sparse_attn_workspace_size(const vsa_layout* layout, int32_t B, int32_t H,
                                          const vsa_params* params, size_t* bytes);

/* vsa_sparse_attn_fwd: exact attention of every query tile over all
 * conditioning key tokens plus the video tiles of its list (EXACT_KV), or over
 * the whole sequence for conditioning query tiles (EXACT_KV_AND_ROWS), or over
 * the tiles of its list only (OFF), then out = o_fine + g * o_coarse[tile] (no
 * coarse term on dense conditioning rows).
 * ("BSAI FastH3 Native VSA (recipe)", "The inputs that matter",
 * sink_conditioning; "ComfyUI-Ref2VA-VSA", "Video-Only Sparse Attention".)
 *
 *  q, k, v, strides : as for vsa_coarse_select.
 *  g                : bf16 gate at element strides g_stride_b, _s, _h, _d:
 *                     [B, S, H] with g_stride_d = 0 (one gate per token and
 *                     head, broadcast over head_dim), or [B, S, H, 128] with
 *                     g_stride_d > 0 (one gate per channel, the output of a
 *                     to_gate_compress projection: "ComfyUI-Ref2VA-VSA",
 *                     "Technical Architecture").
 *  idx, cnt, kmax   : lists from vsa_coarse_select (same params).
 *  o_coarse         : float [B, H, n_tiles, 128] from vsa_coarse_select.
 *  extra_idx,       : the lists of vsa_extra_tokens_select (same params) when
 *  extra_cnt          params->extra_tokens > 0, else NULL; a query tile's
 *                     extra tokens join its exact key set.
 *  out              : [B, S, H, 128] of out_dtype (vsa_out_dtype) at element
 *                     strides out_stride_*, head_dim contiguous; every valid
 *                     token row is written.
 *  workspace        : vsa_sparse_attn_workspace_size bytes, 256-byte aligned.
 *                     A 256-byte header holds this call's status word
 *                     (cleared by the call) and a count of failed calls
 *                     (see vsa_sparse_attn_workspace_init); the rest is
 *                     written by the call before use: a tile-major copy of K
 *                     and V (32 KB per (batch, head, tile); 1.64 GB for the
 *                     24-head 133,696-token shape) and the key-tile schedule
 *                     of every query tile (8 bytes per key tile; about 0.1 GB
 *                     for that shape).
 * Softmax statistics and accumulation are fp32; the probabilities enter the
 * second tensor-core product as bf16. A kernel wait that runs out is recorded
 * in the workspace and reported by vsa_sparse_attn_status. */
vsa_status vsa_sparse_attn_fwd(const vsa_layout* layout, const vsa_params* params,
                               int32_t B, int32_t H,
                               const void* q, const void* k, const void* v,
                               int64_t stride_b, int64_t stride_s, int64_t stride_h,
                               const void* g, int64_t g_stride_b, int64_t g_stride_s,
                               int64_t g_stride_h, int64_t g_stride_d,
                               const int32_t* idx, const int32_t* cnt, int32_t kmax,
                               const float* o_coarse,
                               const int32_t* extra_idx, const int32_t* extra_cnt,
                               void* out, int32_t out_dtype, int64_t out_stride_b,
                               int64_t out_stride_s, int64_t out_stride_h,
                               void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* Zeroes the workspace header, including the count of failed calls that
 * vsa_sparse_attn_failed_calls reads (enqueued on `stream`). Call it once
 * after allocating a workspace; the count is meaningless until then. No
 * counterpart on the pages (error reporting of this library). */
vsa_status vsa_sparse_attn_workspace_init(void* workspace, cudaStream_t stream);

/* Synchronises `stream` and reads, into *count, how many vsa_sparse_attn_fwd
 * calls on this workspace recorded an error (a bounded wait that ran out)
 * since vsa_sparse_attn_workspace_init. Unlike vsa_sparse_attn_status it sees
 * a failure of any earlier call, not only the latest one. */
vsa_status vsa_sparse_attn_failed_calls(const void* workspace, cudaStream_t stream, uint32_t* count);

/* ------------------------------------------------------------------------ */
/* Backward pass                                                             */
/* ------------------------------------------------------------------------ */

vsa_status vsa_sparse_attn_bwd_workspace_size(const vsa_layout* layout, int32_t B, int32_t H,
                                              const vsa_params* params, size_t* bytes);

/* vsa_sparse_attn_bwd: gradients of sum(out * dout) with respect to q, k, v
 * and g, for the forward of vsa_coarse_select + vsa_sparse_attn_fwd with the
 * same params, the block selection held fixed (piecewise constant in the
 * inputs). The pages train and distil checkpoints against these modes ("BSAI
 * FastH3 Native VSA (recipe)"; "ComfyUI-Ref2VA-VSA", "The Solution:
 * Ref2VAVSAGatePatch") without spelling the backward out; this is the exact
 * derivative of the forward: the fine branch's attention backward over each
 * query tile's key set, the gate's product rule, and the coarse branch's
 * tile-level softmax backward flowing back through the mean pooling.
 *
 *  q, k, v, strides : as vsa_coarse_select; g and its strides as
 *                     vsa_sparse_attn_fwd.
 *  idx, cnt, kmax   : the lists of vsa_coarse_select (same params).
 *  o_coarse         : the o_coarse of vsa_coarse_select.
 *  dout             : bf16 [B, S, H, 128] at element strides dout_stride_*.
 *  dq, dk, dv       : fp32 [B, S, H, 128] out at element strides
 *                     grad_stride_* (16-byte multiples), every token written.
 *  dg               : fp32 out shaped like g ([B, S, H] with dg_stride_d = 0,
 *                     or [B, S, H, 128] with dg_stride_d > 0, as g).
 *  workspace        : vsa_sparse_attn_bwd_workspace_size bytes, 256-byte aligned.
 * Errors: UNSUPPORTED for the Spark-Reweight coarse branch and for
 * extra_tokens > 0 (not differentiated on the GPU). A kernel wait that runs
 * out is reported by vsa_sparse_attn_bwd_status. */
vsa_status vsa_sparse_attn_bwd(const vsa_layout* layout, const vsa_params* params,
                               int32_t B, int32_t H, const void* q, const void* k, const void* v,
                               int64_t stride_b, int64_t stride_s, int64_t stride_h,
                               const void* g, int64_t g_stride_b, int64_t g_stride_s,
                               int64_t g_stride_h, int64_t g_stride_d,
                               const int32_t* idx, const int32_t* cnt, int32_t kmax,
                               const float* o_coarse, const void* dout, int64_t dout_stride_b,
                               int64_t dout_stride_s, int64_t dout_stride_h,
                               float* dq, float* dk, float* dv, int64_t grad_stride_b,
                               int64_t grad_stride_s, int64_t grad_stride_h,
                               float* dg, int64_t dg_stride_b, int64_t dg_stride_s,
                               int64_t dg_stride_h, int64_t dg_stride_d,
                               void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* Synchronises `stream` and reads the status a previous vsa_sparse_attn_bwd
 * left in `workspace`: VSA_OK or VSA_ERR_TIMEOUT. No counterpart on the pages
 * (error reporting of this library). */
vsa_status vsa_sparse_attn_bwd_status(const void* workspace, cudaStream_t stream);

/* Synchronises `stream` and reads the error word a previous
 * vsa_sparse_attn_fwd left in `workspace`: VSA_OK, VSA_ERR_TIMEOUT (a bounded
 * wait in the kernel ran out; the output is incomplete) or VSA_ERR_CUDA. */
vsa_status vsa_sparse_attn_status(const void* workspace, cudaStream_t stream);

/* vsa_debug_inject_wait_timeout: failure-injection hook for tests (no
 * counterpart on the pages). While timeout_ns > 0, every vsa_sparse_attn_fwd
 * of this process makes its MMA-issue warp wait, before any work, on a barrier
 * that nothing arrives on, bounded by timeout_ns: the wait runs out, the kernel
 * takes its abort path (drains its copies and MMAs, frees tensor memory, exits)
 * and vsa_sparse_attn_status reports VSA_ERR_TIMEOUT; the output is not
 * written. Nothing faults, traps or hangs, and the CUDA context stays usable.
 * timeout_ns = 0 disarms it. Always returns VSA_OK. */
vsa_status vsa_debug_inject_wait_timeout(uint64_t timeout_ns);

/* vsa_debug_inject_select_wait_timeout: the same hook for the tensor-core
 * kernels of vsa_coarse_select (COARSE_MEAN): while timeout_ns > 0 their
 * MMA-issue warp first waits on a barrier nothing arrives on, bounded by
 * timeout_ns, and vsa_coarse_select_status reports VSA_ERR_TIMEOUT.
 * timeout_ns = 0 disarms it. Always returns VSA_OK. */
vsa_status vsa_debug_inject_select_wait_timeout(uint64_t timeout_ns);

const char* vsa_status_string(vsa_status status);

/* Text of the most recent VSA_ERR_CUDA returned on the calling thread (the
 * failing runtime call and CUDA's error string), or of a shape refused by
 * vsa_coarse_select_noalloc; "" if none yet. The pointer stays valid until
 * the thread's next failing call. */
const char* vsa_last_error_detail(void);

/* Library ABI version, (major << 16) | minor. */
int32_t vsa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* VSA_H_ */
