// Internal definitions shared by the host layout builder and the kernels.
#pragma once

#include <cstddef>
#include <cstdint>
#include <vector>

#include "vsa.h"

namespace vsa {

constexpr int kTile = VSA_TILE;       // tokens per tile
constexpr int kCube = 4;              // 4x4x4 video cubes
constexpr int kHeadDim = VSA_HEAD_DIM;

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Device copy of the geometry map. All arrays live in one caller-owned buffer.
//  perm   [n_tiles*64]  token of (tile, slot), -1 for padding
//  inv    [seq_len]     tile*64 + slot of each token
//  valid  [n_tiles]     bit s set <=> slot s holds a token
//  count  [n_tiles]     popcount(valid)
//  origin [n_tiles]     conditioning tile: (first token, 0, 0, kind)
//                       video tile:        (t0, h0, w0, VSA_SEG_VIDEO)
struct DevLayout {
  const int32_t* perm;
  const int32_t* inv;
  const unsigned long long* valid;
  const int32_t* count;
  const int4* origin;
  int32_t n_cond;
  int32_t n_video;
  int32_t n_tiles;
  int32_t grid_t, grid_h, grid_w;
  int64_t video_start;
  int64_t seq_len;
};

struct TablesOffsets {
  size_t perm, inv, valid, count, origin, total;
};

}  // namespace vsa

struct vsa_layout {
  int64_t seq_len = 0;
  int32_t n_cond = 0, n_video = 0, n_tiles = 0;
  int32_t grid_t = 0, grid_h = 0, grid_w = 0;
  int64_t video_start = 0;
  std::vector<int32_t> perm, inv, count, kind;
  std::vector<unsigned long long> valid;
  std::vector<int32_t> origin;   // 4 per tile
  vsa::TablesOffsets off{};
  void* dev_buf = nullptr;       // caller-owned, set by vsa_layout_upload

  vsa::DevLayout dev() const {
    const char* b = static_cast<const char*>(dev_buf);
    vsa::DevLayout d;
    d.perm = reinterpret_cast<const int32_t*>(b + off.perm);
    d.inv = reinterpret_cast<const int32_t*>(b + off.inv);
    d.valid = reinterpret_cast<const unsigned long long*>(b + off.valid);
    d.count = reinterpret_cast<const int32_t*>(b + off.count);
    d.origin = reinterpret_cast<const int4*>(b + off.origin);
    d.n_cond = n_cond;
    d.n_video = n_video;
    d.n_tiles = n_tiles;
    d.grid_t = grid_t;
    d.grid_h = grid_h;
    d.grid_w = grid_w;
    d.video_start = video_start;
    d.seq_len = seq_len;
    return d;
  }
};

namespace vsa {

// k for top-k selection: max(1, ceil(keep * Nc * (1 - 2^-20))), clamped to Nc.
int32_t topk_count(float keep, int32_t n_cand);

// Candidate key tiles of a sink mode: the video tiles, or every tile with
// VSA_SINK_OFF. Candidate ordinal c is tile id first + c.
struct Candidates {
  int32_t first, count;
};
inline Candidates candidates(const vsa_layout* L, int32_t sink) {
  return sink == VSA_SINK_OFF ? Candidates{0, L->n_tiles} : Candidates{L->n_cond, L->n_video};
}

// Records "where: cuda error string" for vsa_last_error_detail and returns
// VSA_ERR_CUDA; a message-only variant for failures without a cudaError_t.
vsa_status cuda_fail(const char* where, cudaError_t e);
vsa_status cuda_fail(const char* where);
// Records a message for vsa_last_error_detail without a CUDA error.
void set_detail(const char* msg);

// Validation shared by the entry points.
vsa_status check_params(const vsa_params* p);
float effective_scale(const vsa_params* p);
vsa_status check_qkv(const void* q, const void* k, const void* v, int64_t sb, int64_t ss,
                     int64_t sh, int32_t B, int32_t H);

// Workspace layout of vsa_coarse_select. Bytes [0, 256): status word and
// count of failed calls; the pooled means [3, B, H, n_tiles, 128] fp32 follow.
// VSA_COARSE_MEAN runs the tensor-core kernels (vsa_select_tc.cu): Kbar and
// Vbar split into hi/lo bf16 chunks of 64 candidates (32 KB per chunk:
// [term][d half][64][128 B], 128-byte swizzled), per-query-tile max score and
// its candidate, per-block adaptive sums, and per-query-tile selection marks.
// VSA_COARSE_REWEIGHT runs the fp32 kernels of vsa_select.cu over a score
// matrix in the workspace.
constexpr size_t kSelectHeader = 256;
struct SelectWorkspace {
  size_t pooled, scores, stats, total;
  size_t anchor, summaries, bias;   // VSA_COARSE_REWEIGHT only: [B,H,128], [2,B,H,Nc,128], [B,H,Nc]
  size_t ksplit, vsplit, rowmax, rowarg, bits;   // VSA_COARSE_MEAN only
  int32_t n_row_blocks;   // query-tile blocks: 64 per block (fp32 kernels), 128 (tensor-core kernels)
  int32_t ld_scores;      // score row stride: Nc rounded up to 64
  int32_t n_chunks;       // 64-candidate chunks
};
SelectWorkspace select_workspace(const vsa_layout* L, int32_t B, int32_t H, const vsa_params* p);

// The tensor-core coarse branch + selection (VSA_COARSE_MEAN), after the
// pooling kernel filled the pooled means and the split chunks of `ws`.
vsa_status select_tc(const vsa_layout* L, const vsa_params* p, int32_t B, int32_t H, const SelectWorkspace& ws,
                     void* workspace, int32_t* idx, int32_t* cnt, float* o_coarse, uint64_t stall_ns,
                     cudaStream_t stream);
size_t select_tc_smem_bytes();

// Statistics the backward pass needs from a forward call: per query row
// ([B, H, n_tiles, 64], +inf for padding rows) the log2-sum-exp2 of the fine
// branch's scaled logits and D = <dO, o_fine>.
struct AttnStats {
  float* lse;
  float* d;
  const void* dout;          // dO bf16 [B, S, H, 128] at element strides
  int64_t d_sb, d_ss, d_sh;
};

// vsa_sparse_attn_fwd, or with `stats` its statistics instead of the output.
vsa_status attn_forward(const vsa_layout* L, const vsa_params* p, int32_t B, int32_t H, const void* q,
                        const void* k, const void* v, int64_t sb, int64_t ss, int64_t sh, const void* g,
                        int64_t g_sb, int64_t g_ss, int64_t g_sh, int64_t g_sd, const int32_t* idx,
                        const int32_t* cnt, int32_t kmax, const float* o_coarse, const int32_t* extra_idx,
                        const int32_t* extra_cnt, void* out, int32_t out_dtype, int64_t o_sb, int64_t o_ss,
                        int64_t o_sh, const AttnStats* stats, void* workspace, size_t workspace_bytes,
                        cudaStream_t stream);

}  // namespace vsa
