// Geometry mapper: packed [conditioning | video] sequence -> segment-pure tiles.
//
// Conditioning segments (text, reference image, reference audio, ...) are cut
// into contiguous 64-token runs that never cross a segment boundary; the video
// latent grid is cut into 4x4x4 cubes ("Ref2VA VSA : noeud d'attention sparse
// pour le Ref2VA H3", section "Le correctif d'attention a deux niveaux", item 1;
// "ComfyUI-Ref2VA-VSA", sections "Technical Architecture" and "The Solution").
// The map is integer-only and tiny (a few MB at 250k tokens), so it is built on
// the host once per shape and uploaded into caller-owned device memory.

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <new>

#include <cuda_runtime_api.h>

#include "vsa_internal.h"

namespace vsa {

namespace {
thread_local char g_detail[256] = "";
}

vsa_status cuda_fail(const char* where, cudaError_t e) {
  std::snprintf(g_detail, sizeof(g_detail), "%s: %s", where, cudaGetErrorString(e));
  return VSA_ERR_CUDA;
}

vsa_status cuda_fail(const char* where) {
  std::snprintf(g_detail, sizeof(g_detail), "%s", where);
  return VSA_ERR_CUDA;
}

void set_detail(const char* msg) { std::snprintf(g_detail, sizeof(g_detail), "%s", msg); }

int32_t topk_count(float keep, int32_t n_cand) {
  const double prod = static_cast<double>(keep) * static_cast<double>(n_cand) *
                      (1.0 - 1.0 / 1048576.0);
  double k = std::ceil(prod);
  if (k < 1.0) k = 1.0;
  if (k > n_cand) k = n_cand;
  return static_cast<int32_t>(k);
}

vsa_status check_params(const vsa_params* p) {
  if (!p) return VSA_ERR_INVALID_ARG;
  if (p->mode != VSA_SELECT_TOPK && p->mode != VSA_SELECT_ADAPTIVE) return VSA_ERR_INVALID_ARG;
  if (p->sink != VSA_SINK_EXACT_KV && p->sink != VSA_SINK_EXACT_KV_AND_ROWS && p->sink != VSA_SINK_OFF)
    return VSA_ERR_INVALID_ARG;
  if (p->mode == VSA_SELECT_TOPK && !(p->keep > 0.0f && p->keep <= 1.0f)) return VSA_ERR_INVALID_ARG;
  if (p->mode == VSA_SELECT_ADAPTIVE && !(p->tau >= 0.0f && std::isfinite(p->tau)))
    return VSA_ERR_INVALID_ARG;
  if (!std::isfinite(p->scale)) return VSA_ERR_INVALID_ARG;
  if (p->coarse != VSA_COARSE_MEAN && p->coarse != VSA_COARSE_REWEIGHT) return VSA_ERR_INVALID_ARG;
  if (p->extra_tokens < 0 || p->extra_tokens > VSA_MAX_EXTRA_TOKENS) return VSA_ERR_INVALID_ARG;
  return VSA_OK;
}

float effective_scale(const vsa_params* p) {
  return p->scale > 0.0f ? p->scale : static_cast<float>(1.0 / std::sqrt(static_cast<double>(kHeadDim)));
}

vsa_status check_qkv(const void* q, const void* k, const void* v, int64_t sb, int64_t ss,
                     int64_t sh, int32_t B, int32_t H) {
  if (!q || !k || !v) return VSA_ERR_INVALID_ARG;
  if (B <= 0 || H <= 0) return VSA_ERR_INVALID_ARG;
  if (sb < 0 || ss <= 0 || sh <= 0) return VSA_ERR_INVALID_ARG;
  // 16-byte rows: TMA and vector loads need 16-byte aligned bases and strides.
  for (const void* p : {q, k, v})
    if (reinterpret_cast<uintptr_t>(p) % 16) return VSA_ERR_INVALID_ARG;
  if (sb % 8 || ss % 8 || sh % 8) return VSA_ERR_INVALID_ARG;
  if (sh < kHeadDim && H > 1) return VSA_ERR_INVALID_ARG;
  return VSA_OK;
}

SelectWorkspace select_workspace(const vsa_layout* L, int32_t B, int32_t H, const vsa_params* p) {
  SelectWorkspace w{};
  const size_t bh = static_cast<size_t>(B) * H;
  const size_t nt = static_cast<size_t>(L->n_tiles);
  const int32_t nc = candidates(L, p->sink).count;
  const bool tc = p->coarse == VSA_COARSE_MEAN;
  w.n_row_blocks = tc ? (L->n_tiles + 127) / 128 : (L->n_tiles + 63) / 64;
  w.ld_scores = (nc + 63) / 64 * 64;
  w.n_chunks = (nc + 63) / 64;
  size_t off = kSelectHeader;
  w.pooled = off;
  off = align_up(off + 3 * bh * nt * kHeadDim * sizeof(float), 256);
  w.stats = off;
  off = align_up(off + bh * w.n_row_blocks * 2 * sizeof(double), 256);
  w.scores = w.anchor = w.summaries = w.bias = off;
  w.ksplit = w.vsplit = w.rowmax = w.rowarg = w.bits = off;
  if (tc) {
    const size_t chunks = bh * static_cast<size_t>(w.n_chunks) * 32768u;
    w.ksplit = off;
    off = align_up(off + chunks, 256);
    w.vsplit = off;
    off = align_up(off + chunks, 256);
    w.rowmax = off;
    off = align_up(off + bh * nt * sizeof(float), 256);
    w.rowarg = off;
    off = align_up(off + bh * nt * sizeof(int32_t), 256);
    w.bits = off;
    off = align_up(off + bh * nt * 2 * static_cast<size_t>(w.n_chunks) * sizeof(uint32_t), 256);
  } else {
    w.scores = off;
    off = align_up(off + bh * nt * static_cast<size_t>(w.ld_scores) * sizeof(float), 256);
    w.anchor = off;
    off = align_up(off + bh * kHeadDim * sizeof(float), 256);
    w.summaries = off;
    off = align_up(off + 2 * bh * static_cast<size_t>(nc) * kHeadDim * sizeof(float), 256);
    w.bias = off;
    off = align_up(off + bh * static_cast<size_t>(nc) * sizeof(float), 256);
  }
  w.total = off;
  return w;
}

static TablesOffsets tables_offsets(const vsa_layout* L) {
  TablesOffsets o{};
  size_t off = 0;
  o.perm = off;
  off = align_up(off + sizeof(int32_t) * static_cast<size_t>(L->n_tiles) * kTile, 256);
  o.inv = off;
  off = align_up(off + sizeof(int32_t) * static_cast<size_t>(L->seq_len), 256);
  o.valid = off;
  off = align_up(off + sizeof(unsigned long long) * L->n_tiles, 256);
  o.count = off;
  off = align_up(off + sizeof(int32_t) * L->n_tiles, 256);
  o.origin = off;
  off = align_up(off + sizeof(int32_t) * 4 * L->n_tiles, 256);
  o.total = off;
  return o;
}

}  // namespace vsa

using namespace vsa;

extern "C" {

vsa_status vsa_layout_build(const vsa_segment* segs, int32_t n_segs, int64_t seq_len,
                            void* dev_buf, size_t dev_bytes, cudaStream_t stream,
                            vsa_layout** out) {
  if (!out) return VSA_ERR_INVALID_ARG;
  *out = nullptr;
  if (!segs || n_segs < 1 || n_segs > VSA_MAX_SEGMENTS || seq_len <= 0) return VSA_ERR_INVALID_ARG;
  int64_t pos = 0;
  int n_video = 0, vi = -1;
  for (int i = 0; i < n_segs; ++i) {
    const vsa_segment& s = segs[i];
    if (s.start != pos || s.length <= 0) return VSA_ERR_INVALID_ARG;
    if (s.kind < VSA_SEG_TEXT || s.kind > VSA_SEG_VIDEO) return VSA_ERR_INVALID_ARG;
    if (s.kind == VSA_SEG_VIDEO) {
      if (s.grid_t <= 0 || s.grid_h <= 0 || s.grid_w <= 0) return VSA_ERR_INVALID_ARG;
      if (static_cast<int64_t>(s.grid_t) * s.grid_h * s.grid_w != s.length) return VSA_ERR_INVALID_ARG;
      ++n_video;
      vi = i;
    }
    pos += s.length;
  }
  if (pos != seq_len) return VSA_ERR_INVALID_ARG;
  if (n_video != 1) return VSA_ERR_UNSUPPORTED;           // nothing to sparsify: run dense
  if (seq_len >= (int64_t(1) << 31)) return VSA_ERR_UNSUPPORTED;

  vsa_layout* L = new (std::nothrow) vsa_layout;
  if (!L) return VSA_ERR_INVALID_ARG;
  L->seq_len = seq_len;
  const vsa_segment& vs = segs[vi];
  L->grid_t = vs.grid_t;
  L->grid_h = vs.grid_h;
  L->grid_w = vs.grid_w;
  L->video_start = vs.start;

  // Conditioning tiles: 64-token runs per segment, in descriptor order.
  for (int i = 0; i < n_segs; ++i) {
    const vsa_segment& s = segs[i];
    if (s.kind == VSA_SEG_VIDEO) continue;
    for (int64_t r0 = 0; r0 < s.length; r0 += kTile) {
      const int n = static_cast<int>(std::min<int64_t>(kTile, s.length - r0));
      unsigned long long mask = 0;
      for (int j = 0; j < kTile; ++j) {
        if (j < n) {
          L->perm.push_back(static_cast<int32_t>(s.start + r0 + j));
          mask |= 1ull << j;
        } else {
          L->perm.push_back(-1);
        }
      }
      L->valid.push_back(mask);
      L->count.push_back(n);
      L->kind.push_back(s.kind);
      L->origin.insert(L->origin.end(), {static_cast<int32_t>(s.start + r0), 0, 0, s.kind});
    }
  }
  L->n_cond = static_cast<int32_t>(L->count.size());

  // Video cubes in raster order over (t/4, h/4, w/4); slots raster over (t, h, w).
  const int T = vs.grid_t, Hg = vs.grid_h, Wg = vs.grid_w;
  const int na = (T + kCube - 1) / kCube, nb = (Hg + kCube - 1) / kCube, nc = (Wg + kCube - 1) / kCube;
  for (int a = 0; a < na; ++a)
    for (int b = 0; b < nb; ++b)
      for (int c = 0; c < nc; ++c) {
        unsigned long long mask = 0;
        int n = 0;
        for (int dt = 0; dt < kCube; ++dt)
          for (int dh = 0; dh < kCube; ++dh)
            for (int dw = 0; dw < kCube; ++dw) {
              const int t = kCube * a + dt, h = kCube * b + dh, w = kCube * c + dw;
              const int slot = (dt * kCube + dh) * kCube + dw;
              if (t < T && h < Hg && w < Wg) {
                L->perm.push_back(static_cast<int32_t>(vs.start + (static_cast<int64_t>(t) * Hg + h) * Wg + w));
                mask |= 1ull << slot;
                ++n;
              } else {
                L->perm.push_back(-1);
              }
            }
        L->valid.push_back(mask);
        L->count.push_back(n);
        L->kind.push_back(VSA_SEG_VIDEO);
        L->origin.insert(L->origin.end(), {kCube * a, kCube * b, kCube * c, VSA_SEG_VIDEO});
      }
  L->n_tiles = static_cast<int32_t>(L->count.size());
  L->n_video = L->n_tiles - L->n_cond;

  L->inv.assign(static_cast<size_t>(seq_len), -1);
  for (int64_t i = 0; i < static_cast<int64_t>(L->perm.size()); ++i)
    if (L->perm[i] >= 0) L->inv[L->perm[i]] = static_cast<int32_t>(i);
  L->off = tables_offsets(L);

  if (dev_buf) {
    vsa_status st = vsa_layout_upload(L, dev_buf, dev_bytes, stream);
    if (st != VSA_OK) {
      delete L;
      return st;
    }
  }
  *out = L;
  return VSA_OK;
}

vsa_status vsa_layout_upload(vsa_layout* L, void* dev_buf, size_t dev_bytes, cudaStream_t stream) {
  if (!L || !dev_buf) return VSA_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(dev_buf) % 256) return VSA_ERR_INVALID_ARG;
  if (dev_bytes < L->off.total) return VSA_ERR_WORKSPACE_TOO_SMALL;
  char* b = static_cast<char*>(dev_buf);
  struct Piece { size_t off; const void* src; size_t bytes; } pieces[] = {
      {L->off.perm, L->perm.data(), L->perm.size() * sizeof(int32_t)},
      {L->off.inv, L->inv.data(), L->inv.size() * sizeof(int32_t)},
      {L->off.valid, L->valid.data(), L->valid.size() * sizeof(unsigned long long)},
      {L->off.count, L->count.data(), L->count.size() * sizeof(int32_t)},
      {L->off.origin, L->origin.data(), L->origin.size() * sizeof(int32_t)},
  };
  for (const Piece& p : pieces) {
    const cudaError_t e = cudaMemcpyAsync(b + p.off, p.src, p.bytes, cudaMemcpyHostToDevice, stream);
    if (e != cudaSuccess) return cuda_fail("vsa_layout_upload: cudaMemcpyAsync", e);
  }
  L->dev_buf = dev_buf;
  return VSA_OK;
}

vsa_status vsa_layout_query(const vsa_layout* L, vsa_layout_info* info) {
  if (!L || !info) return VSA_ERR_INVALID_ARG;
  info->seq_len = L->seq_len;
  info->n_cond_tiles = L->n_cond;
  info->n_video_tiles = L->n_video;
  info->n_tiles = L->n_tiles;
  info->grid_t = L->grid_t;
  info->grid_h = L->grid_h;
  info->grid_w = L->grid_w;
  info->video_start = L->video_start;
  info->device_bytes = L->off.total;
  return VSA_OK;
}

vsa_status vsa_layout_copy_tables(const vsa_layout* L, int32_t* perm, int32_t* inv,
                                  int32_t* tile_count, int32_t* tile_kind) {
  if (!L) return VSA_ERR_INVALID_ARG;
  if (perm) std::memcpy(perm, L->perm.data(), L->perm.size() * sizeof(int32_t));
  if (inv) std::memcpy(inv, L->inv.data(), L->inv.size() * sizeof(int32_t));
  if (tile_count) std::memcpy(tile_count, L->count.data(), L->count.size() * sizeof(int32_t));
  if (tile_kind) std::memcpy(tile_kind, L->kind.data(), L->kind.size() * sizeof(int32_t));
  return VSA_OK;
}

void vsa_layout_free(vsa_layout* L) { delete L; }

vsa_status vsa_select_kmax(const vsa_layout* L, const vsa_params* p, int32_t* kmax) {
  if (!L || !kmax) return VSA_ERR_INVALID_ARG;
  vsa_status st = check_params(p);
  if (st != VSA_OK) return st;
  const int32_t nc = candidates(L, p->sink).count;
  *kmax = p->mode == VSA_SELECT_TOPK ? topk_count(p->keep, nc) : nc;
  return VSA_OK;
}

const char* vsa_status_string(vsa_status s) {
  switch (s) {
    case VSA_OK: return "ok";
    case VSA_ERR_INVALID_ARG: return "invalid argument";
    case VSA_ERR_UNSUPPORTED: return "unsupported case (run dense attention)";
    case VSA_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case VSA_ERR_CUDA: return "CUDA error";
    case VSA_ERR_TIMEOUT: return "kernel wait timed out";
    case VSA_ERR_NOT_UPLOADED: return "layout has no device tables";
  }
  return "unknown status";
}

int32_t vsa_version(void) { return (1 << 16) | 4; }

const char* vsa_last_error_detail(void) { return g_detail; }

}  // extern "C"
