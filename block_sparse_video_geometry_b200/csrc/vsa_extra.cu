// extra_tokens: the highest-scoring individual tokens beyond the selected tiles
// ("ComfyUI Agrega Nodo Central de Atencion Dispersa y Compilador Comfy",
// section "Atencion dispersa por bloques": extra_tokens adds the best-scoring
// tokens outside the selected blocks to stay closer to dense attention).
//
// Reading (the pages give the knob, not the rule): for every sparsely attended
// query tile qt, the candidate tokens are the valid tokens of the candidate key
// tiles that qt did NOT select; token i scores scale * <Qbar_qt, k_i> (the tile
// score taken at token resolution; the positive scale does not change the
// order); the E highest, ties to the lower token index, join the exact key set
// of every query of the tile. vsa_sparse_attn_fwd attends them as one more key
// tile.
//
// B200 design:
//  * permute_k_kernel: K tile-major, 16 KB 128-byte-swizzled blocks as the
//    attention uses, so that a key tile arrives with one bulk copy.
//  * pool_q_kernel: Qbar, the fp32 mean of the valid tokens of every tile.
//  * extra_select_kernel: one CTA per (batch, head, 128 query tiles). Scoring
//    128 query tiles against a pair of 64-token key tiles is one M = 128,
//    N = 128 tcgen05 product per split term: Qbar = hi + lo in bf16 (hi =
//    bf16(x), lo = bf16(x - hi): x to a relative 2^-17, held in TMEM as the A
//    operand), K exact in bf16, fp32 accumulation, so a score's error stays
//    below 2^-17 of sum_d |q_d k_d|, the size of an fp32 FMA chain's rounding
//    over 128 dims (2 x 8 MMAs per pair; a pair halves the MMA count of one
//    tile at a time, whose N = 64 products ran at a third of the tensor rate).
//    The pairs stream through shared memory (up to four stages; the CTAs of a
//    head start at different tiles). Two sets of 128 threads read the scores:
//    thread r of set s owns query tile r of the block (TMEM lane r) for tile
//    s of every pair, skips the tiles the query tile selected (a bitmap in
//    shared memory), and keeps a running top-E in shared memory (an unordered
//    array plus the position of its weakest entry, which a new token must
//    beat); at the end set 0 offers set 1's entries to its own list.

#include <cuda_runtime.h>

#include <algorithm>
#include <climits>
#include <cmath>

#include "sm100.cuh"
#include "vsa_internal.h"

namespace vsa {
namespace {

using namespace sm100;

constexpr int kXThreads = 320;           // 10 warps: 0 copies, 1 MMAs, 2-9 two sets of one query tile per thread
constexpr int kXRows = 128;
constexpr int kXStagesMax = 4;           // stages of a key tile pair (32 KB each)
constexpr uint32_t kXTmemCols = 512;
constexpr uint32_t kXColA = 0;           // Qbar split terms hi, lo: 64 columns of bf16 pairs each
constexpr uint32_t kXColD = 128;         // two score buffers of 128 fp32 columns (a key tile pair)
constexpr uint32_t kXIdesc = idesc_bf16_f32(128, 128, 0, 0);
constexpr uint64_t kXTimeoutNs = 4000000000ull;
constexpr uint64_t kXDrainNs = 200000000ull;
constexpr size_t kXHeader = 256;         // status word
constexpr uint32_t kXSmemMax = 227u * 1024u;

// Fixed part of the shared memory; the stages, the two sets' top-E lists and
// the selected-tile bitmap follow at offsets XSmemLayout gives.
struct XHead {
  uint64_t k_full[kXStagesMax], k_free[kXStagesMax], d_full[2], d_free[2], a_ready, drain;
  uint32_t tmem_base;
  int abort;
  int cnt1[kXRows];                      // set 1's list length per row, for the merge
};
static_assert(sizeof(XHead) <= 1024, "stages start at byte 1024");

// words of the per-row bitmap of selected candidate tiles
__host__ __device__ inline int x_sel_words(int n_cand) { return (n_cand + 31) / 32; }
// E rounded up to eight: the lists are read eight entries at a time
__host__ __device__ inline int x_pad_e(int E) { return (E + 7) & ~7; }

struct XSmemLayout {
  int stages;
  uint32_t val;                          // set s: scores at val + s * 8 ep * 128, tokens 4 ep * 128 bytes later
  uint32_t sel;                          // bitmap: bit c of word w of row r in word w * 128 + r
  uint32_t total;
};
inline XSmemLayout x_smem_layout(int stages, int E, int n_cand) {
  XSmemLayout l;
  l.stages = stages;
  l.val = 1024u + static_cast<uint32_t>(stages) * 32768u;
  l.sel = l.val + 2u * 8u * static_cast<uint32_t>(x_pad_e(E)) * kXRows;
  l.total = l.sel + 4u * static_cast<uint32_t>(x_sel_words(n_cand)) * kXRows;
  return l;
}

struct XArgs {
  DevLayout L;
  const uint8_t* ktm;                    // tile-major K: ((b * H + h) * n_tiles + tile) * 16 KB
  const float* qbar;                     // [B, H, n_tiles, 128]
  const int32_t* idx;
  const int32_t* cnt;
  int32_t kmax, H, c0, cand0, n_cand, E;
  int32_t stages;
  uint32_t off_val, off_sel;             // XSmemLayout offsets
  int32_t* out_idx;                      // [B, H, n_tiles, E]
  int32_t* out_cnt;                      // [B, H, n_tiles]
  int* err;
};

template <class XS>
__device__ __forceinline__ void x_abort(XS& sm, int* err) {
  atomicExch(err, VSA_ERR_TIMEOUT);
  *reinterpret_cast<volatile int*>(&sm.abort) = 1;
}

template <class XS>
__device__ __forceinline__ bool x_warp_wait(XS& sm, uint64_t& bar, uint32_t parity, int lane, int* err) {
  int ok = 1;
  if (lane == 0) {
    ok = mbar_wait(smem_u32(&bar), parity, &sm.abort, kXTimeoutNs) ? 1 : 0;
    if (!ok) x_abort(sm, err);
  }
  ok = __shfl_sync(0xffffffffu, ok, 0);
  __syncwarp();
  return ok != 0;
}

__device__ __forceinline__ uint32_t bf16_bits(float x) { return __float_as_uint(x) >> 16; }
__device__ __forceinline__ float bf16_round(float x) {
  uint32_t r;
  asm("{\n\t.reg .b16 h;\n\tcvt.rn.bf16.f32 h, %1;\n\tmov.b32 %0, {0, h};\n\t}" : "=r"(r) : "f"(x));
  return __uint_as_float(r);
}

// (v, t) ranks below (wv, wt): lower score, or equal score and higher token
// index. Tokens are distinct, so this is a total order on a row's entries.
__device__ __forceinline__ bool x_weaker(float v, int t, float wv, int wt) { return v < wv || (v == wv && t > wt); }

// The weakest entry of a row's full top-E (entry e at val[e * 128], tok[e * 128]).
// The entries are read eight at a time (independent loads; the arrays hold a
// multiple of eight) and reduced as a tree, so a replacement costs a few load
// latencies, not E of them.
__device__ __forceinline__ void x_find_worst(const float* val, const int* tok, int E, int& worst, float& wv, int& wt) {
  worst = -1;
  wv = INFINITY;
  wt = -1;
  for (int e0 = 0; e0 < E; e0 += 8) {
    float v[8];
    int t[8], w[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const bool in = e0 + j < E;
      v[j] = in ? val[(e0 + j) * kXRows] : INFINITY;
      t[j] = in ? tok[(e0 + j) * kXRows] : -1;
      w[j] = e0 + j;
    }
#pragma unroll
    for (int h = 4; h >= 1; h >>= 1)
#pragma unroll
      for (int j = 0; j < h; ++j)
        if (x_weaker(v[j + h], t[j + h], v[j], t[j])) {
          v[j] = v[j + h];
          t[j] = t[j + h];
          w[j] = w[j + h];
        }
    if (worst < 0 || x_weaker(v[0], t[0], wv, wt)) {
      worst = w[0];
      wv = v[0];
      wt = t[0];
    }
  }
}

// Score of slot i (0..63) of a key tile held in two register arrays, by a
// select tree on the bits of i (depth six, no dynamic register indexing).
__device__ __forceinline__ float x_pick(const float (&x0)[32], const float (&x1)[32], int i) {
  float l[32];
  const bool b5 = (i & 32) != 0;
#pragma unroll
  for (int u = 0; u < 32; ++u) l[u] = b5 ? x1[u] : x0[u];
#pragma unroll
  for (int h = 16; h >= 1; h >>= 1) {
    const bool b = (i & h) != 0;
#pragma unroll
    for (int u = 0; u < h; ++u) l[u] = b ? l[u + h] : l[u];
  }
  return l[0];
}

// Token of slot `slot` of a tile from its origin (conditioning tile: first
// token; video tile: the cube corner), without a memory access.
__device__ __forceinline__ int x_token(const DevLayout& L, int4 org, int slot) {
  if (org.w != VSA_SEG_VIDEO) return org.x + slot;
  const int t = org.x + (slot >> 4), h = org.y + ((slot >> 2) & 3), w = org.z + (slot & 3);
  return static_cast<int>(L.video_start + (static_cast<int64_t>(t) * L.grid_h + h) * L.grid_w + w);
}

// Bit i of the result: slot i's score (x0[i], then x1[i - 32]) is at least
// lim. Built as an OR tree, so no 32-long dependency chain.
__device__ __forceinline__ unsigned long long x_mask_ge(const float (&x0)[32], const float (&x1)[32], float lim) {
  uint32_t mq[16];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    mq[i] = ((x0[4 * i] >= lim ? 1u : 0u) << (4 * i)) | ((x0[4 * i + 1] >= lim ? 1u : 0u) << (4 * i + 1)) |
            ((x0[4 * i + 2] >= lim ? 1u : 0u) << (4 * i + 2)) | ((x0[4 * i + 3] >= lim ? 1u : 0u) << (4 * i + 3));
    mq[8 + i] = ((x1[4 * i] >= lim ? 1u : 0u) << (4 * i)) | ((x1[4 * i + 1] >= lim ? 1u : 0u) << (4 * i + 1)) |
                ((x1[4 * i + 2] >= lim ? 1u : 0u) << (4 * i + 2)) | ((x1[4 * i + 3] >= lim ? 1u : 0u) << (4 * i + 3));
  }
#pragma unroll
  for (int w = 4; w >= 1; w >>= 1)
#pragma unroll
    for (int i = 0; i < w; ++i) {
      mq[i] |= mq[i + w];
      mq[8 + i] |= mq[8 + i + w];
    }
  return static_cast<unsigned long long>(mq[8]) << 32 | mq[0];
}

// Narrows a key tile's candidate slots when more than E of them qualify: a
// slot with at least E candidates of the same tile above it cannot be in the
// top-E after the tile, so any bound lo with at least E candidates at or
// above it filters the rest. lo is found by bisection between the
// candidates' minimum and maximum score (a filter only: ties and the exact
// order are left to the offers).
__device__ __forceinline__ unsigned long long x_narrow(const float (&x0)[32], const float (&x1)[32],
                                                       unsigned long long cand, int E) {
  float t[32];
#pragma unroll
  for (int u = 0; u < 32; ++u)
    t[u] = fminf(((cand >> u) & 1ull) ? x0[u] : INFINITY, ((cand >> (32 + u)) & 1ull) ? x1[u] : INFINITY);
#pragma unroll
  for (int h = 16; h >= 1; h >>= 1)
#pragma unroll
    for (int u = 0; u < h; ++u) t[u] = fminf(t[u], t[u + h]);
  float lo = t[0];
#pragma unroll
  for (int u = 0; u < 32; ++u)
    t[u] = fmaxf(((cand >> u) & 1ull) ? x0[u] : -INFINITY, ((cand >> (32 + u)) & 1ull) ? x1[u] : -INFINITY);
#pragma unroll
  for (int h = 16; h >= 1; h >>= 1)
#pragma unroll
    for (int u = 0; u < h; ++u) t[u] = fmaxf(t[u], t[u + h]);
  float hi = t[0];
  for (int it = 0; it < 10; ++it) {              // invariant: at least E candidates at or above lo
    const float mid = 0.5f * (lo + hi);
    if (__popcll(x_mask_ge(x0, x1, mid) & cand) >= E) lo = mid;
    else hi = mid;
  }
  return x_mask_ge(x0, x1, lo) & cand;
}

// Offers (score, token) to a row's top-E (called for scores that may enter:
// the list is not full, or the score is at least the weakest).
__device__ __forceinline__ void x_offer(float* val, int* tok, int E, float s, int t, int& count, int& worst,
                                        float& wv, int& wt) {
  if (count < E) {
    val[count * kXRows] = s;
    tok[count * kXRows] = t;
    if (++count == E) x_find_worst(val, tok, E, worst, wv, wt);
    return;
  }
  if (x_weaker(wv, wt, s, t)) {
    val[worst * kXRows] = s;
    tok[worst * kXRows] = t;
    x_find_worst(val, tok, E, worst, wv, wt);
  }
}

__device__ __forceinline__ void x_rows_sync() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

// Position t of a CTA's key tile stream -> candidate index (the CTAs of a head
// start at different tiles, spreading their reads of the same tiles in time).
__device__ __forceinline__ int x_rotate(int t, int rot, int n_cand) {
  const int tt = t + rot;
  return tt >= n_cand ? tt - n_cand : tt;
}

__global__ void __launch_bounds__(kXThreads, 1) extra_select_kernel(const __grid_constant__ XArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if (smem_u32(smem_raw) & 1023u) {          // swizzled tiles need 1024-byte alignment
    if (threadIdx.x == 0) atomicExch(a.err, VSA_ERR_UNSUPPORTED);
    return;
  }
  XHead& sm = *reinterpret_cast<XHead*>(smem_raw);
  uint8_t* const stage0 = smem_raw + 1024;
  const int S = a.stages;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const size_t bh = static_cast<size_t>(blockIdx.z) * a.H + blockIdx.y;
  const int qt0 = a.c0 + blockIdx.x * kXRows;
  const int n_tiles = a.L.n_tiles;
  const int n_pairs = (a.n_cand + 1) >> 1;
  const int rot = static_cast<int>((static_cast<long long>(blockIdx.x) * a.n_cand) / gridDim.x);
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(smem_u32(&sm.k_full[s]), 1);
      mbar_init(smem_u32(&sm.k_free[s]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&sm.d_full[i]), 1);
      mbar_init(smem_u32(&sm.d_free[i]), 8);    // one arrival per row warp
    }
    mbar_init(smem_u32(&sm.a_ready), 8);
    mbar_init(smem_u32(&sm.drain), 1);
    sm.abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&sm.tmem_base), kXTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  if (warp == 0) {
    // ------------------------------------------- key tile pair copies
    // stage layout [d half][tile 2p, tile 2p + 1][64 slots][128 B]: each d
    // half of the pair is one 128-row K-major operand of the MMA
    uint32_t issued = 0;
    bool ok = true;
    for (int p = 0; p < n_pairs; ++p) {
      const int st = p % S;
      if (p >= S && !(ok = x_warp_wait(sm, sm.k_free[st], ((p / S) - 1) & 1, lane, a.err))) break;
      if (lane == 0) {
        const uint32_t bar = smem_u32(&sm.k_full[st]);
        const uint32_t dst = smem_u32(stage0 + st * 32768);
        const int nt = 2 * p + 1 < a.n_cand ? 2 : 1;
        mbar_arrive_expect_tx(bar, 16384u * nt);
        for (int j = 0; j < nt; ++j) {
          const uint8_t* src = a.ktm + (bh * n_tiles + a.cand0 + x_rotate(2 * p + j, rot, a.n_cand)) * 16384u;
          bulk_load(dst + 8192u * j, src, 8192, bar);
          bulk_load(dst + 16384u + 8192u * j, src + 8192, 8192, bar);
        }
      }
      __syncwarp();
      ++issued;
    }
    if (!ok && lane == 0) {
      for (uint32_t i = (issued > static_cast<uint32_t>(S) ? issued - S : 0u); i < issued; ++i)
        mbar_wait(smem_u32(&sm.k_full[i % S]), (i / S) & 1, nullptr, kXDrainNs);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMAs
    // D(p) = sum over the two split terms of Qbar_term [K(2p); K(2p+1)]^T into
    // score buffer p & 1, once the row warps have read D(p - 2) out of it.
    // (A missing second tile of an odd count leaves columns 64..127 stale;
    // nothing reads them.)
    if (lane == 0) {
      bool ok = mbar_wait(smem_u32(&sm.a_ready), 0, &sm.abort, kXTimeoutNs);
      for (int p = 0; ok && p < n_pairs; ++p) {
        const int st = p % S;
        if (!(ok = mbar_wait(smem_u32(&sm.k_full[st]), (p / S) & 1, &sm.abort, kXTimeoutNs))) break;
        if (p >= 2 && !(ok = mbar_wait(smem_u32(&sm.d_free[p & 1]), ((p >> 1) - 1) & 1, &sm.abort, kXTimeoutNs)))
          break;
        tc_fence_after();
        const uint64_t kd = smem_desc_sw128(smem_u32(stage0 + st * 32768), 16, 1024);
        const uint32_t d = tmem + kXColD + 128u * (p & 1);
#pragma unroll
        for (int term = 0; term < 2; ++term)
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            umma_ts(d, tmem + kXColA + 64u * term + kk * 8, kd + (kk >> 2) * (16384 >> 4) + (kk & 3) * 2, kXIdesc,
                    (term | kk) ? 1u : 0u);
        umma_commit(smem_u32(&sm.d_full[p & 1]));
        umma_commit(smem_u32(&sm.k_free[st]));
      }
      if (!ok) x_abort(sm, a.err);
      umma_commit(smem_u32(&sm.drain));
      mbar_wait(smem_u32(&sm.drain), 0, nullptr, kXDrainNs);
    }
    __syncwarp();
  } else {
    // -------------------------------- one query tile per thread, two sets
    // set 0 (warps 2-5) scores the first tile of every pair, set 1 (warps
    // 6-9) the second; each keeps its own top-E, merged at the end
    const int set = (warp - 2) >> 2;
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const int qt = qt0 + r;
    const bool row_ok = qt < n_tiles;
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    const size_t row = bh * n_tiles + (row_ok ? qt : 0);
    const int ep = x_pad_e(a.E);
    float* const val = reinterpret_cast<float*>(smem_raw + a.off_val) + set * 2 * ep * kXRows + r;
    int* const tok = reinterpret_cast<int*>(val + ep * kXRows);
    uint32_t* const sel = reinterpret_cast<uint32_t*>(smem_raw + a.off_sel) + r;
    // Qbar of this query tile, split into two bf16 terms, as the A operand:
    // set s writes dims 64 s .. 64 s + 63
    {
      const float* src = a.qbar + row * kHeadDim + 64 * set;
      uint32_t w0[32], w1[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        uint32_t hi[2], lo[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const float x = row_ok ? src[2 * i + e] : 0.f;
          const float hv = bf16_round(x);
          hi[e] = bf16_bits(hv);
          lo[e] = bf16_bits(bf16_round(x - hv));
        }
        w0[i] = hi[0] | (hi[1] << 16);
        w1[i] = lo[0] | (lo[1] << 16);
      }
      tmem_st32x32(lane_addr + kXColA + 0 * 64 + 32 * set, w0);
      tmem_st32x32(lane_addr + kXColA + 1 * 64 + 32 * set, w1);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&sm.a_ready));
    }
    // the tiles this query tile selected, as a bitmap in shared memory (set 0
    // builds it); entries outside [0, n_cand) are ignored
    if (set == 0) {
      const int n_words = x_sel_words(a.n_cand);
      for (int w = 0; w < n_words; ++w) sel[w * kXRows] = 0u;
      const int n_sel = row_ok ? min(max(a.cnt[row], 0), a.kmax) : 0;
      const int32_t* list = a.idx + row * a.kmax;
      for (int i = 0; i < n_sel; ++i) {
        const int cs = list[i];
        if (cs >= 0 && cs < a.n_cand) sel[(cs >> 5) * kXRows] |= 1u << (cs & 31);
      }
    }
    x_rows_sync();
    int count = 0, worst = 0, wt = 0;
    float wv = -INFINITY;
    // the valid-slot mask and origin of this set's tiles, loaded two pairs
    // ahead (a load from L2 takes longer than a pair's scores)
    unsigned long long vm_n[2];
    int4 org_n[2];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int t = 2 * j + set;
      const int tile = a.cand0 + (t < a.n_cand ? x_rotate(t, rot, a.n_cand) : 0);
      vm_n[j] = t < a.n_cand ? a.L.valid[tile] : 0ull;
      org_n[j] = t < a.n_cand ? a.L.origin[tile] : make_int4(0, 0, 0, 0);
    }
    for (int p = 0; p < n_pairs; ++p) {
      const int t = 2 * p + set;
      if (t >= a.n_cand) break;                  // an odd count's last pair has no second tile
      const int tt = x_rotate(t, rot, a.n_cand);
      const unsigned long long vm = vm_n[0];
      const int4 org = org_n[0];
      vm_n[0] = vm_n[1];
      org_n[0] = org_n[1];
      if (t + 4 < a.n_cand) {
        const int tile = a.cand0 + x_rotate(t + 4, rot, a.n_cand);
        vm_n[1] = a.L.valid[tile];
        org_n[1] = a.L.origin[tile];
      }
      if (!x_warp_wait(sm, sm.d_full[p & 1], (p >> 1) & 1, lane, a.err)) break;
      tc_fence_after();
      float x0[32], x1[32];
      const uint32_t dcol = kXColD + 128u * (p & 1) + 64u * set;
      tmem_ld32x32f(lane_addr + dcol, x0);
      tmem_ld32x32f(lane_addr + dcol + 32, x1);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&sm.d_free[p & 1]));
      if (((sel[(tt >> 5) * kXRows] >> (tt & 31)) & 1u) || !row_ok) continue;
      // slots that may enter the top-E: a branch-free mask first (after the
      // first tiles almost none qualify, and a branch per slot costs far more
      // than the compare), then one offer per set bit in slot order
      unsigned long long cand = x_mask_ge(x0, x1, count < a.E ? -INFINITY : wv) & vm;
      if (__popcll(cand) > a.E) cand = x_narrow(x0, x1, cand, a.E);   // early tiles: most slots qualify
      while (cand) {
        const int i = __ffsll(static_cast<long long>(cand)) - 1;
        cand &= cand - 1;
        const float xi = x_pick(x0, x1, i);   // the scores stay in registers
        if (count < a.E || xi >= wv) x_offer(val, tok, a.E, xi, x_token(a.L, org, i), count, worst, wv, wt);
      }
    }
    // merge: set 0 offers set 1's entries to its own list, then writes it out
    if (set == 1) sm.cnt1[r] = count;
    x_rows_sync();
    if (set == 0 && row_ok && !*reinterpret_cast<volatile int*>(&sm.abort)) {
      const float* val1 = val + 2 * ep * kXRows;
      const int* tok1 = tok + 2 * ep * kXRows;
      const int n1 = sm.cnt1[r];
      for (int e = 0; e < n1; ++e) {
        const float s1 = val1[e * kXRows];
        if (count < a.E || s1 >= wv) x_offer(val, tok, a.E, s1, tok1[e * kXRows], count, worst, wv, wt);
      }
      int32_t* dst = a.out_idx + row * a.E;
      for (int e = 0; e < count; ++e) dst[e] = tok[e * kXRows];
      a.out_cnt[row] = count;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kXTmemCols);
  }
}

// K into 16 KB tile-major blocks: [d half][64 slots][128 B], 16-byte chunk c
// of slot r at 16 (c ^ (r & 7)), padding slots zero.
__global__ void __launch_bounds__(256)
permute_k_kernel(DevLayout L, const uint16_t* __restrict__ k, int64_t sb, int64_t ss, int64_t sh, int H,
                 uint8_t* __restrict__ ktm) {
  const int tile = blockIdx.x, b = blockIdx.y;
  __shared__ int tok[kTile];
  for (int i = threadIdx.x; i < kTile; i += blockDim.x) tok[i] = L.perm[tile * kTile + i];
  __syncthreads();
  const int n = H * 1024;   // (head, d-half, row, chunk)
  for (int w = threadIdx.x; w < n; w += blockDim.x) {
    const int pc = w & 7, r = (w >> 3) & 63, j = (w >> 9) & 1, h = w >> 10;
    const int t = tok[r];
    uint4 val = make_uint4(0u, 0u, 0u, 0u);
    if (t >= 0)
      val = __ldg(reinterpret_cast<const uint4*>(k + b * sb + static_cast<int64_t>(t) * ss + h * sh + j * 64 +
                                                 ((pc ^ (r & 7)) << 3)));
    *reinterpret_cast<uint4*>(ktm + ((static_cast<size_t>(b) * H + h) * L.n_tiles + tile) * 16384u + j * 8192 +
                              r * 128 + pc * 16) = val;
  }
}

// Qbar [B, H, n_tiles, 128]: fp32 mean of Q over the valid tokens of each tile.
// grid (n_tiles, B); thread c handles head c / 16, dims 8 (c % 16) .. + 7.
__global__ void __launch_bounds__(1024)
pool_q_kernel(DevLayout L, const uint16_t* __restrict__ q, int64_t sb, int64_t ss, int64_t sh, int H,
              float* __restrict__ qbar) {
  const int tile = blockIdx.x, b = blockIdx.y;
  __shared__ int tok[kTile];
  for (int i = threadIdx.x; i < kTile; i += blockDim.x) tok[i] = L.perm[tile * kTile + i];
  __syncthreads();
  const float n = static_cast<float>(L.count[tile]);
  for (int c = threadIdx.x; c < H * 16; c += blockDim.x) {
    const int h = c >> 4, d0 = (c & 15) * 8;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int s = 0; s < kTile; ++s) {
      const int t = tok[s];
      if (t < 0) continue;
      const uint4 w = __ldg(reinterpret_cast<const uint4*>(q + b * sb + static_cast<int64_t>(t) * ss + h * sh + d0));
      const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        acc[2 * e] += __uint_as_float(u[e] << 16);
        acc[2 * e + 1] += __uint_as_float(u[e] & 0xFFFF0000u);
      }
    }
    float* dst = qbar + (((static_cast<size_t>(b) * H + h) * L.n_tiles + tile) * kHeadDim + d0);
    reinterpret_cast<float4*>(dst)[0] = make_float4(acc[0] / n, acc[1] / n, acc[2] / n, acc[3] / n);
    reinterpret_cast<float4*>(dst)[1] = make_float4(acc[4] / n, acc[5] / n, acc[6] / n, acc[7] / n);
  }
}

struct XWorkspace {
  size_t ktm, qbar, total;
};

XWorkspace x_workspace(const vsa_layout* L, int B, int H) {
  const size_t tiles = static_cast<size_t>(B) * H * L->n_tiles;
  XWorkspace w{};
  w.ktm = kXHeader;
  w.qbar = w.ktm + tiles * 16384u;
  w.total = w.qbar + align_up(tiles * kHeadDim * sizeof(float), 256);
  return w;
}

}  // namespace
}  // namespace vsa

using namespace vsa;

extern "C" {

vsa_status vsa_extra_tokens_workspace_size(const vsa_layout* L, int32_t B, int32_t H, const vsa_params* p,
                                           size_t* bytes) {
  if (!L || !bytes || B <= 0 || H <= 0) return VSA_ERR_INVALID_ARG;
  vsa_status st = check_params(p);
  if (st != VSA_OK) return st;
  *bytes = x_workspace(L, B, H).total;
  return VSA_OK;
}

vsa_status vsa_extra_tokens_select(const vsa_layout* L, const vsa_params* p, int32_t B, int32_t H,
                                   const void* q, const void* k, int64_t sb, int64_t ss, int64_t sh,
                                   const int32_t* idx, const int32_t* cnt, int32_t kmax, int32_t* extra_idx,
                                   int32_t* extra_cnt, void* workspace, size_t workspace_bytes,
                                   cudaStream_t stream) {
  if (!L) return VSA_ERR_INVALID_ARG;
  vsa_status st = check_params(p);
  if (st != VSA_OK) return st;
  if (p->extra_tokens < 1) return VSA_ERR_INVALID_ARG;
  st = check_qkv(q, k, k, sb, ss, sh, B, H);
  if (st != VSA_OK) return st;
  if (!idx || !cnt || !extra_idx || !extra_cnt || !workspace) return VSA_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(workspace) % 256) return VSA_ERR_INVALID_ARG;
  const XWorkspace ws = x_workspace(L, B, H);
  if (workspace_bytes < ws.total) return VSA_ERR_WORKSPACE_TOO_SMALL;
  if (!L->dev_buf) return VSA_ERR_NOT_UPLOADED;
  int32_t want_kmax = 0;
  vsa_select_kmax(L, p, &want_kmax);
  if (kmax != want_kmax) return VSA_ERR_INVALID_ARG;

  const DevLayout D = L->dev();
  const Candidates cand = candidates(L, p->sink);
  uint8_t* w = static_cast<uint8_t*>(workspace);
  XArgs a{};
  a.L = D;
  a.ktm = w + ws.ktm;
  a.qbar = reinterpret_cast<const float*>(w + ws.qbar);
  a.idx = idx;
  a.cnt = cnt;
  a.kmax = kmax;
  a.H = H;
  a.c0 = p->sink == VSA_SINK_EXACT_KV_AND_ROWS ? L->n_cond : 0;   // dense conditioning rows take no extra tokens
  a.cand0 = cand.first;
  a.n_cand = cand.count;
  a.E = p->extra_tokens;
  a.out_idx = extra_idx;
  a.out_cnt = extra_cnt;
  a.err = static_cast<int*>(workspace);

  cudaError_t e = cudaMemsetAsync(workspace, 0, sizeof(int), stream);
  if (e != cudaSuccess) return cuda_fail("vsa_extra_tokens_select: cudaMemsetAsync", e);
  e = cudaMemsetAsync(extra_cnt, 0, static_cast<size_t>(B) * H * L->n_tiles * sizeof(int32_t), stream);
  if (e != cudaSuccess) return cuda_fail("vsa_extra_tokens_select: cudaMemsetAsync(extra_cnt)", e);
  permute_k_kernel<<<dim3(L->n_tiles, B), 256, 0, stream>>>(D, static_cast<const uint16_t*>(k), sb, ss, sh, H,
                                                           w + ws.ktm);
  const int pool_threads = std::min(1024, (16 * H + 31) / 32 * 32);
  pool_q_kernel<<<dim3(L->n_tiles, B), pool_threads, 0, stream>>>(D, static_cast<const uint16_t*>(q), sb, ss, sh,
                                                                  H, reinterpret_cast<float*>(w + ws.qbar));
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail("vsa_extra_tokens_select: permute/pool launch", e);
  const int rows = L->n_tiles - a.c0;
  if (rows > 0) {
    // as many key tile pair stages as fit next to the two top-E lists and the
    // bitmap (the copies take thousands of cycles to land), at most four
    int stages = kXStagesMax;
    while (stages > 1 && x_smem_layout(stages, a.E, cand.count).total > kXSmemMax) --stages;
    const XSmemLayout sl = x_smem_layout(stages, a.E, cand.count);
    if (sl.total > kXSmemMax) {
      set_detail("vsa_extra_tokens_select: the candidate bitmap and the top-E lists exceed shared memory");
      return VSA_ERR_UNSUPPORTED;
    }
    a.stages = stages;
    a.off_val = sl.val;
    a.off_sel = sl.sel;
    e = cudaFuncSetAttribute(extra_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(sl.total));
    if (e != cudaSuccess) return cuda_fail("vsa_extra_tokens_select: cudaFuncSetAttribute", e);
    extra_select_kernel<<<dim3((rows + kXRows - 1) / kXRows, H, B), kXThreads, sl.total, stream>>>(a);
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail("vsa_extra_tokens_select: launch", e);
  }
  return VSA_OK;
}

vsa_status vsa_extra_tokens_status(const void* workspace, cudaStream_t stream) {
  if (!workspace) return VSA_ERR_INVALID_ARG;
  cudaError_t e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return cuda_fail("vsa_extra_tokens_status: cudaStreamSynchronize", e);
  int err = 0;
  e = cudaMemcpy(&err, workspace, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail("vsa_extra_tokens_status: cudaMemcpy", e);
  return err == 0 ? VSA_OK : static_cast<vsa_status>(err);
}

}  // extern "C"
