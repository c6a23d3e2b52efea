// Fine branch of VSA block-sparse attention + gate combine, for sm_100a.
//
// Each query tile attends exactly to every conditioning key token and to the
// video tiles of its selection list ("BSAI FastH3 Native VSA (recipe)", "The
// mechanism, briefly" and "The inputs that matter", sink_conditioning;
// "ComfyUI-Ref2VA-VSA", "Multimodal Dense-Exempt Prefix" and "Video-Only
// Sparse Attention"); with exact_kv_and_rows the conditioning query tiles
// attend the whole sequence. The epilogue writes o_fine + g * o_coarse.
//
// Design (B200). One call runs four kernels:
//  * permute_qkv_kernel rewrites K and V (and, for the pair pass, Q)
//    tile-major into the workspace, each 64-token tile of each head one
//    contiguous 16 KB block already in the 128-byte-swizzled layout of the UMMA
//    descriptors, padding slots zero, so that a step's K or V tile arrives with
//    one bulk copy. schedule_kernel writes every sparse item's key-tile
//    sequence as records, so that the copy warps only stream records (a copy
//    warp shares its scheduler with a softmax warp, and every instruction it
//    needs per step delays the copies).
//  * The pair pass (pairpass::pair_attn_kernel) runs the key tiles that every
//    query tile of a head attends: the conditioning prefix, and for dense
//    conditioning rows the whole sequence. Its work item is a PAIR of query
//    tiles stacked into one M = 128 MMA (full tensor rate, each key tile copied
//    once per two query tiles); it leaves the partial output over the
//    conditioning keys, normalised, with its log-sum-exp (dense rows: the
//    final output).
//  * The sparse pass (vsa_attn_kernel) runs each query tile's own selection
//    list with M = 64 MMAs (the lists of neighbouring query tiles barely
//    overlap, so stacking them would mostly compute masked work) and merges the
//    pair pass's partial result in its epilogue, exactly: the softmax over a
//    union of key sets is the log-sum-exp-weighted combination of the
//    softmaxes over the parts. Two CTAs per SM, each with 256 TMEM columns used
//    in both 16-lane halves of every lane quadrant (an M = 64 operand or
//    accumulator takes 16 lanes of each quadrant): even steps run in lanes
//    0-15, odd steps in lanes 16-31, each half with a copy of Q (the A operand
//    of S = Q K^T), its own O and its own 64-column score buffer, which P of the
//    step overwrites as bf16 pairs (the A operand of O += P V). An MMA with A in
//    TMEM needs A and D in the same lanes, which each half keeps; the output is
//    O(half 0) + O(half 1). Two K and two V stages sit in shared memory.
//  * Sparse pass warps: 0 and 1 copy K (and publish per-step tile info) and V;
//    2 issues the MMAs in the order ..., O += P(j - 1) V, S(j + 1), O += P(j) V,
//    S(j + 2), ... (MMAs from one thread run in issue order, so S(j + 2) cannot
//    overwrite P(j) early, and no issue waits for a completion); 3-6 write each
//    item's Q into both TMEM halves, run the fp32 online softmax and the
//    epilogue: two threads per row (the 16x32bx2 TMEM shape gives the two
//    half-warps the same 16 lanes at two column offsets), 32 keys each per
//    step, exp2. P is computed against the running max; the exact row max of a
//    step is only formed when a row's sum of P exceeds 2^8 (then O and the sum
//    are rescaled and P recomputed), which keeps every P at most 2^8.
//  * Every wait is bounded: a wait that runs out sets an error word in the
//    workspace, raises an abort flag that ends the other roles' loops, drains
//    in-flight copies and MMAs and frees TMEM before the block exits.

#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <climits>
#include <cmath>

#include "sm100.cuh"
#include "vsa_internal.h"

namespace vsa {
namespace {

using namespace sm100;

constexpr int kInfoSlots = 8;        // info of step j is rewritten only after O += P(j) V was issued
constexpr int kThreads = 224;
constexpr int kWarpK = 0, kWarpV = 1, kWarpMma = 2;   // warps 3..6: Q loads, softmax, epilogue
constexpr uint32_t kTmemCols = 256;
// An M = 64 operand or accumulator takes 16 lanes of each 32-lane quadrant
// (row r at lane 32 (r / 16) + r % 16 + lane offset). Both 16-lane halves are
// used: even steps run in half 0 (lane offset 0), odd steps in half 1 (lane
// offset 16). Each half holds a copy of Q (bf16 pairs, 64 columns), the O of
// its own steps (fp32, 128 columns) and the scores S of its current step
// (fp32, 64 columns), overwritten in place by P (bf16 pairs, 32 columns). An
// MMA with A in TMEM needs A and D in the same lanes, which each half keeps;
// the output is O(half 0) + O(half 1).
constexpr uint32_t kColQ = 0, kColO = 64, kColS = 192;
constexpr uint32_t kHalfLanes = 16u << 16;
constexpr uint32_t kTileBytes = 16384;    // one key tile of K or V: [d half 0][d half 1], 64 rows x 128 B
constexpr float kPSumLimit = 256.0f;     // 2^8: see the softmax step
constexpr uint32_t kIdescS = idesc_bf16_f32(64, 64, 0, 0);      // S = Q K^T: Q K-major in TMEM, K K-major
constexpr uint32_t kIdescPV = idesc_bf16_f32(64, 128, 0, 1);    // O = P V, P K-major in TMEM, V MN-major
constexpr uint64_t kTimeoutNs = 4000000000ull;
constexpr uint64_t kDrainNs = 200000000ull;

struct StageInfo {
  int32_t tile;
  int32_t last;   // last key tile of the work item
  unsigned long long valid;
};

// K and V stages and the TMEM halves all go by step parity: stage / half j & 1.
struct AttnSmem {
  uint8_t k[2][kTileBytes];
  uint8_t v[2][kTileBytes];
  StageInfo info[kInfoSlots];
  uint64_t k_full[2], v_full[2], s_full[2], p_full[2], pv_done[2];
  uint64_t info_full[kInfoSlots];
  uint64_t q_full, o_full, drain;
  uint64_t never;                      // nothing arrives on it: the injected wait of vsa_debug_inject_wait_timeout
  uint32_t tmem_base;
  int abort;
  int2 cond[1];                        // conditioning tiles (first token, count); n_cond entries
};

// Dynamic shared memory starts 1024-byte aligned when a kernel has no static
// shared memory (the kernel checks), so no alignment slack is requested.
size_t attn_smem_bytes(int n_cond) {
  return sizeof(AttnSmem) + sizeof(int2) * static_cast<size_t>(std::max(0, n_cond - 1));
}

struct Geom {
  int32_t n_cond, n_video, n_tiles;
  int32_t T, Hg, W;          // video grid
  int32_t ca, cb, cc;        // cubes along t, h, w
  int64_t video_start;
};

struct AttnArgs {
  Geom G;
  const int4* origin;        // device tile table (conditioning tiles are read once)
  const int32_t* count;
  const uint8_t* kv;         // tile-major K/V: ((b * H + h) * n_tiles + tile) * 32 KB, K then V
  const uint16_t* q;         // batch base of Q, element strides q_ss, q_sh
  int64_t q_ss, q_sh;
  int32_t H, b, sink, kmax;
  int32_t c0;                // first query tile of the item range (the rest are dense rows of the pair pass)
  int32_t cand0, n_cand;     // candidate key tiles: tile ids cand0 .. cand0 + n_cand - 1
  int32_t nq, n_items;       // query tiles per head in this pass; items = nq * H
  const int32_t* idx;         // selection lists (read by schedule_kernel)
  const int32_t* cnt;
  const unsigned long long* valid;   // per-tile slot masks
  int2* sched;               // step records: [b][item][max_steps]
  int32_t* nsteps;           // steps per (b, item)
  int32_t max_steps;
  int32_t n_extra;           // extra_tokens E (0: none)
  const int32_t* extra_cnt;  // [B, H, n_tiles] tokens chosen per query tile
  const uint8_t* extra_kv;   // their K and V as one tile-major tile per (b, h, query tile), 32 KB
  int32_t merge_prefix;      // merge the pair pass's partial output over the conditioning keys
  const float* part_o;       // [B, H, n_tiles, 64, 128] normalised partial output
  const float* part_lse;     // [B, H, n_tiles, 64] its log2-sum-exp2 (scaled log2 domain)
  // statistics mode (the backward pass): instead of the output, write each
  // query row's log2-sum-exp2 of the fine branch and D = <dO, o_fine>
  float* st_lse;             // [B, H, n_tiles, 64] (+inf for padding rows), or null
  float* st_d;               // [B, H, n_tiles, 64]
  const uint16_t* dout;      // dO [B, S, H, 128] bf16 at element strides d_sb, d_ss, d_sh
  int64_t d_sb, d_ss, d_sh;
  const float* o_coarse;
  const uint16_t* g;
  int64_t g_sb, g_ss, g_sh, g_sd;   // g_sd = 0: one gate per (token, head)
  void* out;
  int32_t out_bf16;
  int64_t o_sb, o_ss, o_sh;
  float scale_log2;
  int* err;
  uint64_t stall_ns;         // > 0: the S-issue warp first waits this long on a barrier nothing arrives on
};

// Work item = one query tile of one (batch, head).
struct Item {
  int h, qt;
};

__device__ __forceinline__ Item decode_item(const AttnArgs& a, int item) {
  Item it;
  it.h = item / a.nq;
  it.qt = a.c0 + (item - it.h * a.nq);
  return it;
}

// Video cube of ordinal v: origin (t0, h0, w0) and the mask of slots inside the grid.
__device__ __forceinline__ void video_cube(const Geom& G, int v, int& t0, int& h0, int& w0,
                                           unsigned long long& mask) {
  const int per_t = G.cb * G.cc;
  const int a = v / per_t, rem = v - a * per_t;
  const int bb = rem / G.cc, c = rem - bb * G.cc;
  t0 = 4 * a;
  h0 = 4 * bb;
  w0 = 4 * c;
  const int nt = min(4, G.T - t0), nh = min(4, G.Hg - h0), nw = min(4, G.W - w0);
  const uint32_t mw = (1u << nw) - 1u;
  uint32_t m16 = 0;
  for (int i = 0; i < nh; ++i) m16 |= mw << (4 * i);
  mask = 0;
  for (int i = 0; i < nt; ++i) mask |= static_cast<unsigned long long>(m16) << (16 * i);
}

__device__ __forceinline__ unsigned long long tile_mask(const AttnSmem& sm, const Geom& G, int tile) {
  if (tile < G.n_cond) {
    const int n = sm.cond[tile].y;
    return n >= 64 ? ~0ull : ((1ull << n) - 1ull);
  }
  int t0, h0, w0;
  unsigned long long m;
  video_cube(G, tile - G.n_cond, t0, h0, w0, m);
  return m;
}

// Token of (tile, slot); the slot must be valid.
__device__ __forceinline__ int64_t tile_token(const AttnSmem& sm, const Geom& G, int tile, int slot) {
  if (tile < G.n_cond) return sm.cond[tile].x + slot;
  int t0, h0, w0;
  unsigned long long m;
  video_cube(G, tile - G.n_cond, t0, h0, w0, m);
  const int t = t0 + (slot >> 4), h = h0 + ((slot >> 2) & 3), w = w0 + (slot & 3);
  return G.video_start + (static_cast<int64_t>(t) * G.Hg + h) * G.W + w;
}

// err[0]: status of the current call (cleared by each call); err[1]: failed
// calls since the caller last ran vsa_sparse_attn_workspace_init (the first
// block of a call to record an error counts the call).
__device__ __forceinline__ void record_error(int* err, int status) {
  if (atomicExch(err, status) == 0) atomicAdd(err + 1, 1);
}

template <class Smem>
__device__ __forceinline__ void raise_abort(Smem& sm, int* err) {
  record_error(err, VSA_ERR_TIMEOUT);
  *reinterpret_cast<volatile int*>(&sm.abort) = 1;
}

// Lane 0 waits; the result is broadcast so the warp leaves a loop together.
template <class Smem>
__device__ __forceinline__ bool warp_wait(Smem& sm, uint64_t& bar, uint32_t parity, int lane, int* err) {
  int ok = 1;
  if (lane == 0) {
    ok = mbar_wait(smem_u32(&bar), parity, &sm.abort, kTimeoutNs) ? 1 : 0;
    if (!ok) raise_abort(sm, err);
  }
  ok = __shfl_sync(0xffffffffu, ok, 0);
  __syncwarp();
  return ok != 0;
}

// bf16 pairs of P = 2^(x c - ms) for 32 keys; returns the fp32 sum of P.
__device__ __forceinline__ float exp_pass(const float (&x)[32], float c, float ms, uint32_t (&pw)[16]) {
  float ps[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const float p0 = ex2_approx(fmaf(x[2 * i], c, -ms));
    const float p1 = ex2_approx(fmaf(x[2 * i + 1], c, -ms));
    ps[i & 3] += p0 + p1;
    pw[i] = pack_bf16x2(p0, p1);
  }
  return (ps[0] + ps[1]) + (ps[2] + ps[3]);
}

// Q, K and V into tile-major order for the attention kernels:
//   qtm[((b * H + h) * n_tiles + tile) * 16 KB + j * 8 KB + r * 128 B + 16 * (c ^ (r & 7))]
//   kv [((b * H + h) * n_tiles + tile) * 32 KB + which * 16 KB + (same)]   (which = 0: K, 1: V)
// hold 16-byte chunk c of d-half j of slot r, i.e. each 16 KB block is the
// 128-byte-swizzled K-major layout the UMMA descriptors read; padding slots are
// zero. Consecutive threads write consecutive 16-byte chunks and read the
// chunks of one 128-byte row. The tile-major Q feeds the pair pass only (the
// sparse pass loads Q rows straight into tensor memory).
__global__ void __launch_bounds__(256)
permute_qkv_kernel(DevLayout L, const uint16_t* __restrict__ q, const uint16_t* __restrict__ k,
                   const uint16_t* __restrict__ v, int64_t sb, int64_t ss, int64_t sh, int H, int with_q,
                   uint8_t* __restrict__ qtm, uint8_t* __restrict__ kv) {
  const int tile = blockIdx.x, b = blockIdx.y;
  __shared__ int tok[kTile];
  for (int i = threadIdx.x; i < kTile; i += blockDim.x) tok[i] = L.perm[tile * kTile + i];
  __syncthreads();
  const int n_t = with_q ? 3 : 2;
  const int n = H * n_t * 1024;   // (head, tensor, d-half, row, chunk)
  for (int w = threadIdx.x; w < n; w += blockDim.x) {
    const int pc = w & 7, r = (w >> 3) & 63, j = (w >> 9) & 1, rest = w >> 10;
    const int which = rest % n_t + (with_q ? 0 : 1), h = rest / n_t;     // 0: Q, 1: K, 2: V
    const int t = tok[r];
    uint4 val = make_uint4(0u, 0u, 0u, 0u);
    const uint16_t* srcb = which == 0 ? q : (which == 1 ? k : v);
    if (t >= 0) {
      const uint16_t* src = srcb + b * sb + static_cast<int64_t>(t) * ss + h * sh + j * 64 + ((pc ^ (r & 7)) << 3);
      val = __ldg(reinterpret_cast<const uint4*>(src));
    }
    const size_t th = (static_cast<size_t>(b) * H + h) * L.n_tiles + tile;
    uint8_t* dst = which == 0 ? qtm + th * 16384u : kv + th * 32768u + (which - 1) * 16384;
    *reinterpret_cast<uint4*>(dst + j * 8192 + r * 128 + pc * 16) = val;
  }
}

// The extra tokens of each sparsely attended query tile gathered into one
// tile-major K/V tile (same layout as permute_qkv_kernel's; slots past the
// token count zero): extra_kv[((b * H + h) * n_tiles + qt) * 32 KB + ...].
// grid (query tiles from c0, H, B). Token indices outside [0, S) are skipped.
__global__ void __launch_bounds__(256)
gather_extra_kernel(const uint16_t* __restrict__ k, const uint16_t* __restrict__ v, int64_t sb, int64_t ss,
                    int64_t sh, int H, int n_tiles, int c0, int64_t seq_len, const int32_t* __restrict__ extra_idx,
                    const int32_t* __restrict__ extra_cnt, int E, uint8_t* __restrict__ extra_kv) {
  const int qt = c0 + blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const size_t row = (static_cast<size_t>(b) * H + h) * n_tiles + qt;
  __shared__ int tok[kTile];
  const int n = min(max(extra_cnt[row], 0), E);
  for (int i = threadIdx.x; i < kTile; i += blockDim.x) {
    const int t = i < n ? extra_idx[row * E + i] : -1;
    tok[i] = (t >= 0 && t < seq_len) ? t : -1;
  }
  __syncthreads();
  for (int w = threadIdx.x; w < 2048; w += blockDim.x) {   // (tensor, d-half, row, chunk)
    const int pc = w & 7, r = (w >> 3) & 63, j = (w >> 9) & 1, which = w >> 10;
    const int t = tok[r];
    uint4 val = make_uint4(0u, 0u, 0u, 0u);
    if (t >= 0) {
      const uint16_t* src = (which ? v : k) + b * sb + static_cast<int64_t>(t) * ss + h * sh + j * 64 +
                            ((pc ^ (r & 7)) << 3);
      val = __ldg(reinterpret_cast<const uint4*>(src));
    }
    *reinterpret_cast<uint4*>(extra_kv + row * 32768u + which * 16384 + j * 8192 + r * 128 + pc * 16) = val;
  }
}

// Step schedule of each work item, built once per call so that the copy warps
// of the attention kernel only stream records. Record = (key tile, flags): bit 4
// last step of the item, bit 5 the key tile has padding slots. Key tiles are the
// query tile's selection list (ascending candidate ordinals); the conditioning
// keys every query attends are the pair pass's.
constexpr int kSchedThreads = 128;

__global__ void __launch_bounds__(kSchedThreads) schedule_kernel(const __grid_constant__ AttnArgs a) {
  const int item = blockIdx.x, b = blockIdx.y;
  const Geom& G = a.G;
  const Item it = decode_item(a, item);
  const size_t row = (static_cast<size_t>(b) * a.H + it.h) * G.n_tiles + it.qt;
  // lists from vsa_coarse_select hold 1..kmax entries; anything else is clamped
  const int n = min(max(a.cnt[row], 1), a.kmax);
  // extra tokens: one more step over the query tile's gathered tile, whose
  // record holds the token count instead of a tile (flag bit 6)
  const int n_e = a.n_extra > 0 ? min(max(a.extra_cnt[row], 0), a.n_extra) : 0;
  const int total = n + (n_e > 0 ? 1 : 0);
  int2* rec = a.sched + (static_cast<size_t>(b) * a.n_items + item) * a.max_steps;
  for (int r = threadIdx.x; r < total; r += kSchedThreads) {
    uint32_t fl = r == total - 1 ? 16u : 0u;
    int t;
    if (r < n) {
      // entries outside [0, n_cand) (never written by vsa_coarse_select) are clamped: memory stays in bounds
      const int c = a.idx[row * a.kmax + r];
      t = a.cand0 + min(max(c, 0), a.n_cand - 1);
      if (a.valid[t] != ~0ull) fl |= 32u;
    } else {
      t = n_e;
      fl |= 64u;
    }
    rec[r] = make_int2(t, static_cast<int>(fl));
  }
  if (threadIdx.x == 0) a.nsteps[static_cast<size_t>(b) * a.n_items + item] = total;
}

// At most 128 registers per thread: each of an SM's four sub-partitions has its
// own 16K-entry register file, and two CTAs of 7 warps place 4 warps on two of
// them (4 x 32 x 128 = 16K); a higher count leaves room for one CTA per SM.
// kChannelGate: one gate per channel (g_sd > 0), a separate instantiation so
// that the per-token form keeps its register allocation.
template <bool kChannelGate>
__global__ void __maxnreg__(128) vsa_attn_kernel(const __grid_constant__ AttnArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if (smem_u32(smem_raw) & 1023u) {          // swizzled tiles need 1024-byte alignment
    if (threadIdx.x == 0) record_error(a.err, VSA_ERR_UNSUPPORTED);
    return;
  }
  AttnSmem& sm = *reinterpret_cast<AttnSmem*>(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Geom& G = a.G;

  for (int i = threadIdx.x; i < G.n_cond; i += kThreads)
    sm.cond[i] = make_int2(a.origin[i].x, a.count[i]);
  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&sm.k_full[i]), 1);
      mbar_init(smem_u32(&sm.v_full[i]), 1);
      mbar_init(smem_u32(&sm.s_full[i]), 1);
      mbar_init(smem_u32(&sm.p_full[i]), 4);     // one arrival per softmax warp
      mbar_init(smem_u32(&sm.pv_done[i]), 1);
    }
    for (int s = 0; s < kInfoSlots; ++s) mbar_init(smem_u32(&sm.info_full[s]), 1);
    mbar_init(smem_u32(&sm.q_full), 4);
    mbar_init(smem_u32(&sm.o_full), 1);
    mbar_init(smem_u32(&sm.drain), 1);
    mbar_init(smem_u32(&sm.never), 1);
    sm.abort = 0;
    fence_mbar_init();
  }
  if (warp == kWarpMma) {
    tmem_alloc(smem_u32(&sm.tmem_base), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  if (warp == kWarpK || warp == kWarpV) {
    // ----------------------------------------------------------- producers
    // Both stream the item's step records (one key tile each) and copy the
    // tile's 16 KB block of K or V into stage j & 1. A K stage is free again
    // once S of its previous step has completed (s_full), a V stage once O +=
    // P V of its previous step has (pv_done). The K warp also publishes
    // per-step tile info.
    const bool is_k = warp == kWarpK;
    uint64_t* full = is_k ? sm.k_full : sm.v_full;
    uint64_t* freed = is_k ? sm.s_full : sm.pv_done;
    uint32_t step = 0, issued = 0;
    bool ok = true;
    for (int item = blockIdx.x; ok && item < a.n_items; item += gridDim.x) {
      const size_t bi = static_cast<size_t>(a.b) * a.n_items + item;
      const int2* rec = a.sched + bi * a.max_steps;
      const int n = a.nsteps[bi];
      const Item itm = decode_item(a, item);
      const int h = itm.h;
      const uint8_t* head_kv = a.kv + (static_cast<size_t>(a.b) * a.H + h) * G.n_tiles * 32768u + (is_k ? 0u : 16384u);
      const uint8_t* extra_kv = a.n_extra > 0 ? a.extra_kv + ((static_cast<size_t>(a.b) * a.H + h) * G.n_tiles + itm.qt) *
                                                                 32768u + (is_k ? 0u : 16384u)
                                              : nullptr;
      // records 32 at a time, one per lane, the next 32 prefetched
      int2 cur = lane < n ? rec[lane] : make_int2(0, 0);
      int2 nxt = 32 + lane < n ? rec[32 + lane] : make_int2(0, 0);
      for (int jj = 0; jj < n; ++jj) {
        if (jj > 0 && (jj & 31) == 0) {
          cur = nxt;
          nxt = jj + 32 + lane < n ? rec[jj + 32 + lane] : make_int2(0, 0);
        }
        const int tile = __shfl_sync(0xffffffffu, cur.x, jj & 31);
        const int fl = __shfl_sync(0xffffffffu, cur.y, jj & 31);
        const int st = step & 1;
        if (step >= 2 && !(ok = warp_wait(sm, freed[st], ((step >> 1) - 1) & 1, lane, a.err))) break;
        if (lane == 0) {
          const bool extra = (fl & 64) != 0;     // the gathered extra-token tile; `tile` is its token count
          if (is_k) {
            StageInfo& inf = sm.info[step % kInfoSlots];
            inf.tile = tile;
            inf.last = (fl >> 4) & 1;
            inf.valid = extra ? (tile >= 64 ? ~0ull : ((1ull << tile) - 1ull)) : ((fl & 32) ? a.valid[tile] : ~0ull);
            mbar_arrive(smem_u32(&sm.info_full[step % kInfoSlots]));
          }
          const uint32_t bar = smem_u32(&full[st]);
          mbar_arrive_expect_tx(bar, kTileBytes);
          bulk_load(smem_u32(is_k ? sm.k[st] : sm.v[st]),
                    extra ? extra_kv : head_kv + static_cast<size_t>(tile) * 32768u, kTileBytes, bar);
        }
        __syncwarp();
        ++issued;
        ++step;
      }
    }
    if (!ok && lane == 0) {
      // let every issued copy land before the block can exit
      for (uint32_t i = (issued > 2u ? issued - 2u : 0u); i < issued; ++i)
        mbar_wait(smem_u32(&full[i & 1]), (i >> 1) & 1, nullptr, kDrainNs);
    }
  } else if (warp == kWarpMma) {
    // ----------------------------------------------------------------- MMA
    // One thread issues, in the order ..., O += P(j - 1) V, S(j + 1), O += P(j) V,
    // S(j + 2), ... . P(j) sits over the scores of TMEM half j & 1, and MMAs
    // from one thread run in issue order, so S(j + 2) cannot overwrite P(j)
    // before O += P(j) V has read it.
    bool ok = true;
    if (lane == 0) {
      uint32_t j = 0;
      int it_n = 0;
      auto pv = [&](uint32_t t, bool first) -> bool {
        const uint32_t b = t & 1;
        if (!mbar_wait(smem_u32(&sm.p_full[b]), (t >> 1) & 1, &sm.abort, kTimeoutNs)) return false;
        if (!mbar_wait(smem_u32(&sm.v_full[b]), (t >> 1) & 1, &sm.abort, kTimeoutNs)) return false;
        tc_fence_after();
        // V as MN-major B: 64-d blocks 8 KB apart, 16 keys = 2 KB per K step;
        // P (A, in TMEM): 16 keys = 8 columns of bf16 pairs per K step
        const uint64_t vd = smem_desc_sw128(smem_u32(sm.v[b]), 8192, 1024);
        const uint32_t half = tmem + (b ? kHalfLanes : 0u);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          umma_ts(half + kColO, half + kColS + kk * 8, vd + kk * (2048 >> 4), kIdescPV, (first && kk == 0) ? 0u : 1u);
        umma_commit(smem_u32(&sm.pv_done[b]));
        return true;
      };
      // injected failure (vsa_debug_inject_wait_timeout): a bounded wait that runs out
      if (a.stall_ns) ok = mbar_wait(smem_u32(&sm.never), 0, &sm.abort, a.stall_ns);
      for (int item = blockIdx.x; ok && item < a.n_items; item += gridDim.x, ++it_n) {
        if (!(ok = mbar_wait(smem_u32(&sm.q_full), it_n & 1, &sm.abort, kTimeoutNs))) break;
        int jj = 0;
        bool last = false;
        while (!last) {
          const uint32_t b = j & 1;
          if (!(ok = mbar_wait(smem_u32(&sm.k_full[b]), (j >> 1) & 1, &sm.abort, kTimeoutNs))) break;
          tc_fence_after();
          last = sm.info[j % kInfoSlots].last != 0;
          const uint64_t kd = smem_desc_sw128(smem_u32(sm.k[b]), 16, 1024);
          const uint32_t half = tmem + (b ? kHalfLanes : 0u);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            // 16 d per K step: 8 columns of Q pairs; 32 B inside a swizzle
            // row of K's d half kk / 4 (descriptor addresses count 16-byte units)
            umma_ts(half + kColS, half + kColQ + kk * 8, kd + (kk >> 2) * (8192 >> 4) + (kk & 3) * 2, kIdescS,
                    kk > 0 ? 1u : 0u);
          }
          umma_commit(smem_u32(&sm.s_full[b]));
          // the first two steps of an item start the O of their halves
          if (jj > 0 && !(ok = pv(j - 1, jj <= 2))) break;
          ++jj;
          ++j;
        }
        if (!ok) break;
        if (!(ok = pv(j - 1, jj <= 2))) break;
        umma_commit(smem_u32(&sm.o_full));
      }
      if (!ok) raise_abort(sm, a.err);
      // drain: every MMA this thread issued has completed before TMEM is freed
      umma_commit(smem_u32(&sm.drain));
      mbar_wait(smem_u32(&sm.drain), 0, nullptr, kDrainNs);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------ Q / softmax / epilogue
    // M = 64 layout: warp q (TMEM lanes 32q..32q+31) owns rows 16q..16q+15, in
    // lanes 32q..32q+15 for even steps and 32q+16..32q+31 for odd steps;
    // thread t handles row 16q + (t & 15) and the key (or output column) half
    // t >> 4, its partner is thread t ^ 16.
    const int quad = warp & 3;
    const int hf = lane >> 4;                        // 0: keys 0..31 / d 0..63, 1: keys 32..63 / d 64..127
    const int r = quad * 16 + (lane & 15);           // row of the 64-row tile
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    const float c = a.scale_log2;
    uint32_t j = 0;
    int it_n = 0;
    bool ok = true;
    for (int item = blockIdx.x; ok && item < a.n_items; item += gridDim.x, ++it_n) {
      const Item it = decode_item(a, item);
      const bool row_ok = (tile_mask(sm, G, it.qt) >> r) & 1ull;
      const int64_t tok = row_ok ? tile_token(sm, G, it.qt, r) : 0;
      {
        // this row's half of Q (d in [64 hf, 64 hf + 64): columns 32 hf ..
        // 32 hf + 31 of bf16 pairs) into both TMEM halves (every MMA of the
        // previous item has completed)
        const uint4* src = reinterpret_cast<const uint4*>(a.q + tok * a.q_ss + it.h * a.q_sh + 64 * hf);
        uint32_t w[32];
#pragma unroll
        for (int cc = 0; cc < 8; ++cc) {
          const uint4 u = row_ok ? __ldg(src + cc) : make_uint4(0u, 0u, 0u, 0u);
          w[4 * cc] = u.x;
          w[4 * cc + 1] = u.y;
          w[4 * cc + 2] = u.z;
          w[4 * cc + 3] = u.w;
        }
        tmem_st16x2_32<32>(lane_addr + kColQ, w);
        tmem_st16x2_32<32>(lane_addr + kHalfLanes + kColQ, w);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&sm.q_full));
      }
      const uint32_t j0 = j;               // first step of the item
      float ms = -INFINITY, l = 0.f;        // running max (scaled, log2 domain, same in both halves) and half sum
      bool last = false;
      // barrier phases of the next step are tested (without blocking) early in
      // a step and read after its exp2 work, so that their latency is hidden
      bool have_next = false, s_ready = false;
      StageInfo next{};
      while (!last) {
        StageInfo inf;
        if (have_next) {
          inf = next;
        } else {
          if (!(ok = warp_wait(sm, sm.info_full[j % kInfoSlots], (j / kInfoSlots) & 1, lane, a.err))) break;
          inf = sm.info[j % kInfoSlots];
        }
        last = inf.last != 0;
        if (!s_ready && !(ok = warp_wait(sm, sm.s_full[j & 1], (j >> 1) & 1, lane, a.err))) break;
        tc_fence_after();
        uint32_t t_info = 0, t_s = 0;
        if (!last) {
          t_info = mbar_test_wait(smem_u32(&sm.info_full[(j + 1) % kInfoSlots]), ((j + 1) / kInfoSlots) & 1);
          t_s = mbar_test_wait(smem_u32(&sm.s_full[(j + 1) & 1]), ((j + 1) >> 1) & 1);
        }
        const uint32_t scol = lane_addr + ((j & 1) ? kHalfLanes : 0u) + kColS;
        float x[32];
        tmem_ld16x2_32f<32>(scol, x);
        tmem_wait_ld();
        if (inf.valid != ~0ull) {             // padding slots never attend
          const uint32_t vm = static_cast<uint32_t>(inf.valid >> (32 * hf));
#pragma unroll
          for (int i = 0; i < 32; ++i) x[i] = ((vm >> i) & 1u) ? x[i] : -INFINITY;
        }
        // exact row max of the step; O and l rescaled when it raises the running max
        auto exact_max = [&]() -> bool {
          float m = x[0];
#pragma unroll
          for (int i = 1; i < 32; ++i) m = fmaxf(m, x[i]);
          const float mt = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 16)) * c;
          const bool need = ms != -INFINITY && mt > ms;
          if (ms == -INFINITY) ms = mt;       // first key tile of this row: O and l are still zero
          if (__any_sync(0xffffffffu, need)) {
            // rescale this half row of O once every earlier P V has landed (the
            // last one, O += P(j - 1) V, was issued after all the others)
            if (j > 0 && !warp_wait(sm, sm.pv_done[(j - 1) & 1], ((j - 1) >> 1) & 1, lane, a.err)) return false;
            tc_fence_after();
            const float f = need ? ex2_approx(ms - mt) : 1.0f;
            // both halves (a half not yet started by this item holds stale
            // values that its first O += P V overwrites)
#pragma unroll 1
            for (int ch = 0; ch < 4; ++ch) {
              const uint32_t oa = lane_addr + ((ch & 2) ? kHalfLanes : 0u) + kColO + 32 * (ch & 1);
              float u[32];
              tmem_ld16x2_32f<64>(oa, u);
              tmem_wait_ld();
              uint32_t w[32];
#pragma unroll
              for (int i = 0; i < 32; ++i) w[i] = __float_as_uint(u[i] * f);
              tmem_st16x2_32<64>(oa, w);
            }
            tmem_wait_st();
            if (need) {
              l *= f;
              ms = mt;
            }
          }
          return true;
        };
        // P against the running max ms. The softmax does not depend on that
        // reference as long as no P is large, so the exact row max of the step
        // is only formed when a row has no reference yet, or when its P sum
        // exceeds 2^8 (then every P was at most 2^8: fine for bf16 and fp32).
        uint32_t pw[16];
        if (__any_sync(0xffffffffu, ms == -INFINITY) && !(ok = exact_max())) break;
        float psum = exp_pass(x, c, ms, pw);
        if (__any_sync(0xffffffffu, psum + __shfl_xor_sync(0xffffffffu, psum, 16) > kPSumLimit)) {
          if (!(ok = exact_max())) break;
          psum = exp_pass(x, c, ms, pw);     // every P <= 1 now
        }
        l += psum;
        // P(j) over the first 32 score columns of its TMEM half (this half row:
        // keys 32 hf..32 hf + 31 = columns 16 hf..16 hf + 15); the scores were
        // read above. A warp reaches step j + 2 only after S(j + 2), issued after
        // O += P(j) V, which needed every warp's P(j): arrivals on p_full[j & 1]
        // stay in step order.
        tmem_st16x2_16<16>(scol, pw);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&sm.p_full[j & 1]));
        have_next = !last && __all_sync(0xffffffffu, t_info);
        if (have_next) next = sm.info[(j + 1) % kInfoSlots];
        s_ready = !last && __all_sync(0xffffffffu, t_s);
        ++j;
      }
      if (!ok) break;
      // epilogue: out = o_fine + g * o_coarse over this thread's half row (64
      // columns). o_fine merges this pass's O / l with the pair pass's partial
      // output over the conditioning keys, weighted 2^(ms - M) and 2^(lse - M)
      // (the softmax over a union of key sets from the softmaxes of the parts).
      if (!(ok = warp_wait(sm, sm.o_full, it_n & 1, lane, a.err))) break;
      tc_fence_after();
      const float l_row = l + __shfl_xor_sync(0xffffffffu, l, 16);
      const size_t prow = ((static_cast<size_t>(a.b) * a.H + it.h) * G.n_tiles + it.qt) * kTile + r;
      const float lse_c = (a.merge_prefix && row_ok) ? a.part_lse[prow] : -INFINITY;
      const float mx = fmaxf(ms, lse_c);
      const float wf = ex2_approx(ms - mx), wc = lse_c != -INFINITY ? ex2_approx(lse_c - mx) : 0.f;
      const float inv_l = 1.0f / (l_row * wf + wc);
      const float af = wf * inv_l, ac = wc * inv_l;
      const float* pc = a.part_o + prow * kHeadDim + 64 * hf;
      const bool stats = a.st_lse != nullptr;
      const uint16_t* drow = stats && row_ok ? a.dout + a.b * a.d_sb + tok * a.d_ss + it.h * a.d_sh + 64 * hf : nullptr;
      float dsum = 0.f;
      float gate = 0.f;
      const float* oc = nullptr;
      const uint16_t* gp = nullptr;          // per-channel gate of this row (g_sd > 0)
      if (row_ok && !stats) {
        gp = a.g + a.b * a.g_sb + tok * a.g_ss + it.h * a.g_sh;
        gate = __uint_as_float(static_cast<uint32_t>(gp[0]) << 16);
        gp = kChannelGate ? gp + 64 * hf * a.g_sd : nullptr;
        oc = a.o_coarse + ((static_cast<size_t>(a.b) * a.H + it.h) * G.n_tiles + it.qt) * kHeadDim + 64 * hf;
      }
      // O = O(half of step j0) + O(other half) when the item had two steps or more
      const uint32_t o_first = lane_addr + ((j0 & 1) ? kHalfLanes : 0u) + kColO;
      const uint32_t o_second = lane_addr + ((j0 & 1) ? 0u : kHalfLanes) + kColO;
      const bool two_halves = j - j0 >= 2;
#pragma unroll 1
      for (int ch = 0; ch < 2; ++ch) {
        float y[32];
        tmem_ld16x2_32f<64>(o_first + 32 * ch, y);
        if (two_halves) {
          float z[32];
          tmem_ld16x2_32f<64>(o_second + 32 * ch, z);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) y[i] += z[i];
        } else {
          tmem_wait_ld();
        }
        if (row_ok) {
#pragma unroll
          for (int i = 0; i < 32; ++i) y[i] *= af;
          if (ac != 0.f) {
#pragma unroll
            for (int i = 0; i < 32; i += 4) {
              const float4 t = *reinterpret_cast<const float4*>(pc + ch * 32 + i);
              y[i] = fmaf(t.x, ac, y[i]);
              y[i + 1] = fmaf(t.y, ac, y[i + 1]);
              y[i + 2] = fmaf(t.z, ac, y[i + 2]);
              y[i + 3] = fmaf(t.w, ac, y[i + 3]);
            }
          }
          if (stats) {                         // D = <dO, o_fine>: this thread's 32 columns of the chunk
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const uint4 w = __ldg(reinterpret_cast<const uint4*>(drow + ch * 32) + u);
              const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
              for (int e = 0; e < 4; ++e)
                dsum = fmaf(__uint_as_float(wv[e] << 16), y[8 * u + 2 * e],
                            fmaf(__uint_as_float(wv[e] & 0xFFFF0000u), y[8 * u + 2 * e + 1], dsum));
            }
            continue;
          }
          if (kChannelGate && oc) {
            // this chunk's 32 gates as bf16 pairs (vector loads when the channels are contiguous)
            const uint16_t* gc = gp + static_cast<int64_t>(ch) * 32 * a.g_sd;
            uint32_t gw[16];
            if (a.g_sd == 1 && (reinterpret_cast<uintptr_t>(gc) & 15u) == 0) {
#pragma unroll
              for (int u = 0; u < 4; ++u) {
                const uint4 t = __ldg(reinterpret_cast<const uint4*>(gc) + u);
                gw[4 * u] = t.x;
                gw[4 * u + 1] = t.y;
                gw[4 * u + 2] = t.z;
                gw[4 * u + 3] = t.w;
              }
            } else {
#pragma unroll
              for (int u = 0; u < 16; ++u)
                gw[u] = static_cast<uint32_t>(__ldg(gc + 2 * u * a.g_sd)) |
                        (static_cast<uint32_t>(__ldg(gc + (2 * u + 1) * a.g_sd)) << 16);
            }
#pragma unroll
            for (int i = 0; i < 32; i += 4) {
              const float4 cv = *reinterpret_cast<const float4*>(oc + ch * 32 + i);
              const uint32_t g0 = gw[i / 2], g1 = gw[i / 2 + 1];
              y[i] = fmaf(__uint_as_float(g0 << 16), cv.x, y[i]);
              y[i + 1] = fmaf(__uint_as_float(g0 & 0xFFFF0000u), cv.y, y[i + 1]);
              y[i + 2] = fmaf(__uint_as_float(g1 << 16), cv.z, y[i + 2]);
              y[i + 3] = fmaf(__uint_as_float(g1 & 0xFFFF0000u), cv.w, y[i + 3]);
            }
          } else if (oc) {
#pragma unroll
            for (int i = 0; i < 32; i += 4) {
              const float4 cv = *reinterpret_cast<const float4*>(oc + ch * 32 + i);
              y[i] = fmaf(gate, cv.x, y[i]);
              y[i + 1] = fmaf(gate, cv.y, y[i + 1]);
              y[i + 2] = fmaf(gate, cv.z, y[i + 2]);
              y[i + 3] = fmaf(gate, cv.w, y[i + 3]);
            }
          }
          const int64_t off = a.b * a.o_sb + tok * a.o_ss + it.h * a.o_sh + 64 * hf + ch * 32;
          if (a.out_bf16) {
            uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(a.out) + off);
#pragma unroll
            for (int i = 0; i < 32; i += 8)
              dst[i / 8] = make_uint4(pack_bf16x2(y[i], y[i + 1]), pack_bf16x2(y[i + 2], y[i + 3]),
                                      pack_bf16x2(y[i + 4], y[i + 5]), pack_bf16x2(y[i + 6], y[i + 7]));
          } else {
            float4* dst = reinterpret_cast<float4*>(static_cast<float*>(a.out) + off);
#pragma unroll
            for (int i = 0; i < 32; i += 4) dst[i / 4] = make_float4(y[i], y[i + 1], y[i + 2], y[i + 3]);
          }
        }
      }
      if (stats) {
        const float d_row = dsum + __shfl_xor_sync(0xffffffffu, dsum, 16);
        if (hf == 0) {
          a.st_lse[prow] = row_ok ? mx + __log2f(l_row * wf + wc) : INFINITY;
          a.st_d[prow] = row_ok ? d_row : 0.f;
        }
      }
      tc_fence_before();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ------------------------------------------------------------------ pair pass
// The key tiles that every query tile of a head attends (the conditioning
// prefix, and for dense conditioning rows the whole sequence) are run for
// PAIRS of query tiles stacked into one M = 128 MMA: the tensor pipe runs at
// its full rate (an M = 64 MMA takes as long as an M = 128 one) and each key
// tile is copied once per two query tiles. Dense rows are final output; for
// the others the pass leaves the normalised partial output and its log2-sum-
// exp2 for the sparse pass to merge. Same roles as the sparse pass: warps 0
// and 1 copy K and V tiles (warp 0 also the pair's Q, bulk-copied from the
// tile-major copy as the M = 128 A operand), warp 2 issues the MMAs (S from
// shared memory, P V with P in tensor memory), warps 3-10 run the softmax of
// 16 rows each (two threads per row) and the epilogue. Tensor memory: O in
// columns 0-127, two score slots in 128-255; two CTAs per SM.
namespace pairpass {

constexpr int kThreads = 352;
constexpr int kWarpK = 0, kWarpV = 1, kWarpMma = 2, kWarpSoftmax = 3;
constexpr int kInfoSlots = 8;
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kColO = 0, kColS = 128;
constexpr uint32_t kIdescS = idesc_bf16_f32(128, 64, 0, 0);     // S = Q K^T: Q and K K-major in shared memory
constexpr uint32_t kIdescPV = idesc_bf16_f32(128, 128, 0, 1);   // O += P V: P in TMEM, V MN-major

struct Info {
  int32_t flags;                    // bit 0: first step of the item, bit 1: last step
  unsigned long long valid;         // slot mask of the key tile
};

struct Smem {
  uint8_t q[2 * kTileBytes];        // the pair's Q: [d half][128 rows][128 B], rows 64-127 the second tile
  uint8_t k[2][kTileBytes];
  uint8_t v[2][kTileBytes];
  Info info[kInfoSlots];
  uint64_t k_full[2], v_full[2], s_full[2], p_full[2], pv_done[2];
  uint64_t info_full[kInfoSlots];
  uint64_t q_full, q_empty, o_full, drain, never;
  uint32_t tmem_base;
  int abort;
};

struct Args {
  int32_t n_cond, n_tiles;
  const int32_t* perm;              // token of (tile, slot), -1 for padding
  const unsigned long long* valid;  // slot mask of each tile
  const uint8_t* qtm;               // tile-major Q: ((b * H + h) * n_tiles + tile) * 16 KB
  const uint8_t* kv;                // tile-major K, V: ((b * H + h) * n_tiles + tile) * 32 KB
  int32_t H, b;
  int32_t c0;                       // first query tile of the prefix pairs
  int32_t n_dpairs, n_ppairs;       // pairs per head: dense rows (all key tiles), prefix (conditioning key tiles)
  int32_t n_items;
  float* part_o;                    // [B, H, n_tiles, 64, 128] normalised partial output
  float* part_lse;                  // [B, H, n_tiles, 64] its log2-sum-exp2 (scaled log2 domain)
  float* st_lse;                    // statistics mode (see AttnArgs): dense rows' log2-sum-exp2 and D, or null
  float* st_d;
  const uint16_t* dout;
  int64_t d_sb, d_ss, d_sh;
  void* out;
  int32_t out_bf16;
  int64_t o_sb, o_ss, o_sh;
  float scale_log2;
  int* err;
  uint64_t stall_ns;                // > 0: the MMA warp first waits this long on a barrier nothing arrives on
};

struct PItem {
  int h, qa, qb;                    // query tiles of rows 0-63 and 64-127 (qb < 0: none)
  int n;                            // key tiles 0 .. n - 1
  int dense;
};

__device__ __forceinline__ PItem decode(const Args& a, int item) {
  PItem it;
  const int nd = a.H * a.n_dpairs;
  if (item < nd) {
    it.h = item / a.n_dpairs;
    const int p = item - it.h * a.n_dpairs;
    it.qa = 2 * p;
    it.qb = 2 * p + 1 < a.n_cond ? 2 * p + 1 : -1;
    it.n = a.n_tiles;
    it.dense = 1;
  } else {
    const int r = item - nd;
    it.h = r / a.n_ppairs;
    const int p = r - it.h * a.n_ppairs;
    it.qa = a.c0 + 2 * p;
    it.qb = it.qa + 1 < a.n_tiles ? it.qa + 1 : -1;
    it.n = a.n_cond;
    it.dense = 0;
  }
  return it;
}

__global__ void __maxnreg__(80) pair_attn_kernel(const __grid_constant__ Args a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if (smem_u32(smem_raw) & 1023u) {          // swizzled tiles need 1024-byte alignment
    if (threadIdx.x == 0) record_error(a.err, VSA_ERR_UNSUPPORTED);
    return;
  }
  Smem& sm = *reinterpret_cast<Smem*>(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&sm.k_full[i]), 1);
      mbar_init(smem_u32(&sm.v_full[i]), 1);
      mbar_init(smem_u32(&sm.s_full[i]), 1);
      mbar_init(smem_u32(&sm.p_full[i]), 8);      // one arrival per softmax warp
      mbar_init(smem_u32(&sm.pv_done[i]), 1);
    }
    for (int s = 0; s < kInfoSlots; ++s) mbar_init(smem_u32(&sm.info_full[s]), 1);
    mbar_init(smem_u32(&sm.q_full), 1);
    mbar_init(smem_u32(&sm.q_empty), 1);
    mbar_init(smem_u32(&sm.o_full), 1);
    mbar_init(smem_u32(&sm.drain), 1);
    mbar_init(smem_u32(&sm.never), 1);
    sm.abort = 0;
    fence_mbar_init();
  }
  if (warp == kWarpMma) {
    tmem_alloc(smem_u32(&sm.tmem_base), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  const size_t head0 = static_cast<size_t>(a.b) * a.H;

  if (warp == kWarpK || warp == kWarpV) {
    // ----------------------------------------------------------- producers
    // Key tiles 0 .. n - 1 of every item into stage j & 1: a K stage is free
    // again once S of its previous step completed (s_full), a V stage once
    // O += P V of it did (pv_done). The K warp also copies each pair's Q (once
    // the previous pair's S completed) and publishes per-step tile info.
    const bool is_k = warp == kWarpK;
    uint64_t* full = is_k ? sm.k_full : sm.v_full;
    uint64_t* freed = is_k ? sm.s_full : sm.pv_done;
    uint32_t step = 0;
    int it_n = 0, q_last = -1;
    bool ok = true;
    for (int item = blockIdx.x; ok && item < a.n_items; item += gridDim.x, ++it_n) {
      const PItem it = decode(a, item);
      const uint8_t* head_kv = a.kv + (head0 + it.h) * a.n_tiles * 32768u + (is_k ? 0u : 16384u);
      if (is_k) {
        if (it_n >= 1 && !(ok = warp_wait(sm, sm.q_empty, (it_n - 1) & 1, lane, a.err))) break;
        if (lane == 0) {
          const uint8_t* qa = a.qtm + ((head0 + it.h) * a.n_tiles + it.qa) * kTileBytes;
          const uint8_t* qb = a.qtm + ((head0 + it.h) * a.n_tiles + (it.qb >= 0 ? it.qb : it.qa)) * kTileBytes;
          const uint32_t bar = smem_u32(&sm.q_full);
          mbar_arrive_expect_tx(bar, 2 * kTileBytes);
          bulk_load(smem_u32(sm.q), qa, 8192, bar);
          bulk_load(smem_u32(sm.q) + 8192, qb, 8192, bar);
          bulk_load(smem_u32(sm.q) + 16384, qa + 8192, 8192, bar);
          bulk_load(smem_u32(sm.q) + 24576, qb + 8192, 8192, bar);
        }
        q_last = it_n;
        __syncwarp();
      }
      unsigned long long v_cur = 0ull;       // slot masks of key tiles jj .. jj + 31, one per lane
      for (int jj = 0; jj < it.n; ++jj) {
        if (is_k && (jj & 31) == 0) v_cur = jj + lane < it.n ? a.valid[jj + lane] : 0ull;
        const unsigned long long vm = __shfl_sync(0xffffffffu, v_cur, jj & 31);
        const int st = step & 1;
        if (step >= 2 && !(ok = warp_wait(sm, freed[st], ((step >> 1) - 1) & 1, lane, a.err))) break;
        if (lane == 0) {
          if (is_k) {
            Info& inf = sm.info[step % kInfoSlots];
            inf.flags = (jj == 0 ? 1 : 0) | (jj == it.n - 1 ? 2 : 0);
            inf.valid = vm;
            mbar_arrive(smem_u32(&sm.info_full[step % kInfoSlots]));
          }
          const uint32_t bar = smem_u32(&full[st]);
          mbar_arrive_expect_tx(bar, kTileBytes);
          bulk_load(smem_u32(is_k ? sm.k[st] : sm.v[st]), head_kv + static_cast<size_t>(jj) * 32768u, kTileBytes,
                    bar);
        }
        __syncwarp();
        ++step;
      }
    }
    if (!ok && lane == 0) {
      // let every issued copy land before the block can exit
      for (uint32_t i = (step > 2u ? step - 2u : 0u); i < step; ++i)
        mbar_wait(smem_u32(&full[i & 1]), (i >> 1) & 1, nullptr, kDrainNs);
      if (is_k && q_last >= 0) mbar_wait(smem_u32(&sm.q_full), q_last & 1, nullptr, kDrainNs);
    }
  } else if (warp == kWarpMma) {
    // ----------------------------------------------------------------- MMA
    // S(j) once O += P(j - 2) V was issued (its score slot is free: MMAs from
    // one thread run in issue order), the pair's Q and K(j) have landed;
    // O += P(j) V once all softmax warps wrote P(j) and V(j) has landed. The
    // thread issues whichever is ready, S first.
    bool ok = true;
    if (lane == 0) {
      if (a.stall_ns) ok = mbar_wait(smem_u32(&sm.never), 0, &sm.abort, a.stall_ns);   // injected failure
      uint32_t ns = 0, np = 0, ring = 0;
      int s_item = blockIdx.x, s_it = 0;
      bool s_done = s_item >= a.n_items;
      uint64_t t_idle = globaltimer_ns();
      uint32_t spins = 0;
      const uint64_t qd = smem_desc_sw128(smem_u32(sm.q), 16, 1024);
      while (ok) {
        bool progress = false;
        if (!s_done && ns < np + 2 && mbar_test_wait(smem_u32(&sm.k_full[ns & 1]), (ns >> 1) & 1) &&
            (!(sm.info[ns % kInfoSlots].flags & 1) || mbar_test_wait(smem_u32(&sm.q_full), s_it & 1))) {
          tc_fence_after();
          const int fl = sm.info[ns % kInfoSlots].flags;
          // 16 d per K step: 32 B inside a swizzle row of the d half kk / 4
          // (descriptor addresses count 16-byte units)
          const uint64_t kd = smem_desc_sw128(smem_u32(sm.k[ns & 1]), 16, 1024);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            umma_ss(tmem + kColS + 64 * (ns & 1), qd + (kk >> 2) * (16384 >> 4) + (kk & 3) * 2,
                    kd + (kk >> 2) * (8192 >> 4) + (kk & 3) * 2, kIdescS, kk > 0 ? 1u : 0u);
          umma_commit(smem_u32(&sm.s_full[ns & 1]));
          ring = (ring & ~(3u << (2 * (ns & 3)))) | (static_cast<uint32_t>(fl & 3) << (2 * (ns & 3)));
          if (fl & 2) {
            umma_commit(smem_u32(&sm.q_empty));       // the pair's Q may be replaced
            s_item += gridDim.x;
            ++s_it;
            s_done = s_item >= a.n_items;
          }
          ++ns;
          progress = true;
        }
        if (np < ns && mbar_test_wait(smem_u32(&sm.p_full[np & 1]), (np >> 1) & 1) &&
            mbar_test_wait(smem_u32(&sm.v_full[np & 1]), (np >> 1) & 1)) {
          tc_fence_after();
          const uint32_t fl = (ring >> (2 * (np & 3))) & 3u;
          // V as MN-major B: 64-d blocks 8 KB apart, 16 keys = 2 KB per K step;
          // P (A, over its scores in TMEM): 16 keys = 8 columns of bf16 pairs
          const uint64_t vd = smem_desc_sw128(smem_u32(sm.v[np & 1]), 8192, 1024);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_ts(tmem + kColO, tmem + kColS + 64 * (np & 1) + kk * 8, vd + kk * (2048 >> 4), kIdescPV,
                    ((fl & 1) && kk == 0) ? 0u : 1u);
          umma_commit(smem_u32(&sm.pv_done[np & 1]));
          if (fl & 2) umma_commit(smem_u32(&sm.o_full));
          ++np;
          progress = true;
        }
        if (s_done && np == ns) break;
        if (progress) {
          spins = 0;
        } else if ((++spins & 255u) == 0) {
          const uint64_t now = globaltimer_ns();
          if (spins == 256u) t_idle = now;
          if (*reinterpret_cast<volatile int*>(&sm.abort) || now - t_idle > kTimeoutNs) ok = false;
        }
      }
      if (!ok) raise_abort(sm, a.err);
      // drain: every MMA this thread issued has completed before TMEM is freed
      umma_commit(smem_u32(&sm.drain));
      mbar_wait(smem_u32(&sm.drain), 0, nullptr, kDrainNs);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------ softmax / epilogue
    // Warp w owns TMEM lanes 32 (w & 3) + 16 s .. + 15 (s = (w - 3) / 4), i.e.
    // rows of the M = 128 pair (row r in lane r: rows 0-63 the first query
    // tile, 64-127 the second). Thread t handles row t & 15 of them and the key
    // (or output column) half hf = t >> 4; its partner is thread t ^ 16.
    const int quad = warp & 3;
    const int sub = (warp - kWarpSoftmax) >> 2;
    const int hf = lane >> 4;
    const int prow = quad * 32 + sub * 16 + (lane & 15);
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(quad * 32 + sub * 16) << 16);
    const float c = a.scale_log2;
    uint32_t j = 0;
    int it_n = 0;
    bool ok = true;
    for (int item = blockIdx.x; ok && item < a.n_items; item += gridDim.x, ++it_n) {
      const PItem it = decode(a, item);
      const int qtile = prow < 64 ? it.qa : it.qb;
      const int slot = prow & 63;
      const int tok = qtile >= 0 ? a.perm[qtile * kTile + slot] : -1;
      const bool row_ok = tok >= 0;
      const uint32_t j0 = j, jend = j + it.n;
      float ms = -INFINITY, l = 0.f;
      bool have_next = false, s_ready = false;
      Info next{};
      for (; j < jend; ++j) {
        Info inf;
        if (have_next) {
          inf = next;
        } else {
          if (!(ok = warp_wait(sm, sm.info_full[j % kInfoSlots], (j / kInfoSlots) & 1, lane, a.err))) break;
          inf = sm.info[j % kInfoSlots];
        }
        if (!s_ready && !(ok = warp_wait(sm, sm.s_full[j & 1], (j >> 1) & 1, lane, a.err))) break;
        tc_fence_after();
        const bool more = j + 1 < jend;
        uint32_t t_info = 0, t_s = 0;
        if (more) {
          t_info = mbar_test_wait(smem_u32(&sm.info_full[(j + 1) % kInfoSlots]), ((j + 1) / kInfoSlots) & 1);
          t_s = mbar_test_wait(smem_u32(&sm.s_full[(j + 1) & 1]), ((j + 1) >> 1) & 1);
        }
        const uint32_t scol = lane_addr + kColS + 64 * (j & 1);
        float x[32];
        tmem_ld16x2_32f<32>(scol, x);
        tmem_wait_ld();
        if (inf.valid != ~0ull) {             // padding slots never attend
          const uint32_t vm = static_cast<uint32_t>(inf.valid >> (32 * hf));
#pragma unroll
          for (int i = 0; i < 32; ++i) x[i] = ((vm >> i) & 1u) ? x[i] : -INFINITY;
        }
        // exact row max; O and l rescaled when it raises the running max
        auto exact_max = [&]() -> bool {
          float m = x[0];
#pragma unroll
          for (int i = 1; i < 32; ++i) m = fmaxf(m, x[i]);
          const float mt = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 16)) * c;
          const bool need = ms != -INFINITY && mt > ms;
          if (ms == -INFINITY) ms = mt;       // first key tile of the item: O and l are still zero
          if (__any_sync(0xffffffffu, need)) {
            // rescale once the last O += P V (of step j - 1) has landed
            if (j > j0 && !warp_wait(sm, sm.pv_done[(j - 1) & 1], ((j - 1) >> 1) & 1, lane, a.err)) return false;
            tc_fence_after();
            const float f = need ? ex2_approx(ms - mt) : 1.0f;
#pragma unroll 1
            for (int ch = 0; ch < 4; ++ch) {
              const uint32_t oa = lane_addr + kColO + 16 * ch;
              float u[16];
              tmem_ld16x2_16f<64>(oa, u);
              tmem_wait_ld();
              uint32_t w[16];
#pragma unroll
              for (int i = 0; i < 16; ++i) w[i] = __float_as_uint(u[i] * f);
              tmem_st16x2_16<64>(oa, w);
            }
            tmem_wait_st();
            if (need) {
              l *= f;
              ms = mt;
            }
          }
          return true;
        };
        // P against the running max; the exact max only when a row has no
        // reference yet or its sum of P exceeds 2^8 (every P stays <= 2^8)
        uint32_t pw[16];
        if (__any_sync(0xffffffffu, ms == -INFINITY) && !(ok = exact_max())) break;
        float psum = exp_pass(x, c, ms, pw);
        if (__any_sync(0xffffffffu, psum + __shfl_xor_sync(0xffffffffu, psum, 16) > kPSumLimit)) {
          if (!(ok = exact_max())) break;
          psum = exp_pass(x, c, ms, pw);
        }
        l += psum;
        tmem_st16x2_16<16>(scol, pw);          // P(j) over the first 32 columns of its slot
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&sm.p_full[j & 1]));
        have_next = more && __all_sync(0xffffffffu, t_info);
        if (have_next) next = sm.info[(j + 1) % kInfoSlots];
        s_ready = more && __all_sync(0xffffffffu, t_s);
      }
      if (!ok) break;
      // epilogue: dense rows -> out = O / l (no coarse term); prefix rows ->
      // the normalised partial output and its log2-sum-exp2
      if (!(ok = warp_wait(sm, sm.o_full, it_n & 1, lane, a.err))) break;
      tc_fence_after();
      const float l_row = l + __shfl_xor_sync(0xffffffffu, l, 16);
      const float inv_l = 1.0f / l_row;
      const size_t poff = ((head0 + it.h) * a.n_tiles + (qtile >= 0 ? qtile : 0)) * kTile + slot;
      if (row_ok && !it.dense && hf == 0) a.part_lse[poff] = ms + __log2f(l_row);
      const bool stats = it.dense && a.st_lse != nullptr;
      const uint16_t* drow = stats && row_ok ? a.dout + a.b * a.d_sb + tok * a.d_ss + it.h * a.d_sh + 64 * hf : nullptr;
      float dsum = 0.f;
#pragma unroll 1
      for (int ch = 0; ch < 4; ++ch) {
        float y[16];
        tmem_ld16x2_16f<64>(lane_addr + kColO + 16 * ch, y);
        tmem_wait_ld();
        if (!row_ok) continue;
#pragma unroll
        for (int i = 0; i < 16; ++i) y[i] *= inv_l;
        const int col = 64 * hf + 16 * ch;
        if (stats) {                           // D = <dO, o_fine> over this thread's columns
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const uint4 w = __ldg(reinterpret_cast<const uint4*>(drow + 16 * ch) + u);
            const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int e = 0; e < 4; ++e)
              dsum = fmaf(__uint_as_float(wv[e] << 16), y[8 * u + 2 * e],
                          fmaf(__uint_as_float(wv[e] & 0xFFFF0000u), y[8 * u + 2 * e + 1], dsum));
          }
        } else if (!it.dense) {
          float4* dst = reinterpret_cast<float4*>(a.part_o + poff * kHeadDim + col);
#pragma unroll
          for (int i = 0; i < 16; i += 4) dst[i / 4] = make_float4(y[i], y[i + 1], y[i + 2], y[i + 3]);
        } else {
          const int64_t off = a.b * a.o_sb + tok * a.o_ss + it.h * a.o_sh + col;
          if (a.out_bf16) {
            uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(a.out) + off);
#pragma unroll
            for (int i = 0; i < 16; i += 8)
              dst[i / 8] = make_uint4(pack_bf16x2(y[i], y[i + 1]), pack_bf16x2(y[i + 2], y[i + 3]),
                                      pack_bf16x2(y[i + 4], y[i + 5]), pack_bf16x2(y[i + 6], y[i + 7]));
          } else {
            float4* dst = reinterpret_cast<float4*>(static_cast<float*>(a.out) + off);
#pragma unroll
            for (int i = 0; i < 16; i += 4) dst[i / 4] = make_float4(y[i], y[i + 1], y[i + 2], y[i + 3]);
          }
        }
      }
      if (stats && qtile >= 0) {
        const float d_row = dsum + __shfl_xor_sync(0xffffffffu, dsum, 16);
        if (hf == 0) {
          a.st_lse[poff] = row_ok ? ms + __log2f(l_row) : INFINITY;
          a.st_d[poff] = row_ok ? d_row : 0.f;
        }
      }
      // the next item's first O += P V overwrites O only after every softmax
      // warp's P of that step, i.e. after every warp finished reading O here
      tc_fence_before();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace pairpass

// ------------------------------------------------------------------ host side
int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return n;
}

constexpr size_t kAttnHeader = 256;   // status word, failed-call count

std::atomic<uint64_t> g_stall_ns{0};   // vsa_debug_inject_wait_timeout
constexpr size_t kMaxAttnSmem = 227 * 1024;

// Work decomposition shared by the host and the kernels (see decode_item and
// pairpass::decode). The conditioning keys that every query attends go to the
// pair pass (dense rows: all keys); the sparse pass walks the selection lists.
struct Passes {
  int32_t c0, nq, max_steps;           // sparse pass: query tiles [c0, n_tiles); steps per item <= max_steps
  int32_t n_dpairs, n_ppairs;          // pair pass, per head
  int32_t merge_prefix;                // the sparse epilogue merges the pair pass's partial output
};

Passes passes(const vsa_layout* L, const vsa_params* p, int32_t kmax) {
  Passes s{};
  const bool rows = p->sink == VSA_SINK_EXACT_KV_AND_ROWS;
  s.c0 = rows ? L->n_cond : 0;
  s.nq = L->n_tiles - s.c0;
  s.max_steps = std::max(1, std::min(kmax, candidates(L, p->sink).count)) + (p->extra_tokens > 0 ? 1 : 0);
  s.n_dpairs = rows ? (L->n_cond + 1) / 2 : 0;
  s.n_ppairs = (p->sink != VSA_SINK_OFF && L->n_cond > 0) ? (s.nq + 1) / 2 : 0;
  s.merge_prefix = s.n_ppairs > 0;
  return s;
}

// [header][tile-major K/V][tile-major Q][step records][steps per item][partial output][partial log-sum-exp]
// [extra-token tiles]
struct AttnWorkspace {
  size_t kv, qtm, sched, nsteps, part_o, part_lse, extra_kv, total;
};

AttnWorkspace attn_workspace(const vsa_layout* L, int B, int H, const vsa_params* p) {
  int32_t kmax = 0;
  vsa_select_kmax(L, p, &kmax);
  const Passes s = passes(L, p, kmax);
  const bool pairs = s.n_dpairs + s.n_ppairs > 0;
  const size_t tiles = static_cast<size_t>(B) * H * L->n_tiles;
  const size_t items = static_cast<size_t>(B) * H * s.nq;
  AttnWorkspace w{};
  w.kv = kAttnHeader;
  w.qtm = w.kv + tiles * 2 * kTileBytes;
  w.sched = w.qtm + (pairs ? tiles * kTileBytes : 0);
  w.nsteps = w.sched + align_up(items * s.max_steps * sizeof(int2), 256);
  w.part_o = w.nsteps + align_up(items * sizeof(int32_t), 256);
  w.part_lse = w.part_o + (s.merge_prefix ? tiles * kTile * kHeadDim * sizeof(float) : 0);
  w.extra_kv = w.part_lse + align_up(s.merge_prefix ? tiles * kTile * sizeof(float) : 0, 256);
  w.total = w.extra_kv + (p->extra_tokens > 0 ? tiles * 2 * kTileBytes : 0);
  return w;
}

}  // namespace
}  // namespace vsa

using namespace vsa;

extern "C" {

vsa_status vsa_sparse_attn_workspace_size(const vsa_layout* L, int32_t B, int32_t H,
                                          const vsa_params* p, size_t* bytes) {
  if (!L || !bytes || B <= 0 || H <= 0) return VSA_ERR_INVALID_ARG;
  vsa_status st = check_params(p);
  if (st != VSA_OK) return st;
  *bytes = attn_workspace(L, B, H, p).total;
  return VSA_OK;
}

}  // extern "C"

// The forward call; with `stats` (the backward pass) it writes each query
// row's log2-sum-exp2 and D = <dO, o_fine> instead of the output (g, o_coarse
// and out are then not read and may be null).
vsa_status vsa::attn_forward(const vsa_layout* L, const vsa_params* p, int32_t B, int32_t H, const void* q,
                             const void* k, const void* v, int64_t sb, int64_t ss, int64_t sh, const void* g,
                             int64_t g_sb, int64_t g_ss, int64_t g_sh, int64_t g_sd, const int32_t* idx,
                             const int32_t* cnt, int32_t kmax, const float* o_coarse, const int32_t* extra_idx,
                             const int32_t* extra_cnt, void* out, int32_t out_dtype, int64_t o_sb, int64_t o_ss,
                             int64_t o_sh, const AttnStats* stats, void* workspace, size_t workspace_bytes,
                             cudaStream_t stream) {
  if (!L) return VSA_ERR_INVALID_ARG;
  vsa_status st = check_params(p);
  if (st != VSA_OK) return st;
  st = check_qkv(q, k, v, sb, ss, sh, B, H);
  if (st != VSA_OK) return st;
  if (!idx || !cnt || !workspace) return VSA_ERR_INVALID_ARG;
  if (stats) {
    // only the statistics are written: any aligned non-null stand-ins for the rest
    static const uint16_t kZero[8] = {0};
    if (!stats->lse || !stats->d || !stats->dout) return VSA_ERR_INVALID_ARG;
    g = kZero;
    g_sb = 0;
    g_ss = g_sh = 1;
    g_sd = 0;
    o_coarse = reinterpret_cast<const float*>(workspace);
    out = workspace;
    out_dtype = VSA_OUT_F32;
    o_sb = 0;
    o_ss = o_sh = 4;
  }
  if (!g || !o_coarse || !out) return VSA_ERR_INVALID_ARG;
  if (p->extra_tokens > 0 && (!extra_idx || !extra_cnt)) return VSA_ERR_INVALID_ARG;
  if (out_dtype != VSA_OUT_F32 && out_dtype != VSA_OUT_BF16) return VSA_ERR_INVALID_ARG;
  if (g_sb < 0 || g_ss <= 0 || g_sh <= 0 || g_sd < 0 || o_sb < 0 || o_ss <= 0 || o_sh <= 0)
    return VSA_ERR_INVALID_ARG;
  const int elem = out_dtype == VSA_OUT_F32 ? 4 : 2;
  if (reinterpret_cast<uintptr_t>(out) % 16 || (o_sb * elem) % 16 || (o_ss * elem) % 16 ||
      (o_sh * elem) % 16)
    return VSA_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(o_coarse) % 16 || reinterpret_cast<uintptr_t>(workspace) % 256)
    return VSA_ERR_INVALID_ARG;
  const AttnWorkspace ws = attn_workspace(L, B, H, p);
  if (workspace_bytes < ws.total) return VSA_ERR_WORKSPACE_TOO_SMALL;
  if (!L->dev_buf) return VSA_ERR_NOT_UPLOADED;
  int32_t want_kmax = 0;
  vsa_select_kmax(L, p, &want_kmax);
  if (kmax != want_kmax) return VSA_ERR_INVALID_ARG;
  const size_t smem = attn_smem_bytes(L->n_cond);
  if (smem > kMaxAttnSmem) return VSA_ERR_UNSUPPORTED;   // thousands of conditioning tiles
  const int n_sm = sm_count();
  if (n_sm <= 0) return cuda_fail("vsa_sparse_attn_fwd: no current CUDA device");

  const DevLayout D = L->dev();
  AttnArgs a{};
  a.G.n_cond = L->n_cond;
  a.G.n_video = L->n_video;
  a.G.n_tiles = L->n_tiles;
  a.G.T = L->grid_t;
  a.G.Hg = L->grid_h;
  a.G.W = L->grid_w;
  a.G.ca = (L->grid_t + 3) / 4;
  a.G.cb = (L->grid_h + 3) / 4;
  a.G.cc = (L->grid_w + 3) / 4;
  a.G.video_start = L->video_start;
  a.origin = D.origin;
  a.count = D.count;
  a.q_ss = ss;
  a.q_sh = sh;
  a.H = H;
  a.sink = p->sink;
  a.kmax = kmax;
  const Passes ps = passes(L, p, kmax);
  a.c0 = ps.c0;
  const Candidates cand = candidates(L, p->sink);
  a.cand0 = cand.first;
  a.n_cand = cand.count;
  a.nq = ps.nq;
  a.n_items = ps.nq * H;
  a.max_steps = ps.max_steps;
  a.merge_prefix = ps.merge_prefix;
  a.n_extra = p->extra_tokens;
  a.extra_cnt = extra_cnt;
  a.valid = D.valid;
  a.idx = idx;
  a.cnt = cnt;
  a.o_coarse = o_coarse;
  a.g = static_cast<const uint16_t*>(g);
  a.g_sb = g_sb;
  a.g_ss = g_ss;
  a.g_sh = g_sh;
  a.g_sd = g_sd;
  a.out = out;
  a.out_bf16 = out_dtype == VSA_OUT_BF16;
  a.o_sb = o_sb;
  a.o_ss = o_ss;
  a.o_sh = o_sh;
  a.scale_log2 = effective_scale(p) * 1.4426950408889634f;
  a.err = static_cast<int*>(workspace);
  a.stall_ns = g_stall_ns.load(std::memory_order_relaxed);

  uint8_t* wsb = static_cast<uint8_t*>(workspace);
  a.kv = wsb + ws.kv;
  a.sched = reinterpret_cast<int2*>(wsb + ws.sched);
  a.nsteps = reinterpret_cast<int32_t*>(wsb + ws.nsteps);
  a.part_o = reinterpret_cast<const float*>(wsb + ws.part_o);
  a.part_lse = reinterpret_cast<const float*>(wsb + ws.part_lse);
  a.extra_kv = wsb + ws.extra_kv;

  pairpass::Args pa{};
  pa.n_cond = L->n_cond;
  pa.n_tiles = L->n_tiles;
  pa.perm = D.perm;
  pa.valid = D.valid;
  pa.qtm = wsb + ws.qtm;
  pa.kv = wsb + ws.kv;
  pa.H = H;
  pa.c0 = ps.c0;
  pa.n_dpairs = ps.n_dpairs;
  pa.n_ppairs = ps.n_ppairs;
  pa.n_items = H * (ps.n_dpairs + ps.n_ppairs);
  pa.part_o = reinterpret_cast<float*>(wsb + ws.part_o);
  pa.part_lse = reinterpret_cast<float*>(wsb + ws.part_lse);
  pa.out = out;
  pa.out_bf16 = a.out_bf16;
  pa.o_sb = o_sb;
  pa.o_ss = o_ss;
  pa.o_sh = o_sh;
  pa.scale_log2 = a.scale_log2;
  pa.err = a.err;
  pa.stall_ns = a.stall_ns;
  if (stats) {
    a.st_lse = pa.st_lse = stats->lse;
    a.st_d = pa.st_d = stats->d;
    a.dout = pa.dout = static_cast<const uint16_t*>(stats->dout);
    a.d_sb = pa.d_sb = stats->d_sb;
    a.d_ss = pa.d_ss = stats->d_ss;
    a.d_sh = pa.d_sh = stats->d_sh;
  }

  auto attn_kernel = g_sd > 0 ? vsa_attn_kernel<true> : vsa_attn_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return cuda_fail("vsa_sparse_attn_fwd: cudaFuncSetAttribute", e);
  const size_t pair_smem = sizeof(pairpass::Smem);
  e = cudaFuncSetAttribute(pairpass::pair_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(pair_smem));
  if (e != cudaSuccess) return cuda_fail("vsa_sparse_attn_fwd: cudaFuncSetAttribute(pair)", e);
  e = cudaMemsetAsync(workspace, 0, sizeof(int), stream);   // this call's status word only
  if (e != cudaSuccess) return cuda_fail("vsa_sparse_attn_fwd: cudaMemsetAsync", e);
  permute_qkv_kernel<<<dim3(L->n_tiles, B), 256, 0, stream>>>(
      D, static_cast<const uint16_t*>(q), static_cast<const uint16_t*>(k), static_cast<const uint16_t*>(v), sb, ss,
      sh, H, pa.n_items > 0 ? 1 : 0, wsb + ws.qtm, wsb + ws.kv);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail("vsa_sparse_attn_fwd: permute launch", e);
  if (a.n_extra > 0 && ps.nq > 0) {
    gather_extra_kernel<<<dim3(ps.nq, H, B), 256, 0, stream>>>(
        static_cast<const uint16_t*>(k), static_cast<const uint16_t*>(v), sb, ss, sh, H, L->n_tiles, ps.c0,
        L->seq_len, extra_idx, extra_cnt, a.n_extra, wsb + ws.extra_kv);
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail("vsa_sparse_attn_fwd: extra-token gather launch", e);
  }
  schedule_kernel<<<dim3(a.n_items, B), kSchedThreads, 0, stream>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail("vsa_sparse_attn_fwd: schedule launch", e);
  for (int b = 0; b < B; ++b) {
    if (pa.n_items > 0) {
      pa.b = b;
      pairpass::pair_attn_kernel<<<std::max(1, std::min(pa.n_items, 2 * n_sm)), pairpass::kThreads, pair_smem,
                                   stream>>>(pa);
      e = cudaGetLastError();
      if (e != cudaSuccess) return cuda_fail("vsa_sparse_attn_fwd: pair pass launch", e);
    }
    a.b = b;
    a.q = static_cast<const uint16_t*>(q) + b * sb;
    // two CTAs per SM, 256 TMEM columns each
    attn_kernel<<<std::max(1, std::min(a.n_items, 2 * n_sm)), kThreads, smem, stream>>>(a);
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail("vsa_sparse_attn_fwd: launch", e);
  }
  return VSA_OK;
}

extern "C" {

vsa_status vsa_sparse_attn_fwd(const vsa_layout* L, const vsa_params* p, int32_t B, int32_t H,
                               const void* q, const void* k, const void* v, int64_t sb, int64_t ss,
                               int64_t sh, const void* g, int64_t g_sb, int64_t g_ss, int64_t g_sh,
                               int64_t g_sd, const int32_t* idx, const int32_t* cnt, int32_t kmax,
                               const float* o_coarse, const int32_t* extra_idx, const int32_t* extra_cnt,
                               void* out, int32_t out_dtype, int64_t o_sb,
                               int64_t o_ss, int64_t o_sh, void* workspace, size_t workspace_bytes,
                               cudaStream_t stream) {
  if (!g || !o_coarse || !out) return VSA_ERR_INVALID_ARG;
  return attn_forward(L, p, B, H, q, k, v, sb, ss, sh, g, g_sb, g_ss, g_sh, g_sd, idx, cnt, kmax, o_coarse,
                      extra_idx, extra_cnt, out, out_dtype, o_sb, o_ss, o_sh, nullptr, workspace, workspace_bytes,
                      stream);
}

vsa_status vsa_debug_inject_wait_timeout(uint64_t timeout_ns) {
  g_stall_ns.store(timeout_ns, std::memory_order_relaxed);
  return VSA_OK;
}

vsa_status vsa_sparse_attn_workspace_init(void* workspace, cudaStream_t stream) {
  if (!workspace || reinterpret_cast<uintptr_t>(workspace) % 256) return VSA_ERR_INVALID_ARG;
  cudaError_t e = cudaMemsetAsync(workspace, 0, kAttnHeader, stream);
  if (e != cudaSuccess) return cuda_fail("vsa_sparse_attn_workspace_init: cudaMemsetAsync", e);
  return VSA_OK;
}

vsa_status vsa_sparse_attn_failed_calls(const void* workspace, cudaStream_t stream, uint32_t* count) {
  if (!workspace || !count) return VSA_ERR_INVALID_ARG;
  cudaError_t e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return cuda_fail("vsa_sparse_attn_failed_calls: cudaStreamSynchronize", e);
  e = cudaMemcpy(count, static_cast<const int*>(workspace) + 1, sizeof(uint32_t), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail("vsa_sparse_attn_failed_calls: cudaMemcpy", e);
  return VSA_OK;
}

vsa_status vsa_sparse_attn_status(const void* workspace, cudaStream_t stream) {
  if (!workspace) return VSA_ERR_INVALID_ARG;
  cudaError_t e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return cuda_fail("vsa_sparse_attn_status: cudaStreamSynchronize", e);
  int err = 0;
  e = cudaMemcpy(&err, workspace, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail("vsa_sparse_attn_status: cudaMemcpy", e);
  return err == 0 ? VSA_OK : static_cast<vsa_status>(err);
}

}  // extern "C"
