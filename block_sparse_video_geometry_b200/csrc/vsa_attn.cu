// Fine branch of VSA block-sparse attention + gate combine, for sm_100a.
//
// Each query tile attends exactly to every conditioning key token and to the
// video tiles of its selection list ("BSAI FastH3 Native VSA (recipe)", "The
// mechanism, briefly" and "The inputs that matter", sink_conditioning;
// "ComfyUI-Ref2VA-VSA", "Multimodal Dense-Exempt Prefix" and "Video-Only
// Sparse Attention"); with exact_kv_and_rows the conditioning query tiles
// attend the whole sequence. The epilogue writes o_fine + g * o_coarse.
//
// Design (B200):
//  * Work item = two query tiles of one (batch, head) stacked into a 128-row
//    tcgen05 tile (M = 128). The key tiles of the item are the union of the two
//    tiles' key lists; each 128x64 score block is masked per 64-row half for
//    key tiles that only one of the two tiles selected. Conditioning key tiles
//    are shared by every query tile, so they run at full M = 128 efficiency.
//  * Q, K, V are read straight from the natural [B, S, H, 128] layout by TMA
//    (no multicast): a 3-D map (d, head, token) for 64-token conditioning runs
//    and a 5-D map (d, head, w, h, t) over the video latent grid whose 4x4x4
//    box lands a video cube in shared memory in slot order; cubes cut by the
//    grid edge are zero-filled by the TMA unit and masked in the softmax. Each
//    64-key step gathers 256 rows of 128 B; a TMA issue occupies its warp for
//    a few hundred cycles, so K and V have a producer warp each, and two CTAs
//    per SM keep the TMA unit busy.
//  * Warp roles per CTA: warp 0 walks the merged key list, loads Q and K and
//    publishes per-step tile info; warp 1 loads V; warp 2 owns TMEM and issues
//    tcgen05.mma (S = Q K^T into one of two TMEM score buffers; O += P V with P
//    read from TMEM); warps 3-6 run the fp32 online softmax (exp2, lazy rescale
//    of O in TMEM when the running max grows by more than 2^8), write P as bf16
//    over the score buffer with tcgen05.st, and run the epilogue. About 100 KB
//    of shared memory and 256 TMEM columns per CTA: two CTAs share an SM so
//    that one's softmax overlaps the other's tensor work.
//  * Every wait is bounded: a wait that runs out sets an error word in the
//    workspace, raises an abort flag that ends the other roles' loops, drains
//    in-flight TMA and MMA work and frees TMEM before the block exits.

#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <climits>
#include <cmath>
#include <mutex>

#include "sm100.cuh"
#include "vsa_internal.h"

namespace vsa {
namespace {

using namespace sm100;

constexpr int kKStages = 2;
constexpr int kVStages = 2;
static_assert(kKStages == kVStages, "the producers share one stage counter");
constexpr int kInfoSlots = 4;
constexpr int kThreads = 224;
constexpr int kWarpK = 0, kWarpV = 1, kWarpMma = 2;   // warps 3..6: softmax / epilogue
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kColO = 0, kColS0 = 128, kColS1 = 192;   // P (bf16) overwrites S columns 0..31
constexpr float kRescaleLog2 = 8.0f;
constexpr uint32_t kIdescS = idesc_bf16_f32(128, 64, 0, 0);    // S = Q K^T, both K-major
constexpr uint32_t kIdescPV = idesc_bf16_f32(128, 128, 0, 1);  // O = P V, V is MN-major
constexpr uint64_t kTimeoutNs = 4000000000ull;
constexpr uint64_t kDrainNs = 200000000ull;

struct StageInfo {
  int32_t tile;
  int32_t mask;   // bit 0: first query tile lists it, bit 1: second query tile lists it
  int32_t last;   // last key tile of the work item
  int32_t pad;
  unsigned long long valid;
};

struct AttnSmem {
  uint8_t q[2][128 * 128];             // [d half][128 rows x 128 B], SW128
  uint8_t k[kKStages][2][64 * 128];    // [stage][d half][64 keys x 128 B], SW128
  uint8_t v[kVStages][2][64 * 128];
  StageInfo info[kInfoSlots];
  uint64_t k_full[kKStages], k_empty[kKStages], v_full[kVStages], v_empty[kVStages];
  uint64_t info_full[kInfoSlots];
  uint64_t q_full, q_empty, s_full[2], p_full[2], o_done, o_full, o_empty, drain;
  uint32_t tmem_base;
  int abort;
  int2 cond[1];                        // conditioning tiles (first token, count); n_cond entries
};

size_t attn_smem_bytes(int n_cond) {
  return sizeof(AttnSmem) + sizeof(int2) * static_cast<size_t>(std::max(0, n_cond - 1)) + 1024;
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
  int32_t H, b, sink, kmax;
  int32_t c0;                // first query tile of the sparse item range
  int32_t np_dense, np_sparse, n_dense_items, n_items;
  const int32_t* idx;
  const int32_t* cnt;
  const float* o_coarse;
  const uint16_t* g;
  int64_t g_sb, g_ss, g_sh;
  void* out;
  int32_t out_bf16;
  int64_t o_sb, o_ss, o_sh;
  float scale_log2;
  int* err;
};

struct Item {
  int h, qa, qb, dense;
};

__device__ __forceinline__ Item decode_item(const AttnArgs& a, int item) {
  Item it;
  if (item < a.n_dense_items) {
    it.h = item / a.np_dense;
    it.qa = 2 * (item % a.np_dense);
    it.qb = it.qa + 1 < a.G.n_cond ? it.qa + 1 : -1;
    it.dense = 1;
  } else {
    const int r = item - a.n_dense_items;
    it.h = r / a.np_sparse;
    it.qa = a.c0 + 2 * (r % a.np_sparse);
    it.qb = it.qa + 1 < a.G.n_tiles ? it.qa + 1 : -1;
    it.dense = 0;
  }
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

// One 64x128 tile (two 64-column halves) of Q, K or V into shared memory.
__device__ __forceinline__ void load_tile(const AttnSmem& sm, const Geom& G, const CUtensorMap* mc,
                                          const CUtensorMap* mv, int tile, int h, uint32_t dst0,
                                          uint32_t dst1, uint32_t bar) {
  if (tile < G.n_cond) {
    const int tok = sm.cond[tile].x;
    tma_load_3d(dst0, mc, bar, 0, h, tok);
    tma_load_3d(dst1, mc, bar, 64, h, tok);
  } else {
    int t0, h0, w0;
    unsigned long long m;
    video_cube(G, tile - G.n_cond, t0, h0, w0, m);
    tma_load_5d(dst0, mv, bar, 0, h, w0, h0, t0);
    tma_load_5d(dst1, mv, bar, 64, h, w0, h0, t0);
  }
}

// Ascending list of video ordinals, read 32 at a time by the whole warp with
// the next chunk prefetched; every lane sees the same sequence.
struct ListReader {
  const int32_t* base;
  int n, pos;
  int32_t chunk, pre;
  __device__ __forceinline__ void init(const int32_t* b, int len, int lane) {
    base = b;
    n = len;
    pos = 0;
    chunk = lane < n ? b[lane] : INT_MAX;
    pre = 32 + lane < n ? b[32 + lane] : INT_MAX;
  }
  __device__ __forceinline__ int32_t peek() const {
    const int32_t x = __shfl_sync(0xffffffffu, chunk, pos & 31);
    return pos < n ? x : INT_MAX;
  }
  __device__ __forceinline__ void pop(int lane) {
    ++pos;
    if ((pos & 31) == 0) {
      chunk = pre;
      const int nx = pos + 32 + lane;
      pre = nx < n ? base[nx] : INT_MAX;
    }
  }
};

__device__ __forceinline__ void raise_abort(AttnSmem& sm, int* err) {
  atomicExch(err, VSA_ERR_TIMEOUT);
  *reinterpret_cast<volatile int*>(&sm.abort) = 1;
}

// Lane 0 waits; the result is broadcast so the warp leaves a loop together.
__device__ __forceinline__ bool warp_wait(AttnSmem& sm, uint64_t& bar, uint32_t parity, int lane,
                                          int* err) {
  int ok = 1;
  if (lane == 0) {
    ok = mbar_wait(smem_u32(&bar), parity, &sm.abort, kTimeoutNs) ? 1 : 0;
    if (!ok) raise_abort(sm, err);
  }
  ok = __shfl_sync(0xffffffffu, ok, 0);
  __syncwarp();
  return ok != 0;
}

// Pairwise tree reductions over 64 values: short dependency chains.
__device__ __forceinline__ float tree_max64(const float (&x)[64]) {
  float t[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) t[i] = fmaxf(x[i], x[i + 32]);
#pragma unroll
  for (int w = 16; w >= 1; w >>= 1)
#pragma unroll
    for (int i = 0; i < w; ++i) t[i] = fmaxf(t[i], t[i + w]);
  return t[0];
}

__global__ void __launch_bounds__(kThreads, 2)
vsa_attn_kernel(const __grid_constant__ AttnArgs a, const __grid_constant__ CUtensorMap tq_c,
                const __grid_constant__ CUtensorMap tq_v, const __grid_constant__ CUtensorMap tk_c,
                const __grid_constant__ CUtensorMap tk_v, const __grid_constant__ CUtensorMap tv_c,
                const __grid_constant__ CUtensorMap tv_v) {
  extern __shared__ uint8_t smem_raw[];
  AttnSmem& sm = *reinterpret_cast<AttnSmem*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Geom& G = a.G;

  for (int i = threadIdx.x; i < G.n_cond; i += kThreads)
    sm.cond[i] = make_int2(a.origin[i].x, a.count[i]);
  if (threadIdx.x == 0) {
    for (int s = 0; s < kKStages; ++s) {
      mbar_init(smem_u32(&sm.k_full[s]), 1);
      mbar_init(smem_u32(&sm.k_empty[s]), 1);
    }
    for (int s = 0; s < kVStages; ++s) {
      mbar_init(smem_u32(&sm.v_full[s]), 1);
      mbar_init(smem_u32(&sm.v_empty[s]), 1);
    }
    for (int s = 0; s < kInfoSlots; ++s) mbar_init(smem_u32(&sm.info_full[s]), 1);
    mbar_init(smem_u32(&sm.q_full), 1);
    mbar_init(smem_u32(&sm.q_empty), 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&sm.s_full[i]), 1);
      mbar_init(smem_u32(&sm.p_full[i]), 4);     // one arrival per softmax warp
    }
    mbar_init(smem_u32(&sm.o_done), 1);
    mbar_init(smem_u32(&sm.o_full), 1);
    mbar_init(smem_u32(&sm.o_empty), 4);
    mbar_init(smem_u32(&sm.drain), 1);
    sm.abort = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    for (const CUtensorMap* m : {&tq_c, &tq_v, &tk_c, &tk_v}) tma_prefetch_desc(m);
  }
  if (warp == kWarpV && lane == 0) {
    tma_prefetch_desc(&tv_c);
    tma_prefetch_desc(&tv_v);
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
    // Both producer warps walk the same key list; the K warp also loads Q and
    // publishes the per-step tile info.
    const bool is_k = warp == kWarpK;
    const CUtensorMap* mc = is_k ? &tk_c : &tv_c;
    const CUtensorMap* mv = is_k ? &tk_v : &tv_v;
    uint64_t* full = is_k ? sm.k_full : sm.v_full;
    uint64_t* empty = is_k ? sm.k_empty : sm.v_empty;
    uint32_t step = 0, issued = 0;
    int it_n = 0, q_loads = 0;
    bool ok = true;
    for (int item = blockIdx.x; ok && item < a.n_items; item += gridDim.x, ++it_n) {
      const Item it = decode_item(a, item);
      if (is_k) {
        if (!(ok = warp_wait(sm, sm.q_empty, (it_n & 1) ^ 1, lane, a.err))) break;
        if (lane == 0) {
          const uint32_t bar = smem_u32(&sm.q_full);
          mbar_arrive_expect_tx(bar, (it.qb >= 0 ? 2u : 1u) * 16384u);
          load_tile(sm, G, &tq_c, &tq_v, it.qa, it.h, smem_u32(sm.q[0]), smem_u32(sm.q[1]), bar);
          if (it.qb >= 0)
            load_tile(sm, G, &tq_c, &tq_v, it.qb, it.h, smem_u32(sm.q[0] + 8192),
                      smem_u32(sm.q[1] + 8192), bar);
        }
        ++q_loads;
      }
      const int both = it.qb >= 0 ? 3 : 1;
      const int n_dense = it.dense ? G.n_tiles : G.n_cond;
      ListReader la, lb;
      const size_t row = (static_cast<size_t>(a.b) * a.H + it.h) * G.n_tiles;
      const int na = it.dense ? 0 : a.cnt[row + it.qa];
      const int nb = (it.dense || it.qb < 0) ? 0 : a.cnt[row + it.qb];
      la.init(a.idx + (row + it.qa) * a.kmax, na, lane);
      lb.init(a.idx + (row + (it.qb >= 0 ? it.qb : it.qa)) * a.kmax, nb, lane);
      int j = 0;
      // next key tile of the item: the dense part first, then the merged lists
      auto next = [&](int& tile, int& mask) -> bool {
        if (j < n_dense) {
          tile = j++;
          mask = both;
          return true;
        }
        const int32_t x0 = la.peek(), y0 = lb.peek();
        if (x0 == INT_MAX && y0 == INT_MAX) return false;
        const int32_t t = min(x0, y0);
        mask = (x0 == t ? 1 : 0) | (y0 == t ? 2 : 0);
        if (x0 == t) la.pop(lane);
        if (y0 == t) lb.pop(lane);
        tile = G.n_cond + t;
        return true;
      };
      int tile, mask, ntile, nmask;
      bool have = next(tile, mask);
      while (have) {
        const bool more = next(ntile, nmask);
        const int st = step % kKStages;
        if (!(ok = warp_wait(sm, empty[st], ((step / kKStages) & 1) ^ 1, lane, a.err))) break;
        if (is_k && lane == 0) {
          StageInfo& inf = sm.info[step % kInfoSlots];
          inf.tile = tile;
          inf.mask = mask;
          inf.last = more ? 0 : 1;
          inf.valid = tile_mask(sm, G, tile);
          mbar_arrive(smem_u32(&sm.info_full[step % kInfoSlots]));
        }
        if (lane == 0) {
          uint8_t (*buf)[64 * 128] = is_k ? sm.k[st] : sm.v[st];
          mbar_arrive_expect_tx(smem_u32(&full[st]), 16384u);
          load_tile(sm, G, mc, mv, tile, it.h, smem_u32(buf[0]), smem_u32(buf[1]), smem_u32(&full[st]));
        }
        __syncwarp();
        ++issued;
        ++step;
        tile = ntile;
        mask = nmask;
        have = more;
      }
    }
    if (!ok && lane == 0) {
      // let every issued TMA load land before the block can exit: the last
      // fill of each stage, and the last Q load
      for (uint32_t i = (issued > kKStages ? issued - kKStages : 0); i < issued; ++i)
        mbar_wait(smem_u32(&full[i % kKStages]), (i / kKStages) & 1, nullptr, kDrainNs);
      if (is_k && q_loads > 0) mbar_wait(smem_u32(&sm.q_full), (q_loads - 1) & 1, nullptr, kDrainNs);
    }
  } else if (warp == kWarpMma) {
    // ----------------------------------------------------------------- MMA
    bool ok = true;
    if (lane == 0) {
      uint32_t step = 0;
      int it_n = 0;
      auto pv = [&](uint32_t st, bool first) -> bool {
        if (!mbar_wait(smem_u32(&sm.p_full[st & 1]), (st >> 1) & 1, &sm.abort, kTimeoutNs)) return false;
        if (first && !mbar_wait(smem_u32(&sm.o_empty), (it_n & 1) ^ 1, &sm.abort, kTimeoutNs)) return false;
        const int vs = st % kVStages;
        if (!mbar_wait(smem_u32(&sm.v_full[vs]), (st / kVStages) & 1, &sm.abort, kTimeoutNs)) return false;
        tc_fence_after();
        const uint32_t pcol = tmem + ((st & 1) ? kColS1 : kColS0);
        const uint32_t vbase = smem_u32(sm.v[vs][0]);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t bd = smem_desc_sw128(vbase + kk * 2048, 8192, 1024);
          umma_ts(tmem + kColO, pcol + kk * 8, bd, kIdescPV, (first && kk == 0) ? 0u : 1u);
        }
        umma_commit(smem_u32(&sm.v_empty[vs]));
        umma_commit(smem_u32(&sm.o_done));
        return true;
      };
      for (int item = blockIdx.x; ok && item < a.n_items; item += gridDim.x, ++it_n) {
        if (!(ok = mbar_wait(smem_u32(&sm.q_full), it_n & 1, &sm.abort, kTimeoutNs))) break;
        int j = 0;
        bool last = false;
        while (!last) {
          const int ks = step % kKStages;
          if (!(ok = mbar_wait(smem_u32(&sm.k_full[ks]), (step / kKStages) & 1, &sm.abort, kTimeoutNs))) break;
          tc_fence_after();
          last = sm.info[step % kInfoSlots].last != 0;
          const uint32_t qbase = smem_u32(sm.q[0]);
          const uint32_t kbase = smem_u32(sm.k[ks][0]);
          const uint32_t dS = tmem + ((step & 1) ? kColS1 : kColS0);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = (kk & 3) * 32;   // 16 bf16 = 32 B K step inside a swizzle row
            const uint64_t ad = smem_desc_sw128(qbase + (kk >> 2) * 16384 + off, 16, 1024);
            const uint64_t bd = smem_desc_sw128(kbase + (kk >> 2) * 8192 + off, 16, 1024);
            umma_ss(dS, ad, bd, kIdescS, kk > 0 ? 1u : 0u);
          }
          umma_commit(smem_u32(&sm.k_empty[ks]));
          umma_commit(smem_u32(&sm.s_full[step & 1]));
          if (last) umma_commit(smem_u32(&sm.q_empty));
          if (j > 0 && !(ok = pv(step - 1, j == 1))) break;
          ++j;
          ++step;
        }
        if (!ok) break;
        if (!(ok = pv(step - 1, j == 1))) break;
        umma_commit(smem_u32(&sm.o_full));
      }
      if (!ok) raise_abort(sm, a.err);
      // drain: every MMA issued so far has completed before TMEM is freed
      umma_commit(smem_u32(&sm.drain));
      mbar_wait(smem_u32(&sm.drain), 0, nullptr, kDrainNs);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------ softmax / epilogue
    const int quad = warp & 3;              // TMEM lane quadrant of this warp
    const int r = quad * 32 + lane;         // row of the 128-row tile
    const int half = r >> 6;                // 0: first query tile, 1: second
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    const float c = a.scale_log2;
    uint32_t step = 0;
    int it_n = 0;
    bool ok = true;
    for (int item = blockIdx.x; ok && item < a.n_items; item += gridDim.x, ++it_n) {
      const Item it = decode_item(a, item);
      float ms = -INFINITY, l = 0.f;        // running max (scaled, log2 domain) and sum
      bool last = false;
      while (!last) {
        if (!(ok = warp_wait(sm, sm.info_full[step % kInfoSlots], (step / kInfoSlots) & 1, lane, a.err))) break;
        const StageInfo inf = sm.info[step % kInfoSlots];
        last = inf.last != 0;
        if (!(ok = warp_wait(sm, sm.s_full[step & 1], (step >> 1) & 1, lane, a.err))) break;
        tc_fence_after();
        const uint32_t scol = lane_addr + ((step & 1) ? kColS1 : kColS0);
        uint32_t pw[32];
        if ((inf.mask >> half) & 1) {
          float x[64];
          {
            uint32_t u0[32], u1[32];
            tmem_ld32(scol, u0);
            tmem_ld32(scol + 32, u1);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              x[i] = __uint_as_float(u0[i]);
              x[32 + i] = __uint_as_float(u1[i]);
            }
          }
          if (inf.valid != ~0ull) {           // partial tile: padded keys never attend
            const uint32_t lo = static_cast<uint32_t>(inf.valid), hi = static_cast<uint32_t>(inf.valid >> 32);
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              x[i] = ((lo >> i) & 1u) ? x[i] : -INFINITY;
              x[32 + i] = ((hi >> i) & 1u) ? x[32 + i] : -INFINITY;
            }
          }
          const float mt = tree_max64(x) * c;
          const bool need = ms != -INFINITY && mt > ms + kRescaleLog2;
          if (ms == -INFINITY) ms = mt;       // first key tile of this row: O and l are still zero
          if (__any_sync(0xffffffffu, need)) {
            // rescale this warp's rows of O once the previous P V has landed
            if (!(ok = warp_wait(sm, sm.o_done, (step - 1) & 1, lane, a.err))) break;
            tc_fence_after();
            const float f = need ? ex2_approx(ms - mt) : 1.0f;
#pragma unroll 1
            for (int ch = 0; ch < 4; ++ch) {
              uint32_t u[32];
              tmem_ld32(lane_addr + kColO + ch * 32, u);
              tmem_wait_ld();
#pragma unroll
              for (int i = 0; i < 32; ++i) u[i] = __float_as_uint(__uint_as_float(u[i]) * f);
              tmem_st32(lane_addr + kColO + ch * 32, u);
            }
            tmem_wait_st();
            if (need) {
              l *= f;
              ms = mt;
            }
          }
          float ps[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float p0 = ex2_approx(fmaf(x[2 * i], c, -ms));
            const float p1 = ex2_approx(fmaf(x[2 * i + 1], c, -ms));
            ps[i & 3] += p0 + p1;
            pw[i] = pack_bf16x2(p0, p1);
          }
          l += (ps[0] + ps[1]) + (ps[2] + ps[3]);
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) pw[i] = 0u;     // rows of the other query tile
        }
        tmem_st32(scol, pw);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&sm.p_full[step & 1]));
        ++step;
      }
      if (!ok) break;
      // epilogue: out = O / l + g * o_coarse
      if (!(ok = warp_wait(sm, sm.o_full, it_n & 1, lane, a.err))) break;
      tc_fence_after();
      const int qt = half ? it.qb : it.qa;
      const int slot = r & 63;
      bool row_ok = qt >= 0;
      int64_t tok = 0;
      float gate = 0.f;
      const float* oc = nullptr;
      if (row_ok) row_ok = (tile_mask(sm, G, qt) >> slot) & 1ull;
      if (row_ok) {
        tok = tile_token(sm, G, qt, slot);
        const bool coarse = !(a.sink == VSA_SINK_EXACT_KV_AND_ROWS && qt < G.n_cond);
        if (coarse) {
          gate = __uint_as_float(static_cast<uint32_t>(a.g[a.b * a.g_sb + tok * a.g_ss + it.h * a.g_sh]) << 16);
          oc = a.o_coarse + ((static_cast<size_t>(a.b) * a.H + it.h) * G.n_tiles + qt) * kHeadDim;
        }
      }
      const float inv_l = 1.0f / l;
#pragma unroll 1
      for (int ch = 0; ch < 4; ++ch) {
        uint32_t u[32];
        tmem_ld32(lane_addr + kColO + ch * 32, u);
        tmem_wait_ld();
        if (row_ok) {
          float y[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) y[i] = __uint_as_float(u[i]) * inv_l;
          if (oc) {
#pragma unroll
            for (int i = 0; i < 32; i += 4) {
              const float4 cv = *reinterpret_cast<const float4*>(oc + ch * 32 + i);
              y[i] = fmaf(gate, cv.x, y[i]);
              y[i + 1] = fmaf(gate, cv.y, y[i + 1]);
              y[i + 2] = fmaf(gate, cv.z, y[i + 2]);
              y[i + 3] = fmaf(gate, cv.w, y[i + 3]);
            }
          }
          const int64_t off = a.b * a.o_sb + tok * a.o_ss + it.h * a.o_sh + ch * 32;
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
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&sm.o_empty));
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ------------------------------------------------------------------ host side
PFN_cuTensorMapEncodeTiled_v12000 get_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 3-D map (d, head, token) over a [S, H, 128] bf16 slab; box 64 x 1 x 64.
bool make_cond_map(CUtensorMap* m, const void* base, int64_t S, int H, int64_t ss, int64_t sh) {
  auto enc = get_encoder();
  if (!enc) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(kHeadDim), static_cast<cuuint64_t>(H),
                        static_cast<cuuint64_t>(S)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(sh * 2), static_cast<cuuint64_t>(ss * 2)};
  cuuint32_t box[3] = {64, 1, 64};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 5-D map (d, head, w, h, t) over the video latent grid; box 64 x 1 x 4 x 4 x 4.
bool make_video_map(CUtensorMap* m, const void* base, int T, int Hg, int W, int H, int64_t ss,
                    int64_t sh) {
  auto enc = get_encoder();
  if (!enc) return false;
  cuuint64_t dims[5] = {static_cast<cuuint64_t>(kHeadDim), static_cast<cuuint64_t>(H),
                        static_cast<cuuint64_t>(W), static_cast<cuuint64_t>(Hg),
                        static_cast<cuuint64_t>(T)};
  cuuint64_t strides[4] = {static_cast<cuuint64_t>(sh * 2), static_cast<cuuint64_t>(ss * 2),
                           static_cast<cuuint64_t>(ss * 2 * W),
                           static_cast<cuuint64_t>(ss * 2 * W * Hg)};
  cuuint32_t box[5] = {64, 1, 4, 4, 4};
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return n;
}

constexpr size_t kAttnWorkspace = 256;   // error word
constexpr size_t kMaxAttnSmem = 227 * 1024;

}  // namespace
}  // namespace vsa

using namespace vsa;

extern "C" {

vsa_status vsa_sparse_attn_workspace_size(const vsa_layout* L, int32_t B, int32_t H,
                                          const vsa_params* p, size_t* bytes) {
  if (!L || !bytes || B <= 0 || H <= 0) return VSA_ERR_INVALID_ARG;
  vsa_status st = check_params(p);
  if (st != VSA_OK) return st;
  *bytes = kAttnWorkspace;
  return VSA_OK;
}

vsa_status vsa_sparse_attn_fwd(const vsa_layout* L, const vsa_params* p, int32_t B, int32_t H,
                               const void* q, const void* k, const void* v, int64_t sb, int64_t ss,
                               int64_t sh, const void* g, int64_t g_sb, int64_t g_ss, int64_t g_sh,
                               const int32_t* idx, const int32_t* cnt, int32_t kmax,
                               const float* o_coarse, void* out, int32_t out_dtype, int64_t o_sb,
                               int64_t o_ss, int64_t o_sh, void* workspace, size_t workspace_bytes,
                               cudaStream_t stream) {
  if (!L) return VSA_ERR_INVALID_ARG;
  vsa_status st = check_params(p);
  if (st != VSA_OK) return st;
  st = check_qkv(q, k, v, sb, ss, sh, B, H);
  if (st != VSA_OK) return st;
  if (!g || !idx || !cnt || !o_coarse || !out || !workspace) return VSA_ERR_INVALID_ARG;
  if (out_dtype != VSA_OUT_F32 && out_dtype != VSA_OUT_BF16) return VSA_ERR_INVALID_ARG;
  if (g_sb < 0 || g_ss <= 0 || g_sh <= 0 || o_sb < 0 || o_ss <= 0 || o_sh <= 0) return VSA_ERR_INVALID_ARG;
  const int elem = out_dtype == VSA_OUT_F32 ? 4 : 2;
  if (reinterpret_cast<uintptr_t>(out) % 16 || (o_sb * elem) % 16 || (o_ss * elem) % 16 ||
      (o_sh * elem) % 16)
    return VSA_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(o_coarse) % 16 || reinterpret_cast<uintptr_t>(workspace) % 256)
    return VSA_ERR_INVALID_ARG;
  if (workspace_bytes < kAttnWorkspace) return VSA_ERR_WORKSPACE_TOO_SMALL;
  if (!L->dev_buf) return VSA_ERR_NOT_UPLOADED;
  int32_t want_kmax = 0;
  vsa_select_kmax(L, p, &want_kmax);
  if (kmax != want_kmax) return VSA_ERR_INVALID_ARG;
  const size_t smem = attn_smem_bytes(L->n_cond);
  if (smem > kMaxAttnSmem) return VSA_ERR_UNSUPPORTED;   // more than ~16k conditioning tiles
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
  a.H = H;
  a.sink = p->sink;
  a.kmax = kmax;
  const bool rows = p->sink == VSA_SINK_EXACT_KV_AND_ROWS;
  a.c0 = rows ? L->n_cond : 0;
  a.np_dense = rows ? (L->n_cond + 1) / 2 : 0;
  a.np_sparse = (L->n_tiles - a.c0 + 1) / 2;
  a.n_dense_items = a.np_dense * H;
  a.n_items = a.n_dense_items + a.np_sparse * H;
  a.idx = idx;
  a.cnt = cnt;
  a.o_coarse = o_coarse;
  a.g = static_cast<const uint16_t*>(g);
  a.g_sb = g_sb;
  a.g_ss = g_ss;
  a.g_sh = g_sh;
  a.out = out;
  a.out_bf16 = out_dtype == VSA_OUT_BF16;
  a.o_sb = o_sb;
  a.o_ss = o_ss;
  a.o_sh = o_sh;
  a.scale_log2 = effective_scale(p) * 1.4426950408889634f;
  a.err = static_cast<int*>(workspace);

  cudaError_t e = cudaFuncSetAttribute(vsa_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return cuda_fail("vsa_sparse_attn_fwd: cudaFuncSetAttribute", e);
  // Two CTAs per SM when their shared memory fits (TMEM holds two 256-column
  // CTAs); registers are bounded for two by __launch_bounds__.
  int dev = 0, smem_sm = 0, smem_resv = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev);
  cudaDeviceGetAttribute(&smem_resv, cudaDevAttrReservedSharedMemoryPerBlock, dev);
  const int per_sm = 2 * (smem + smem_resv) <= static_cast<size_t>(smem_sm) ? 2 : 1;
  e = cudaFuncSetAttribute(vsa_attn_kernel, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
  if (e != cudaSuccess) return cuda_fail("vsa_sparse_attn_fwd: cudaFuncSetAttribute(carveout)", e);
  e = cudaMemsetAsync(workspace, 0, kAttnWorkspace, stream);
  if (e != cudaSuccess) return cuda_fail("vsa_sparse_attn_fwd: cudaMemsetAsync", e);
  const int grid = std::max(1, std::min(a.n_items, n_sm * per_sm));
  const uint16_t* qq = static_cast<const uint16_t*>(q);
  const uint16_t* kk = static_cast<const uint16_t*>(k);
  const uint16_t* vv = static_cast<const uint16_t*>(v);
  for (int b = 0; b < B; ++b) {
    CUtensorMap m[6];
    const int64_t vo = L->video_start * ss;
    const uint16_t* bases[3] = {qq + b * sb, kk + b * sb, vv + b * sb};
    for (int t = 0; t < 3; ++t) {
      if (!make_cond_map(&m[2 * t], bases[t], L->seq_len, H, ss, sh))
        return cuda_fail("vsa_sparse_attn_fwd: cuTensorMapEncodeTiled (token map)");
      if (!make_video_map(&m[2 * t + 1], bases[t] + vo, L->grid_t, L->grid_h, L->grid_w, H, ss, sh))
        return cuda_fail("vsa_sparse_attn_fwd: cuTensorMapEncodeTiled (video grid map)");
    }
    a.b = b;
    vsa_attn_kernel<<<grid, kThreads, smem, stream>>>(a, m[0], m[1], m[2], m[3], m[4], m[5]);
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail("vsa_sparse_attn_fwd: launch", e);
  }
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
