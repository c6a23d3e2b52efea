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
//    128 query tiles against one 64-token key tile is one M = 128, N = 64
//    tcgen05 product per split term: Qbar = hi + mid + lo in bf16 (24 mantissa
//    bits, held in TMEM as the A operand), K exact in bf16, fp32 accumulation,
//    so the scores carry fp32 rounding only (3 x 8 MMAs per key tile). The key
//    tiles stream through shared memory in candidate order (four stages); each
//    of 128 threads owns one query tile (TMEM lane r = query tile r of the
//    block), skips the tiles its ascending selection list holds (a pointer
//    walks the list), and keeps a running top-E in shared memory (an unordered
//    array plus the position of its weakest entry, which a new token must beat).

#include <cuda_runtime.h>

#include <algorithm>
#include <climits>
#include <cmath>

#include "sm100.cuh"
#include "vsa_internal.h"

namespace vsa {
namespace {

using namespace sm100;

constexpr int kXThreads = 192;           // 6 warps: 0 copies, 1 MMAs, 2-5 one query tile per thread
constexpr int kXRows = 128;
constexpr int kXStages = 4;
constexpr int kXMaxE = VSA_MAX_EXTRA_TOKENS;
constexpr uint32_t kXTmemCols = 512;
constexpr uint32_t kXColA = 0;           // Qbar split terms: 64 columns of bf16 pairs each
constexpr uint32_t kXColD = 192;         // two score buffers of 64 fp32 columns
constexpr uint32_t kXIdesc = idesc_bf16_f32(128, 64, 0, 0);
constexpr uint64_t kXTimeoutNs = 4000000000ull;
constexpr uint64_t kXDrainNs = 200000000ull;
constexpr size_t kXHeader = 256;         // status word

struct XSmem {
  uint8_t k[kXStages][16384];
  float val[kXMaxE * kXRows];            // top-E scores: entry e of row r at e * 128 + r
  int32_t tok[kXMaxE * kXRows];
  uint64_t k_full[kXStages], k_free[kXStages], d_full[2], d_free[2], a_ready, drain;
  uint32_t tmem_base;
  int abort;
};

struct XArgs {
  DevLayout L;
  const uint8_t* ktm;                    // tile-major K: ((b * H + h) * n_tiles + tile) * 16 KB
  const float* qbar;                     // [B, H, n_tiles, 128]
  const int32_t* idx;
  const int32_t* cnt;
  int32_t kmax, H, c0, cand0, n_cand, E;
  int32_t* out_idx;                      // [B, H, n_tiles, E]
  int32_t* out_cnt;                      // [B, H, n_tiles]
  int* err;
};

__device__ __forceinline__ void x_abort(XSmem& sm, int* err) {
  atomicExch(err, VSA_ERR_TIMEOUT);
  *reinterpret_cast<volatile int*>(&sm.abort) = 1;
}

__device__ __forceinline__ bool x_warp_wait(XSmem& sm, uint64_t& bar, uint32_t parity, int lane, int* err) {
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

// The weakest entry of a row's full top-E: lowest score, and among equal
// lowest scores the highest token index.
__device__ __noinline__ void x_find_worst(const XSmem& sm, int r, int E, int& worst, float& wv, int& wt) {
  worst = 0;
  wv = sm.val[r];
  wt = sm.tok[r];
  for (int e = 1; e < E; ++e) {
    const float v = sm.val[e * kXRows + r];
    const int t = sm.tok[e * kXRows + r];
    if (v < wv || (v == wv && t > wt)) {
      worst = e;
      wv = v;
      wt = t;
    }
  }
}

// Offers (score, slot of key tile) to row r's top-E (called for scores that
// may enter: the list is not full, or the score is at least the weakest).
__device__ __noinline__ void x_offer(XSmem& sm, const int32_t* perm_tile, int r, int E, float s, int slot,
                                     int& count, int& worst, float& wv, int& wt) {
  const int t = perm_tile[slot];
  if (count < E) {
    sm.val[count * kXRows + r] = s;
    sm.tok[count * kXRows + r] = t;
    if (++count == E) x_find_worst(sm, r, E, worst, wv, wt);
    return;
  }
  if (s > wv || (s == wv && t < wt)) {
    sm.val[worst * kXRows + r] = s;
    sm.tok[worst * kXRows + r] = t;
    x_find_worst(sm, r, E, worst, wv, wt);
  }
}

__global__ void __launch_bounds__(kXThreads, 1) extra_select_kernel(const __grid_constant__ XArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if (smem_u32(smem_raw) & 1023u) {          // swizzled tiles need 1024-byte alignment
    if (threadIdx.x == 0) atomicExch(a.err, VSA_ERR_UNSUPPORTED);
    return;
  }
  XSmem& sm = *reinterpret_cast<XSmem*>(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const size_t bh = static_cast<size_t>(blockIdx.z) * a.H + blockIdx.y;
  const int qt0 = a.c0 + blockIdx.x * kXRows;
  const int n_tiles = a.L.n_tiles;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kXStages; ++s) {
      mbar_init(smem_u32(&sm.k_full[s]), 1);
      mbar_init(smem_u32(&sm.k_free[s]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&sm.d_full[i]), 1);
      mbar_init(smem_u32(&sm.d_free[i]), 4);    // one arrival per row warp
    }
    mbar_init(smem_u32(&sm.a_ready), 4);
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
    // ---------------------------------------------------- key tile copies
    uint32_t issued = 0;
    bool ok = true;
    for (int t = 0; t < a.n_cand; ++t) {
      const int st = t % kXStages;
      if (t >= kXStages && !(ok = x_warp_wait(sm, sm.k_free[st], ((t / kXStages) - 1) & 1, lane, a.err))) break;
      if (lane == 0) {
        const uint32_t bar = smem_u32(&sm.k_full[st]);
        mbar_arrive_expect_tx(bar, 16384);
        bulk_load(smem_u32(sm.k[st]), a.ktm + (bh * n_tiles + a.cand0 + t) * 16384u, 16384, bar);
      }
      __syncwarp();
      ++issued;
    }
    if (!ok && lane == 0) {
      for (uint32_t i = (issued > kXStages ? issued - kXStages : 0u); i < issued; ++i)
        mbar_wait(smem_u32(&sm.k_full[i % kXStages]), (i / kXStages) & 1, nullptr, kXDrainNs);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMAs
    // D(t) = sum over the three split terms of Qbar_term K(t)^T into score
    // buffer t & 1, once the row warps have read D(t - 2) out of it.
    if (lane == 0) {
      bool ok = mbar_wait(smem_u32(&sm.a_ready), 0, &sm.abort, kXTimeoutNs);
      for (int t = 0; ok && t < a.n_cand; ++t) {
        const int st = t % kXStages;
        if (!(ok = mbar_wait(smem_u32(&sm.k_full[st]), (t / kXStages) & 1, &sm.abort, kXTimeoutNs))) break;
        if (t >= 2 && !(ok = mbar_wait(smem_u32(&sm.d_free[t & 1]), ((t >> 1) - 1) & 1, &sm.abort, kXTimeoutNs)))
          break;
        tc_fence_after();
        const uint64_t kd = smem_desc_sw128(smem_u32(sm.k[st]), 16, 1024);
        const uint32_t d = tmem + kXColD + 64u * (t & 1);
#pragma unroll
        for (int term = 0; term < 3; ++term)
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            umma_ts(d, tmem + kXColA + 64u * term + kk * 8, kd + (kk >> 2) * (8192 >> 4) + (kk & 3) * 2, kXIdesc,
                    (term | kk) ? 1u : 0u);
        umma_commit(smem_u32(&sm.d_full[t & 1]));
        umma_commit(smem_u32(&sm.k_free[st]));
      }
      if (!ok) x_abort(sm, a.err);
      umma_commit(smem_u32(&sm.drain));
      mbar_wait(smem_u32(&sm.drain), 0, nullptr, kXDrainNs);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------ one query tile per thread
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const int qt = qt0 + r;
    const bool row_ok = qt < n_tiles;
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    const size_t row = bh * n_tiles + (row_ok ? qt : 0);
    // Qbar of this query tile, split into three bf16 terms, as the A operand
    {
      const float* src = a.qbar + row * kHeadDim;
#pragma unroll 1
      for (int c = 0; c < 2; ++c) {            // 64 dims = 32 bf16 pairs = 32 columns per chunk
        uint32_t w0[32], w1[32], w2[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          uint32_t hi[2], mid[2], lo[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const float x = row_ok ? src[64 * c + 2 * i + e] : 0.f;
            const float hv = bf16_round(x);
            const float mv = bf16_round(x - hv);
            const float lv = bf16_round(x - hv - mv);
            hi[e] = bf16_bits(hv);
            mid[e] = bf16_bits(mv);
            lo[e] = bf16_bits(lv);
          }
          w0[i] = hi[0] | (hi[1] << 16);
          w1[i] = mid[0] | (mid[1] << 16);
          w2[i] = lo[0] | (lo[1] << 16);
        }
        tmem_st32x32(lane_addr + kXColA + 0 * 64 + 32 * c, w0);
        tmem_st32x32(lane_addr + kXColA + 1 * 64 + 32 * c, w1);
        tmem_st32x32(lane_addr + kXColA + 2 * 64 + 32 * c, w2);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&sm.a_ready));
    }
    // walk the candidate key tiles; skip the ones this query tile selected
    const int n_sel = row_ok ? min(max(a.cnt[row], 0), a.kmax) : 0;
    const int32_t* list = a.idx + row * a.kmax;
    int p = 0;
    int nxt = n_sel > 0 ? list[0] : INT_MAX;
    int count = 0, worst = 0, wt = 0;
    float wv = -INFINITY;
    bool ok = true;
    for (int t = 0; t < a.n_cand; ++t) {
      if (!(ok = x_warp_wait(sm, sm.d_full[t & 1], (t >> 1) & 1, lane, a.err))) break;
      tc_fence_after();
      float x0[32], x1[32];
      tmem_ld32x32f(lane_addr + kXColD + 64u * (t & 1), x0);
      tmem_ld32x32f(lane_addr + kXColD + 64u * (t & 1) + 32, x1);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&sm.d_free[t & 1]));
      while (nxt < t) nxt = ++p < n_sel ? list[p] : INT_MAX;   // lists are ascending (anything else is skipped over)
      if (nxt == t) {
        nxt = ++p < n_sel ? list[p] : INT_MAX;
        continue;
      }
      if (!row_ok) continue;
      const int tile = a.cand0 + t;
      const unsigned long long vm = a.L.valid[tile];
      const int32_t* perm_tile = a.L.perm + tile * kTile;
      // slots that may enter the top-E: a branch-free mask first (after the
      // first tiles almost none qualify, and a branch per slot costs far more
      // than the compare), then one offer per set bit in slot order
      const float lim = count < a.E ? -INFINITY : wv;
      uint32_t m0 = 0, m1 = 0;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        m0 |= (x0[i] >= lim ? 1u : 0u) << i;
        m1 |= (x1[i] >= lim ? 1u : 0u) << i;
      }
      unsigned long long cand = (static_cast<unsigned long long>(m1) << 32 | m0) & vm;
      while (cand) {
        const int i = __ffsll(static_cast<long long>(cand)) - 1;
        cand &= cand - 1;
        // the scores stay in registers: pick slot i's without dynamic indexing
        float xi = 0.f;
#pragma unroll
        for (int u = 0; u < 32; ++u) {
          xi = (i == u) ? x0[u] : xi;
          xi = (i == 32 + u) ? x1[u] : xi;
        }
        if (count < a.E || xi >= wv) x_offer(sm, perm_tile, r, a.E, xi, i, count, worst, wv, wt);
      }
    }
    if (ok && row_ok) {
      int32_t* dst = a.out_idx + row * a.E;
      for (int e = 0; e < count; ++e) dst[e] = sm.tok[e * kXRows + r];
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
    const size_t smem = sizeof(XSmem);
    e = cudaFuncSetAttribute(extra_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return cuda_fail("vsa_extra_tokens_select: cudaFuncSetAttribute", e);
    extra_select_kernel<<<dim3((rows + kXRows - 1) / kXRows, H, B), kXThreads, smem, stream>>>(a);
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
