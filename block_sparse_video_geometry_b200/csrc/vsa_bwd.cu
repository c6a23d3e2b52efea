// Backward pass of the VSA block-sparse attention: gradients of <out, dO> with
// respect to q, k, v and the gate, the block selection held fixed (it is a
// piecewise-constant function of the inputs). The pages train and distil
// checkpoints against these modes ("BSAI FastH3 Native VSA (recipe)" and
// "ComfyUI-Ref2VA-VSA", "The Solution: Ref2VAVSAGatePatch"); they do not spell
// the backward out, so this is the exact derivative of the forward as the
// forward kernels compute it (mean-pooled coarse branch).
//
// out_i = o_fine_i + cr_i g_i o_coarse[tile(i)]   (cr_i = 0 on dense conditioning rows)
//  * gate:   dg_i = cr_i <dO_i, o_coarse[tile(i)]> (per channel: the products).
//  * fine:   exact attention over each query tile's key set: with the row
//            log2-sum-exp2 and D_i = <dO_i, o_fine_i> from a forward pass in
//            statistics mode, P = 2^(c s - lse), dS = P (dO V^T - D),
//            dq = scale dS K, dk = scale dS^T q, dv = P^T dO.
//  * coarse: o_coarse[t] = softmax_c(scale <Qbar_t, Kbar_c>) Vbar over the
//            candidate tiles; dOc[t] = sum over the tile's rows of cr g dO;
//            the tile-level softmax backward gives dQbar, dKbar, dVbar, which
//            flow back through the pooling (1 / tile count to every valid token).
//
// B200 design:
//  * dq_kernel: one CTA per (batch, head, query tile) walking its selection
//    list; per key tile S = Q K^T and dP = dO V^T are M = 64 tcgen05 MMAs
//    with Q and dO in TMEM and K, V bulk-copied tiles (the forward's
//    tile-major copies), the fp32 elementwise step writes dS as bf16 over S
//    in TMEM, and dQ += dS K accumulates in TMEM (K as the MN-major B
//    operand). dq_pair_kernel runs the key tiles every query tile shares (the
//    conditioning tiles; all tiles for dense conditioning rows) for two query
//    tiles at a time as M = 128 products and writes dQ first; dq_kernel adds.
//  * dkv_kernel: one CTA per (batch, head, candidate key tile) walking the
//    query tiles that attend it (dense conditioning rows plus the transpose of
//    the selection lists, built on the GPU by a counting sort); S^T = K Q^T
//    and dP^T = V dO^T with K, V, Q and dO as bulk-copied shared-memory tiles,
//    then dV += P^T dO and dK += dS^T Q with P^T, dS^T (bf16) in TMEM.
//  * dkv_pair_kernel: the conditioning key tiles (sink on), which every query
//    tile attends, two per CTA as M = 128 products over the same query steps.
//  * All four are warp-specialised pipelines: a copy warp keeps four 32 KB
//    stages in flight; the MMAs are spread over several issuing warps (each
//    tcgen05.mma holds its thread for tens of cycles, so one thread issuing a
//    step's 20-24 MMAs was the bound; dq: S, dP and dQ on three warps, dkv:
//    S^T with dV and dP^T with dK on two); the products of step j + 1 and the
//    accumulations of step j run while eight warps do the elementwise step of
//    the other of two TMEM score buffers (two per TMEM lane quadrant, each
//    half of a row's columns). A product rewrites its buffer only after the
//    accumulation that read it two steps earlier has completed (dq: acc_a) or
//    was issued before it by the same thread (dkv).
//  * The coarse branch runs on CUDA cores in fp32 (like its forward):
//    dOc and dg in one pass over the tokens, a row pass per 64 query tiles
//    (softmax statistics, P, dS, dQbar), a column pass per 64 candidate tiles
//    (dKbar, dVbar), and a scatter through the pooling.

#include <cuda_runtime.h>

#include <algorithm>
#include <climits>
#include <cmath>

#include "sm100.cuh"
#include "vsa_internal.h"

namespace vsa {
namespace {

using namespace sm100;

constexpr int kBThreads = 416;           // warp 0 copies, warps 1 and 10-12 MMAs, warps 2-9 the elementwise step
constexpr int kBStages = 4;              // copy stages of 32 KB
constexpr uint32_t kBTmemCols = 512;
constexpr uint32_t kTB = 16384;          // one tile of Q, K, V or dO: [d half][64 rows][128 B]
constexpr uint64_t kBTimeoutNs = 4000000000ull;
constexpr uint64_t kBDrainNs = 200000000ull;
constexpr size_t kBHeader = 256;         // status word

// TMEM columns (lanes 0-15 of every quadrant: M = 64); S and dP are double
// buffered so that step j + 1's products run during step j's elementwise work
//  dq_kernel : Q 0-63, dO 64-127, S / dS [b] 128 + 128 b, dP [b] 192 + 128 b, dQ 384-511
//  dkv_kernel: S^T / P^T [b] 128 b, dP^T / dS^T [b] 64 + 128 b, dK 256-383, dV 384-511
//              (K and V stay in shared memory as A operands)
constexpr uint32_t kQColQ = 0, kQColDO = 64, kQColS = 128, kQColP = 192, kQColAcc = 384;
constexpr uint32_t kKColS = 0, kKColP = 64, kKColDK = 256, kKColDV = 384;

// Shared memory: this header, then (1024-byte aligned) the tiles.
//  dq_kernel : stage s (K then V of a key tile) at 1024 + 32 KB s
//  dkv_kernel: the key tile's K and V at 1024, stage s (Q then dO of a query
//              tile) at 1024 + 32 KB (s + 1), then the stages' row statistics
struct BHead {
  uint64_t full[kBStages], free_[kBStages], s_full[2], p_full[2], ds_ready[2], acc_a[2], a_ready, acc_done;
  uint64_t qpair[4];                     // dkv_pair_kernel: the two warps of a lane quadrant, once per step
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(BHead) <= 1024, "tiles start at byte 1024");
constexpr size_t kDqSmem = 1024 + kBStages * 2 * kTB;
constexpr size_t kDkvSmem = 1024 + 2 * kTB + kBStages * 2 * kTB + kBStages * 2 * 64 * sizeof(float);

struct BArgs {
  DevLayout L;
  int32_t H, sink, n_cond, cand0, n_cand, kmax, c0;     // c0 = dense conditioning rows (0 unless rows mode)
  const uint16_t* q;                     // natural layout [B, S, H, 128]
  const uint16_t* dout;
  int64_t sb, ss, sh;                    // strides of q, k, v
  int64_t d_sb, d_ss, d_sh;              // strides of dO
  const uint8_t* kv;                     // tile-major K, V: ((b * H + h) * n_tiles + t) * 32 KB
  const uint8_t* qtm;                    // tile-major Q, dO: ((b * H + h) * n_tiles + t) * 16 KB
  const uint8_t* dotm;
  const float* lse;                      // [B, H, n_tiles, 64]
  const float* dd;                       // [B, H, n_tiles, 64]
  const int32_t* idx;
  const int32_t* cnt;
  const int32_t* csr_off;                // [B, H, n_cand + 1]
  const int32_t* csr_list;               // query tiles per candidate
  float* dq;                             // fp32 [B, S, H, 128] at element strides o_sb, o_ss, o_sh
  float* dk;
  float* dv;
  int64_t o_sb, o_ss, o_sh;
  float scale, c_log2;
  int32_t dq_add;                        // dq_kernel adds to the dQ dq_pair_kernel wrote
  int* err;
};

// 16 lanes x 8 consecutive 32-bit columns per half-warp (16x32bx2 shape: the
// upper half-warp at column offset `split`)
template <int split>
__device__ __forceinline__ void tmem_st16x2_8(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile(
      "tcgen05.st.sync.aligned.16x32bx2.x8.b32 [%0], %1, {%2, %3, %4, %5, %6, %7, %8, %9};" ::"r"(taddr), "n"(split),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
      : "memory");
}

__device__ __forceinline__ void b_abort(BHead& sm, int* err) {
  atomicExch(err, VSA_ERR_TIMEOUT);
  *reinterpret_cast<volatile int*>(&sm.abort) = 1;
}

// the calling threads wait (bounded) on a barrier phase; a phase that has
// already completed is taken with a non-suspending test first (a try_wait on
// it still costs a few hundred cycles)
__device__ __forceinline__ bool b_wait(BHead& sm, uint64_t& bar, uint32_t parity, int* err) {
  if (mbar_test_wait(smem_u32(&bar), parity)) return true;
  const bool ok = mbar_wait(smem_u32(&bar), parity, &sm.abort, kBTimeoutNs);
  if (!ok) b_abort(sm, err);
  return ok;
}

// a_ready_count: arrivals that complete a_ready (dq: the eight elementwise
// warps after writing Q and dO into TMEM; dkv: the copy of K and V);
// free_count: MMA warps whose accumulation reads a stage
__device__ __forceinline__ void b_init(BHead& sm, uint32_t a_ready_count, uint32_t free_count) {
  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kBStages; ++s) {
      mbar_init(smem_u32(&sm.full[s]), 1);
      mbar_init(smem_u32(&sm.free_[s]), free_count);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&sm.s_full[i]), 1);
      mbar_init(smem_u32(&sm.p_full[i]), 1);
      mbar_init(smem_u32(&sm.acc_a[i]), 1);      // dq: dQ of the step that used buffer i completed
      mbar_init(smem_u32(&sm.ds_ready[i]), 8);   // one arrival per elementwise warp
    }
    mbar_init(smem_u32(&sm.a_ready), a_ready_count);
    for (int i = 0; i < 4; ++i) mbar_init(smem_u32(&sm.qpair[i]), 2);
    mbar_init(smem_u32(&sm.acc_done), 4);       // the four MMA warps, after their last MMA
    sm.abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&sm.tmem_base), kBTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
}

// Copy-warp loop (lane 0): step j's tiles into stage j % kBStages once the
// MMAs of step j - kBStages released it; on a failed wait, lets the copies in
// flight land before returning.
template <class Issue>
__device__ __forceinline__ void b_copy_loop(BHead& sm, int n, int* err, Issue issue) {
  int issued = 0;
  bool ok = true;
  for (int j = 0; j < n; ++j) {
    const int st = j % kBStages;
    if (j >= kBStages && !(ok = b_wait(sm, sm.free_[st], ((j / kBStages) - 1) & 1, err))) break;
    issue(j, st, smem_u32(&sm.full[st]));
    ++issued;
  }
  if (!ok)
    for (int i = max(0, issued - kBStages); i < issued; ++i)
      mbar_wait(smem_u32(&sm.full[i % kBStages]), (i / kBStages) & 1, nullptr, kBDrainNs);
}

// 64-row tile of a natural-layout [B, S, H, 128] tensor into TMEM as an M = 64
// A operand (bf16 pairs, 64 columns): thread (row r, half hf) its 64 dims.
__device__ __forceinline__ void rows_to_tmem(const uint16_t* base, const int32_t* perm_tile, int64_t ss, int r, int hf,
                                             uint32_t taddr) {
  const int t = perm_tile[r];
  const uint4* src = reinterpret_cast<const uint4*>(base + static_cast<int64_t>(t) * ss + 64 * hf);
  uint32_t w[32];
#pragma unroll
  for (int cc = 0; cc < 8; ++cc) {
    const uint4 u = t >= 0 ? __ldg(src + cc) : make_uint4(0u, 0u, 0u, 0u);
    w[4 * cc] = u.x;
    w[4 * cc + 1] = u.y;
    w[4 * cc + 2] = u.z;
    w[4 * cc + 3] = u.w;
  }
  tmem_st16x2_32<32>(taddr, w);
}

// Key tile of step jj of query tile row's selection list.
__device__ __forceinline__ int dq_step_tile(const BArgs& a, size_t row, int jj) {
  const int c = a.idx[row * a.kmax + jj];
  return a.cand0 + min(max(c, 0), a.n_cand - 1);
}

// Query tile of step jj of candidate key tile kt's attending set: the dense
// conditioning rows, then the query tiles whose lists hold the tile.
__device__ __forceinline__ int dkv_step_tile(const BArgs& a, const int32_t* list, int jj) {
  return jj < a.c0 ? jj : list[jj - a.c0];
}

// -------------------------------------------------------------------- dQ
// Per step j (key tile t_j): S = Q K^T and dP = dO V^T into buffer j & 1;
// the elementwise warps turn them into dS = P (dP - D) (bf16, over S); then
// dQ += dS K. The MMA warp issues S(j), dP(j) before dQ(j - 1), so the tensor
// pipe has the next products queued while the elementwise step runs.
__global__ void __launch_bounds__(kBThreads, 1) dq_kernel(const __grid_constant__ BArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if (smem_u32(smem_raw) & 1023u) {
    if (threadIdx.x == 0) atomicExch(a.err, VSA_ERR_UNSUPPORTED);
    return;
  }
  BHead& sm = *reinterpret_cast<BHead*>(smem_raw);
  uint8_t* const stage0 = smem_raw + 1024;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qt = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  if (qt < a.c0) return;                           // dense conditioning rows: dq_pair_kernel
  const size_t bh = static_cast<size_t>(b) * a.H + h;
  const size_t row = bh * a.L.n_tiles + qt;
  const int n = min(max(a.cnt[row], 1), a.kmax);   // the selection list (the shared key tiles: dq_pair_kernel)
  b_init(sm, 8, 1);
  const uint32_t tmem = sm.tmem_base;

  if (warp == 0) {
    if (lane == 0) {
      const uint8_t* head_kv = a.kv + bh * a.L.n_tiles * 32768u;
      b_copy_loop(sm, n, a.err, [&](int j, int st, uint32_t bar) {
        const int t = dq_step_tile(a, row, j);
        const uint32_t dst = smem_u32(stage0 + st * 2 * kTB);
        mbar_arrive_expect_tx(bar, 2 * kTB);
        bulk_load(dst, head_kv + static_cast<size_t>(t) * 32768u, kTB, bar);
        bulk_load(dst + kTB, head_kv + static_cast<size_t>(t) * 32768u + kTB, kTB, bar);
      });
    }
    __syncwarp();
  } else if (warp == 1 || warp >= 10) {
    // one issuing thread per MMA chain: warp 1 S = Q K^T, warp 10 dP = dO V^T
    // (V K-major like K: [keys][d]), warp 11 dQ += dS K (K as the MN-major B
    // operand); warp 12 has nothing to issue here. S(j) overwrites dS(j - 2):
    // it waits for dQ(j - 2) to complete (acc_a); dP(j) overwrites dP(j - 2):
    // it waits for the elementwise step to release it (ds_ready).
    if (lane == 0) {
      constexpr uint32_t kIdS = idesc_bf16_f32(64, 64, 0, 0), kIdQ = idesc_bf16_f32(64, 128, 0, 1);
      bool ok = b_wait(sm, sm.a_ready, 0, a.err);
      if (warp == 1 || warp == 10) {
        const bool is_s = warp == 1;
        for (int j = 0; ok && j < n; ++j) {
          const int st = j % kBStages;
          const uint32_t bs = 128u * (j & 1);
          if (!(ok = b_wait(sm, sm.full[st], (j / kBStages) & 1, a.err))) break;
          if (j >= 2 && !(ok = b_wait(sm, is_s ? sm.acc_a[j & 1] : sm.ds_ready[j & 1], ((j >> 1) - 1) & 1, a.err)))
            break;
          tc_fence_after();
          const uint64_t bd = smem_desc_sw128(smem_u32(stage0 + st * 2 * kTB + (is_s ? 0u : kTB)), 16, 1024);
          const uint32_t dcol = (is_s ? kQColS : kQColP) + bs, acol = is_s ? kQColQ : kQColDO;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            umma_ts(tmem + dcol, tmem + acol + kk * 8, bd + (kk >> 2) * (8192 >> 4) + (kk & 3) * 2, kIdS, kk > 0);
          umma_commit(smem_u32(is_s ? &sm.s_full[j & 1] : &sm.p_full[j & 1]));
        }
      } else if (warp == 11) {
        for (int j = 0; ok && j < n; ++j) {
          const int st = j % kBStages;
          if (!(ok = b_wait(sm, sm.ds_ready[j & 1], (j >> 1) & 1, a.err))) break;
          tc_fence_after();
          const uint64_t kmn = smem_desc_sw128(smem_u32(stage0 + st * 2 * kTB), 8192, 1024);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_ts(tmem + kQColAcc, tmem + kQColS + 128u * (j & 1) + kk * 8, kmn + kk * (2048 >> 4), kIdQ,
                    (j > 0 || kk > 0) ? 1u : 0u);
          umma_commit(smem_u32(&sm.acc_a[j & 1]));
          umma_commit(smem_u32(&sm.free_[st]));   // S(j), dP(j) completed before the elementwise step released it
        }
      }
      umma_commit(smem_u32(&sm.acc_done));     // every MMA issued, also on a failed wait
      mbar_wait(smem_u32(&sm.acc_done), 0, nullptr, kBDrainNs);
    }
    __syncwarp();
  } else {
    // thread (row r, half hf) of column set cs: keys 32 hf + 16 cs .. + 15
    const int qd = warp & 3, hf = lane >> 4, cs = (warp - 2) >> 2;
    const int r = qd * 16 + (lane & 15);
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(qd * 32) << 16);   // lanes 32 qd .. 32 qd + 15
    const int32_t* perm_q = a.L.perm + qt * kTile;
    if (cs == 0) rows_to_tmem(a.q + b * a.sb + h * a.sh, perm_q, a.ss, r, hf, lane_addr + kQColQ);
    else rows_to_tmem(a.dout + b * a.d_sb + h * a.d_sh, perm_q, a.d_ss, r, hf, lane_addr + kQColDO);
    tmem_wait_st();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_u32(&sm.a_ready));
    const float lse = a.lse[row * kTile + r];
    const float dd = a.dd[row * kTile + r];
    unsigned long long vm_next = a.L.valid[dq_step_tile(a, row, 0)];
    bool ok = true;
    for (int j = 0; j < n; ++j) {
      const unsigned long long vm = vm_next;
      if (j + 1 < n) vm_next = a.L.valid[dq_step_tile(a, row, j + 1)];
      const uint32_t bs = 128u * (j & 1);
      if (!(ok = b_wait(sm, sm.s_full[j & 1], (j >> 1) & 1, a.err))) break;
      if (!(ok = b_wait(sm, sm.p_full[j & 1], (j >> 1) & 1, a.err))) break;
      tc_fence_after();
      float s[16], dp[16];
      tmem_ld16x2_16f<32>(lane_addr + kQColS + bs + 16 * cs, s);
      tmem_ld16x2_16f<32>(lane_addr + kQColP + bs + 16 * cs, dp);
      tmem_wait_ld();
      const uint32_t vbits = static_cast<uint32_t>(vm >> (32 * hf + 16 * cs));
      uint32_t w[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        float ds[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int key = 2 * i + e;
          const float p = ((vbits >> key) & 1u) ? ex2_approx(fmaf(s[key], a.c_log2, -lse)) : 0.f;
          ds[e] = p * (dp[key] - dd);
        }
        w[i] = pack_bf16x2(ds[0], ds[1]);
      }
      tmem_st16x2_8<16>(lane_addr + kQColS + bs + 8 * cs, w);    // dS (bf16 pairs) over S
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&sm.ds_ready[j & 1]));
    }
    if (ok && (ok = b_wait(sm, sm.acc_done, 0, a.err))) {
      tc_fence_after();
      const int tok = perm_q[r];
      const int ch = cs;                               // dims 64 hf + 32 cs .. + 31
      float y[32];
      tmem_ld16x2_32f<64>(lane_addr + kQColAcc + 32 * ch, y);
      tmem_wait_ld();
      if (tok >= 0) {
        float4* dst = reinterpret_cast<float4*>(a.dq + b * a.o_sb + static_cast<int64_t>(tok) * a.o_ss +
                                                h * a.o_sh + 64 * hf + 32 * ch);
#pragma unroll
        for (int i = 0; i < 32; i += 4) {
          float4 v = make_float4(y[i] * a.scale, y[i + 1] * a.scale, y[i + 2] * a.scale, y[i + 3] * a.scale);
          if (a.dq_add) {
            const float4 u = dst[i / 4];
            v.x += u.x;
            v.y += u.y;
            v.z += u.z;
            v.w += u.w;
          }
          dst[i / 4] = v;
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kBTmemCols);
  }
}

// -------------------------------------------------------------- dK and dV
// Per step j (query tile q_j): S^T = K Q^T and dP^T = V dO^T into buffer
// j & 1 (K and V of this CTA's key tile in shared memory as A operands); the
// elementwise warps write P^T and dS^T = P^T (dP^T - D) (bf16, in place); then
// dV += P^T dO and dK += dS^T Q, issued after the next step's products.
__global__ void __launch_bounds__(kBThreads, 1) dkv_kernel(const __grid_constant__ BArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if (smem_u32(smem_raw) & 1023u) {
    if (threadIdx.x == 0) atomicExch(a.err, VSA_ERR_UNSUPPORTED);
    return;
  }
  BHead& sm = *reinterpret_cast<BHead*>(smem_raw);
  uint8_t* const kvt = smem_raw + 1024;
  uint8_t* const stage0 = kvt + 2 * kTB;
  float* const rowstat = reinterpret_cast<float*>(stage0 + kBStages * 2 * kTB);   // [stage][lse, D][64]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kt = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  if (a.sink != VSA_SINK_OFF && kt < a.n_cond) return;   // dkv_pair_kernel's key tiles
  const size_t bh = static_cast<size_t>(b) * a.H + h;
  const int n_tiles = a.L.n_tiles;
  const int c = kt - a.cand0;                       // candidate ordinal
  const int32_t* off = a.csr_off + bh * (a.n_cand + 1);
  const int32_t* list = a.csr_list + off[c];
  const int n = a.c0 + (off[c + 1] - off[c]);
  b_init(sm, 1, 2);
  const uint32_t tmem = sm.tmem_base;

  if (warp == 0) {
    if (lane == 0) {
      // K and V of the key tile once (a_ready), then Q, dO and the row
      // statistics of every attending query tile
      mbar_arrive_expect_tx(smem_u32(&sm.a_ready), 2 * kTB);
      bulk_load(smem_u32(kvt), a.kv + (bh * n_tiles + kt) * 32768u, 2 * kTB, smem_u32(&sm.a_ready));
      b_copy_loop(sm, n, a.err, [&](int j, int st, uint32_t bar) {
        const size_t tq = bh * n_tiles + dkv_step_tile(a, list, j);
        const uint32_t dst = smem_u32(stage0 + st * 2 * kTB);
        mbar_arrive_expect_tx(bar, 2 * kTB + 2 * 256);
        bulk_load(dst, a.qtm + tq * kTB, kTB, bar);
        bulk_load(dst + kTB, a.dotm + tq * kTB, kTB, bar);
        bulk_load(smem_u32(rowstat + st * 128), a.lse + tq * kTile, 256, bar);
        bulk_load(smem_u32(rowstat + st * 128 + 64), a.dd + tq * kTile, 256, bar);
      });
    }
    __syncwarp();
  } else if (warp == 1 || warp >= 10) {
    // two MMA issuers: warp 1 S^T = K Q^T and dV += P^T dO, warp 10
    // dP^T = V dO^T and dK += dS^T Q (K, V, Q and dO K-major in shared memory
    // for the products; dO and Q as MN-major B operands, [queries][d], for
    // the accumulations); each rewrites its half of buffer j & 1 only after
    // its own accumulation of step j - 2 (one thread's MMAs run in issue
    // order), and both release a stage. (Separate warps for the
    // accumulations made the products wait for their completion: slower.)
    // Warps 11 and 12 have nothing to issue here.
    if (lane == 0 && (warp == 1 || warp == 10)) {
      constexpr uint32_t kIdS = idesc_bf16_f32(64, 64, 0, 0), kIdA = idesc_bf16_f32(64, 128, 0, 1);
      const bool is_s = warp == 1;
      const uint64_t ad = smem_desc_sw128(smem_u32(kvt + (is_s ? 0u : kTB)), 16, 1024);
      bool ok = b_wait(sm, sm.a_ready, 0, a.err);
      for (int j = 0; ok && j <= n; ++j) {
        if (j < n) {
          const int st = j % kBStages;
          const uint32_t bs = 128u * (j & 1);
          if (!(ok = b_wait(sm, sm.full[st], (j / kBStages) & 1, a.err))) break;
          tc_fence_after();
          const uint64_t bd = smem_desc_sw128(smem_u32(stage0 + st * 2 * kTB + (is_s ? 0u : kTB)), 16, 1024);
          const uint32_t dcol = (is_s ? kKColS : kKColP) + bs;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint64_t off = (kk >> 2) * (8192 >> 4) + (kk & 3) * 2;
            umma_ss(tmem + dcol, ad + off, bd + off, kIdS, kk > 0);
          }
          umma_commit(smem_u32(is_s ? &sm.s_full[j & 1] : &sm.p_full[j & 1]));
        }
        if (j >= 1) {
          const int jp = j - 1, stp = jp % kBStages;
          const uint32_t bp = 128u * (jp & 1);
          if (!(ok = b_wait(sm, sm.ds_ready[jp & 1], (jp >> 1) & 1, a.err))) break;
          tc_fence_after();
          // warp 1: dV += P^T dO; warp 10: dK += dS^T Q
          const uint64_t bmn = smem_desc_sw128(smem_u32(stage0 + stp * 2 * kTB + (is_s ? kTB : 0u)), 8192, 1024);
          const uint32_t acc = is_s ? kKColDV : kKColDK, acol = (is_s ? kKColS : kKColP) + bp;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_ts(tmem + acc, tmem + acol + kk * 8, bmn + kk * (2048 >> 4), kIdA, (jp > 0 || kk > 0) ? 1u : 0u);
          umma_commit(smem_u32(&sm.free_[stp]));
        }
      }
      umma_commit(smem_u32(&sm.acc_done));     // every MMA issued, also on a failed wait
      mbar_wait(smem_u32(&sm.acc_done), 0, nullptr, kBDrainNs);
    } else if (lane == 0) {
      umma_commit(smem_u32(&sm.acc_done));     // no MMAs: arrives at once
      mbar_wait(smem_u32(&sm.acc_done), 0, nullptr, kBDrainNs);
    }
    __syncwarp();
  } else {
    // thread (key slot r, half hf) of column set cs: queries 32 hf + 16 cs .. + 15
    const int qd = warp & 3, hf = lane >> 4, cs = (warp - 2) >> 2;
    const int r = qd * 16 + (lane & 15);
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(qd * 32) << 16);
    bool ok = true;
    for (int j = 0; j < n; ++j) {
      const int st = j % kBStages;
      const uint32_t bs = 128u * (j & 1);
      if (!(ok = b_wait(sm, sm.s_full[j & 1], (j >> 1) & 1, a.err))) break;
      if (!(ok = b_wait(sm, sm.p_full[j & 1], (j >> 1) & 1, a.err))) break;
      tc_fence_after();
      float s[16], dp[16];
      tmem_ld16x2_16f<32>(lane_addr + kKColS + bs + 16 * cs, s);
      tmem_ld16x2_16f<32>(lane_addr + kKColP + bs + 16 * cs, dp);
      tmem_wait_ld();
      uint32_t wp[8], wd[8];
      const float* lse = rowstat + st * 128 + 32 * hf + 16 * cs;     // the queries of this thread's columns
      const float* dd = rowstat + st * 128 + 64 + 32 * hf + 16 * cs;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        float p[2], ds[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int qi = 2 * i + e;
          p[e] = ex2_approx(fmaf(s[qi], a.c_log2, -lse[qi]));    // padding query rows: lse = +inf, P = 0
          ds[e] = p[e] * (dp[qi] - dd[qi]);
        }
        wp[i] = pack_bf16x2(p[0], p[1]);
        wd[i] = pack_bf16x2(ds[0], ds[1]);
      }
      tmem_st16x2_8<16>(lane_addr + kKColS + bs + 8 * cs, wp);     // P^T over S^T
      tmem_st16x2_8<16>(lane_addr + kKColP + bs + 8 * cs, wd);     // dS^T over dP^T
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&sm.ds_ready[j & 1]));
    }
    if (ok && (ok = b_wait(sm, sm.acc_done, 0, a.err))) {
      tc_fence_after();
      const int tok = a.L.perm[kt * kTile + r];
      {
        const int which = cs;                            // set 0: dK (scaled), set 1: dV
        float* dst_base = which == 0 ? a.dk : a.dv;
        const float f = which == 0 ? a.scale : 1.0f;
#pragma unroll 1
        for (int ch = 0; ch < 2; ++ch) {
          float y[32];
          if (n > 0) {
            tmem_ld16x2_32f<64>(lane_addr + (which == 0 ? kKColDK : kKColDV) + 32 * ch, y);
            tmem_wait_ld();
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) y[i] = 0.f;
          }
          if (tok >= 0) {
            float4* dst = reinterpret_cast<float4*>(dst_base + b * a.o_sb + static_cast<int64_t>(tok) * a.o_ss +
                                                    h * a.o_sh + 64 * hf + 32 * ch);
#pragma unroll
            for (int i = 0; i < 32; i += 4)
              dst[i / 4] = make_float4(y[i] * f, y[i + 1] * f, y[i + 2] * f, y[i + 3] * f);
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kBTmemCols);
  }
}

// ----------------------------- dK and dV of the conditioning key tiles, in pairs
// Every query tile attends the conditioning key tiles (sink on), so two of
// them share each step as one M = 128 product: rows 0-63 are key tile kt0,
// rows 64-127 key tile kt0 + 1 (an odd last tile leaves rows 64-127 unused;
// rows never mix in these products, and nothing reads those rows back). An
// M = 128 MMA takes about as long as an M = 64 MMA of the same N, so a pair
// costs about one dkv_kernel step. Same roles and barriers as dkv_kernel;
// TMEM lane = key row (M = 128 layout). The two warps of a lane quadrant split
// a row's 64 query columns and meet at a barrier between reading S^T, dP^T
// and writing P^T, dS^T (bf16 pairs) over them, since the pairs of the second
// warp's columns land in fp32 columns the first warp reads.
constexpr size_t kDkvPairSmem = 1024 + 4 * kTB + kBStages * 2 * kTB + kBStages * 2 * 64 * sizeof(float);

// 32 lanes x 16 consecutive 32-bit columns (one lane per thread)
__device__ __forceinline__ void tmem_st32x32_16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

__global__ void __launch_bounds__(kBThreads, 1) dkv_pair_kernel(const __grid_constant__ BArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if (smem_u32(smem_raw) & 1023u) {
    if (threadIdx.x == 0) atomicExch(a.err, VSA_ERR_UNSUPPORTED);
    return;
  }
  BHead& sm = *reinterpret_cast<BHead*>(smem_raw);
  uint8_t* const kp = smem_raw + 1024;              // K of the pair: [d half][128 rows][128 B]
  uint8_t* const vp = kp + 2 * kTB;                 // V of the pair, same layout
  uint8_t* const stage0 = vp + 2 * kTB;
  float* const rowstat = reinterpret_cast<float*>(stage0 + kBStages * 2 * kTB);   // [stage][lse, D][64]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kt0 = 2 * blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int nk = min(2, a.n_cond - kt0);            // key tiles of this pair
  const size_t bh = static_cast<size_t>(b) * a.H + h;
  const int n_tiles = a.L.n_tiles;
  const int n = n_tiles;                            // every query tile attends them
  b_init(sm, 1, 2);
  const uint32_t tmem = sm.tmem_base;

  if (warp == 0) {
    if (lane == 0) {
      mbar_arrive_expect_tx(smem_u32(&sm.a_ready), 4u * 8192u * nk);
      for (int i = 0; i < nk; ++i) {
        const uint8_t* src = a.kv + (bh * n_tiles + kt0 + i) * 32768u;
        for (int dh = 0; dh < 2; ++dh) {
          bulk_load(smem_u32(kp + dh * kTB + i * 8192), src + dh * 8192, 8192, smem_u32(&sm.a_ready));
          bulk_load(smem_u32(vp + dh * kTB + i * 8192), src + kTB + dh * 8192, 8192, smem_u32(&sm.a_ready));
        }
      }
      b_copy_loop(sm, n, a.err, [&](int j, int st, uint32_t bar) {
        const size_t tq = bh * n_tiles + j;
        const uint32_t dst = smem_u32(stage0 + st * 2 * kTB);
        mbar_arrive_expect_tx(bar, 2 * kTB + 2 * 256);
        bulk_load(dst, a.qtm + tq * kTB, kTB, bar);
        bulk_load(dst + kTB, a.dotm + tq * kTB, kTB, bar);
        bulk_load(smem_u32(rowstat + st * 128), a.lse + tq * kTile, 256, bar);
        bulk_load(smem_u32(rowstat + st * 128 + 64), a.dd + tq * kTile, 256, bar);
      });
    }
    __syncwarp();
  } else if (warp == 1 || warp >= 10) {
    // as dkv_kernel: warp 1 S^T and dV, warp 10 dP^T and dK, M = 128
    if (lane == 0 && (warp == 1 || warp == 10)) {
      constexpr uint32_t kIdS = idesc_bf16_f32(128, 64, 0, 0), kIdA = idesc_bf16_f32(128, 128, 0, 1);
      const bool is_s = warp == 1;
      const uint64_t ad = smem_desc_sw128(smem_u32(is_s ? kp : vp), 16, 1024);
      bool ok = b_wait(sm, sm.a_ready, 0, a.err);
      for (int j = 0; ok && j <= n; ++j) {
        if (j < n) {
          const int st = j % kBStages;
          const uint32_t bs = 128u * (j & 1);
          if (!(ok = b_wait(sm, sm.full[st], (j / kBStages) & 1, a.err))) break;
          tc_fence_after();
          const uint64_t bd = smem_desc_sw128(smem_u32(stage0 + st * 2 * kTB + (is_s ? 0u : kTB)), 16, 1024);
          const uint32_t dcol = (is_s ? kKColS : kKColP) + bs;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            umma_ss(tmem + dcol, ad + (kk >> 2) * (16384 >> 4) + (kk & 3) * 2, bd + (kk >> 2) * (8192 >> 4) + (kk & 3) * 2,
                    kIdS, kk > 0);
          umma_commit(smem_u32(is_s ? &sm.s_full[j & 1] : &sm.p_full[j & 1]));
        }
        if (j >= 1) {
          const int jp = j - 1, stp = jp % kBStages;
          const uint32_t bp = 128u * (jp & 1);
          if (!(ok = b_wait(sm, sm.ds_ready[jp & 1], (jp >> 1) & 1, a.err))) break;
          tc_fence_after();
          const uint64_t bmn = smem_desc_sw128(smem_u32(stage0 + stp * 2 * kTB + (is_s ? kTB : 0u)), 8192, 1024);
          const uint32_t acc = is_s ? kKColDV : kKColDK, acol = (is_s ? kKColS : kKColP) + bp;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_ts(tmem + acc, tmem + acol + kk * 8, bmn + kk * (2048 >> 4), kIdA, (jp > 0 || kk > 0) ? 1u : 0u);
          umma_commit(smem_u32(&sm.free_[stp]));
        }
      }
      umma_commit(smem_u32(&sm.acc_done));     // every MMA issued, also on a failed wait
      mbar_wait(smem_u32(&sm.acc_done), 0, nullptr, kBDrainNs);
    } else if (lane == 0) {
      umma_commit(smem_u32(&sm.acc_done));     // no MMAs: arrives at once
      mbar_wait(smem_u32(&sm.acc_done), 0, nullptr, kBDrainNs);
    }
    __syncwarp();
  } else {
    // thread (key row r = 32 qd + lane) of column set cs: queries 32 cs .. 32 cs + 31
    const int qd = warp & 3, cs = (warp - 2) >> 2;
    const int r = 32 * qd + lane;
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(qd * 32) << 16);
    bool ok = true;
    for (int j = 0; j < n; ++j) {
      const int st = j % kBStages;
      const uint32_t bs = 128u * (j & 1);
      if (!(ok = b_wait(sm, sm.s_full[j & 1], (j >> 1) & 1, a.err))) break;
      if (!(ok = b_wait(sm, sm.p_full[j & 1], (j >> 1) & 1, a.err))) break;
      tc_fence_after();
      float s[32], dp[32];
      tmem_ld32x32f(lane_addr + kKColS + bs + 32 * cs, s);
      tmem_ld32x32f(lane_addr + kKColP + bs + 32 * cs, dp);
      tmem_wait_ld();
      // both column sets of this quadrant have read their scores (a bounded
      // barrier wait, so that a warp leaving on a failed wait strands no one)
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&sm.qpair[qd]));
      if (!(ok = b_wait(sm, sm.qpair[qd], j & 1, a.err))) break;
      uint32_t wp[16], wd[16];
      const float* lse = rowstat + st * 128 + 32 * cs;
      const float* dd = rowstat + st * 128 + 64 + 32 * cs;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        float p[2], ds[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int qi = 2 * i + e;
          p[e] = ex2_approx(fmaf(s[qi], a.c_log2, -lse[qi]));    // padding query rows: lse = +inf, P = 0
          ds[e] = p[e] * (dp[qi] - dd[qi]);
        }
        wp[i] = pack_bf16x2(p[0], p[1]);
        wd[i] = pack_bf16x2(ds[0], ds[1]);
      }
      tmem_st32x32_16(lane_addr + kKColS + bs + 16 * cs, wp);     // P^T over S^T
      tmem_st32x32_16(lane_addr + kKColP + bs + 16 * cs, wd);     // dS^T over dP^T
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&sm.ds_ready[j & 1]));
    }
    if (ok && (ok = b_wait(sm, sm.acc_done, 0, a.err))) {
      tc_fence_after();
      const int i = r >> 6;                        // key tile kt0 + i, slot r & 63
      const int tok = i < nk ? a.L.perm[(kt0 + i) * kTile + (r & 63)] : -1;
      float* dst_base = cs == 0 ? a.dk : a.dv;     // set 0: dK (scaled), set 1: dV
      const float f = cs == 0 ? a.scale : 1.0f;
#pragma unroll 1
      for (int ch = 0; ch < 4; ++ch) {
        float y[32];
        tmem_ld32x32f(lane_addr + (cs == 0 ? kKColDK : kKColDV) + 32 * ch, y);
        tmem_wait_ld();
        if (tok >= 0) {
          float4* dst = reinterpret_cast<float4*>(dst_base + b * a.o_sb + static_cast<int64_t>(tok) * a.o_ss +
                                                  h * a.o_sh + 32 * ch);
#pragma unroll
          for (int k4 = 0; k4 < 32; k4 += 4)
            dst[k4 / 4] = make_float4(y[k4] * f, y[k4 + 1] * f, y[k4 + 2] * f, y[k4 + 3] * f);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kBTmemCols);
  }
}

// ------------------------------- dQ of the shared key tiles, query tiles in pairs
// Every query tile attends the conditioning key tiles (sink on), and a dense
// conditioning row attends every tile, so two query tiles share each of those
// steps as one M = 128 product: rows 0-63 query tile qa, rows 64-127 query
// tile qb (missing at an odd end: its rows hold zero Q and dO and an infinite
// log-sum, so P and dS vanish there). Pairs are formed among the dense rows
// (all tiles) and among the other query tiles (the conditioning tiles); the
// kernel writes dQ of those steps and dq_kernel adds the selection-list steps
// of the non-dense tiles. Same roles and barriers as dq_kernel with TMEM lane =
// query row; the two warps of a lane quadrant split the 64 key columns and
// meet at a bounded barrier before writing dS (bf16 pairs) over the scores.
constexpr size_t kDqPairSmem = 1024 + kBStages * 2 * kTB;

// One row (64 tokens' worth of bf16 pairs: 64 columns) of a natural-layout
// [B, S, H, 128] tensor into TMEM lane `taddr` (32x32b shape: one lane per
// thread), zeros for a missing token.
__device__ __forceinline__ void row_to_tmem32(const uint16_t* base, int tok, int64_t ss, uint32_t taddr) {
  const uint4* src = reinterpret_cast<const uint4*>(base + static_cast<int64_t>(tok) * ss);
#pragma unroll 1
  for (int half = 0; half < 2; ++half) {
    uint32_t w[32];
#pragma unroll
    for (int cc = 0; cc < 8; ++cc) {
      const uint4 u = tok >= 0 ? __ldg(src + 8 * half + cc) : make_uint4(0u, 0u, 0u, 0u);
      w[4 * cc] = u.x;
      w[4 * cc + 1] = u.y;
      w[4 * cc + 2] = u.z;
      w[4 * cc + 3] = u.w;
    }
    tmem_st32x32(taddr + 32 * half, w);
  }
}

__global__ void __launch_bounds__(kBThreads, 1) dq_pair_kernel(const __grid_constant__ BArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if (smem_u32(smem_raw) & 1023u) {
    if (threadIdx.x == 0) atomicExch(a.err, VSA_ERR_UNSUPPORTED);
    return;
  }
  BHead& sm = *reinterpret_cast<BHead*>(smem_raw);
  uint8_t* const stage0 = smem_raw + 1024;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y, b = blockIdx.z;
  const int n_tiles = a.L.n_tiles;
  const int n_dense_pairs = (a.c0 + 1) / 2;
  int qa, qb, n;                                   // the pair's query tiles (qb < 0: none) and steps
  if (static_cast<int>(blockIdx.x) < n_dense_pairs) {
    qa = 2 * blockIdx.x;
    qb = qa + 1 < a.c0 ? qa + 1 : -1;
    n = n_tiles;
  } else {
    qa = a.c0 + 2 * (blockIdx.x - n_dense_pairs);
    qb = qa + 1 < n_tiles ? qa + 1 : -1;
    n = a.n_cond;
  }
  const size_t bh = static_cast<size_t>(b) * a.H + h;
  b_init(sm, 8, 1);
  const uint32_t tmem = sm.tmem_base;

  if (warp == 0) {
    if (lane == 0) {                               // step j: key tile j
      const uint8_t* head_kv = a.kv + bh * n_tiles * 32768u;
      b_copy_loop(sm, n, a.err, [&](int j, int st, uint32_t bar) {
        const uint32_t dst = smem_u32(stage0 + st * 2 * kTB);
        mbar_arrive_expect_tx(bar, 2 * kTB);
        bulk_load(dst, head_kv + static_cast<size_t>(j) * 32768u, kTB, bar);
        bulk_load(dst + kTB, head_kv + static_cast<size_t>(j) * 32768u + kTB, kTB, bar);
      });
    }
    __syncwarp();
  } else if (warp == 1 || warp >= 10) {
    // as dq_kernel, M = 128: warp 1 S, warp 10 dP, warp 11 dQ
    if (lane == 0) {
      constexpr uint32_t kIdS = idesc_bf16_f32(128, 64, 0, 0), kIdQ = idesc_bf16_f32(128, 128, 0, 1);
      bool ok = b_wait(sm, sm.a_ready, 0, a.err);
      if (warp == 1 || warp == 10) {
        const bool is_s = warp == 1;
        for (int j = 0; ok && j < n; ++j) {
          const int st = j % kBStages;
          const uint32_t bs = 128u * (j & 1);
          if (!(ok = b_wait(sm, sm.full[st], (j / kBStages) & 1, a.err))) break;
          if (j >= 2 && !(ok = b_wait(sm, is_s ? sm.acc_a[j & 1] : sm.ds_ready[j & 1], ((j >> 1) - 1) & 1, a.err)))
            break;
          tc_fence_after();
          const uint64_t bd = smem_desc_sw128(smem_u32(stage0 + st * 2 * kTB + (is_s ? 0u : kTB)), 16, 1024);
          const uint32_t dcol = (is_s ? kQColS : kQColP) + bs, acol = is_s ? kQColQ : kQColDO;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            umma_ts(tmem + dcol, tmem + acol + kk * 8, bd + (kk >> 2) * (8192 >> 4) + (kk & 3) * 2, kIdS, kk > 0);
          umma_commit(smem_u32(is_s ? &sm.s_full[j & 1] : &sm.p_full[j & 1]));
        }
      } else if (warp == 11) {
        for (int j = 0; ok && j < n; ++j) {
          const int st = j % kBStages;
          if (!(ok = b_wait(sm, sm.ds_ready[j & 1], (j >> 1) & 1, a.err))) break;
          tc_fence_after();
          const uint64_t kmn = smem_desc_sw128(smem_u32(stage0 + st * 2 * kTB), 8192, 1024);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_ts(tmem + kQColAcc, tmem + kQColS + 128u * (j & 1) + kk * 8, kmn + kk * (2048 >> 4), kIdQ,
                    (j > 0 || kk > 0) ? 1u : 0u);
          umma_commit(smem_u32(&sm.acc_a[j & 1]));
          umma_commit(smem_u32(&sm.free_[st]));
        }
      }
      umma_commit(smem_u32(&sm.acc_done));     // every MMA issued, also on a failed wait
      mbar_wait(smem_u32(&sm.acc_done), 0, nullptr, kBDrainNs);
    }
    __syncwarp();
  } else {
    // thread (query row r = 32 qd + lane) of column set cs: keys 32 cs .. 32 cs + 31
    const int qd = warp & 3, cs = (warp - 2) >> 2;
    const int r = 32 * qd + lane;
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(qd * 32) << 16);
    const int qt = r < 64 ? qa : qb;
    const int tok = qt >= 0 ? a.L.perm[qt * kTile + (r & 63)] : -1;
    if (cs == 0) row_to_tmem32(a.q + b * a.sb + h * a.sh, tok, a.ss, lane_addr + kQColQ);
    else row_to_tmem32(a.dout + b * a.d_sb + h * a.d_sh, tok, a.d_ss, lane_addr + kQColDO);
    tmem_wait_st();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_u32(&sm.a_ready));
    const size_t srow = (bh * n_tiles + (qt >= 0 ? qt : 0)) * kTile + (r & 63);
    const float lse = qt >= 0 ? a.lse[srow] : INFINITY;
    const float dd = qt >= 0 ? a.dd[srow] : 0.f;
    unsigned long long vm_next = a.L.valid[0];
    bool ok = true;
    for (int j = 0; j < n; ++j) {
      const unsigned long long vm = vm_next;
      if (j + 1 < n) vm_next = a.L.valid[j + 1];
      const uint32_t bs = 128u * (j & 1);
      if (!(ok = b_wait(sm, sm.s_full[j & 1], (j >> 1) & 1, a.err))) break;
      if (!(ok = b_wait(sm, sm.p_full[j & 1], (j >> 1) & 1, a.err))) break;
      tc_fence_after();
      float s[32], dp[32];
      tmem_ld32x32f(lane_addr + kQColS + bs + 32 * cs, s);
      tmem_ld32x32f(lane_addr + kQColP + bs + 32 * cs, dp);
      tmem_wait_ld();
      // both column sets of this quadrant have read their scores (bounded)
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&sm.qpair[qd]));
      if (!(ok = b_wait(sm, sm.qpair[qd], j & 1, a.err))) break;
      const uint32_t vbits = static_cast<uint32_t>(vm >> (32 * cs));
      uint32_t w[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        float ds[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int key = 2 * i + e;
          const float p = ((vbits >> key) & 1u) ? ex2_approx(fmaf(s[key], a.c_log2, -lse)) : 0.f;
          ds[e] = p * (dp[key] - dd);
        }
        w[i] = pack_bf16x2(ds[0], ds[1]);
      }
      tmem_st32x32_16(lane_addr + kQColS + bs + 16 * cs, w);    // dS (bf16 pairs) over S
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&sm.ds_ready[j & 1]));
    }
    if (ok && (ok = b_wait(sm, sm.acc_done, 0, a.err))) {
      tc_fence_after();
#pragma unroll 1
      for (int ch = 2 * cs; ch < 2 * cs + 2; ++ch) {   // dims 32 ch .. 32 ch + 31
        float y[32];
        tmem_ld32x32f(lane_addr + kQColAcc + 32 * ch, y);
        tmem_wait_ld();
        if (tok >= 0) {
          float4* dst = reinterpret_cast<float4*>(a.dq + b * a.o_sb + static_cast<int64_t>(tok) * a.o_ss +
                                                  h * a.o_sh + 32 * ch);
#pragma unroll
          for (int i = 0; i < 32; i += 4)
            dst[i / 4] = make_float4(y[i] * a.scale, y[i + 1] * a.scale, y[i + 2] * a.scale, y[i + 3] * a.scale);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kBTmemCols);
  }
}

// ------------------------------------------- transpose of the selection lists
// grid (sparse query tiles, H, B): counts of query tiles per candidate tile
__global__ void csr_count_kernel(const int32_t* __restrict__ idx, const int32_t* __restrict__ cnt, int kmax,
                                 int n_cand, int n_tiles, int c0, int H, int32_t* __restrict__ counts) {
  const int qt = c0 + blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const size_t bh = static_cast<size_t>(b) * H + h;
  const size_t row = bh * n_tiles + qt;
  const int n = min(max(cnt[row], 1), kmax);
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const int c = min(max(idx[row * kmax + i], 0), n_cand - 1);
    atomicAdd(&counts[bh * (n_cand + 1) + c], 1);
  }
}

// grid (H, B), 1024 threads: exclusive scan of the counts of one (b, h) into
// offsets (n_cand + 1 entries, relative to the head's list base bh * n_tiles *
// kmax); the cursors for the fill start at the offsets.
__global__ void __launch_bounds__(1024) csr_scan_kernel(int32_t* __restrict__ counts_off, int32_t* __restrict__ cursor,
                                                        int n_cand, int n_tiles, int kmax, int H) {
  const size_t bh = static_cast<size_t>(blockIdx.y) * H + blockIdx.x;
  int32_t* c = counts_off + bh * (n_cand + 1);
  int32_t* cur = cursor + bh * (n_cand + 1);
  __shared__ int32_t part[1024];
  const int per = (n_cand + blockDim.x - 1) / blockDim.x;
  const int lo = threadIdx.x * per, hi = min(n_cand, lo + per);
  int sum = 0;
  for (int i = lo; i < hi; ++i) sum += c[i];
  part[threadIdx.x] = sum;
  __syncthreads();
  for (int off = 1; off < static_cast<int>(blockDim.x); off <<= 1) {
    const int v = threadIdx.x >= static_cast<unsigned>(off) ? part[threadIdx.x - off] : 0;
    __syncthreads();
    part[threadIdx.x] += v;
    __syncthreads();
  }
  int run = static_cast<int>(bh * static_cast<size_t>(n_tiles) * kmax) + part[threadIdx.x] - sum;
  for (int i = lo; i < hi; ++i) {
    const int ci = c[i];
    c[i] = run;
    cur[i] = run;
    run += ci;
  }
  if (threadIdx.x == blockDim.x - 1) c[n_cand] = run;
}

__global__ void csr_fill_kernel(const int32_t* __restrict__ idx, const int32_t* __restrict__ cnt, int kmax,
                                int n_cand, int n_tiles, int c0, int H, int32_t* __restrict__ cursor,
                                int32_t* __restrict__ list) {
  const int qt = c0 + blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const size_t bh = static_cast<size_t>(b) * H + h;
  const size_t row = bh * n_tiles + qt;
  const int n = min(max(cnt[row], 1), kmax);
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const int c = min(max(idx[row * kmax + i], 0), n_cand - 1);
    list[atomicAdd(&cursor[bh * (n_cand + 1) + c], 1)] = qt;
  }
}

// One tensor of [B, S, H, 128] into tile-major 16 KB blocks (as the forward's).
__global__ void __launch_bounds__(256)
permute_one_kernel(DevLayout L, const uint16_t* __restrict__ x, int64_t sb, int64_t ss, int64_t sh, int H,
                   uint8_t* __restrict__ xtm) {
  const int tile = blockIdx.x, b = blockIdx.y;
  __shared__ int tok[kTile];
  for (int i = threadIdx.x; i < kTile; i += blockDim.x) tok[i] = L.perm[tile * kTile + i];
  __syncthreads();
  for (int w = threadIdx.x; w < H * 1024; w += blockDim.x) {
    const int pc = w & 7, r = (w >> 3) & 63, j = (w >> 9) & 1, h = w >> 10;
    const int t = tok[r];
    uint4 val = make_uint4(0u, 0u, 0u, 0u);
    if (t >= 0)
      val = __ldg(reinterpret_cast<const uint4*>(x + b * sb + static_cast<int64_t>(t) * ss + h * sh + j * 64 +
                                                 ((pc ^ (r & 7)) << 3)));
    *reinterpret_cast<uint4*>(xtm + ((static_cast<size_t>(b) * H + h) * L.n_tiles + tile) * 16384u + j * 8192 +
                              r * 128 + pc * 16) = val;
  }
}

// ---------------------------------------------------------- coarse branch
// Pooled means of Q, K, V: [3, B, H, n_tiles, 128]; grid (n_tiles, B, 3).
__global__ void __launch_bounds__(1024)
pool3_kernel(DevLayout L, const uint16_t* __restrict__ q, const uint16_t* __restrict__ k,
             const uint16_t* __restrict__ v, int64_t sb, int64_t ss, int64_t sh, int H, int B,
             float* __restrict__ pooled) {
  const int tile = blockIdx.x, b = blockIdx.y, which = blockIdx.z;
  const uint16_t* x = which == 0 ? q : (which == 1 ? k : v);
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
      const uint4 w = __ldg(reinterpret_cast<const uint4*>(x + b * sb + static_cast<int64_t>(t) * ss + h * sh + d0));
      const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        acc[2 * e] += __uint_as_float(u[e] << 16);
        acc[2 * e + 1] += __uint_as_float(u[e] & 0xFFFF0000u);
      }
    }
    float* dst = pooled + ((((static_cast<size_t>(which) * B + b) * H + h) * L.n_tiles + tile) * kHeadDim + d0);
#pragma unroll
    for (int e = 0; e < 8; ++e) dst[e] = acc[e] / n;
  }
}

// dOc[b, h, t] = sum over the valid rows i of tile t of cr_i g_i dO_i (per
// channel: g_{i,d} dO_{i,d}); dg_i = cr_i <dO_i, o_coarse[t]> (per channel:
// cr_i dO_{i,d} o_coarse[t, d]). cr = 0 on dense conditioning rows.
// grid (n_tiles, B), thread c: head c / 16, dims 8 (c % 16) .. + 7.
__global__ void __launch_bounds__(1024)
gate_bwd_kernel(DevLayout L, const uint16_t* __restrict__ dout, int64_t d_sb, int64_t d_ss, int64_t d_sh,
                const uint16_t* __restrict__ g, int64_t g_sb, int64_t g_ss, int64_t g_sh, int64_t g_sd,
                const float* __restrict__ o_coarse, int H, int c0, float* __restrict__ doc, float* __restrict__ dg,
                int64_t dg_sb, int64_t dg_ss, int64_t dg_sh, int64_t dg_sd) {
  const int tile = blockIdx.x, b = blockIdx.y;
  __shared__ int tok[kTile];
  for (int i = threadIdx.x; i < kTile; i += blockDim.x) tok[i] = L.perm[tile * kTile + i];
  __syncthreads();
  const bool cr = tile >= c0;
  // every lane of a warp runs the loop (the shuffle-sum below needs them all);
  // threads past the last head compute on head 0 and write nothing
  for (int cb = 0; cb < H * 16; cb += blockDim.x) {
    const int c = cb + threadIdx.x;
    const bool act = c < H * 16;
    const int h = act ? c >> 4 : 0, d0 = (c & 15) * 8, part = c & 15;
    const size_t th = (static_cast<size_t>(b) * H + h) * L.n_tiles + tile;
    const float* oc = o_coarse + th * kHeadDim + d0;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int s = 0; s < kTile; ++s) {
      const int t = tok[s];
      if (t < 0) continue;     // uniform over the block: every thread sees the same token list
      const uint4 w = __ldg(reinterpret_cast<const uint4*>(dout + b * d_sb + static_cast<int64_t>(t) * d_ss +
                                                           h * d_sh + d0));
      const uint32_t u[4] = {w.x, w.y, w.z, w.w};
      float dov[8];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        dov[2 * e] = __uint_as_float(u[e] << 16);
        dov[2 * e + 1] = __uint_as_float(u[e] & 0xFFFF0000u);
      }
      const uint16_t* gp = g + b * g_sb + static_cast<int64_t>(t) * g_ss + h * g_sh;
      float* dgp = dg + b * dg_sb + static_cast<int64_t>(t) * dg_ss + h * dg_sh;
      if (g_sd > 0) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float ge = __uint_as_float(static_cast<uint32_t>(gp[(d0 + e) * g_sd]) << 16);
          acc[e] = fmaf(cr ? ge : 0.f, dov[e], acc[e]);
          if (act) dgp[(d0 + e) * dg_sd] = cr ? dov[e] * oc[e] : 0.f;
        }
      } else {
        const float ge = cr ? __uint_as_float(static_cast<uint32_t>(gp[0]) << 16) : 0.f;
        float dot = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          acc[e] = fmaf(ge, dov[e], acc[e]);
          dot = fmaf(dov[e], oc[e], dot);
        }
        // the 16 threads of a head hold the 16 parts of <dO, o_coarse>: shuffle-sum
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
        if (act && part == 0) dgp[0] = cr ? dot : 0.f;
      }
    }
    if (act) {
      float* dst = doc + th * kHeadDim + d0;
#pragma unroll
      for (int e = 0; e < 8; ++e) dst[e] = acc[e];
    }
  }
}

// Row pass of the coarse softmax backward: per block of 64 query tiles of one
// (b, h), two sweeps over the candidate tiles: (1) row max and sum of
// s = scale <Qbar, Kbar>; (2) P = softmax, dP = <dOc, Vbar>, dS = P (dP - D)
// with D = <dOc, o_coarse>, dQbar += scale dS Kbar; P and dS are stored for the
// column pass. Thread (ty, tx) = (tid / 16, tid % 16): rows 4 ty .. 4 ty + 3,
// candidate columns 4 tx .. 4 tx + 3 of a chunk, output dims 8 tx .. 8 tx + 7.
constexpr int kCR = 64, kCC = 64, kCThreads = 256;

struct CRSmem {
  float qT[kHeadDim][kCR];               // Qbar rows, transposed
  float gT[kHeadDim][kCR];               // dOc rows, transposed
  float kT[kHeadDim][kCC];               // Kbar chunk, transposed
  float vT[kHeadDim][kCC];               // Vbar chunk, transposed
  float kr[kCC][kHeadDim];               // Kbar chunk, rows (for dQbar)
  float ds[kCR][kCC + 4];
  float dsum[kCR];                       // D per row
};

__global__ void __launch_bounds__(kCThreads)
coarse_bwd_rows_kernel(int n_tiles, int cand0, int n_cand, int H, int B, const float* __restrict__ pooled,
                       const float* __restrict__ doc, const float* __restrict__ o_coarse, float scale,
                       float* __restrict__ pm, float* __restrict__ dsm, int ld, float* __restrict__ dqbar) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  CRSmem& sm = *reinterpret_cast<CRSmem*>(smem_raw);
  const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
  const int qt0 = blockIdx.x * kCR, h = blockIdx.y, b = blockIdx.z;
  const size_t bh = static_cast<size_t>(b) * H + h;
  const size_t plane = static_cast<size_t>(B) * H * n_tiles * kHeadDim;
  const float* qbar = pooled + bh * n_tiles * kHeadDim;
  const float* kbar = pooled + plane + (bh * n_tiles + cand0) * kHeadDim;
  const float* vbar = pooled + 2 * plane + (bh * n_tiles + cand0) * kHeadDim;
  for (int f = tid; f < kCR * kHeadDim; f += kCThreads) {
    const int r = f % kCR, d = f / kCR;
    const bool in = qt0 + r < n_tiles;
    sm.qT[d][r] = in ? qbar[static_cast<size_t>(qt0 + r) * kHeadDim + d] : 0.f;
    sm.gT[d][r] = in ? doc[(bh * n_tiles + qt0 + r) * kHeadDim + d] : 0.f;
  }
  if (tid < kCR) {
    float s = 0.f;
    if (qt0 + tid < n_tiles)
      for (int d = 0; d < kHeadDim; ++d)
        s += doc[(bh * n_tiles + qt0 + tid) * kHeadDim + d] * o_coarse[(bh * n_tiles + qt0 + tid) * kHeadDim + d];
    sm.dsum[tid] = s;
  }
  float m[4], l[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    m[i] = -INFINITY;
    l[i] = 0.f;
  }
  float acc[4][8];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[i][e] = 0.f;
  for (int pass = 0; pass < 2; ++pass) {
    for (int c0 = 0; c0 < n_cand; c0 += kCC) {
      __syncthreads();
      for (int f = tid; f < kCC * kHeadDim; f += kCThreads) {
        const int cc = f / kHeadDim, d = f % kHeadDim;
        const bool in = c0 + cc < n_cand;
        const float kv = in ? kbar[static_cast<size_t>(c0 + cc) * kHeadDim + d] : 0.f;
        sm.kT[d][cc] = kv;
        sm.kr[cc][d] = kv;
        sm.vT[d][cc] = in ? vbar[static_cast<size_t>(c0 + cc) * kHeadDim + d] : 0.f;
      }
      __syncthreads();
      float s[4][4], dp[4][4];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) s[i][j] = dp[i][j] = 0.f;
      for (int d = 0; d < kHeadDim; ++d) {
        float qa[4], kb[4], ga[4], vb[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          qa[i] = sm.qT[d][4 * ty + i];
          ga[i] = sm.gT[d][4 * ty + i];
          kb[i] = sm.kT[d][4 * tx + i];
          vb[i] = sm.vT[d][4 * tx + i];
        }
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            s[i][j] = fmaf(qa[i], kb[j], s[i][j]);
            if (pass) dp[i][j] = fmaf(ga[i], vb[j], dp[i][j]);
          }
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) s[i][j] = (c0 + 4 * tx + j < n_cand) ? s[i][j] * scale : -INFINITY;
      if (pass == 0) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          float cm = fmaxf(fmaxf(s[i][0], s[i][1]), fmaxf(s[i][2], s[i][3]));
#pragma unroll
          for (int off = 1; off < 16; off <<= 1) cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, off));
          const float mn = fmaxf(m[i], cm);
          float ps = 0.f;
#pragma unroll
          for (int j = 0; j < 4; ++j) ps += expf(s[i][j] - mn);
#pragma unroll
          for (int off = 1; off < 16; off <<= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
          l[i] = l[i] * expf(m[i] - mn) + ps;
          m[i] = mn;
        }
      } else {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int rr = 4 * ty + i, row = qt0 + rr;
          const float dsum = sm.dsum[rr];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int col = c0 + 4 * tx + j;
            const float p = col < n_cand ? expf(s[i][j] - m[i]) / l[i] : 0.f;
            const float dsv = p * (dp[i][j] - dsum);
            sm.ds[rr][4 * tx + j] = dsv;
            if (row < n_tiles && col < n_cand) {
              pm[(bh * n_tiles + row) * ld + col] = p;
              dsm[(bh * n_tiles + row) * ld + col] = dsv;
            }
          }
        }
        __syncthreads();
        for (int cc = 0; cc < kCC; ++cc) {
          float dsr[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) dsr[i] = sm.ds[4 * ty + i][cc];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float kv = sm.kr[cc][8 * tx + e];
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[i][e] = fmaf(dsr[i], kv, acc[i][e]);
          }
        }
      }
    }
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int row = qt0 + 4 * ty + i;
    if (row < n_tiles)
#pragma unroll
      for (int e = 0; e < 8; ++e) dqbar[(bh * n_tiles + row) * kHeadDim + 8 * tx + e] = acc[i][e] * scale;
  }
}

// Column pass: per block of 64 candidate tiles, dKbar = scale dS^T Qbar and
// dVbar = P^T dOc over all query tiles. Thread (ty, tx): candidates 4 ty ..,
// dims 8 tx ...
struct CCSmem {
  float ds[kCR][kCC + 4];
  float p[kCR][kCC + 4];
  float q[kCR][kHeadDim];
  float g[kCR][kHeadDim];
};

__global__ void __launch_bounds__(kCThreads)
coarse_bwd_cols_kernel(int n_tiles, int n_cand, int H, int B, const float* __restrict__ pooled,
                       const float* __restrict__ doc, float scale, const float* __restrict__ pm,
                       const float* __restrict__ dsm, int ld, float* __restrict__ dkbar, float* __restrict__ dvbar) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  CCSmem& sm = *reinterpret_cast<CCSmem*>(smem_raw);
  const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
  const int c0 = blockIdx.x * kCC, h = blockIdx.y, b = blockIdx.z;
  const size_t bh = static_cast<size_t>(b) * H + h;
  const float* qbar = pooled + bh * n_tiles * kHeadDim;
  float ak[4][8], av[4][8];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int e = 0; e < 8; ++e) ak[i][e] = av[i][e] = 0.f;
  for (int r0 = 0; r0 < n_tiles; r0 += kCR) {
    __syncthreads();
    for (int f = tid; f < kCR * kCC; f += kCThreads) {
      const int rr = f / kCC, cc = f % kCC;
      const bool in = r0 + rr < n_tiles && c0 + cc < n_cand;
      sm.ds[rr][cc] = in ? dsm[(bh * n_tiles + r0 + rr) * ld + c0 + cc] : 0.f;
      sm.p[rr][cc] = in ? pm[(bh * n_tiles + r0 + rr) * ld + c0 + cc] : 0.f;
    }
    for (int f = tid; f < kCR * kHeadDim; f += kCThreads) {
      const int rr = f / kHeadDim, d = f % kHeadDim;
      const bool in = r0 + rr < n_tiles;
      sm.q[rr][d] = in ? qbar[static_cast<size_t>(r0 + rr) * kHeadDim + d] : 0.f;
      sm.g[rr][d] = in ? doc[(bh * n_tiles + r0 + rr) * kHeadDim + d] : 0.f;
    }
    __syncthreads();
    for (int rr = 0; rr < kCR; ++rr) {
      float dsr[4], pr[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        dsr[i] = sm.ds[rr][4 * ty + i];
        pr[i] = sm.p[rr][4 * ty + i];
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float qv = sm.q[rr][8 * tx + e], gv = sm.g[rr][8 * tx + e];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          ak[i][e] = fmaf(dsr[i], qv, ak[i][e]);
          av[i][e] = fmaf(pr[i], gv, av[i][e]);
        }
      }
    }
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int c = c0 + 4 * ty + i;
    if (c < n_cand)
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        dkbar[(bh * n_cand + c) * kHeadDim + 8 * tx + e] = ak[i][e] * scale;
        dvbar[(bh * n_cand + c) * kHeadDim + 8 * tx + e] = av[i][e];
      }
  }
}

// The pooled gradients back to the tokens: dq += dQbar[t] / n_t for every
// valid token of tile t, dk += dKbar / n_t, dv += dVbar / n_t for candidate
// tiles. grid (n_tiles, B).
__global__ void __launch_bounds__(1024)
pool_scatter_kernel(DevLayout L, int H, int cand0, int n_cand, const float* __restrict__ dqbar,
                    const float* __restrict__ dkbar, const float* __restrict__ dvbar, float* __restrict__ dq,
                    float* __restrict__ dk, float* __restrict__ dv, int64_t o_sb, int64_t o_ss, int64_t o_sh) {
  const int tile = blockIdx.x, b = blockIdx.y;
  __shared__ int tok[kTile];
  for (int i = threadIdx.x; i < kTile; i += blockDim.x) tok[i] = L.perm[tile * kTile + i];
  __syncthreads();
  const float inv_n = 1.0f / static_cast<float>(L.count[tile]);
  const int c = tile - cand0;
  const bool cand = c >= 0 && c < n_cand;
  for (int w = threadIdx.x; w < H * kHeadDim; w += blockDim.x) {
    const int h = w / kHeadDim, d = w % kHeadDim;
    const size_t bh = static_cast<size_t>(b) * H + h;
    const float gq = dqbar[(bh * L.n_tiles + tile) * kHeadDim + d] * inv_n;
    const float gk = cand ? dkbar[(bh * n_cand + c) * kHeadDim + d] * inv_n : 0.f;
    const float gv = cand ? dvbar[(bh * n_cand + c) * kHeadDim + d] * inv_n : 0.f;
    for (int s = 0; s < kTile; ++s) {
      const int t = tok[s];
      if (t < 0) continue;
      const int64_t off = b * o_sb + static_cast<int64_t>(t) * o_ss + h * o_sh + d;
      dq[off] += gq;
      if (cand) {
        dk[off] += gk;
        dv[off] += gv;
      }
    }
  }
}

// [header][attention workspace][lse][D][tile-major Q][tile-major dO][CSR offsets][CSR cursors][CSR lists]
// [pooled Q, K, V][dOc][P][dS][dQbar][dKbar][dVbar]
struct BWorkspace {
  size_t attn, attn_bytes, lse, dd, qtm, dotm, off, cur, list, pooled, doc, pm, dsm, dqbar, dkbar, dvbar, total;
  int32_t ld;
};

BWorkspace b_workspace(const vsa_layout* L, int B, int H, const vsa_params* p) {
  BWorkspace w{};
  const size_t bh = static_cast<size_t>(B) * H;
  const size_t tiles = bh * L->n_tiles;
  const Candidates cand = candidates(L, p->sink);
  int32_t kmax = 0;
  vsa_select_kmax(L, p, &kmax);
  size_t attn_bytes = 0;
  vsa_sparse_attn_workspace_size(L, B, H, p, &attn_bytes);
  w.ld = (cand.count + 3) / 4 * 4;
  size_t o = kBHeader;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o = align_up(o + bytes, 256);
    return at;
  };
  w.attn = take(attn_bytes);
  w.attn_bytes = attn_bytes;
  w.lse = take(tiles * kTile * sizeof(float));
  w.dd = take(tiles * kTile * sizeof(float));
  w.qtm = take(tiles * kTB);
  w.dotm = take(tiles * kTB);
  w.off = take(bh * (cand.count + 1) * sizeof(int32_t));
  w.cur = take(bh * (cand.count + 1) * sizeof(int32_t));
  w.list = take(tiles * static_cast<size_t>(kmax) * sizeof(int32_t));
  w.pooled = take(3 * tiles * kHeadDim * sizeof(float));
  w.doc = take(tiles * kHeadDim * sizeof(float));
  w.pm = take(tiles * static_cast<size_t>(w.ld) * sizeof(float));
  w.dsm = take(tiles * static_cast<size_t>(w.ld) * sizeof(float));
  w.dqbar = take(tiles * kHeadDim * sizeof(float));
  w.dkbar = take(bh * cand.count * kHeadDim * sizeof(float));
  w.dvbar = take(bh * cand.count * kHeadDim * sizeof(float));
  w.total = o;
  return w;
}

}  // namespace
}  // namespace vsa

using namespace vsa;

extern "C" {

vsa_status vsa_sparse_attn_bwd_workspace_size(const vsa_layout* L, int32_t B, int32_t H, const vsa_params* p,
                                              size_t* bytes) {
  if (!L || !bytes || B <= 0 || H <= 0) return VSA_ERR_INVALID_ARG;
  vsa_status st = check_params(p);
  if (st != VSA_OK) return st;
  *bytes = b_workspace(L, B, H, p).total;
  return VSA_OK;
}

vsa_status vsa_sparse_attn_bwd(const vsa_layout* L, const vsa_params* p, int32_t B, int32_t H, const void* q,
                               const void* k, const void* v, int64_t sb, int64_t ss, int64_t sh, const void* g,
                               int64_t g_sb, int64_t g_ss, int64_t g_sh, int64_t g_sd, const int32_t* idx,
                               const int32_t* cnt, int32_t kmax, const float* o_coarse, const void* dout,
                               int64_t d_sb, int64_t d_ss, int64_t d_sh, float* dq, float* dk, float* dv,
                               int64_t o_sb, int64_t o_ss, int64_t o_sh, float* dg, int64_t dg_sb, int64_t dg_ss,
                               int64_t dg_sh, int64_t dg_sd, void* workspace, size_t workspace_bytes,
                               cudaStream_t stream) {
  if (!L) return VSA_ERR_INVALID_ARG;
  vsa_status st = check_params(p);
  if (st != VSA_OK) return st;
  if (p->coarse != VSA_COARSE_MEAN || p->extra_tokens != 0) return VSA_ERR_UNSUPPORTED;
  st = check_qkv(q, k, v, sb, ss, sh, B, H);
  if (st != VSA_OK) return st;
  st = check_qkv(dout, dout, dout, d_sb, d_ss, d_sh, B, H);
  if (st != VSA_OK) return st;
  if (!g || !idx || !cnt || !o_coarse || !dq || !dk || !dv || !dg || !workspace) return VSA_ERR_INVALID_ARG;
  if (g_sb < 0 || g_ss <= 0 || g_sh <= 0 || g_sd < 0 || dg_sb < 0 || dg_ss <= 0 || dg_sh <= 0 || dg_sd < 0 ||
      (g_sd > 0) != (dg_sd > 0))
    return VSA_ERR_INVALID_ARG;
  if (o_sb < 0 || o_ss <= 0 || o_sh <= 0 || (o_sb * 4) % 16 || (o_ss * 4) % 16 || (o_sh * 4) % 16 ||
      reinterpret_cast<uintptr_t>(dq) % 16 || reinterpret_cast<uintptr_t>(dk) % 16 ||
      reinterpret_cast<uintptr_t>(dv) % 16 || reinterpret_cast<uintptr_t>(workspace) % 256 ||
      reinterpret_cast<uintptr_t>(o_coarse) % 16)
    return VSA_ERR_INVALID_ARG;
  const BWorkspace ws = b_workspace(L, B, H, p);
  if (workspace_bytes < ws.total) return VSA_ERR_WORKSPACE_TOO_SMALL;
  if (!L->dev_buf) return VSA_ERR_NOT_UPLOADED;
  int32_t want_kmax = 0;
  vsa_select_kmax(L, p, &want_kmax);
  if (kmax != want_kmax) return VSA_ERR_INVALID_ARG;

  uint8_t* w = static_cast<uint8_t*>(workspace);
  const DevLayout D = L->dev();
  const Candidates cand = candidates(L, p->sink);
  const int c0 = p->sink == VSA_SINK_EXACT_KV_AND_ROWS ? L->n_cond : 0;
  const float scale = effective_scale(p);
  cudaError_t e = cudaMemsetAsync(workspace, 0, sizeof(int), stream);
  if (e != cudaSuccess) return cuda_fail("vsa_sparse_attn_bwd: cudaMemsetAsync", e);

  // 1. the forward's row statistics (log2-sum-exp2, D = <dO, o_fine>)
  AttnStats stats{};
  stats.lse = reinterpret_cast<float*>(w + ws.lse);
  stats.d = reinterpret_cast<float*>(w + ws.dd);
  stats.dout = dout;
  stats.d_sb = d_sb;
  stats.d_ss = d_ss;
  stats.d_sh = d_sh;
  st = attn_forward(L, p, B, H, q, k, v, sb, ss, sh, nullptr, 0, 0, 0, 0, idx, cnt, kmax, nullptr, nullptr,
                    nullptr, nullptr, VSA_OUT_F32, 0, 0, 0, &stats, w + ws.attn, ws.attn_bytes, stream);
  if (st != VSA_OK) return st;
  // the attention workspace now holds the tile-major K and V right after its 256-byte header
  const uint8_t* kv = w + ws.attn + 256;

  // 2. tile-major Q and dO; the transpose of the selection lists
  permute_one_kernel<<<dim3(L->n_tiles, B), 256, 0, stream>>>(D, static_cast<const uint16_t*>(q), sb, ss, sh, H,
                                                             w + ws.qtm);
  permute_one_kernel<<<dim3(L->n_tiles, B), 256, 0, stream>>>(D, static_cast<const uint16_t*>(dout), d_sb, d_ss,
                                                             d_sh, H, w + ws.dotm);
  int32_t* off = reinterpret_cast<int32_t*>(w + ws.off);
  int32_t* cur = reinterpret_cast<int32_t*>(w + ws.cur);
  int32_t* list = reinterpret_cast<int32_t*>(w + ws.list);
  e = cudaMemsetAsync(off, 0, static_cast<size_t>(B) * H * (cand.count + 1) * sizeof(int32_t), stream);
  if (e != cudaSuccess) return cuda_fail("vsa_sparse_attn_bwd: cudaMemsetAsync(csr)", e);
  const int nq = L->n_tiles - c0;
  if (nq > 0) csr_count_kernel<<<dim3(nq, H, B), 128, 0, stream>>>(idx, cnt, kmax, cand.count, L->n_tiles, c0, H, off);
  csr_scan_kernel<<<dim3(H, B), 1024, 0, stream>>>(off, cur, cand.count, L->n_tiles, kmax, H);
  if (nq > 0)
    csr_fill_kernel<<<dim3(nq, H, B), 128, 0, stream>>>(idx, cnt, kmax, cand.count, L->n_tiles, c0, H, cur, list);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail("vsa_sparse_attn_bwd: permute/transpose launch", e);

  // 3. the fine branch: dq, then dk and dv (each written once per token)
  BArgs a{};
  a.L = D;
  a.H = H;
  a.sink = p->sink;
  a.n_cond = L->n_cond;
  a.cand0 = cand.first;
  a.n_cand = cand.count;
  a.kmax = kmax;
  a.c0 = c0;
  a.q = static_cast<const uint16_t*>(q);
  a.dout = static_cast<const uint16_t*>(dout);
  a.sb = sb;
  a.ss = ss;
  a.sh = sh;
  a.d_sb = d_sb;
  a.d_ss = d_ss;
  a.d_sh = d_sh;
  a.kv = kv;
  a.qtm = w + ws.qtm;
  a.dotm = w + ws.dotm;
  a.lse = stats.lse;
  a.dd = stats.d;
  a.idx = idx;
  a.cnt = cnt;
  a.csr_off = off;
  a.csr_list = list;
  a.dq = dq;
  a.dk = dk;
  a.dv = dv;
  a.o_sb = o_sb;
  a.o_ss = o_ss;
  a.o_sh = o_sh;
  a.scale = scale;
  a.c_log2 = scale * 1.4426950408889634f;
  a.err = static_cast<int*>(workspace);
  a.dq_add = (p->sink != VSA_SINK_OFF && L->n_cond > 0) ? 1 : 0;
  e = cudaFuncSetAttribute(dq_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(kDqPairSmem));
  if (e != cudaSuccess) return cuda_fail("vsa_sparse_attn_bwd: cudaFuncSetAttribute(dq pair)", e);
  e = cudaFuncSetAttribute(dq_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kDqSmem));
  if (e != cudaSuccess) return cuda_fail("vsa_sparse_attn_bwd: cudaFuncSetAttribute(dq)", e);
  e = cudaFuncSetAttribute(dkv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kDkvSmem));
  if (e != cudaSuccess) return cuda_fail("vsa_sparse_attn_bwd: cudaFuncSetAttribute(dkv)", e);
  e = cudaFuncSetAttribute(dkv_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(kDkvPairSmem));
  if (e != cudaSuccess) return cuda_fail("vsa_sparse_attn_bwd: cudaFuncSetAttribute(dkv pair)", e);
  if (a.dq_add)
    dq_pair_kernel<<<dim3((c0 + 1) / 2 + (L->n_tiles - c0 + 1) / 2, H, B), kBThreads, kDqPairSmem, stream>>>(a);
  dq_kernel<<<dim3(L->n_tiles, H, B), kBThreads, kDqSmem, stream>>>(a);
  if (p->sink != VSA_SINK_OFF && L->n_cond > 0)
    dkv_pair_kernel<<<dim3((L->n_cond + 1) / 2, H, B), kBThreads, kDkvPairSmem, stream>>>(a);
  dkv_kernel<<<dim3(L->n_tiles, H, B), kBThreads, kDkvSmem, stream>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail("vsa_sparse_attn_bwd: fine-branch launch", e);

  // 4. gate and coarse branch, then the pooled gradients back to the tokens
  float* pooled = reinterpret_cast<float*>(w + ws.pooled);
  float* doc = reinterpret_cast<float*>(w + ws.doc);
  const int pool_threads = std::min(1024, (16 * H + 31) / 32 * 32);
  pool3_kernel<<<dim3(L->n_tiles, B, 3), pool_threads, 0, stream>>>(
      D, static_cast<const uint16_t*>(q), static_cast<const uint16_t*>(k), static_cast<const uint16_t*>(v), sb, ss,
      sh, H, B, pooled);
  gate_bwd_kernel<<<dim3(L->n_tiles, B), pool_threads, 0, stream>>>(
      D, static_cast<const uint16_t*>(dout), d_sb, d_ss, d_sh, static_cast<const uint16_t*>(g), g_sb, g_ss, g_sh,
      g_sd, o_coarse, H, c0, doc, dg, dg_sb, dg_ss, dg_sh, dg_sd);
  float* pm = reinterpret_cast<float*>(w + ws.pm);
  float* dsm = reinterpret_cast<float*>(w + ws.dsm);
  float* dqbar = reinterpret_cast<float*>(w + ws.dqbar);
  float* dkbar = reinterpret_cast<float*>(w + ws.dkbar);
  float* dvbar = reinterpret_cast<float*>(w + ws.dvbar);
  e = cudaFuncSetAttribute(coarse_bwd_rows_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(sizeof(CRSmem)));
  if (e != cudaSuccess) return cuda_fail("vsa_sparse_attn_bwd: cudaFuncSetAttribute(rows)", e);
  e = cudaFuncSetAttribute(coarse_bwd_cols_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(sizeof(CCSmem)));
  if (e != cudaSuccess) return cuda_fail("vsa_sparse_attn_bwd: cudaFuncSetAttribute(cols)", e);
  coarse_bwd_rows_kernel<<<dim3((L->n_tiles + kCR - 1) / kCR, H, B), kCThreads, sizeof(CRSmem), stream>>>(
      L->n_tiles, cand.first, cand.count, H, B, pooled, doc, o_coarse, scale, pm, dsm, ws.ld, dqbar);
  coarse_bwd_cols_kernel<<<dim3((cand.count + kCC - 1) / kCC, H, B), kCThreads, sizeof(CCSmem), stream>>>(
      L->n_tiles, cand.count, H, B, pooled, doc, scale, pm, dsm, ws.ld, dkbar, dvbar);
  pool_scatter_kernel<<<dim3(L->n_tiles, B), 1024, 0, stream>>>(D, H, cand.first, cand.count, dqbar, dkbar, dvbar,
                                                               dq, dk, dv, o_sb, o_ss, o_sh);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail("vsa_sparse_attn_bwd: coarse-branch launch", e);
  return VSA_OK;
}

vsa_status vsa_sparse_attn_bwd_status(const void* workspace, cudaStream_t stream) {
  if (!workspace) return VSA_ERR_INVALID_ARG;
  cudaError_t e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return cuda_fail("vsa_sparse_attn_bwd_status: cudaStreamSynchronize", e);
  // word 0: the backward kernels; the attention workspace (right after the
  // 256-byte header) holds the status of the forward pass in statistics mode
  int err[2] = {0, 0};
  e = cudaMemcpy(&err[0], workspace, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail("vsa_sparse_attn_bwd_status: cudaMemcpy", e);
  e = cudaMemcpy(&err[1], static_cast<const uint8_t*>(workspace) + kBHeader, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail("vsa_sparse_attn_bwd_status: cudaMemcpy", e);
  const int st = err[0] != 0 ? err[0] : err[1];
  return st == 0 ? VSA_OK : static_cast<vsa_status>(st);
}

}  // extern "C"
