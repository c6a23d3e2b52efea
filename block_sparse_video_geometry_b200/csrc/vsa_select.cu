// Coarse branch and block selection: the entry points, the pooling kernel,
// and the fp32 kernels of the Spark-Reweight coarse branch.
//
// 1. pool_kernel      : mean of Q, K, V over the valid tokens of every tile
//                       (fp32), read straight from the natural [B, S, H, 128]
//                       layout through the tile's token list. For
//                       VSA_COARSE_MEAN it also writes Kbar and Vbar of the
//                       candidate tiles as hi/lo bf16 chunks for the tensor-core
//                       kernels of vsa_select_tc.cu, which then do the scores,
//                       the selection and the coarse softmax on chip.
// VSA_COARSE_REWEIGHT runs:
// 2. anchor_kernel, reweight_kernel: the Spark-Reweight summaries.
// 3. coarse_kernel    : for a block of 64 query tiles of one (batch, head):
//                       s = scale * Qbar Kbar^T against every candidate
//                       key tile (the video tiles, or every tile with
//                       VSA_SINK_OFF), in fp32 FMA; the scores go to the
//                       workspace for selection, and the reweighted logits feed
//                       an online softmax against V~ that yields o_coarse. With
//                       the adaptive threshold it also sums s and s^2 in fp64
//                       per block.
// 4. select_kernel    : one warp per query tile: radix select of the k-th
//                       largest score (ties -> lower tile) or the adaptive
//                       threshold mean + tau * std, emitted as an ascending
//                       list of candidate ordinals.
// Pages: "BSAI FastH3 Native VSA (recipe)", "The mechanism, briefly" (tiles
// are scored and only the top slice is attended exactly); "ComfyUI Agrega Nodo
// Central de Atencion Dispersa y Compilador Comfy", "Atencion dispersa por
// bloques" (top-k keep percent; Sol-Attn per-head threshold in sigmas; VSA
// coarse compression branch); "Spark-H3 ...", "Que cambia Spark-Attn" (the
// compressed branch summarises K/V by mean pooling, Spark-Reweight by anchor
// weights).
//
// Pooling is bound by HBM (it reads Q, K, V once). Scores stay fp32-accurate
// end to end so that the selected sets match an fp64 evaluation except on
// near-ties.

#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cfloat>
#include <cmath>

#include "vsa_internal.h"

namespace vsa {

namespace {

constexpr int kPoolMaxThreads = 1024;
std::atomic<uint64_t> g_select_stall_ns{0};   // vsa_debug_inject_select_wait_timeout
constexpr int kCoarseRows = 64;       // query tiles per coarse block
constexpr int kCoarseCols = 64;       // candidate key tiles per streamed chunk
constexpr int kCoarseThreads = 256;
constexpr int kSelectWarps = 4;

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// ------------------------------------------------------------------ pooling
// The split Kbar / Vbar chunks of the tensor-core kernels (VSA_COARSE_MEAN):
// candidate c of (b, h) is row c % 64 of chunk c / 64; a chunk is
// [term: hi, lo][d half][64 rows][128 B] with 16-byte unit u of a row at
// 16 (u ^ (row & 7)) (the 128-byte swizzle the MMA descriptors expect).
struct SplitOut {
  uint8_t* kv[2];           // K, V chunks, or null (fp32 kernels)
  int32_t cand0, n_cand, n_chunks;
};

__device__ __forceinline__ uint32_t bf16_pair_rn(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %2, %1;" : "=r"(r) : "f"(lo), "f"(hi));
  return r;
}

// grid (n_tiles + pad, B, 3), block = min(1024, 16 * H) rounded up to a warp.
// Thread c handles head c / 16, dims 8 * (c % 16) .. + 7. Blocks past n_tiles
// (split output only) zero the pad rows of the last chunk. Block (0, 0, 0)
// also clears the call's status word.
__global__ void __launch_bounds__(kPoolMaxThreads)
pool_kernel(DevLayout L, const uint16_t* __restrict__ q, const uint16_t* __restrict__ k,
            const uint16_t* __restrict__ v, int64_t sb, int64_t ss, int64_t sh, int H, int B,
            float* __restrict__ pooled, SplitOut so, int* __restrict__ status) {
  const int tile = blockIdx.x, b = blockIdx.y, which = blockIdx.z;
  if (tile == 0 && b == 0 && which == 0 && threadIdx.x == 0) status[0] = 0;
  const int nchunks = H * 16;
  if (tile >= L.n_tiles) {
    if (which == 0) return;
    const int c = so.n_cand + (tile - L.n_tiles);
    for (int t = threadIdx.x; t < nchunks; t += blockDim.x) {
      const int h = t >> 4, d0 = (t & 15) * 8, r = c & 63, u = (d0 & 63) >> 3;
      uint8_t* dst = so.kv[which - 1] + ((static_cast<size_t>(b) * H + h) * so.n_chunks + (c >> 6)) * 32768u +
                     (d0 >> 6) * 8192 + r * 128 + ((u ^ (r & 7)) << 4);
      *reinterpret_cast<uint4*>(dst) = make_uint4(0u, 0u, 0u, 0u);
      *reinterpret_cast<uint4*>(dst + 16384) = make_uint4(0u, 0u, 0u, 0u);
    }
    return;
  }
  const uint16_t* x = which == 0 ? q : (which == 1 ? k : v);
  __shared__ int tok[kTile];
  for (int i = threadIdx.x; i < kTile; i += blockDim.x) tok[i] = L.perm[tile * kTile + i];
  __syncthreads();
  const float n = static_cast<float>(L.count[tile]);
  const int cand = tile - so.cand0;
  const bool split = which > 0 && so.kv[0] != nullptr && cand >= 0 && cand < so.n_cand;
  for (int c = threadIdx.x; c < nchunks; c += blockDim.x) {
    const int h = c >> 4, d0 = (c & 15) * 8;
    const uint16_t* base = x + b * sb + h * sh + d0;
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;
#pragma unroll 8
    for (int s = 0; s < kTile; ++s) {
      const int t = tok[s];
      if (t >= 0) {
        const uint4 w = __ldg(reinterpret_cast<const uint4*>(base + static_cast<int64_t>(t) * ss));
        acc[0] += bf16lo(w.x); acc[1] += bf16hi(w.x);
        acc[2] += bf16lo(w.y); acc[3] += bf16hi(w.y);
        acc[4] += bf16lo(w.z); acc[5] += bf16hi(w.z);
        acc[6] += bf16lo(w.w); acc[7] += bf16hi(w.w);
      }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] /= n;
    float* dst = pooled + ((((static_cast<size_t>(which) * B + b) * H + h) * L.n_tiles + tile) * kHeadDim + d0);
    reinterpret_cast<float4*>(dst)[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
    reinterpret_cast<float4*>(dst)[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
    if (split) {
      uint32_t hi[4], lo[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        hi[e] = bf16_pair_rn(acc[2 * e], acc[2 * e + 1]);
        lo[e] = bf16_pair_rn(acc[2 * e] - __uint_as_float(hi[e] << 16),
                             acc[2 * e + 1] - __uint_as_float(hi[e] & 0xFFFF0000u));
      }
      const int r = cand & 63, u = (d0 & 63) >> 3;
      uint8_t* o = so.kv[which - 1] + ((static_cast<size_t>(b) * H + h) * so.n_chunks + (cand >> 6)) * 32768u +
                   (d0 >> 6) * 8192 + r * 128 + ((u ^ (r & 7)) << 4);
      *reinterpret_cast<uint4*>(o) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
      *reinterpret_cast<uint4*>(o + 16384) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
    }
  }
}

// --------------------------------------------------------- Spark-Reweight
// Anchor of each (batch, head): the mean query of the video tokens, from the
// pooled tile means weighted by the tiles' token counts (fp64 sums).
// grid (H, B), 128 threads (one per dim).
__global__ void __launch_bounds__(kHeadDim) anchor_kernel(DevLayout L, int H, const float* __restrict__ pooled_q,
                                                          float* __restrict__ anchor) {
  const int h = blockIdx.x, b = blockIdx.y, d = threadIdx.x;
  const size_t bh = static_cast<size_t>(b) * H + h;
  double acc = 0.0, n = 0.0;
#pragma unroll 4
  for (int t = L.n_cond; t < L.n_tiles; ++t) {
    const double c = static_cast<double>(L.count[t]);
    acc += c * static_cast<double>(pooled_q[(bh * L.n_tiles + t) * kHeadDim + d]);
    n += c;
  }
  anchor[bh * kHeadDim + d] = static_cast<float>(acc / n);
}

// Weighted summaries and log-mass bias of every candidate key tile: with the
// anchor logits x_i = scale <a, k_i> of the tile's valid tokens,
//   K~ = sum w_i k_i, V~ = sum w_i v_i, w = softmax(x), b = log(mean exp(x)) - scale <a, K~>.
// grid (n_cand, B), 256 threads; warp w handles heads w, w + 8, ...; lane l
// handles dims 4l .. 4l + 3 (one 8-byte load per token row and tensor).
constexpr int kReweightThreads = 256;

__global__ void __launch_bounds__(kReweightThreads)
reweight_kernel(DevLayout L, int cand0, int n_cand, const uint16_t* __restrict__ k, const uint16_t* __restrict__ v,
                int64_t sb, int64_t ss, int64_t sh, int H, int B, float scale, const float* __restrict__ anchor,
                float* __restrict__ summaries, float* __restrict__ bias) {
  const int c = blockIdx.x, b = blockIdx.y, tile = cand0 + c;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __shared__ int tok[kTile];
  __shared__ float xs[kReweightThreads / 32][kTile];
  for (int i = threadIdx.x; i < kTile; i += kReweightThreads) tok[i] = L.perm[tile * kTile + i];
  __syncthreads();
  const float n = static_cast<float>(L.count[tile]);
  for (int h = warp; h < H; h += kReweightThreads / 32) {
    const size_t bh = static_cast<size_t>(b) * H + h;
    const float4 a = reinterpret_cast<const float4*>(anchor + bh * kHeadDim)[lane];
    const uint16_t* kb = k + b * sb + h * sh + 4 * lane;
    const uint16_t* vb = v + b * sb + h * sh + 4 * lane;
    float m = -INFINITY;
    for (int s = 0; s < kTile; ++s) {
      const int t = tok[s];
      float x = -INFINITY;
      if (t >= 0) {
        const uint2 w = __ldg(reinterpret_cast<const uint2*>(kb + static_cast<int64_t>(t) * ss));
        float part = a.x * bf16lo(w.x) + a.y * bf16hi(w.x) + a.z * bf16lo(w.y) + a.w * bf16hi(w.y);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
        x = part * scale;
      }
      if (lane == 0) xs[warp][s] = x;
      m = fmaxf(m, x);
    }
    __syncwarp();
    float z = 0.f, ks[4] = {0.f, 0.f, 0.f, 0.f}, vs[4] = {0.f, 0.f, 0.f, 0.f};
    for (int s = 0; s < kTile; ++s) {
      const int t = tok[s];
      if (t < 0) continue;
      const float e = expf(xs[warp][s] - m);
      z += e;
      const uint2 kw = __ldg(reinterpret_cast<const uint2*>(kb + static_cast<int64_t>(t) * ss));
      const uint2 vw = __ldg(reinterpret_cast<const uint2*>(vb + static_cast<int64_t>(t) * ss));
      ks[0] = fmaf(e, bf16lo(kw.x), ks[0]); ks[1] = fmaf(e, bf16hi(kw.x), ks[1]);
      ks[2] = fmaf(e, bf16lo(kw.y), ks[2]); ks[3] = fmaf(e, bf16hi(kw.y), ks[3]);
      vs[0] = fmaf(e, bf16lo(vw.x), vs[0]); vs[1] = fmaf(e, bf16hi(vw.x), vs[1]);
      vs[2] = fmaf(e, bf16lo(vw.y), vs[2]); vs[3] = fmaf(e, bf16hi(vw.y), vs[3]);
    }
    const float inv = 1.0f / z;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      ks[e] *= inv;
      vs[e] *= inv;
    }
    float part = a.x * ks[0] + a.y * ks[1] + a.z * ks[2] + a.w * ks[3];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
    const size_t plane = static_cast<size_t>(B) * H * n_cand * kHeadDim;
    float* kd = summaries + (bh * n_cand + c) * kHeadDim;
    reinterpret_cast<float4*>(kd)[lane] = make_float4(ks[0], ks[1], ks[2], ks[3]);
    reinterpret_cast<float4*>(kd + plane)[lane] = make_float4(vs[0], vs[1], vs[2], vs[3]);
    if (lane == 0) bias[bh * n_cand + c] = m + logf(z / n) - scale * part;
    __syncwarp();   // xs[warp] is rewritten by the next head
  }
}

// ------------------------------------------------------- scores + coarse
// grid (ceil(n_tiles / 64), H, B), 256 threads. Thread (ty, tx) = (tid / 16,
// tid % 16) owns query rows 4*ty .. 4*ty+3; in the score block it owns candidate
// columns 4*tx .. 4*tx+3 of the chunk, in the coarse product dims 8*tx .. +7.
struct CoarseSmem {
  float qT[kHeadDim][kCoarseRows];        // pooled Q, transposed
  float kv[kCoarseCols * kHeadDim];       // Kbar chunk transposed [d][c], then Vbar chunk [c][d]
  float p[kCoarseRows][kCoarseCols + 4];  // probabilities of the chunk
};

// With kReweight the selection scores still use the mean-pooled K, and the
// coarse softmax uses scale <Qbar, K~> + b against V~ (Spark-Reweight).
template <bool kStats, bool kReweight>
__global__ void __launch_bounds__(kCoarseThreads, 2)
coarse_kernel(int n_tiles, int cand0, int n_cand, int H, int B, const float* __restrict__ pooled,
              float scale, float* __restrict__ scores, int ld_scores, float* __restrict__ o_coarse,
              double* __restrict__ stats, const float* __restrict__ summaries, const float* __restrict__ rbias) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  CoarseSmem& sm = *reinterpret_cast<CoarseSmem*>(smem_raw);
  const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
  const int qt0 = blockIdx.x * kCoarseRows, h = blockIdx.y, b = blockIdx.z;
  const size_t bh = static_cast<size_t>(b) * H + h;
  const size_t plane = static_cast<size_t>(B) * H * n_tiles * kHeadDim;
  const float* qbar = pooled + bh * n_tiles * kHeadDim;
  const float* kbar = pooled + plane + (bh * n_tiles + cand0) * kHeadDim;
  const float* vbar = pooled + 2 * plane + (bh * n_tiles + cand0) * kHeadDim;
  const size_t rplane = static_cast<size_t>(B) * H * n_cand * kHeadDim;
  const float* ktil = kReweight ? summaries + bh * n_cand * kHeadDim : nullptr;
  const float* vsum = kReweight ? summaries + rplane + bh * n_cand * kHeadDim : vbar;

  // pooled Q rows of this block, transposed; rows past n_tiles are zero
  for (int f = tid; f < kCoarseRows * kHeadDim / 4; f += kCoarseThreads) {
    const int r = f % kCoarseRows, d4 = f / kCoarseRows;
    float4 val = make_float4(0.f, 0.f, 0.f, 0.f);
    if (qt0 + r < n_tiles) val = reinterpret_cast<const float4*>(qbar + static_cast<size_t>(qt0 + r) * kHeadDim)[d4];
    sm.qT[4 * d4 + 0][r] = val.x;
    sm.qT[4 * d4 + 1][r] = val.y;
    sm.qT[4 * d4 + 2][r] = val.z;
    sm.qT[4 * d4 + 3][r] = val.w;
  }

  float m[4], l[4], o[4][8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    m[i] = -INFINITY;
    l[i] = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) o[i][e] = 0.f;
  }
  double s1 = 0.0, s2 = 0.0;

  for (int c0 = 0; c0 < n_cand; c0 += kCoarseCols) {
    // chunk of key summaries (rows c0 .. c0 + 63 of src) into sm.kv, transposed
    // [d][c], then acc = Qbar K^T for this thread's 4 x 4 block
    float acc[4][4];
    auto chunk_dots = [&](const float* src) {
      __syncthreads();  // previous readers of sm.kv are done
      for (int f = tid; f < kCoarseCols * kHeadDim / 4; f += kCoarseThreads) {
        const int c = f % kCoarseCols, d4 = f / kCoarseCols;
        float4 val = make_float4(0.f, 0.f, 0.f, 0.f);
        if (c0 + c < n_cand) val = reinterpret_cast<const float4*>(src + static_cast<size_t>(c0 + c) * kHeadDim)[d4];
        sm.kv[(4 * d4 + 0) * kCoarseCols + c] = val.x;
        sm.kv[(4 * d4 + 1) * kCoarseCols + c] = val.y;
        sm.kv[(4 * d4 + 2) * kCoarseCols + c] = val.z;
        sm.kv[(4 * d4 + 3) * kCoarseCols + c] = val.w;
      }
      __syncthreads();
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
#pragma unroll 4
      for (int d = 0; d < kHeadDim; ++d) {
        const float4 a = *reinterpret_cast<const float4*>(&sm.qT[d][4 * ty]);
        const float4 bb = *reinterpret_cast<const float4*>(&sm.kv[d * kCoarseCols + 4 * tx]);
        const float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {bb.x, bb.y, bb.z, bb.w};
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
      }
    };
    chunk_dots(kbar);

    // scale, write the selection scores, statistics
    float s[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int row = qt0 + 4 * ty + i;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int col = c0 + 4 * tx + j;
        s[i][j] = col < n_cand ? acc[i][j] * scale : -INFINITY;
        if (kStats && col < n_cand && row < n_tiles) {
          s1 += static_cast<double>(s[i][j]);
          s2 += static_cast<double>(s[i][j]) * static_cast<double>(s[i][j]);
        }
      }
      if (row < n_tiles) {
        float4* dst = reinterpret_cast<float4*>(scores + (bh * n_tiles + row) * ld_scores + c0 + 4 * tx);
        *dst = make_float4(s[i][0], s[i][1], s[i][2], s[i][3]);
      }
    }
    if (kReweight) {
      // the coarse logits: scale <Qbar, K~> + b
      chunk_dots(ktil);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int col = c0 + 4 * tx + j;
        const float bj = col < n_cand ? rbias[bh * n_cand + col] : 0.f;
#pragma unroll
        for (int i = 0; i < 4; ++i) s[i][j] = col < n_cand ? fmaf(acc[i][j], scale, bj) : -INFINITY;
      }
    }

    // online softmax of the chunk
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float cm = fmaxf(fmaxf(s[i][0], s[i][1]), fmaxf(s[i][2], s[i][3]));
#pragma unroll
      for (int off = 1; off < 16; off <<= 1) cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, off));
      const float mn = fmaxf(m[i], cm);
      const float corr = expf(m[i] - mn);
      float ps = 0.f;
      float pv[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        pv[j] = expf(s[i][j] - mn);
        ps += pv[j];
      }
#pragma unroll
      for (int off = 1; off < 16; off <<= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
      l[i] = l[i] * corr + ps;
      m[i] = mn;
#pragma unroll
      for (int e = 0; e < 8; ++e) o[i][e] *= corr;
      *reinterpret_cast<float4*>(&sm.p[4 * ty + i][4 * tx]) = make_float4(pv[0], pv[1], pv[2], pv[3]);
    }
    __syncthreads();  // the dots consumed sm.kv; p is complete

    // Vbar (or V~) chunk [c][d] into the same buffer
    for (int f = tid; f < kCoarseCols * kHeadDim / 4; f += kCoarseThreads) {
      const int c = f / (kHeadDim / 4), d4 = f % (kHeadDim / 4);
      float4 val = make_float4(0.f, 0.f, 0.f, 0.f);
      if (c0 + c < n_cand) val = reinterpret_cast<const float4*>(vsum + static_cast<size_t>(c0 + c) * kHeadDim)[d4];
      reinterpret_cast<float4*>(sm.kv)[f] = val;
    }
    __syncthreads();
#pragma unroll 2
    for (int c = 0; c < kCoarseCols; c += 4) {
      float pr[4][4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float4 t = *reinterpret_cast<const float4*>(&sm.p[4 * ty + i][c]);
        pr[i][0] = t.x; pr[i][1] = t.y; pr[i][2] = t.z; pr[i][3] = t.w;
      }
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        const float4 v0 = *reinterpret_cast<const float4*>(&sm.kv[(c + cc) * kHeadDim + 8 * tx]);
        const float4 v1 = *reinterpret_cast<const float4*>(&sm.kv[(c + cc) * kHeadDim + 8 * tx + 4]);
        const float vv[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int e = 0; e < 8; ++e) o[i][e] = fmaf(pr[i][cc], vv[e], o[i][e]);
      }
    }
  }

#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int row = qt0 + 4 * ty + i;
    if (row < n_tiles) {
      float* dst = o_coarse + (bh * n_tiles + row) * kHeadDim + 8 * tx;
      const float inv = 1.0f / l[i];
      reinterpret_cast<float4*>(dst)[0] = make_float4(o[i][0] * inv, o[i][1] * inv, o[i][2] * inv, o[i][3] * inv);
      reinterpret_cast<float4*>(dst)[1] = make_float4(o[i][4] * inv, o[i][5] * inv, o[i][6] * inv, o[i][7] * inv);
    }
  }

  if (kStats) {
    __shared__ double red[2][kCoarseThreads / 32];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      s1 += __shfl_xor_sync(0xffffffffu, s1, off);
      s2 += __shfl_xor_sync(0xffffffffu, s2, off);
    }
    if ((tid & 31) == 0) {
      red[0][tid >> 5] = s1;
      red[1][tid >> 5] = s2;
    }
    __syncthreads();
    if (tid == 0) {
      double a = 0.0, c = 0.0;
      for (int w = 0; w < kCoarseThreads / 32; ++w) {
        a += red[0][w];
        c += red[1][w];
      }
      stats[(bh * gridDim.x + blockIdx.x) * 2 + 0] = a;
      stats[(bh * gridDim.x + blockIdx.x) * 2 + 1] = c;
    }
  }
}

// ---------------------------------------------------------------- selection
__device__ __forceinline__ uint32_t ordered_key(float f) {
  const uint32_t u = __float_as_uint(f + 0.0f);   // -0 -> +0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// grid (ceil(n_tiles / rows_per_block), H, B), rows_per_block warps.
template <bool kAdaptive>
__global__ void select_kernel(int n_tiles, int n_cand, int H, const float* __restrict__ scores,
                              int ld_scores, int k, float tau, const double* __restrict__ stats,
                              int n_row_blocks, int32_t* __restrict__ idx, int kmax,
                              int32_t* __restrict__ cnt) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float* row = reinterpret_cast<float*>(smem_raw) + static_cast<size_t>(warp) * ld_scores;
  uint32_t* hist = reinterpret_cast<uint32_t*>(reinterpret_cast<float*>(smem_raw) +
                                               static_cast<size_t>(blockDim.x >> 5) * ld_scores) +
                   warp * 256;
  const int qt = blockIdx.x * (blockDim.x >> 5) + warp;
  if (qt >= n_tiles) return;
  const int h = blockIdx.y, b = blockIdx.z;
  const size_t bh = static_cast<size_t>(b) * H + h;
  const float* src = scores + (bh * n_tiles + qt) * ld_scores;
  for (int i = lane; i < n_cand; i += 32) row[i] = src[i];
  __syncwarp();
  int32_t* out = idx + (bh * n_tiles + qt) * kmax;
  const uint32_t lt_mask = (1u << lane) - 1u;

  if (!kAdaptive) {
    // radix select of the k-th largest key, 8 bits per round from the top
    uint32_t prefix = 0, pmask = 0;
    int krem = k;
    for (int shift = 24; shift >= 0; shift -= 8) {
      for (int i = lane; i < 256; i += 32) hist[i] = 0;
      __syncwarp();
      for (int i = lane; i < n_cand; i += 32) {
        const uint32_t key = ordered_key(row[i]);
        if ((key & pmask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
      }
      __syncwarp();
      int c8[8], tot = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        c8[j] = static_cast<int>(hist[255 - (lane * 8 + j)]);
        tot += c8[j];
      }
      int incl = tot;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += y;
      }
      const int excl = incl - tot;
      const uint32_t hit = __ballot_sync(0xffffffffu, excl < krem && krem <= incl);
      const int src_lane = __ffs(hit) - 1;
      int bin = 0, before = 0;
      if (lane == src_lane) {
        int run = excl;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (run + c8[j] >= krem) {
            bin = 255 - (lane * 8 + j);
            before = run;
            break;
          }
          run += c8[j];
        }
      }
      bin = __shfl_sync(0xffffffffu, bin, src_lane);
      before = __shfl_sync(0xffffffffu, before, src_lane);
      krem -= before;
      prefix |= static_cast<uint32_t>(bin) << shift;
      pmask |= 0xFFu << shift;
      __syncwarp();
    }
    // prefix is the k-th largest key; krem of its equals are taken, lowest ordinals first
    int pos = 0, eq_seen = 0;
    for (int base = 0; base < n_cand; base += 32) {
      const int i = base + lane;
      const uint32_t key = i < n_cand ? ordered_key(row[i]) : 0u;
      const bool eq = i < n_cand && key == prefix;
      const uint32_t eqb = __ballot_sync(0xffffffffu, eq);
      const int eq_rank = eq_seen + __popc(eqb & lt_mask);
      const bool sel = i < n_cand && (key > prefix || (eq && eq_rank < krem));
      const uint32_t selb = __ballot_sync(0xffffffffu, sel);
      if (sel) out[pos + __popc(selb & lt_mask)] = i;
      pos += __popc(selb);
      eq_seen += __popc(eqb);
    }
    if (lane == 0) cnt[bh * n_tiles + qt] = pos;
  } else {
    // per-(batch, head) threshold from the block partial sums, fixed order
    double a = 0.0, c = 0.0;
    for (int i = lane; i < n_row_blocks; i += 32) {
      a += stats[(bh * n_row_blocks + i) * 2 + 0];
      c += stats[(bh * n_row_blocks + i) * 2 + 1];
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      a += __shfl_xor_sync(0xffffffffu, a, off);
      c += __shfl_xor_sync(0xffffffffu, c, off);
    }
    const double nn = static_cast<double>(n_tiles) * static_cast<double>(n_cand);
    const double mean = a / nn;
    const double var = fmax(c / nn - mean * mean, 0.0);
    const double thr = mean + static_cast<double>(tau) * sqrt(var);
    int pos = 0;
    for (int base = 0; base < n_cand; base += 32) {
      const int i = base + lane;
      const bool sel = i < n_cand && static_cast<double>(row[i]) >= thr;
      const uint32_t selb = __ballot_sync(0xffffffffu, sel);
      if (sel) out[pos + __popc(selb & lt_mask)] = i;
      pos += __popc(selb);
    }
    if (pos == 0) {  // keep the argmax (lowest ordinal among equal maxima)
      float best = -INFINITY;
      int bi = 0x7fffffff;
      for (int i = lane; i < n_cand; i += 32) {
        if (row[i] > best) {
          best = row[i];
          bi = i;
        }
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        const float ob = __shfl_xor_sync(0xffffffffu, best, off);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
        if (ob > best || (ob == best && oi < bi)) {
          best = ob;
          bi = oi;
        }
      }
      if (lane == 0) out[0] = bi;
      pos = 1;
    }
    if (lane == 0) cnt[bh * n_tiles + qt] = pos;
  }
}

}  // namespace

}  // namespace vsa

using namespace vsa;

extern "C" {

vsa_status vsa_coarse_select_workspace_size(const vsa_layout* L, int32_t B, int32_t H,
                                            const vsa_params* p, size_t* bytes) {
  if (!L || !bytes || B <= 0 || H <= 0) return VSA_ERR_INVALID_ARG;
  vsa_status st = check_params(p);
  if (st != VSA_OK) return st;
  *bytes = select_workspace(L, B, H, p).total;
  return VSA_OK;
}

vsa_status vsa_coarse_select(const vsa_layout* L, const vsa_params* p, int32_t B, int32_t H,
                             const void* q, const void* k, const void* v, int64_t sb, int64_t ss,
                             int64_t sh, int32_t* idx, int32_t* cnt, float* o_coarse,
                             void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  if (!L) return VSA_ERR_INVALID_ARG;
  vsa_status st = check_params(p);
  if (st != VSA_OK) return st;
  st = check_qkv(q, k, v, sb, ss, sh, B, H);
  if (st != VSA_OK) return st;
  if (!idx || !cnt || !o_coarse || !workspace) return VSA_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(o_coarse) % 16 || reinterpret_cast<uintptr_t>(workspace) % 256)
    return VSA_ERR_INVALID_ARG;
  if (!L->dev_buf) return VSA_ERR_NOT_UPLOADED;
  const SelectWorkspace ws = select_workspace(L, B, H, p);
  const Candidates cand = candidates(L, p->sink);
  if (workspace_bytes < ws.total) return VSA_ERR_WORKSPACE_TOO_SMALL;
  const bool reweight = p->coarse == VSA_COARSE_REWEIGHT;
  if (!reweight && cand.count > 65535) {   // 16-bit histogram counters of the tensor-core kernel
    set_detail("vsa_coarse_select: more than 65535 candidate key tiles");
    return VSA_ERR_UNSUPPORTED;
  }

  const int ld = ws.ld_scores;
  const size_t row_bytes = static_cast<size_t>(ld) * sizeof(float);
  const int rows_per_block = static_cast<int>(std::min<size_t>(kSelectWarps, (200u << 10) / row_bytes));
  if (reweight && rows_per_block < 1) return VSA_ERR_UNSUPPORTED;   // more than 51200 candidate tiles

  char* w = static_cast<char*>(workspace);
  float* pooled = reinterpret_cast<float*>(w + ws.pooled);
  float* scores = reinterpret_cast<float*>(w + ws.scores);
  double* stats = reinterpret_cast<double*>(w + ws.stats);
  const DevLayout D = L->dev();
  const bool adaptive = p->mode == VSA_SELECT_ADAPTIVE;
  const float scale = effective_scale(p);
  int32_t kmax = 0;
  vsa_select_kmax(L, p, &kmax);

  SplitOut so{};
  so.kv[0] = reweight ? nullptr : reinterpret_cast<uint8_t*>(w + ws.ksplit);
  so.kv[1] = reweight ? nullptr : reinterpret_cast<uint8_t*>(w + ws.vsplit);
  so.cand0 = cand.first;
  so.n_cand = cand.count;
  so.n_chunks = ws.n_chunks;
  const int pad = reweight ? 0 : ws.n_chunks * 64 - cand.count;
  const int pool_threads = std::min(kPoolMaxThreads, (16 * H + 31) / 32 * 32);
  pool_kernel<<<dim3(L->n_tiles + pad, B, 3), pool_threads, 0, stream>>>(
      D, static_cast<const uint16_t*>(q), static_cast<const uint16_t*>(k),
      static_cast<const uint16_t*>(v), sb, ss, sh, H, B, pooled, so, static_cast<int*>(workspace));
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail("vsa_coarse_select: pool launch", e);
  if (!reweight)
    return select_tc(L, p, B, H, ws, workspace, idx, cnt, o_coarse, g_select_stall_ns.load(std::memory_order_relaxed),
                     stream);

  float* anchor = reinterpret_cast<float*>(w + ws.anchor);
  float* summaries = reinterpret_cast<float*>(w + ws.summaries);
  float* rbias = reinterpret_cast<float*>(w + ws.bias);
  anchor_kernel<<<dim3(H, B), kHeadDim, 0, stream>>>(D, H, pooled, anchor);
  reweight_kernel<<<dim3(cand.count, B), kReweightThreads, 0, stream>>>(
      D, cand.first, cand.count, static_cast<const uint16_t*>(k), static_cast<const uint16_t*>(v), sb, ss, sh, H,
      B, scale, anchor, summaries, rbias);

  const size_t coarse_smem = sizeof(CoarseSmem);
  auto ck = adaptive ? coarse_kernel<true, true> : coarse_kernel<false, true>;
  e = cudaFuncSetAttribute(ck, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(coarse_smem));
  if (e != cudaSuccess) return cuda_fail("vsa_coarse_select: cudaFuncSetAttribute(coarse)", e);
  ck<<<dim3(ws.n_row_blocks, H, B), kCoarseThreads, coarse_smem, stream>>>(
      L->n_tiles, cand.first, cand.count, H, B, pooled, scale, scores, ld, o_coarse, stats, summaries, rbias);

  const size_t sel_smem = rows_per_block * row_bytes + rows_per_block * 256 * sizeof(uint32_t);
  auto sk = adaptive ? select_kernel<true> : select_kernel<false>;
  e = cudaFuncSetAttribute(sk, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(sel_smem));
  if (e != cudaSuccess) return cuda_fail("vsa_coarse_select: cudaFuncSetAttribute(select)", e);
  sk<<<dim3((L->n_tiles + rows_per_block - 1) / rows_per_block, H, B), 32 * rows_per_block, sel_smem,
       stream>>>(L->n_tiles, cand.count, H, scores, ld, kmax, p->tau, stats, ws.n_row_blocks, idx,
                 kmax, cnt);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail("vsa_coarse_select: launch", e);
  return VSA_OK;
}

vsa_status vsa_coarse_select_workspace_init(void* workspace, cudaStream_t stream) {
  if (!workspace || reinterpret_cast<uintptr_t>(workspace) % 256) return VSA_ERR_INVALID_ARG;
  cudaError_t e = cudaMemsetAsync(workspace, 0, kSelectHeader, stream);
  if (e != cudaSuccess) return cuda_fail("vsa_coarse_select_workspace_init: cudaMemsetAsync", e);
  return VSA_OK;
}

vsa_status vsa_coarse_select_status(const void* workspace, cudaStream_t stream) {
  if (!workspace) return VSA_ERR_INVALID_ARG;
  cudaError_t e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return cuda_fail("vsa_coarse_select_status: cudaStreamSynchronize", e);
  int err = 0;
  e = cudaMemcpy(&err, workspace, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail("vsa_coarse_select_status: cudaMemcpy", e);
  return err == 0 ? VSA_OK : static_cast<vsa_status>(err);
}

vsa_status vsa_coarse_select_failed_calls(const void* workspace, cudaStream_t stream, uint32_t* count) {
  if (!workspace || !count) return VSA_ERR_INVALID_ARG;
  cudaError_t e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return cuda_fail("vsa_coarse_select_failed_calls: cudaStreamSynchronize", e);
  e = cudaMemcpy(count, static_cast<const int*>(workspace) + 1, sizeof(uint32_t), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail("vsa_coarse_select_failed_calls: cudaMemcpy", e);
  return VSA_OK;
}

vsa_status vsa_debug_inject_select_wait_timeout(uint64_t timeout_ns) {
  g_select_stall_ns.store(timeout_ns, std::memory_order_relaxed);
  return VSA_OK;
}

}  // extern "C"

// -------------------------------------------------------------------------
// Allocation-free variant of vsa_coarse_select.
//
// Some callers cannot hand this library a workspace: code running inside a
// host framework that plans every device allocation ahead of time and forbids
// allocations outside its plan, or callers that must not pay the device-wide
// synchronisation and latency of cudaMalloc in the middle of a step. For them
// the selection scratch (status words, pooled means, split chunks, marks)
// lives in the fixed buffer below, which is part of the library's device
// image: every GPU that loads libvsa holds these 32 MiB until the process
// exits. Workloads whose scratch does not fit are refused, not truncated.
// -------------------------------------------------------------------------
#include <cstdio>
#include <mutex>

namespace vsa {
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;
constexpr int kNoAllocMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kNoAllocMaxDevices] = {};

// The built-in buffer's device address on the current device, looked up once
// per device with that device current (host code must not use the array's
// name as a device address). A process that resets a device with
// cudaDeviceReset must not call the allocation-free entry points afterwards:
// the cached address belongs to the destroyed context.
vsa_status noalloc_scratch(void** scratch) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail("vsa_coarse_select_noalloc: cudaGetDevice", e);
  if (dev < 0 || dev >= kNoAllocMaxDevices) {
    set_detail("vsa_coarse_select_noalloc: device ordinal beyond 63");
    return VSA_ERR_UNSUPPORTED;
  }
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    e = cudaGetSymbolAddress(&g_noalloc_ptr[dev], g_noalloc_scratch);
    if (e != cudaSuccess) {
      g_noalloc_ptr[dev] = nullptr;
      return cuda_fail("vsa_coarse_select_noalloc: cudaGetSymbolAddress", e);
    }
  }
  *scratch = g_noalloc_ptr[dev];
  return VSA_OK;
}

}  // namespace
}  // namespace vsa

extern "C" vsa_status vsa_coarse_select_noalloc(const vsa_layout* L, const vsa_params* p, int32_t B,
                                                int32_t H, const void* q, const void* k, const void* v,
                                                int64_t sb, int64_t ss, int64_t sh, int32_t* idx,
                                                int32_t* cnt, float* o_coarse, cudaStream_t stream) {
  if (!L || B <= 0 || H <= 0) return VSA_ERR_INVALID_ARG;
  vsa_status st = check_params(p);
  if (st != VSA_OK) return st;
  const size_t need = select_workspace(L, B, H, p).total;
  if (need > kNoAllocScratchBytes) {
    char msg[160];
    std::snprintf(msg, sizeof(msg),
                  "vsa_coarse_select_noalloc: this shape needs %zu bytes of scratch, the built-in buffer "
                  "holds %zu",
                  need, kNoAllocScratchBytes);
    set_detail(msg);
    return VSA_ERR_UNSUPPORTED;
  }
  void* scratch = nullptr;
  st = noalloc_scratch(&scratch);
  if (st != VSA_OK) return st;
  return vsa_coarse_select(L, p, B, H, q, k, v, sb, ss, sh, idx, cnt, o_coarse, scratch,
                           kNoAllocScratchBytes, stream);
}

extern "C" vsa_status vsa_coarse_select_noalloc_status(cudaStream_t stream) {
  void* scratch = nullptr;
  vsa_status st = noalloc_scratch(&scratch);
  if (st != VSA_OK) return st;
  return vsa_coarse_select_status(scratch, stream);
}
