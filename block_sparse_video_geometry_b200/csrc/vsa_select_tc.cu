// Coarse branch and block selection on the tensor cores (VSA_COARSE_MEAN).
//
// Pages: "BSAI FastH3 Native VSA (recipe)", "The mechanism, briefly" (tiles are
// scored by their pooled summaries and only the top slice is attended
// exactly); "ComfyUI Agrega Nodo Central de Atencion Dispersa y Compilador
// Comfy", "Atencion dispersa por bloques" (top-k keep percent; the Sol-Attn
// per-head threshold mean + tau * std; the VSA coarse compression branch).
//
// One CTA owns 128 query tiles of one (batch, head): TMEM lane r holds query
// tile r of the block. The tile scores s = scale * <Qbar, Kbar> of the block
// against every candidate key tile are formed by tcgen05 MMAs, 64 candidates
// (one chunk) at a time, and never leave the chip: the score matrix is
// recomputed when a later pass needs it again (an M = 128, N = 64 score chunk
// costs 24 MMAs; writing it to HBM and reading it back would cost more).
//
// Precision. Qbar, Kbar and Vbar are fp32 means. Each is split as hi + lo with
// hi = bf16(x) and lo = bf16(x - hi) (x - hi is exact; the pair holds x to a
// relative 2^-17), and products take the three leading terms
//   Qhi Khi + Qhi Klo + Qlo Khi
// with fp32 accumulation. The dropped Qlo Klo and the split residuals are below
// 3 * 2^-17 of |q_d k_d| per term, the size of the rounding of an fp32 FMA chain
// over 128 dims, so the scores carry fp32-class error and the selected sets
// match an fp64 evaluation except on near-ties. P V uses the same three terms
// of P (in [0, 1]) and Vbar.
//
// Passes over the candidate chunks (each one streams Kbar through shared
// memory and recomputes the scores):
//  * range    : per query tile the maximum score (first maximal candidate),
//               the minimum, and (adaptive mode) the fp64 sum and sum of
//               squares of the block's scores;
//  * softmax  : P = exp2((s - max) log2 e) with the exact row maximum, so no
//               rescaling; P overwrites its scores in TMEM as hi/lo bf16 pairs
//               and O += P V accumulates in TMEM; o_coarse = O / sum P. Top-k:
//               every score also lands in a 256-bin histogram of its row over
//               [min, max] (bins are a monotone function of the score, so each
//               bin is an interval of values). Adaptive: the scores at or above
//               the head's threshold are marked;
//  * collect  : (top-k) the bin holding the k-th largest score is known from
//               the histogram; candidates in higher bins are selected, the
//               boundary bin's members (at most 64, normally a handful) are
//               kept with their ordinals and ranked exactly (score descending,
//               lower ordinal first);
//  * radix x4, emit : (top-k, only when some row's boundary bin holds more than
//               64 members, e.g. rows of equal scores) an exact radix select of
//               the 32-bit order-preserving keys of that bin's members, 8 bits
//               per pass, then a pass that marks the members above the found
//               key and the first equal ones by ordinal.
// Marks are bitmaps per query tile in the workspace; the CTA turns them into
// ascending candidate lists at the end (one warp per query tile).
//
// Top-k runs range, softmax and collect in one launch. The adaptive threshold
// needs the statistics of the whole head, so it takes two launches: range with
// statistics, then softmax with the threshold marks.
//
// Warp roles: 0 issues the bulk copies of the Kbar (and Vbar) chunks, 1 issues
// the MMAs (whichever of the next score chunk or the next P V product is ready),
// 2-9 own the query tiles, two threads per tile (TMEM lane quadrant = warp % 4;
// warps 2-5 take candidates 0-31 of each chunk, 6-9 candidates 32-63). Every wait
// is bounded; a wait that runs out records VSA_ERR_TIMEOUT, raises an abort
// flag that ends the other roles' loops, drains the copies and MMAs in flight
// and frees TMEM.

#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "sm100.cuh"
#include "vsa_internal.h"

namespace vsa {
namespace {

using namespace sm100;

constexpr int kRows = 128;               // query tiles per CTA
constexpr int kChunk = 64;               // candidates per chunk
constexpr int kKStages = 2;
constexpr int kVStages = 2;
constexpr int kSBufs = 4;                // score buffers in TMEM
constexpr int kBins = 256;
constexpr int kHistPairs = kBins / 2 + 1;   // histogram words per row (two 16-bit counters each) + one for
                                            // the dummy bin 256 that scores outside the candidates go to
constexpr int kCap = 64;                 // boundary-bin members ranked directly per row
constexpr int kHalfCap = kCap / 2;       // of which each of the row's two threads keeps up to 32
constexpr int kQStride = 528;            // staged Qbar rows: 512 bytes + 16 (conflict-free column reads)
constexpr int kRowWarps = 8;             // two threads per query tile
constexpr int kThreads = 64 + 32 * kRowWarps;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColQ = 0;            // Qbar hi (64 columns of bf16 pairs), lo (64)
constexpr uint32_t kColS = 128;          // 4 score buffers of 64 fp32 columns; P overwrites them as bf16 pairs
constexpr uint32_t kColO = 384;          // coarse output accumulator, 128 fp32 columns
constexpr uint32_t kTermBytes = 16384;   // one split term of a chunk: [d half][64 rows][128 B], swizzled
constexpr uint32_t kChunkBytes = 2 * kTermBytes;
constexpr uint32_t kIdescS = idesc_bf16_f32(128, 64, 0, 0);     // S = Qbar Kbar^T, both K-major
constexpr uint32_t kIdescPV = idesc_bf16_f32(128, 128, 0, 1);   // O += P Vbar, Vbar MN-major
constexpr uint64_t kTimeoutNs = 2000000000ull;
constexpr uint64_t kDrainNs = 200000000ull;
constexpr float kLog2e = 1.4426950408889634f;

enum : int { kModeTopk = 0, kModeStats = 1, kModeThresh = 2 };
enum : int { kPassRange = 0, kPassSoftmax = 1, kPassCollect = 2, kPassRadix = 3, kPassEmit = 4 };
constexpr int kFallbackPasses = 5;       // radix x 4 + emit

template <int kMode>
__device__ __forceinline__ int pass_kind(int p) {
  if (kMode == kModeStats) return kPassRange;
  if (kMode == kModeThresh) return kPassSoftmax;
  return p < 3 ? p : (p < 7 ? kPassRadix : kPassEmit);
}

struct SelArgs {
  const float* qbar;        // pooled Q [B, H, n_tiles, 128]
  const uint8_t* ksplit;    // [B, H, n_chunks] chunks of kChunkBytes: hi term, lo term
  const uint8_t* vsplit;
  int32_t n_tiles, H, n_cand, n_chunks, n_qblocks;
  int32_t k;                // top-k count
  float scale, tau;
  float* rowmax;            // [B, H, n_tiles]: written by the statistics launch, read by the threshold launch
  int32_t* rowarg;
  double* stats;            // [B, H, n_qblocks, 2]
  uint32_t* bits;           // [B, H, n_tiles, 2 * n_chunks] marks
  float* o_coarse;          // [B, H, n_tiles, 128]
  int32_t* idx;             // [B, H, n_tiles, kmax]
  int32_t* cnt;
  int32_t kmax;
  int* err;                 // status word, failed-call count
  uint64_t stall_ns;        // > 0: the MMA warp first waits this long on a barrier nothing arrives on
};

struct SelSmem {
  uint8_t k[kKStages][kChunkBytes];
  uint8_t v[kVStages][kChunkBytes];
  // One region, three uses in turn: the staged Qbar rows of the block (start),
  // the row histograms [bin pair][row] (softmax and radix passes: lane r always
  // hits bank r), the boundary members [slot][row] (collect pass).
  union {
    uint8_t q[kRows * kQStride];
    uint32_t hist[kHistPairs * kRows];
    float2 member[kCap * kRows];
  } u;
  float xmx[2][kRows], xmn[2][kRows], xl[2][kRows];   // the two threads of a row exchange their partial results
  int xarg[2][kRows], xcnt[2][kRows];
  uint64_t k_full[kKStages], k_free[kKStages], v_full[kVStages], v_free[kVStages];
  uint64_t s_full[kSBufs], s_free[kSBufs], p_full[kSBufs], pv_done[kSBufs];
  uint64_t o_full, q_full, q_ready, decide, drain, never;
  uint32_t tmem_base;
  int abort;
  int more;                              // top-k: the fallback passes run
  double red[2][kRowWarps];
};

__device__ __forceinline__ void record_error(int* err, int status) {
  if (atomicExch(err, status) == 0) atomicAdd(err + 1, 1);
}

__device__ __forceinline__ void raise_abort(SelSmem& sm, int* err) {
  record_error(err, VSA_ERR_TIMEOUT);
  *reinterpret_cast<volatile int*>(&sm.abort) = 1;
}

__device__ __forceinline__ bool aborted(const SelSmem& sm) {
  return *reinterpret_cast<const volatile int*>(&sm.abort) != 0;
}

// Lane 0 waits; the warp leaves together.
__device__ __forceinline__ bool warp_wait(SelSmem& sm, uint64_t& bar, uint32_t parity, int lane, int* err) {
  int ok = 1;
  if (lane == 0) {
    ok = mbar_wait(smem_u32(&bar), parity, &sm.abort, kTimeoutNs) ? 1 : 0;
    if (!ok) raise_abort(sm, err);
  }
  ok = __shfl_sync(0xffffffffu, ok, 0);
  __syncwarp();
  return ok != 0;
}

// Named barriers of the eight row warps (ids 1 and 2; 256 threads).
__device__ __forceinline__ int rows_any(int pred) {
  int r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.s32 p, %1, 0;\n\tbar.red.or.pred q, 1, 256, p;\n\t"
      "selp.s32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(pred)
      : "memory");
  return r;
}

__device__ __forceinline__ void rows_sync() { asm volatile("bar.sync 2, 256;" ::: "memory"); }

__device__ __forceinline__ uint32_t ordered_key(float f) {
  const uint32_t u = __float_as_uint(f + 0.0f);   // -0 -> +0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// hi = bf16(x) pair and lo = bf16(x - hi) pair of (x0, x1), element 0 in the low half.
__device__ __forceinline__ void split_pair(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  hi = pack_bf16x2(x0, x1);
  lo = pack_bf16x2(x0 - __uint_as_float(hi << 16), x1 - __uint_as_float(hi & 0xFFFF0000u));
}

// Row histograms: two 16-bit counters per word (bin 2i in the low half), so
// that the two threads of a row add with shared-memory atomics (no return
// value: nothing waits on them); counts stay below 65536.
// h points at the row's first word; its words are kRows apart.
__device__ __forceinline__ void hist_add(uint32_t* h, uint32_t bin) {
  atomicAdd(h + (bin >> 1) * kRows, 1u << ((bin & 1u) << 4));
}
__device__ __forceinline__ int hist_count(const uint32_t* h, int bin) {
  return static_cast<int>((h[(bin >> 1) * kRows] >> ((bin & 1) << 4)) & 0xFFFFu);
}

__device__ __forceinline__ void tmem_st32x16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

// Histogram bin of a score: a monotone non-decreasing function of s.
__device__ __forceinline__ int score_bin(float s, float inv_w, float off) {
  const float t = fmaf(s, inv_w, off);
  return static_cast<int>(fminf(fmaxf(t, 0.f), static_cast<float>(kBins - 1)));
}

template <int kMode>
__global__ void __launch_bounds__(kThreads, 1) select_tc_kernel(const __grid_constant__ SelArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if (smem_u32(smem_raw) & 1023u) {          // swizzled chunks need 1024-byte alignment
    if (threadIdx.x == 0) record_error(a.err, VSA_ERR_UNSUPPORTED);
    return;
  }
  SelSmem& sm = *reinterpret_cast<SelSmem*>(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const size_t bh = static_cast<size_t>(blockIdx.z) * a.H + blockIdx.y;
  const int n_chunks = a.n_chunks;
  // The CTAs of a head start their passes at different chunks (the fallback
  // passes, which count equal keys in candidate order, do not rotate).
  const int rot = static_cast<int>((static_cast<long long>(blockIdx.x) * n_chunks) / gridDim.x);
  auto chunk_at = [&](int kind, int i) { return kind >= kPassRadix ? i : (i + rot) % n_chunks; };
  constexpr int kBasePasses = kMode == kModeTopk ? 3 : 1;
  constexpr int kSoftPass = kMode == kModeTopk ? 1 : (kMode == kModeThresh ? 0 : -1);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kKStages; ++s) {
      mbar_init(smem_u32(&sm.k_full[s]), 1);
      mbar_init(smem_u32(&sm.k_free[s]), 1);
    }
    for (int s = 0; s < kVStages; ++s) {
      mbar_init(smem_u32(&sm.v_full[s]), 1);
      mbar_init(smem_u32(&sm.v_free[s]), 1);
    }
    for (int b = 0; b < kSBufs; ++b) {
      mbar_init(smem_u32(&sm.s_full[b]), 1);
      mbar_init(smem_u32(&sm.s_free[b]), kRowWarps);   // one arrival per row warp
      mbar_init(smem_u32(&sm.p_full[b]), kRowWarps);
      mbar_init(smem_u32(&sm.pv_done[b]), 1);
    }
    mbar_init(smem_u32(&sm.o_full), 1);
    mbar_init(smem_u32(&sm.q_full), 1);
    mbar_init(smem_u32(&sm.q_ready), kRowWarps);
    mbar_init(smem_u32(&sm.decide), 1);
    mbar_init(smem_u32(&sm.drain), 1);
    mbar_init(smem_u32(&sm.never), 1);
    sm.abort = 0;
    sm.more = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&sm.tmem_base), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  if (warp == 0) {
    // ----------------------------------------------------------- copies
    // Qbar rows of the block (512 bytes each) at a padded stride
    const int n_rows = min(kRows, a.n_tiles - static_cast<int>(blockIdx.x) * kRows);
    if (lane == 0) mbar_arrive_expect_tx(smem_u32(&sm.q_full), static_cast<uint32_t>(n_rows) * 512u);
    __syncwarp();
    for (int i = lane; i < n_rows; i += 32)
      bulk_load(smem_u32(sm.u.q + i * kQStride), a.qbar + (bh * a.n_tiles + blockIdx.x * kRows + i) * kHeadDim, 512,
                smem_u32(&sm.q_full));
    __syncwarp();
    if (lane == 0) {
      const uint8_t* kb = a.ksplit + bh * n_chunks * kChunkBytes;
      const uint8_t* vb = a.vsplit + bh * n_chunks * kChunkBytes;
      uint32_t gk = 0, gv = 0;
      bool ok = true;
      int n_passes = kBasePasses;
      for (int p = 0; ok && p < n_passes; ++p) {
        const int kind = pass_kind<kMode>(p);
        const bool soft = kind == kPassSoftmax;
        for (int i = 0; i < n_chunks; ++i) {
          const int c = chunk_at(kind, i);
          const uint32_t st = gk % kKStages;
          if (gk >= kKStages &&
              !(ok = mbar_wait(smem_u32(&sm.k_free[st]), ((gk / kKStages) - 1) & 1, &sm.abort, kTimeoutNs)))
            break;
          mbar_arrive_expect_tx(smem_u32(&sm.k_full[st]), kChunkBytes);
          bulk_load(smem_u32(sm.k[st]), kb + static_cast<size_t>(c) * kChunkBytes, kChunkBytes,
                    smem_u32(&sm.k_full[st]));
          ++gk;
          if (soft) {
            const uint32_t sv = gv % kVStages;
            if (gv >= kVStages &&
                !(ok = mbar_wait(smem_u32(&sm.v_free[sv]), ((gv / kVStages) - 1) & 1, &sm.abort, kTimeoutNs)))
              break;
            mbar_arrive_expect_tx(smem_u32(&sm.v_full[sv]), kChunkBytes);
            bulk_load(smem_u32(sm.v[sv]), vb + static_cast<size_t>(c) * kChunkBytes, kChunkBytes,
                      smem_u32(&sm.v_full[sv]));
            ++gv;
          }
        }
        if (kMode == kModeTopk && p == 2 && ok) {
          if (!(ok = mbar_wait(smem_u32(&sm.decide), 0, &sm.abort, kTimeoutNs))) break;
          if (*reinterpret_cast<volatile int*>(&sm.more)) n_passes = kBasePasses + kFallbackPasses;
        }
      }
      if (!ok) {
        raise_abort(sm, a.err);
        mbar_wait(smem_u32(&sm.q_full), 0, nullptr, kDrainNs);
        for (uint32_t i = (gk > kKStages ? gk - kKStages : 0u); i < gk; ++i)
          mbar_wait(smem_u32(&sm.k_full[i % kKStages]), (i / kKStages) & 1, nullptr, kDrainNs);
        for (uint32_t i = (gv > kVStages ? gv - kVStages : 0u); i < gv; ++i)
          mbar_wait(smem_u32(&sm.v_full[i % kVStages]), (i / kVStages) & 1, nullptr, kDrainNs);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMAs
    // Issues the next score chunk S(ns) when its Kbar chunk has landed and its
    // TMEM buffer is free (its previous chunk was read out, or in the softmax
    // pass consumed by P V), and the next O += P V when P and Vbar are ready.
    if (lane == 0) {
      bool ok = true;
      if (a.stall_ns) ok = mbar_wait(smem_u32(&sm.never), 0, &sm.abort, a.stall_ns);   // injected failure
      if (ok) ok = mbar_wait(smem_u32(&sm.q_ready), 0, &sm.abort, kTimeoutNs);
      const uint32_t soft0 = kSoftPass >= 0 ? static_cast<uint32_t>(kSoftPass * n_chunks) : 0u;
      const uint32_t n_pv = kSoftPass >= 0 ? static_cast<uint32_t>(n_chunks) : 0u;
      uint32_t total = static_cast<uint32_t>(kBasePasses * n_chunks);
      bool decided = kMode != kModeTopk;
      uint32_t ns = 0, np = 0, ph_sf = 0, ph_pv = 0, ph_pf = 0, spins = 0;
      uint64_t t0 = 0;
      while (ok) {
        bool progress = false;
        if (ns < total) {
          const uint32_t st = ns % kKStages, b = ns % kSBufs;
          bool ready = mbar_test_wait(smem_u32(&sm.k_full[st]), (ns / kKStages) & 1) != 0;
          bool prev_soft = false;
          if (ready && ns >= kSBufs) {
            const uint32_t prev = ns - kSBufs;
            prev_soft = kSoftPass >= 0 && prev - soft0 < n_pv;   // unsigned: false below soft0
            ready = prev_soft ? mbar_test_wait(smem_u32(&sm.pv_done[b]), (ph_pv >> b) & 1) != 0
                              : mbar_test_wait(smem_u32(&sm.s_free[b]), (ph_sf >> b) & 1) != 0;
            if (ready) {
              if (prev_soft) ph_pv ^= 1u << b;
              else ph_sf ^= 1u << b;
            }
          }
          if (ready) {
            tc_fence_after();
            const uint64_t kh = smem_desc_sw128(smem_u32(sm.k[st]), 16, 1024);
            const uint64_t kl = smem_desc_sw128(smem_u32(sm.k[st] + kTermBytes), 16, 1024);
            const uint32_t d = tmem + kColS + 64u * b;
            // K steps of 16 dims: 8 columns of the A operand, 32 bytes inside a
            // 64-dim half of the chunk, the second half 8 KB on
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              umma_ts(d, tmem + kColQ + kk * 8, kh + (kk >> 2) * (8192 >> 4) + (kk & 3) * 2, kIdescS, kk ? 1u : 0u);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              umma_ts(d, tmem + kColQ + kk * 8, kl + (kk >> 2) * (8192 >> 4) + (kk & 3) * 2, kIdescS, 1u);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              umma_ts(d, tmem + kColQ + 64 + kk * 8, kh + (kk >> 2) * (8192 >> 4) + (kk & 3) * 2, kIdescS, 1u);
            umma_commit(smem_u32(&sm.s_full[b]));
            umma_commit(smem_u32(&sm.k_free[st]));
            ++ns;
            progress = true;
          }
        }
        if constexpr (kSoftPass >= 0) {
          if (np < n_pv && soft0 + np < ns) {
            const uint32_t b = (soft0 + np) % kSBufs, sv = np % kVStages;
            if (mbar_test_wait(smem_u32(&sm.p_full[b]), (ph_pf >> b) & 1) &&
                mbar_test_wait(smem_u32(&sm.v_full[sv]), (np / kVStages) & 1)) {
              ph_pf ^= 1u << b;
              tc_fence_after();
              // Vbar as MN-major B: 64-dim blocks 8 KB apart, 16 candidates = 2 KB
              // per K step. P (A) over its scores: candidates 32 h .. + 31 as hi
              // pairs at columns 32 h .. + 15 and lo pairs at 32 h + 16 .. + 31;
              // K step kk (16 candidates, 8 columns) of hi starts at column
              // 32 (kk >> 1) + 8 (kk & 1), of lo 16 columns later
              const uint64_t vh = smem_desc_sw128(smem_u32(sm.v[sv]), 8192, 1024);
              const uint64_t vl = smem_desc_sw128(smem_u32(sm.v[sv] + kTermBytes), 8192, 1024);
              const uint32_t pa = tmem + kColS + 64u * b;
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                umma_ts(tmem + kColO, pa + 32 * (kk >> 1) + 8 * (kk & 1), vh + kk * (2048 >> 4), kIdescPV,
                        (np == 0 && kk == 0) ? 0u : 1u);
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                umma_ts(tmem + kColO, pa + 32 * (kk >> 1) + 8 * (kk & 1), vl + kk * (2048 >> 4), kIdescPV, 1u);
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                umma_ts(tmem + kColO, pa + 32 * (kk >> 1) + 16 + 8 * (kk & 1), vh + kk * (2048 >> 4), kIdescPV, 1u);
              umma_commit(smem_u32(&sm.pv_done[b]));
              umma_commit(smem_u32(&sm.v_free[sv]));
              if (np + 1 == n_pv) umma_commit(smem_u32(&sm.o_full));
              ++np;
              progress = true;
            }
          }
        }
        if (ns == total && np == n_pv) {
          if (decided) break;
          if (mbar_test_wait(smem_u32(&sm.decide), 0)) {
            decided = true;
            if (*reinterpret_cast<volatile int*>(&sm.more)) total += static_cast<uint32_t>(kFallbackPasses * n_chunks);
            progress = true;
          }
        }
        if (progress) {
          spins = 0;
          t0 = 0;
        } else if (++spins > 4) {
          __nanosleep(32);   // nothing ready: leave the issue slots to the row warps sharing this sub-partition
        }
        if (!progress && (spins & 255u) == 0) {
          if (aborted(sm)) {
            ok = false;
          } else {
            const uint64_t now = globaltimer_ns();
            if (t0 == 0) t0 = now;
            else if (now - t0 > kTimeoutNs) ok = false;
          }
        }
      }
      if (!ok) raise_abort(sm, a.err);
      umma_commit(smem_u32(&sm.drain));
      mbar_wait(smem_u32(&sm.drain), 0, nullptr, kDrainNs);
    }
    __syncwarp();
  } else {
    // ------------------------------------------ two threads per query tile
    // Warp 2 + 4 half + i covers TMEM lane quadrant (2 + i) % 4 and candidates
    // 32 half .. 32 half + 31 of every chunk.
    const int quad = warp & 3;
    const int half = (warp - 2) >> 2;
    const int r = quad * 32 + lane;
    const int qt = blockIdx.x * kRows + r;
    const bool row_ok = qt < a.n_tiles;
    const size_t row = bh * a.n_tiles + (row_ok ? qt : 0);
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    const int n_words = 2 * n_chunks;
    uint32_t* bits_row = a.bits + row * n_words;
    uint32_t* hist = sm.u.hist + r;
    float2* member = sm.u.member;   // collect pass: (score, ordinal) of slot e of row r at e * 128 + r
    const int et = threadIdx.x - 64;   // 0 .. 255 over the row warps

    bool ok = true;
    // Qbar dims 64 half .. + 63 of this query tile, split hi / lo, as the A
    // operand (rows past the end are zero: their scores are 0 and nothing of
    // theirs is written)
    {
      ok = warp_wait(sm, sm.q_full, 0, lane, a.err);
      const float4* src = reinterpret_cast<const float4*>(sm.u.q + r * kQStride + 256 * half);
      uint32_t wh[32], wl[32];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float4 x = row_ok ? src[i] : make_float4(0.f, 0.f, 0.f, 0.f);
        split_pair(x.x, x.y, wh[2 * i], wl[2 * i]);
        split_pair(x.z, x.w, wh[2 * i + 1], wl[2 * i + 1]);
      }
      tmem_st32x32(lane_addr + kColQ + 32 * half, wh);
      tmem_st32x32(lane_addr + kColQ + 64 + 32 * half, wl);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&sm.q_ready));
    }

    uint32_t gs = 0;
    float mx = -INFINITY, mn = INFINITY, lq[4] = {0.f, 0.f, 0.f, 0.f};
    int arg = 0;
    double s1 = 0.0, s2 = 0.0, s1b = 0.0, s2b = 0.0, thr = 0.0;
    float inv_w = 0.f, off = 0.f;
    int bstar = 0, krem = 0, nmem = 0, eq_seen = 0, n_loc = 0;
    bool fb = false;
    uint32_t prefix = 0, pmask = 0;

    if (kMode == kModeThresh) {
      mx = row_ok ? a.rowmax[row] : 0.f;
      arg = row_ok ? a.rowarg[row] : 0;
      double sa = 0.0, sb = 0.0;
      for (int i = 0; i < a.n_qblocks; ++i) {
        sa += a.stats[(bh * a.n_qblocks + i) * 2 + 0];
        sb += a.stats[(bh * a.n_qblocks + i) * 2 + 1];
      }
      const double nn = static_cast<double>(a.n_tiles) * static_cast<double>(a.n_cand);
      const double mean = sa / nn;
      const double var = fmax(sb / nn - mean * mean, 0.0);
      thr = mean + static_cast<double>(a.tau) * sqrt(var);
    }

    int n_passes = kBasePasses;
    for (int p = 0; p < n_passes; ++p) {
      const int kind = pass_kind<kMode>(p);
      const int shift = 24 - 8 * (p - 3);   // radix passes 3..6
      // the fallback passes are rare: the first thread of a row takes all 64 candidates of each chunk
      const bool solo = kind == kPassRadix || kind == kPassEmit;
      if ((kMode == kModeTopk && kind == kPassSoftmax) || kind == kPassRadix) {
        // every thread is done with the region (the previous pass's counts and scans, the staged Qbar)
        rows_sync();
        uint4* h4 = reinterpret_cast<uint4*>(sm.u.hist);
        for (int i = et; i < kHistPairs * kRows / 4; i += 32 * kRowWarps) h4[i] = make_uint4(0u, 0u, 0u, 0u);
        rows_sync();
      }
      for (int ci = 0; ci < n_chunks; ++ci, ++gs) {
        const int c = chunk_at(kind, ci);
        const uint32_t b = gs % kSBufs;
        if (ok) ok = warp_wait(sm, sm.s_full[b], (gs / kSBufs) & 1, lane, a.err);
        if (!ok) continue;
        tc_fence_after();
        const uint32_t sbuf = lane_addr + kColS + 64u * b;
        if (solo) {
          float x[64];
          if (half == 0) {
            float x0[32], x1[32];
            tmem_ld32x32f(sbuf, x0);
            tmem_ld32x32f(sbuf + 32, x1);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              x[j] = x0[j];
              x[32 + j] = x1[j];
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(&sm.s_free[b]));
          if (half == 0 && fb) {
            const int n_valid = min(kChunk, a.n_cand - c * kChunk);
            uint32_t w0 = 0, w1 = 0;
#pragma unroll
            for (int j = 0; j < 64; ++j) {
              const float s = x[j] * a.scale;
              if (j < n_valid && score_bin(s, inv_w, off) == bstar) {
                const uint32_t key = ordered_key(s);
                if (kind == kPassRadix) {
                  if ((key & pmask) == prefix) hist_add(hist, (key >> shift) & 255u);
                } else if (key > prefix || (key == prefix && eq_seen < krem)) {
                  if (key == prefix) ++eq_seen;
                  if (j < 32) w0 |= 1u << j;
                  else w1 |= 1u << (j - 32);
                }
              }
            }
            if (kind == kPassEmit && row_ok && (w0 | w1)) {
              uint2* wp = reinterpret_cast<uint2*>(bits_row + 2 * c);
              const uint2 cur = *wp;
              *wp = make_uint2(cur.x | w0, cur.y | w1);
            }
          }
          continue;
        }
        float x[32];
        tmem_ld32x32f(sbuf + 32 * half, x);
        tmem_wait_ld();
        if (kind != kPassSoftmax) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(&sm.s_free[b]));
        }
        const int o0 = c * kChunk + 32 * half;   // candidate of x[0]
        const int n_valid = a.n_cand - o0;        // x[j] is a candidate for j < n_valid
        uint32_t word = 0;                        // marks of candidates o0 .. o0 + 31
        // The per-score work avoids long serial chains (tree reductions,
        // bit masks, several accumulators): two row warps per scheduler hide
        // little latency.
        if (kind == kPassRange) {
          float hv[32], lv[32];
          int hi_[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const float s = x[j] * a.scale;
            const bool v = j < n_valid;
            hv[j] = v ? s : -INFINITY;
            lv[j] = v ? s : INFINITY;
            hi_[j] = j;
            if (kMode == kModeStats) {
              const double sd = v ? static_cast<double>(s) : 0.0;
              if (j & 1) {
                s2 = fma(sd, sd, s2);
                s1 += sd;
              } else {
                s2b = fma(sd, sd, s2b);
                s1b += sd;
              }
            }
          }
          // maximum with the lowest index among equal maxima, and minimum, as trees
#pragma unroll
          for (int w = 16; w >= 1; w >>= 1) {
#pragma unroll
            for (int j = 0; j < w; ++j) {
              const bool tb = hv[j + w] > hv[j];      // the upper half wins only when strictly larger
              hv[j] = tb ? hv[j + w] : hv[j];
              hi_[j] = tb ? hi_[j + w] : hi_[j];
              lv[j] = fminf(lv[j], lv[j + w]);
            }
          }
          // the first maximal candidate in any visiting order
          const bool better = hv[0] > mx || (hv[0] == mx && o0 + hi_[0] < arg);
          mx = better ? hv[0] : mx;
          arg = better ? o0 + hi_[0] : arg;
          mn = fminf(mn, lv[0]);
        } else if (kind == kPassSoftmax) {
          uint32_t wh[16], wl[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float sa = x[2 * i] * a.scale, sb = x[2 * i + 1] * a.scale;
            const bool va = 2 * i < n_valid, vb = 2 * i + 1 < n_valid;
            const float pa = va ? ex2_approx((sa - mx) * kLog2e) : 0.f;
            const float pb = vb ? ex2_approx((sb - mx) * kLog2e) : 0.f;
            lq[i & 3] += pa + pb;
            split_pair(pa, pb, wh[i], wl[i]);
            if (kMode == kModeTopk) {
              hist_add(hist, va ? score_bin(sa, inv_w, off) : kBins);
              hist_add(hist, vb ? score_bin(sb, inv_w, off) : kBins);
            } else {
              word |= (va && static_cast<double>(sa) >= thr ? 1u : 0u) << (2 * i);
              word |= (vb && static_cast<double>(sb) >= thr ? 1u : 0u) << (2 * i + 1);
            }
          }
          // P of candidates 32 half .. + 31 over this thread's own score columns 32 half .. + 31
          // (the other warp of the row may still be reading its half): hi pairs first, then lo pairs
          tmem_st32x16(sbuf + 32 * half, wh);
          tmem_st32x16(sbuf + 32 * half + 16, wl);
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(&sm.p_full[b]));
          if (kMode == kModeThresh && row_ok) bits_row[2 * c + half] = word;
        } else {   // collect
          uint32_t memb = 0;
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const float s = x[j] * a.scale;
            const bool v = j < n_valid;
            const int bn = score_bin(s, inv_w, off);
            word |= (v && bn > bstar ? 1u : 0u) << j;
            memb |= (v && bn == bstar ? 1u : 0u) << j;
          }
          // boundary members (a handful per row over the whole pass)
          if (!fb) {
            while (memb) {
              const int j = __ffs(memb) - 1;
              memb &= memb - 1;
              float xj = 0.f;
#pragma unroll
              for (int u = 0; u < 32; ++u) xj = (u == j) ? x[u] : xj;
              if (n_loc < kHalfCap)
                member[(kHalfCap * half + n_loc) * kRows + r] = make_float2(xj * a.scale, __int_as_float(o0 + j));
              ++n_loc;
            }
          }
          if (row_ok) bits_row[2 * c + half] = word;
        }
      }

      // ---- end of a pass
      if (kind == kPassRange) {
        if (kMode != kModeThresh) {
          // the row's maximum (first maximal candidate) and minimum from its two threads
          sm.xmx[half][r] = mx;
          sm.xarg[half][r] = arg;
          sm.xmn[half][r] = mn;
          rows_sync();
          const float m0 = sm.xmx[0][r], m1 = sm.xmx[1][r];
          const int a0 = sm.xarg[0][r], a1 = sm.xarg[1][r];
          mx = m0;
          arg = a0;
          if (m1 > m0 || (m1 == m0 && a1 < a0)) {
            mx = m1;
            arg = a1;
          }
          mn = fminf(sm.xmn[0][r], sm.xmn[1][r]);
        }
        if (kMode == kModeTopk) {
          // histogram bins over [min, max]; a zero-width or unrepresentable range puts every score in bin 0
          inv_w = mx > mn ? static_cast<float>(kBins) / (mx - mn) : 0.f;
          if (!(inv_w < INFINITY)) inv_w = 0.f;
          off = -mn * inv_w;
          if (!(fabsf(off) < INFINITY)) inv_w = off = 0.f;
        } else if (kMode == kModeStats) {
          if (ok && row_ok && half == 0) {
            a.rowmax[row] = mx;
            a.rowarg[row] = arg;
          }
          s1 += s1b;
          s2 += s2b;
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) {
            s1 += __shfl_xor_sync(0xffffffffu, s1, o);
            s2 += __shfl_xor_sync(0xffffffffu, s2, o);
          }
          if (lane == 0) {
            sm.red[0][warp - 2] = s1;
            sm.red[1][warp - 2] = s2;
          }
          rows_sync();
          if (warp == 2 && lane == 0 && ok) {
            double t1 = 0.0, t2 = 0.0;
            for (int w = 0; w < kRowWarps; ++w) {
              t1 += sm.red[0][w];
              t2 += sm.red[1][w];
            }
            a.stats[(bh * a.n_qblocks + blockIdx.x) * 2 + 0] = t1;
            a.stats[(bh * a.n_qblocks + blockIdx.x) * 2 + 1] = t2;
          }
        }
      } else if (kind == kPassSoftmax) {
        sm.xl[half][r] = (lq[0] + lq[1]) + (lq[2] + lq[3]);
        rows_sync();                              // also: every histogram count of the pass has landed
        const float l = sm.xl[0][r] + sm.xl[1][r];
        if (ok) ok = warp_wait(sm, sm.o_full, 0, lane, a.err);
        if (ok) {
          tc_fence_after();
          const float inv_l = 1.0f / l;
          float4* dst = reinterpret_cast<float4*>(a.o_coarse + row * kHeadDim + 64 * half);
#pragma unroll 1
          for (int c = 0; c < 2; ++c) {
            float o[32];
            tmem_ld32x32f(lane_addr + kColO + 64 * half + 32 * c, o);
            tmem_wait_ld();
            if (row_ok) {
#pragma unroll
              for (int i = 0; i < 8; ++i)
                dst[8 * c + i] = make_float4(o[4 * i] * inv_l, o[4 * i + 1] * inv_l, o[4 * i + 2] * inv_l,
                                             o[4 * i + 3] * inv_l);
            }
          }
        }
        if (kMode == kModeTopk && row_ok) {
          // the bin of the k-th largest score and how many of its members are taken
          int above = 0;
          for (int bn = kBins - 1; bn >= 0; --bn) {
            const int h = hist_count(hist, bn);
            if (above + h >= a.k) {
              bstar = bn;
              krem = a.k - above;
              nmem = h;
              break;
            }
            above += h;
          }
          fb = nmem > kCap;
        }
        if (kMode == kModeTopk) rows_sync();   // every row's scan is done: the members overlay the histograms
      } else if (kind == kPassCollect) {
        sm.xcnt[half][r] = n_loc;
        rows_sync();                              // members and marks of both threads of every row are in
        const int n0 = sm.xcnt[0][r], n1 = sm.xcnt[1][r];
        if (n0 > kHalfCap || n1 > kHalfCap) fb = true;   // a thread's share overflowed: the exact passes rank the row
        // rank the boundary members (score descending, lower ordinal first); take krem
        if (ok && row_ok && !fb && half == 0) {
          const int n_got = n0 + n1;
          auto slot = [&](int e) { return e < n0 ? e : kHalfCap + (e - n0); };
          for (int e = 0; e < n_got; ++e) {
            const float2 me = member[slot(e) * kRows + r];
            const int oe = __float_as_int(me.y);
            int rank = 0;
            for (int f = 0; f < n_got; ++f) {
              const float2 mf = member[slot(f) * kRows + r];
              const int of = __float_as_int(mf.y);
              rank += (mf.x > me.x || (mf.x == me.x && of < oe)) ? 1 : 0;
            }
            if (rank < krem) bits_row[oe >> 5] |= 1u << (oe & 31);
          }
        }
        const int any = rows_any(row_ok && fb ? 1 : 0);
        if (warp == 2 && lane == 0) {
          sm.more = any;
          mbar_arrive(smem_u32(&sm.decide));
        }
        if (any) n_passes = kBasePasses + kFallbackPasses;
      } else if (kind == kPassRadix && fb && ok && half == 0) {
        int above = 0;
        for (int bn = 255; bn >= 0; --bn) {
          const int h = hist_count(hist, bn);
          if (above + h >= krem) {
            prefix |= static_cast<uint32_t>(bn) << shift;
            pmask |= 0xFFu << shift;
            krem -= above;
            break;
          }
          above += h;
        }
      }
    }

    // ---- marks -> ascending candidate lists, one warp per query tile
    __threadfence();
    rows_sync();
    if (!aborted(sm) && kMode != kModeStats) {
      for (int i = 0; i < 16; ++i) {
        const int rr = quad * 32 + half * 16 + i;
        const int qq = blockIdx.x * kRows + rr;
        if (qq >= a.n_tiles) break;
        const size_t rw = bh * a.n_tiles + qq;
        const uint32_t* br = a.bits + rw * n_words;
        int32_t* out = a.idx + rw * a.kmax;
        int pos = 0;
        for (int w0 = 0; w0 < n_words; w0 += 32) {
          const int w = w0 + lane;
          uint32_t word = w < n_words ? __ldcg(br + w) : 0u;
          const int n = __popc(word);
          int incl = n;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
          }
          int q = pos + incl - n;
          while (word) {
            const int bit = __ffs(word) - 1;
            word &= word - 1;
            if (q < a.kmax) out[q] = 32 * w + bit;
            ++q;
          }
          pos += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) {
          if (kMode == kModeThresh && pos == 0) {   // nothing reaches the threshold: keep the argmax
            out[0] = a.rowarg[rw];
            pos = 1;
          }
          a.cnt[rw] = min(pos, a.kmax);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

size_t select_tc_smem_bytes() { return sizeof(SelSmem); }

vsa_status select_tc(const vsa_layout* L, const vsa_params* p, int32_t B, int32_t H, const SelectWorkspace& ws,
                     void* workspace, int32_t* idx, int32_t* cnt, float* o_coarse, uint64_t stall_ns,
                     cudaStream_t stream) {
  const Candidates cand = candidates(L, p->sink);
  uint8_t* w = static_cast<uint8_t*>(workspace);
  SelArgs a{};
  a.qbar = reinterpret_cast<const float*>(w + ws.pooled);
  a.ksplit = w + ws.ksplit;
  a.vsplit = w + ws.vsplit;
  a.n_tiles = L->n_tiles;
  a.H = H;
  a.n_cand = cand.count;
  a.n_chunks = ws.n_chunks;
  a.n_qblocks = ws.n_row_blocks;
  int32_t kmax = 0;
  vsa_select_kmax(L, p, &kmax);
  a.k = kmax;
  a.kmax = kmax;
  a.scale = effective_scale(p);
  a.tau = p->tau;
  a.rowmax = reinterpret_cast<float*>(w + ws.rowmax);
  a.rowarg = reinterpret_cast<int32_t*>(w + ws.rowarg);
  a.stats = reinterpret_cast<double*>(w + ws.stats);
  a.bits = reinterpret_cast<uint32_t*>(w + ws.bits);
  a.o_coarse = o_coarse;
  a.idx = idx;
  a.cnt = cnt;
  a.err = static_cast<int*>(workspace);
  a.stall_ns = stall_ns;

  const size_t smem = sizeof(SelSmem);
  const dim3 grid(ws.n_row_blocks, H, B);
  auto launch = [&](auto kernel, const char* what) -> vsa_status {
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return cuda_fail(what, e);
    kernel<<<grid, kThreads, smem, stream>>>(a);
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(what, e);
    return VSA_OK;
  };
  if (p->mode == VSA_SELECT_TOPK) return launch(select_tc_kernel<kModeTopk>, "vsa_coarse_select: top-k launch");
  vsa_status st = launch(select_tc_kernel<kModeStats>, "vsa_coarse_select: statistics launch");
  if (st != VSA_OK) return st;
  return launch(select_tc_kernel<kModeThresh>, "vsa_coarse_select: threshold launch");
}

}  // namespace vsa
