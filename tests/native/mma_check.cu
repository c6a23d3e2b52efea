// Test-only check of the tcgen05 building blocks the attention kernels use, in
// the same forms (one CTA, 4 warps):
//  * bulk copies of 16 KB tile-major operand tiles ([d half][64 rows][128 B],
//    128-byte swizzled) and of a query-tile pair as four 8 KB pieces into the
//    [d half][128 rows][128 B] layout;
//  * S = Q K^T with M = 64 (Q and K from shared memory) into TMEM lane half 0
//    and lane half 1 (address lane field 0 and 16), and with M = 128 on a pair;
//  * P written into TMEM as bf16 pairs with the 16x32bx2 store shape, then
//    O = P V with P as the A operand in TMEM and V MN-major from shared memory,
//    for M = 64 in lane half 1 and for M = 128;
//  * every read-back with the 16x32bx2 load shape.
// Results go to global memory for the host to compare with plain matmuls.
#include <cuda_runtime.h>

#include <cstdint>

#include "sm100.cuh"

using namespace vsa::sm100;

namespace {

constexpr uint32_t kCols = 512;
constexpr uint64_t kWaitNs = 1000000000ull;

struct Smem {
  uint8_t q[16384];
  uint8_t qp[32768];
  uint8_t k[16384];
  uint8_t v[16384];
  uint64_t bar_load, bar_mma;
  uint32_t tmem;
  int fail;
};

// bf16 bits of a row-major [rows, 64] P (keys 32 hf .. + 31 of row r) as 16 pairs
__device__ void load_p_pairs(const uint16_t* p, int r, int hf, uint32_t (&w)[16]) {
  const uint16_t* src = p + r * 64 + 32 * hf;
#pragma unroll
  for (int i = 0; i < 16; ++i) w[i] = static_cast<uint32_t>(src[2 * i]) | (static_cast<uint32_t>(src[2 * i + 1]) << 16);
}

// rows (lanes base .. base + 15 of warp w) x 64 fp32 columns from TMEM, split 32
__device__ void store_rows64(uint32_t taddr, float* out, int row0, int ld) {
  const int lane = threadIdx.x & 31;
  float x[32];
  tmem_ld16x2_32f<32>(taddr, x);
  tmem_wait_ld();
  float* dst = out + (row0 + (lane & 15)) * ld + 32 * (lane >> 4);
  for (int i = 0; i < 32; ++i) dst[i] = x[i];
}

// same rows x 128 fp32 columns, split 64 (two loads of 32)
__device__ void store_rows128(uint32_t taddr, float* out, int row0) {
  const int lane = threadIdx.x & 31;
  for (int ch = 0; ch < 2; ++ch) {
    float x[32];
    tmem_ld16x2_32f<64>(taddr + 32 * ch, x);
    tmem_wait_ld();
    float* dst = out + (row0 + (lane & 15)) * 128 + 64 * (lane >> 4) + 32 * ch;
    for (int i = 0; i < 32; ++i) dst[i] = x[i];
  }
}

__global__ void __launch_bounds__(128, 1)
mma_check_kernel(const uint8_t* q, const uint8_t* qa, const uint8_t* qb, const uint8_t* k, const uint8_t* v,
                 const uint16_t* p64, const uint16_t* p128, float* s64_0, float* s64_1, float* s128, float* o64,
                 float* o128, int* err) {
  extern __shared__ __align__(1024) uint8_t raw[];
  if (smem_u32(raw) & 1023u) {
    if (threadIdx.x == 0) *err = 99;
    return;
  }
  Smem& sm = *reinterpret_cast<Smem*>(raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&sm.bar_load), 1);
    mbar_init(smem_u32(&sm.bar_mma), 1);
    sm.fail = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(&sm.tmem), kCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = sm.tmem;

  if (threadIdx.x == 0) {
    const uint32_t bar = smem_u32(&sm.bar_load);
    mbar_arrive_expect_tx(bar, 16384u * 5);
    bulk_load(smem_u32(sm.q), q, 16384, bar);
    bulk_load(smem_u32(sm.qp), qa, 8192, bar);
    bulk_load(smem_u32(sm.qp) + 8192, qb, 8192, bar);
    bulk_load(smem_u32(sm.qp) + 16384, qa + 8192, 8192, bar);
    bulk_load(smem_u32(sm.qp) + 24576, qb + 8192, 8192, bar);
    bulk_load(smem_u32(sm.k), k, 16384, bar);
    bulk_load(smem_u32(sm.v), v, 16384, bar);
    if (!mbar_wait(bar, 0, nullptr, kWaitNs)) sm.fail = 1;
    tc_fence_after();
    if (!sm.fail) {
      const uint64_t qd = smem_desc_sw128(smem_u32(sm.q), 16, 1024);
      const uint64_t pd = smem_desc_sw128(smem_u32(sm.qp), 16, 1024);
      const uint64_t kd = smem_desc_sw128(smem_u32(sm.k), 16, 1024);
      for (int kk = 0; kk < 8; ++kk) {
        const uint64_t ko = (kk >> 2) * (8192 >> 4) + (kk & 3) * 2;
        umma_ss(tm + 0, qd + ko, kd + ko, idesc_bf16_f32(64, 64, 0, 0), kk > 0);                     // half 0, cols 0-63
        umma_ss(tm + (16u << 16) + 64, qd + ko, kd + ko, idesc_bf16_f32(64, 64, 0, 0), kk > 0);      // half 1, cols 64-127
        umma_ss(tm + 128, pd + (kk >> 2) * (16384 >> 4) + (kk & 3) * 2, kd + ko, idesc_bf16_f32(128, 64, 0, 0),
                kk > 0);                                                                                // M = 128, cols 128-191
      }
      umma_commit(smem_u32(&sm.bar_mma));
      if (!mbar_wait(smem_u32(&sm.bar_mma), 0, nullptr, kWaitNs)) sm.fail = 2;
    }
  }
  __syncthreads();
  tc_fence_after();
  if (sm.fail) {
    if (threadIdx.x == 0) *err = sm.fail;
  } else {
    const uint32_t q0 = tm + (static_cast<uint32_t>(warp * 32) << 16);
    store_rows64(q0 + 0, s64_0, 16 * warp, 64);                        // M = 64: rows 16 w .. in lanes 32 w ..
    store_rows64(q0 + (16u << 16) + 64, s64_1, 16 * warp, 64);
    store_rows64(q0 + 128, s128, 32 * warp, 64);                       // M = 128: row r in lane r
    store_rows64(q0 + (16u << 16) + 128, s128, 32 * warp + 16, 64);
    // P into TMEM: M = 64 in lane half 1 at columns 256-287, M = 128 at 320-351
    uint32_t w[16];
    load_p_pairs(p64, 16 * warp + (lane & 15), lane >> 4, w);
    tmem_st16x2_16<16>(q0 + (16u << 16) + 256, w);
    load_p_pairs(p128, 32 * warp + (lane & 15), lane >> 4, w);
    tmem_st16x2_16<16>(q0 + 320, w);
    load_p_pairs(p128, 32 * warp + 16 + (lane & 15), lane >> 4, w);
    tmem_st16x2_16<16>(q0 + (16u << 16) + 320, w);
    tmem_wait_st();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (threadIdx.x == 0 && !sm.fail) {
    const uint64_t vd = smem_desc_sw128(smem_u32(sm.v), 8192, 1024);
    for (int kk = 0; kk < 4; ++kk) {
      umma_ts(tm + (16u << 16) + 384, tm + (16u << 16) + 256 + kk * 8, vd + kk * (2048 >> 4),
              idesc_bf16_f32(64, 128, 0, 1), kk > 0);                                   // O64, lane half 1, cols 384-511
      umma_ts(tm + 0, tm + 320 + kk * 8, vd + kk * (2048 >> 4), idesc_bf16_f32(128, 128, 0, 1), kk > 0);   // O128, cols 0-127
    }
    umma_commit(smem_u32(&sm.bar_mma));
    if (!mbar_wait(smem_u32(&sm.bar_mma), 1, nullptr, kWaitNs)) sm.fail = 3;
  }
  __syncthreads();
  tc_fence_after();
  if (sm.fail) {
    if (threadIdx.x == 0) *err = sm.fail;
  } else {
    const uint32_t q0 = tm + (static_cast<uint32_t>(warp * 32) << 16);
    store_rows128(q0 + (16u << 16) + 384, o64, 16 * warp);
    store_rows128(q0 + 0, o128, 32 * warp);
    store_rows128(q0 + (16u << 16) + 0, o128, 32 * warp + 16);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tm, kCols);
  }
}

}  // namespace

extern "C" int mma_check_run(const void* q, const void* qa, const void* qb, const void* k, const void* v,
                             const void* p64, const void* p128, float* s64_0, float* s64_1, float* s128, float* o64,
                             float* o128, int* err) {
  const int smem = static_cast<int>(sizeof(Smem));
  if (cudaFuncSetAttribute(mma_check_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return 1;
  mma_check_kernel<<<1, 128, smem>>>(static_cast<const uint8_t*>(q), static_cast<const uint8_t*>(qa),
                                     static_cast<const uint8_t*>(qb), static_cast<const uint8_t*>(k),
                                     static_cast<const uint8_t*>(v), static_cast<const uint16_t*>(p64),
                                     static_cast<const uint16_t*>(p128), s64_0, s64_1, s128, o64, o128, err);
  if (cudaGetLastError() != cudaSuccess) return 2;
  if (cudaDeviceSynchronize() != cudaSuccess) return 3;
  return 0;
}
