// Test harness (not part of libvsa): runs the attention kernel's tcgen05
// building blocks once on small inputs so that tests can compare each against
// a torch matmul:
//   S1 = Q K^T   Q [128 x 128] and K [64 x 128] loaded by the 3-D token map
//   S2 = Q Kc^T  Kc = one 4x4x4 cube gathered by the 5-D video-grid map
//   O  = P V     P [128 x 64] written to 128B-swizzled smem by threads,
//                V [64 x 128] loaded by the 3-D map, used as an MN-major operand
//   O2 = P V     the same product with P written to TMEM by tcgen05.st
//                (row i in lane i, bf16 pairs per column) and read as A from TMEM
// Same descriptors, swizzle and TMEM access pattern as vsa_attn.cu. All waits
// are bounded; a wait that runs out writes 1 to *err.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include "sm100.cuh"

using namespace vsa::sm100;

namespace {

struct __align__(1024) CheckSmem {
  uint8_t q[2][128 * 128];
  uint8_t k[2][64 * 128];
  uint8_t kc[2][64 * 128];
  uint8_t v[2][64 * 128];
  uint8_t p[128 * 128];
  uint64_t bar_load, bar_mma, bar_ts;
  uint32_t tmem_base;
};

constexpr uint64_t kTimeout = 2000000000ull;

__global__ void __launch_bounds__(128, 1)
check_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
             const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tgrid,
             int cube_t0, int cube_h0, int cube_w0, int cube_head, const uint16_t* p_in,
             float* s1_out, float* s2_out, float* o_out, float* o2_out, int* err) {
  extern __shared__ uint8_t raw[];
  CheckSmem& sm = *reinterpret_cast<CheckSmem*>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    mbar_init(smem_u32(&sm.bar_load), 1);
    mbar_init(smem_u32(&sm.bar_mma), 1);
    mbar_init(smem_u32(&sm.bar_ts), 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(&sm.tmem_base), 512);
    tmem_relinquish();
  }
  // P: row r = thread, 64 bf16, written in the 128B-swizzled K-major layout
  {
    const uint4* src = reinterpret_cast<const uint4*>(p_in + tid * 64);
    for (int ch = 0; ch < 8; ++ch)
      *reinterpret_cast<uint4*>(sm.p + tid * 128 + ((ch ^ (tid & 7)) << 4)) = src[ch];
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  bool ok = true;
  if (tid == 0) {
    const uint32_t bar = smem_u32(&sm.bar_load);
    mbar_arrive_expect_tx(bar, 32768 + 16384 * 3);
    tma_load_3d(smem_u32(sm.q[0]), &tq, bar, 0, 0, 0);
    tma_load_3d(smem_u32(sm.q[0] + 8192), &tq, bar, 0, 0, 64);
    tma_load_3d(smem_u32(sm.q[1]), &tq, bar, 64, 0, 0);
    tma_load_3d(smem_u32(sm.q[1] + 8192), &tq, bar, 64, 0, 64);
    tma_load_3d(smem_u32(sm.k[0]), &tk, bar, 0, 0, 0);
    tma_load_3d(smem_u32(sm.k[1]), &tk, bar, 64, 0, 0);
    tma_load_3d(smem_u32(sm.v[0]), &tv, bar, 0, 0, 0);
    tma_load_3d(smem_u32(sm.v[1]), &tv, bar, 64, 0, 0);
    tma_load_5d(smem_u32(sm.kc[0]), &tgrid, bar, 0, cube_head, cube_w0, cube_h0, cube_t0);
    tma_load_5d(smem_u32(sm.kc[1]), &tgrid, bar, 64, cube_head, cube_w0, cube_h0, cube_t0);
    ok = mbar_wait(bar, 0, nullptr, kTimeout);
    if (ok) {
      tc_fence_after();
      const uint32_t idS = idesc_bf16_f32(128, 64, 0, 0);
      const uint32_t idPV = idesc_bf16_f32(128, 128, 0, 1);
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t off = (kk & 3) * 32;
        const uint64_t ad = smem_desc_sw128(smem_u32(sm.q[0]) + (kk >> 2) * 16384 + off, 16, 1024);
        umma_ss(tmem + 128, ad, smem_desc_sw128(smem_u32(sm.k[0]) + (kk >> 2) * 8192 + off, 16, 1024),
                idS, kk > 0);
        umma_ss(tmem + 192, ad, smem_desc_sw128(smem_u32(sm.kc[0]) + (kk >> 2) * 8192 + off, 16, 1024),
                idS, kk > 0);
      }
      for (int kk = 0; kk < 4; ++kk)
        umma_ss(tmem, smem_desc_sw128(smem_u32(sm.p) + kk * 32, 16, 1024),
                smem_desc_sw128(smem_u32(sm.v[0]) + kk * 2048, 8192, 1024), idPV, kk > 0);
      umma_commit(smem_u32(&sm.bar_mma));
      ok = mbar_wait(smem_u32(&sm.bar_mma), 0, nullptr, kTimeout);
    }
    if (!ok) *err = 1;
  }
  __syncthreads();
  ok = *reinterpret_cast<volatile int*>(err) == 0;
  const uint32_t la = tmem + (static_cast<uint32_t>(warp * 32) << 16);
  if (ok) {
    // P into TMEM columns 384..415 of this thread's lane, then O2 = P V from TMEM
    tc_fence_after();
    uint32_t w[32];
    const uint32_t* src = reinterpret_cast<const uint32_t*>(p_in + tid * 64);
    for (int c = 0; c < 32; ++c) w[c] = src[c];
    tmem_st32(la + 384, w);
    tmem_wait_st();
  }
  tc_fence_before();
  __syncthreads();
  if (ok && tid == 0) {
    tc_fence_after();
    const uint32_t idPV = idesc_bf16_f32(128, 128, 0, 1);
    for (int kk = 0; kk < 4; ++kk)
      umma_ts(tmem + 256, tmem + 384 + kk * 8, smem_desc_sw128(smem_u32(sm.v[0]) + kk * 2048, 8192, 1024),
              idPV, kk > 0);
    umma_commit(smem_u32(&sm.bar_ts));
    if (!mbar_wait(smem_u32(&sm.bar_ts), 0, nullptr, kTimeout)) *err = 1;
  }
  __syncthreads();
  ok = *reinterpret_cast<volatile int*>(err) == 0;
  if (ok) {
    tc_fence_after();
    uint32_t u[32];
    for (int ch = 0; ch < 2; ++ch) {
      tmem_ld32(la + 128 + ch * 32, u);
      tmem_wait_ld();
      for (int c = 0; c < 32; ++c) s1_out[tid * 64 + ch * 32 + c] = __uint_as_float(u[c]);
      tmem_ld32(la + 192 + ch * 32, u);
      tmem_wait_ld();
      for (int c = 0; c < 32; ++c) s2_out[tid * 64 + ch * 32 + c] = __uint_as_float(u[c]);
    }
    for (int ch = 0; ch < 4; ++ch) {
      tmem_ld32(la + ch * 32, u);
      tmem_wait_ld();
      for (int c = 0; c < 32; ++c) o_out[tid * 128 + ch * 32 + c] = __uint_as_float(u[c]);
      tmem_ld32(la + 256 + ch * 32, u);
      tmem_wait_ld();
      for (int c = 0; c < 32; ++c) o2_out[tid * 128 + ch * 32 + c] = __uint_as_float(u[c]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

PFN_cuTensorMapEncodeTiled_v12000 encoder() {
  void* p = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess)
    return nullptr;
  return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
}

bool encode(CUtensorMap* m, int rank, const void* base, const cuuint64_t* dims, const cuuint64_t* strides,
            const cuuint32_t* box) {
  auto enc = encoder();
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  return enc && enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), dims, strides, box,
                    estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

// q [128, 128], k [64, 128], v [64, 128], p [128, 64] bf16 row-major;
// grid [T, Hg, W, 2 heads, 128] bf16; outputs fp32 s1 [128, 64], s2 [128, 64], o and o2 [128, 128].
// Returns 0 on success, 1 for a wait that ran out, 2 for a CUDA error.
extern "C" int mma_check_run(const void* q, const void* k, const void* v, const void* p, const void* grid,
                             int T, int Hg, int W, int cube_t0, int cube_h0, int cube_w0, int cube_head,
                             float* s1, float* s2, float* o, float* o2, int* err_dev) {
  CUtensorMap tq, tk, tv, tg;
  const cuuint32_t box3[3] = {64, 1, 64};
  const cuuint64_t dq[3] = {128, 1, 128}, dk[3] = {128, 1, 64};
  const cuuint64_t st3[2] = {256, 256};
  if (!encode(&tq, 3, q, dq, st3, box3) || !encode(&tk, 3, k, dk, st3, box3) || !encode(&tv, 3, v, dk, st3, box3))
    return 2;
  const cuuint64_t dg[5] = {128, 2, static_cast<cuuint64_t>(W), static_cast<cuuint64_t>(Hg), static_cast<cuuint64_t>(T)};
  const cuuint64_t sg[4] = {256, 512, 512ull * W, 512ull * W * Hg};
  const cuuint32_t box5[5] = {64, 1, 4, 4, 4};
  if (!encode(&tg, 5, grid, dg, sg, box5)) return 2;
  const size_t smem = sizeof(CheckSmem) + 1024;
  if (cudaFuncSetAttribute(check_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) !=
      cudaSuccess)
    return 2;
  cudaMemset(err_dev, 0, sizeof(int));
  check_kernel<<<1, 128, smem>>>(tq, tk, tv, tg, cube_t0, cube_h0, cube_w0, cube_head,
                                 static_cast<const uint16_t*>(p), s1, s2, o, o2, err_dev);
  if (cudaDeviceSynchronize() != cudaSuccess) return 2;
  int err = 0;
  cudaMemcpy(&err, err_dev, sizeof(int), cudaMemcpyDeviceToHost);
  return err;
}
