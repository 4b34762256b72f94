// selftest.cu -- checks of the two tcgen05 operand forms the prefill kernel uses,
// on single tiles whose products the tests recompute on the host:
//   mode 0: D[128x128] = A[128x128] * B[128x128]^T, A and B K-major in shared memory
//           (two 64-column swizzled chunks each), as for S = Q K^T.
//   mode 1: D[128x64] = P[128x128] * V[128x64], P written to tensor memory as bf16
//           pairs by tcgen05.st, V MN-major in shared memory, as for O += P V.
//   mode 2: D[128x128] = P[128x128] * V[128x128], V as two 64-column MN-major chunks
//           16 KB apart (the descriptor's leading byte offset), as for a 128-column
//           share of an N = 256 paired PV product.
#include "common.cuh"
#include "kernels.h"

namespace gattn {

__global__ void __launch_bounds__(128, 1)
umma_selftest_kernel(const __grid_constant__ CUtensorMap a_map, const __grid_constant__ CUtensorMap b_map,
                     const uint16_t* p_global, float* d_out, int mode) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* a_s = smem;              // 2 x 16 KB
  uint8_t* b_s = smem + 32768;      // 2 x 16 KB
  __shared__ __align__(8) uint64_t bar_load, bar_mma, bar_p;
  __shared__ uint32_t tmem_base;
  __shared__ int abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(&bar_load, 1);
    mbar_init(&bar_mma, 1);
    mbar_init(&bar_p, 128);
    abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0) { tmem_alloc(&tmem_base, 256); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base;
  const uint32_t lane_off = (uint32_t)(warp * 32) << 16;

  if (threadIdx.x == 0) {
    if (mode == 0) {
      mbar_arrive_expect_tx(&bar_load, 65536);
      for (int c = 0; c < 2; ++c) {
        tma_load_3d(a_s + c * 16384, &a_map, &bar_load, c * 64, 0, 0);
        tma_load_3d(b_s + c * 16384, &b_map, &bar_load, c * 64, 0, 0);
      }
    } else {
      const int nchunks = mode == 1 ? 1 : 2;
      mbar_arrive_expect_tx(&bar_load, 16384u * nchunks);
      for (int c = 0; c < nchunks; ++c) tma_load_3d(b_s + c * 16384, &b_map, &bar_load, c * 64, 0, 0);
    }
  }
  if (mode != 0) {
    // row `threadIdx.x` of P into TMEM columns [128, 192) as bf16 pairs
    const int row = warp * 32 + lane;
    uint32_t pk[64];
    for (int c = 0; c < 64; ++c)
      pk[c] = (uint32_t)p_global[row * 128 + 2 * c] | ((uint32_t)p_global[row * 128 + 2 * c + 1] << 16);
    tmem_st_x32(tmem + lane_off + 128, pk);
    tmem_st_x32(tmem + lane_off + 160, pk + 32);
    tmem_st_wait();
    tc_fence_before();
    mbar_arrive(&bar_p);
  }
  if (threadIdx.x == 0) {
    volatile int* ab = &abort_flag;
    bool ok = mbar_wait(&bar_load, 0, ab);
    if (ok && mode != 0) ok = mbar_wait(&bar_p, 0, ab);
    tc_fence_after();
    if (ok) {
      if (mode == 0) {
        const uint32_t idesc = umma_idesc_bf16(128, 128, 0, 0);
        for (int c = 0; c < 2; ++c)
          for (int kk = 0; kk < 4; ++kk) {
            uint64_t ad = sdesc_sw128(smem_u32(a_s + c * 16384) + kk * 32, 16, 1024);
            uint64_t bd = sdesc_sw128(smem_u32(b_s + c * 16384) + kk * 32, 16, 1024);
            umma_ss(tmem, ad, bd, idesc, (c | kk) != 0);
          }
      } else {
        const uint32_t idesc = umma_idesc_bf16(128, mode == 1 ? 64 : 128, 0, 1);
        for (int kk = 0; kk < 8; ++kk) {
          uint64_t bd = sdesc_sw128(smem_u32(b_s) + kk * 2048, 16384, 1024);
          umma_ts(tmem, tmem + 128 + kk * 8, bd, idesc, kk != 0);
        }
      }
    }
    umma_commit(&bar_mma);
  }
  __syncwarp();
  volatile int* ab = &abort_flag;
  bool ok = mbar_wait(&bar_mma, 0, ab);
  ok = __all_sync(0xffffffffu, ok);
  tc_fence_after();
  const int ncol = mode == 1 ? 64 : 128;
  const int row = warp * 32 + lane;
  if (ok) {
    for (int c = 0; c < ncol / 32; ++c) {
      uint32_t r[32];
      tmem_ld_x32(tmem + lane_off + c * 32, r);
      tmem_ld_wait();
      for (int i = 0; i < 32; ++i) d_out[row * ncol + c * 32 + i] = __uint_as_float(r[i]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

cudaError_t launch_umma_selftest(const CUtensorMap& a, const CUtensorMap& b, const uint16_t* p, float* d,
                                 int mode, cudaStream_t stream) {
  const int smem = 65536 + 1024;
  cudaError_t e = cudaFuncSetAttribute(umma_selftest_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  umma_selftest_kernel<<<1, 128, smem, stream>>>(a, b, p, d, mode);
  return cudaGetLastError();
}

}  // namespace gattn

namespace gattn {

// One CTA waits on an mbarrier that nothing arrives at. The bounded wait gives up after
// its limit, records a timeout in the device status word and the kernel returns: the
// path every pipeline wait takes when a peer role never signals.
__global__ void timeout_selftest_kernel(int* gave_up) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const bool ok = mbar_wait(&bar, 0, &abort_flag);
    *gave_up = ok ? 0 : 1;
  }
}

cudaError_t launch_timeout_selftest(int* gave_up, cudaStream_t stream) {
  timeout_selftest_kernel<<<1, 32, 0, stream>>>(gave_up);
  return cudaGetLastError();
}

}  // namespace gattn
