// diag.cu -- tensor-core throughput probe: back-to-back tcgen05.mma from
// shared-memory operands into tensor memory, no loads, no epilogue, one CTA
// per SM.  It measures the MMA rate per SM per clock that the attention and
// linear kernels are bounded by (kind::i8 for QK^T, kind::f8f6f4 for P.V,
// kind::f16 for the BF16 path), independent of the clock the SM runs at.
#include <cuda_runtime.h>

#include <cstdint>

#include "internal.h"
#include "sm100.cuh"

namespace sage {

namespace {

// One "block" = 4 MMAs of M=128 x N x 32 bytes of K into alternating accumulators.
template <int KIND, int N>
__global__ void __launch_bounds__(128, 1) mma_peak_kernel(long long* cycles, int iters, uint32_t* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ uint64_t done;
  __shared__ uint32_t slot;
  __shared__ int abort_s;
  const int warp = threadIdx.x >> 5;
  for (int i = threadIdx.x; i < (128 + N) * 128 / 16; i += 128) reinterpret_cast<uint4*>(smem)[i] = make_uint4(0, 0, 0, 0);
  fence_proxy_async_smem();
  if (threadIdx.x == 0) {
    mbar_init(&done, 1);
    abort_s = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = slot;
  if (threadIdx.x == 0) {
    const uint32_t a_s = smem_u32(smem), b_s = a_s + 128 * 128;
    constexpr uint32_t idesc = KIND == kKindI8      ? make_idesc(kFmtS32Acc, kFmtS8, kFmtS8, 0, 128, N)
                               : KIND == kKindF16   ? make_idesc(kFmtF32Acc, kFmtBF16, kFmtBF16, 0, 128, N)
                                                    : make_idesc(kFmtF32Acc, kFmtE4M3, kFmtE4M3, 0, 128, N);
    const long long c0 = clock64();
    for (int it = 0; it < iters; ++it) {
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const uint64_t ad = make_sdesc(a_s + k * 32, 16, 1024, kLayoutSW128);
        const uint64_t bd = make_sdesc(b_s + k * 32, 16, 1024, kLayoutSW128);
        mma_ss<KIND>(tmem + (uint32_t)(it & 1) * 256, ad, bd, idesc, 1u);
      }
    }
    mma_commit(&done);
    const bool ok = mbar_wait(&done, 0, &abort_s, kDefaultTimeoutCycles);
    cycles[blockIdx.x] = clock64() - c0;
    if (!ok) atomicOr(status, kStatusTimeout);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

template <int KIND, int N>
cudaError_t launch_one(long long* cycles, int iters, uint32_t* status, int grid, cudaStream_t stream) {
  const int smem = (128 + N) * 128 + 1024;
  cudaError_t e = cudaFuncSetAttribute(mma_peak_kernel<KIND, N>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  mma_peak_kernel<KIND, N><<<grid, 128, smem, stream>>>(cycles, iters, status);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_mma_peak(int kind, int n, int iters, long long* cycles, uint32_t* status, int grid,
                            cudaStream_t stream) {
  if (kind == kKindI8) return n == 256 ? launch_one<kKindI8, 256>(cycles, iters, status, grid, stream)
                                       : launch_one<kKindI8, 128>(cycles, iters, status, grid, stream);
  if (kind == kKindF16) return n == 256 ? launch_one<kKindF16, 256>(cycles, iters, status, grid, stream)
                                        : launch_one<kKindF16, 128>(cycles, iters, status, grid, stream);
  return n == 256 ? launch_one<kKindF8F6F4, 256>(cycles, iters, status, grid, stream)
                  : launch_one<kKindF8F6F4, 128>(cycles, iters, status, grid, stream);
}

}  // namespace sage
