// calib.cu -- per-layer error statistics for choosing the layers that stay at
// full precision (page 1 of the TMAP write-up, "Attention performance
// optimisation / keeping video quality": the attention error of each layer
// was measured over the denoising iterations; layers whose error was large in
// every iteration keep the original precision, the rest are quantized).
//
// sage_attn_error_stats: for two bf16 tensors a (e.g. the quantized output)
// and b (e.g. the BF16 output) of shape [B,H,N,d], per head, in fp64:
//   sum (a-b)^2, sum b^2, sum a*b, sum a^2.
// Two kernels: per (head, slice) partial sums with a fixed per-thread order
// and a fixed shared-memory tree, then per head the slices in ascending order,
// so the result is deterministic.
// sage_attn_rel_l2: the same partial sums, then one thread adds every head's
// (a-b)^2 and b^2 slices in ascending order and writes sqrt(num / den).
// sage_select_full_precision_layers: the selection rule, on the host: a layer
// stays at full precision when its error is above the threshold at every
// iteration (the page's "large in every iteration"), or, with the mean rule,
// when its mean error over the iterations is.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "../../include/sage.h"
#include "internal.h"

namespace sage {
namespace {

constexpr int kErrThreads = 256;
constexpr int kErrSlices = 8;

__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// grid (kErrSlices, BH): slice s of head bh covers uint4 words [s*per, (s+1)*per)
__global__ void __launch_bounds__(kErrThreads) err_partial_kernel(const uint4* __restrict__ a, const uint4* __restrict__ b,
                                                                  long long words_per_head, double* __restrict__ partial) {
  const int s = blockIdx.x, bh = blockIdx.y;
  const long long per = (words_per_head + kErrSlices - 1) / kErrSlices;
  const long long w0 = (long long)s * per;
  const long long w1 = min(words_per_head, w0 + per);
  const uint4* ah = a + (long long)bh * words_per_head;
  const uint4* bh_ = b + (long long)bh * words_per_head;
  double acc[4] = {0.0, 0.0, 0.0, 0.0};
  for (long long w = w0 + threadIdx.x; w < w1; w += kErrThreads) {
    const uint4 ua = ah[w], ub = bh_[w];
    const uint32_t wa[4] = {ua.x, ua.y, ua.z, ua.w}, wb[4] = {ub.x, ub.y, ub.z, ub.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const double x0 = bf_lo(wa[i]), x1 = bf_hi(wa[i]), y0 = bf_lo(wb[i]), y1 = bf_hi(wb[i]);
      acc[0] += (x0 - y0) * (x0 - y0) + (x1 - y1) * (x1 - y1);
      acc[1] += y0 * y0 + y1 * y1;
      acc[2] += x0 * y0 + x1 * y1;
      acc[3] += x0 * x0 + x1 * x1;
    }
  }
  __shared__ double red[4][kErrThreads];
#pragma unroll
  for (int k = 0; k < 4; ++k) red[k][threadIdx.x] = acc[k];
  __syncthreads();
  for (int stride = kErrThreads / 2; stride > 0; stride >>= 1) {
    if (threadIdx.x < stride)
#pragma unroll
      for (int k = 0; k < 4; ++k) red[k][threadIdx.x] += red[k][threadIdx.x + stride];
    __syncthreads();
  }
  if (threadIdx.x < 4) partial[((long long)bh * kErrSlices + s) * 4 + threadIdx.x] = red[threadIdx.x][0];
}

// one thread per (head, quantity): the slices in ascending order
__global__ void err_final_kernel(const double* __restrict__ partial, int BH, double* __restrict__ stats) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= BH * 4) return;
  const int bh = i / 4, k = i % 4;
  double sum = 0.0;
  for (int s = 0; s < kErrSlices; ++s) sum += partial[((long long)bh * kErrSlices + s) * 4 + k];
  stats[i] = sum;
}

// one thread: every head's slices in ascending order, then the relative L2 error
__global__ void rel_l2_final_kernel(const double* __restrict__ partial, int BH, double* __restrict__ out) {
  if (blockIdx.x != 0 || threadIdx.x != 0) return;
  double num = 0.0, den = 0.0;
  for (int bh = 0; bh < BH; ++bh)
    for (int s = 0; s < kErrSlices; ++s) {
      num += partial[((long long)bh * kErrSlices + s) * 4 + 0];
      den += partial[((long long)bh * kErrSlices + s) * 4 + 1];
    }
  *out = den == 0.0 ? (num == 0.0 ? 0.0 : (double)INFINITY) : sqrt(num / den);
}

int check_err_args(const void* a, const void* b, int B, int H, int N, int d, const void* out, const void* scratch,
                   size_t scratch_bytes) {
  if (B < 1 || H < 1 || N < 1 || d < 8 || (d % 8) != 0) return SAGE_EINVAL;
  if ((long long)B * H > 65535) return SAGE_EINVAL;
  const void* ptrs[] = {a, b, out, scratch};
  for (const void* p : ptrs)
    if (!p || (reinterpret_cast<uintptr_t>(p) & 15u) != 0) return SAGE_EINVAL;
  if (scratch_bytes < (size_t)B * H * kErrSlices * 4 * sizeof(double)) return SAGE_EWORKSPACE;
  return SAGE_OK;
}

}  // namespace
}  // namespace sage

using namespace sage;

extern "C" size_t sage_error_scratch_bytes(int B, int H) {
  if (B < 1 || H < 1 || (long long)B * H > 65535) return 0;
  return (size_t)B * H * kErrSlices * 4 * sizeof(double);
}

extern "C" int sage_attn_error_stats(const void* a, const void* b, int B, int H, int N, int d, double* stats,
                                     void* scratch, size_t scratch_bytes, void* stream) {
  const int rc = check_err_args(a, b, B, H, N, d, stats, scratch, scratch_bytes);
  if (rc != SAGE_OK) return rc;
  const int BH = B * H;
  const long long words = (long long)N * d / 8;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  double* partial = static_cast<double*>(scratch);
  err_partial_kernel<<<dim3(kErrSlices, BH), kErrThreads, 0, st>>>(static_cast<const uint4*>(a),
                                                                   static_cast<const uint4*>(b), words, partial);
  err_final_kernel<<<(BH * 4 + 127) / 128, 128, 0, st>>>(partial, BH, stats);
  return cudaGetLastError() == cudaSuccess ? SAGE_OK : SAGE_ELAUNCH;
}

extern "C" int sage_attn_rel_l2(const void* a, const void* b, int B, int H, int N, int d, double* out, void* scratch,
                                size_t scratch_bytes, void* stream) {
  if (out && (reinterpret_cast<uintptr_t>(out) & 7u) != 0) return SAGE_EINVAL;
  // out needs only 8-byte alignment: check the others with a 16-byte aligned stand-in
  const int rc = check_err_args(a, b, B, H, N, d, out ? scratch : nullptr, scratch, scratch_bytes);
  if (rc != SAGE_OK) return rc;
  const int BH = B * H;
  const long long words = (long long)N * d / 8;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  double* partial = static_cast<double*>(scratch);
  err_partial_kernel<<<dim3(kErrSlices, BH), kErrThreads, 0, st>>>(static_cast<const uint4*>(a),
                                                                   static_cast<const uint4*>(b), words, partial);
  rel_l2_final_kernel<<<1, 32, 0, st>>>(partial, BH, out);
  return cudaGetLastError() == cudaSuccess ? SAGE_OK : SAGE_ELAUNCH;
}

extern "C" int sage_select_full_precision_layers(const double* layer_err, int num_layers, int num_iters,
                                                 double threshold, int rule, int* layers_out, int* n_out) {
  if (num_layers < 0 || num_iters < 1 || !n_out || (num_layers > 0 && (!layer_err || !layers_out))) return SAGE_EINVAL;
  if (rule != SAGE_SELECT_EVERY_ITERATION && rule != SAGE_SELECT_MEAN) return SAGE_EINVAL;
  int n = 0;
  for (int l = 0; l < num_layers; ++l) {
    bool every = true;
    double sum = 0.0;
    for (int i = 0; i < num_iters; ++i) {
      const double e = layer_err[(long long)l * num_iters + i];
      if (!std::isfinite(e)) return SAGE_EINVAL;
      every = every && e > threshold;
      sum += e;
    }
    const bool pick = rule == SAGE_SELECT_EVERY_ITERATION ? every : sum / num_iters > threshold;
    if (pick) layers_out[n++] = l;
  }
  *n_out = n;
  return SAGE_OK;
}
