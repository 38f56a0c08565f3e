// noalloc.cu -- sage_quantize_qk_noalloc: the quantization prepass with its
// scratch (the per-block partial sums, minima, maxima and absmax values) kept
// in a fixed device array owned by this library, for callers that cannot
// allocate device memory.
//
// Who needs this: callers that must not allocate device memory while they
// run -- a service that reserved all of HBM up front for its own pool (so a
// cudaMalloc here would fail or fragment that pool), or a latency-critical
// loop that cannot afford the implicit synchronisation cudaMalloc / cudaFree
// may cause.  They pass inputs and outputs and nothing else.
//
// The array lives for as long as the library is loaded and is held on every
// device that loads the library (kScratchBytes each).  Host code cannot use
// the array's name as a device address, so the address is looked up with
// cudaGetSymbolAddress on the first call made on a device and cached together
// with the unique id of the CUDA context it belongs to.  A call in another
// context (after cudaDeviceReset, or a destroyed and re-created primary
// context, which reloads the module at a new address) looks it up again.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "../../include/sage.h"
#include "internal.h"

namespace sage {
namespace {

constexpr size_t kScratchBytes = SAGE_NOALLOC_SCRATCH_BYTES;
static_assert(kScratchBytes % 256 == 0, "scratch size must keep 256-byte alignment");

static __device__ __align__(256) unsigned char g_prepass_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};
unsigned long long g_scratch_ctx[kMaxDevices] = {};

// Device address of g_prepass_scratch on the current device, looked up with
// that device current the first time it is needed in the current context.
// nullptr on failure.
void* scratch_address(int dev) {
  const unsigned long long ctx = current_context_id();
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_ptr[dev] || ctx == 0 || ctx != g_scratch_ctx[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_prepass_scratch) != cudaSuccess) return nullptr;
    g_scratch_ptr[dev] = p;
    g_scratch_ctx[dev] = ctx;
  }
  return g_scratch_ptr[dev];
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace sage

extern "C" int sage_quantize_qk_noalloc(const void* q, const void* k, const void* v, int B, int H, int N, int d,
                                        int8_t* q_i8, float* q_scale, int8_t* k_i8, float* k_scale, float* k_mean,
                                        uint8_t* v_f8t, float* v_scale, void* stream) {
  using namespace sage;
  if (B < 1 || H < 1 || N < 1) return SAGE_EINVAL;
  if (d != 64 && d != 128) return SAGE_EUNSUPPORTED;
  if ((long long)B * H > 65535) return SAGE_EINVAL;
  if ((long long)B * H * num_tiles(N) * kTile * d >= (1LL << 31)) return SAGE_EINVAL;
  const void* ptrs[] = {q, k, v, q_i8, q_scale, k_i8, k_scale, k_mean, v_f8t, v_scale};
  for (const void* p : ptrs)
    if (!p || !aligned16(p)) return SAGE_EINVAL;
  // the fixed scratch must hold this problem's partials
  if (prepass_scratch_bytes(B * H, N, d) > kScratchBytes) return SAGE_EWORKSPACE;
  int dev = 0, major = 0, minor = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SAGE_ELAUNCH;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
    return SAGE_ELAUNCH;
  if (major != 10 || minor != 0) return SAGE_EUNSUPPORTED;
  void* base = scratch_address(dev);
  if (!base) return SAGE_ELAUNCH;
  // Every partial the kernels read is written earlier in the same call, so
  // nothing in the scratch has to start at zero.
  const PrepassScratch s = prepass_scratch_carve(base, B * H, N, d);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const cudaError_t e = launch_prepass(q, k, v, B * H, N, d, q_i8, q_scale, k_i8, k_scale, k_mean, v_f8t, v_scale, s,
                                       st);
  return debug_collect(st, e == cudaSuccess ? SAGE_OK : SAGE_ELAUNCH);
}
