// api.cu -- the extern "C" entry points declared in include/sage.h: argument
// validation, workspace layout, TMA tensor-map encoding and kernel launches.
// Marshalling only; every step of the computation runs in the kernels of
// prepass.cu and attention.cu.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <algorithm>
#include <cstring>
#include <mutex>

#include "../../include/sage.h"
#include "internal.h"

namespace sage {

unsigned long long current_context_id() {
  static PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
  static PFN_cuCtxGetId_v12000 get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Side streams and events of sage_attn_fwd_host, made on first use per device
// (and again in a new CUDA context) and kept for the life of the process.  A
// call holds its device's lock, so host calls on one device run one after
// the other.
struct HostPipe {
  std::mutex mu;
  unsigned long long ctx = 0;
  cudaStream_t s_in = nullptr, s_out = nullptr, s_alt = nullptr;
  cudaEvent_t ev_start = nullptr, ev_in = nullptr, ev_done = nullptr;
};
constexpr int kMaxHostDevices = 64;
HostPipe g_pipes[kMaxHostDevices];

// Makes the pipe's handles in the current context if they are missing or
// belong to an earlier one.  Called with p.mu held.
bool pipe_ready(HostPipe& p) {
  const unsigned long long ctx = current_context_id();
  if (p.s_in && ctx != 0 && ctx == p.ctx) return true;
  // handles of an earlier context are gone with it
  p.s_in = p.s_out = p.s_alt = nullptr;
  p.ev_start = p.ev_in = p.ev_done = nullptr;
  bool ok = cudaStreamCreateWithFlags(&p.s_in, cudaStreamNonBlocking) == cudaSuccess &&
            cudaStreamCreateWithFlags(&p.s_out, cudaStreamNonBlocking) == cudaSuccess &&
            cudaStreamCreateWithFlags(&p.s_alt, cudaStreamNonBlocking) == cudaSuccess &&
            cudaEventCreateWithFlags(&p.ev_start, cudaEventDisableTiming) == cudaSuccess &&
            cudaEventCreateWithFlags(&p.ev_in, cudaEventDisableTiming) == cudaSuccess &&
            cudaEventCreateWithFlags(&p.ev_done, cudaEventDisableTiming) == cudaSuccess;
  if (!ok) {
    if (p.s_in) cudaStreamDestroy(p.s_in);
    if (p.s_out) cudaStreamDestroy(p.s_out);
    if (p.s_alt) cudaStreamDestroy(p.s_alt);
    if (p.ev_start) cudaEventDestroy(p.ev_start);
    if (p.ev_in) cudaEventDestroy(p.ev_in);
    if (p.ev_done) cudaEventDestroy(p.ev_done);
    p.s_in = p.s_out = p.s_alt = nullptr;
    p.ev_start = p.ev_in = p.ev_done = nullptr;
    return false;
  }
  p.ctx = ctx;
  return true;
}

// Workspace layout of the INT8/FP8 mode; every region 256-byte aligned.
struct Layout {
  size_t status, q_i8, k_i8, v_f8t, q_scale, k_scale, k_mean, v_scale, scratch, total;
};

Layout layout(int B, int H, int N, int d, bool q_per_token = false) {
  const size_t BH = (size_t)B * H, nT = num_tiles(N), Npad = nT * kTile;
  Layout L;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off += align_up(bytes, 256);
    return at;
  };
  L.status = take(256);
  L.q_i8 = take(BH * Npad * d);
  L.k_i8 = take(BH * Npad * d);
  L.v_f8t = take(BH * d * Npad);
  L.q_scale = take(BH * (q_per_token ? Npad : nT) * 4);
  L.k_scale = take(BH * nT * 4);
  L.k_mean = take(BH * d * 4);
  L.v_scale = take(BH * d * 4);
  L.scratch = take(prepass_scratch_bytes((int)BH, N, d));
  L.total = off;
  return L;
}

int check_shape(int B, int H, int N, int d) {
  if (B < 1 || H < 1 || N < 1) return SAGE_EINVAL;
  if (d != 64 && d != 128) return SAGE_EUNSUPPORTED;
  const long long BH = (long long)B * H;
  if (BH > 65535) return SAGE_EINVAL;                       // grid.y limit
  const long long Npad = (long long)num_tiles(N) * kTile;
  if (BH * Npad * d >= (1LL << 31)) return SAGE_EINVAL;     // 32-bit TMA coordinates / offsets
  return SAGE_OK;
}

int check_device() {
  int dev = 0, major = 0, minor = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SAGE_ELAUNCH;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
    return SAGE_ELAUNCH;
  return (major == 10 && minor == 0) ? SAGE_OK : SAGE_EUNSUPPORTED;
}

int launch_status(cudaError_t e) {
  if (e == cudaSuccess) return SAGE_OK;
  if (e == cudaErrorInvalidValue) return SAGE_EINVAL;
  return SAGE_ELAUNCH;
}


}  // namespace

#ifdef SAGE_DEBUG
std::mutex g_debug_mu;
unsigned long long g_debug_first = 0;   // site << 48 | index of the last reported failure
#endif

// Debug build: waits for the call's work and turns any failed device-side
// bounds check into SAGE_EBOUNDS.  Release build: returns rc unchanged.
int debug_collect(cudaStream_t st, int rc) {
#ifdef SAGE_DEBUG
  if (rc != SAGE_OK) return rc;
  if (cudaStreamSynchronize(st) != cudaSuccess) return SAGE_ELAUNCH;
  std::lock_guard<std::mutex> lock(g_debug_mu);
  unsigned long long first = 0;
  const unsigned w = debug_take_prepass(&first) | debug_take_attention(&first) | debug_take_ulysses(&first);
  if (w) {
    g_debug_first = first;
    return SAGE_EBOUNDS;
  }
#else
  (void)st;
#endif
  return rc;
}

bool encode_tmap_2d(void* map, CUtensorMapDataType dtype, const void* base, uint64_t inner, uint64_t outer,
                    uint64_t outer_stride_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swizzle) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {outer_stride_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  return fn(static_cast<CUtensorMap*>(map), dtype, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool encode_tmap_3d(void* map, CUtensorMapDataType dtype, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
                    uint64_t stride1_bytes, uint64_t stride2_bytes, uint32_t box0, uint32_t box1, uint32_t box2,
                    CUtensorMapSwizzle swizzle) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {stride1_bytes, stride2_bytes};
  cuuint32_t box[3] = {box0, box1, box2};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(static_cast<CUtensorMap*>(map), dtype, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace sage

using namespace sage;

extern "C" {

size_t sage_workspace_bytes(int B, int H, int N, int d, int mode) {
  if (check_shape(B, H, N, d) != SAGE_OK) return 0;
  if (mode == SAGE_MODE_BF16) return 256;
  if (mode == SAGE_MODE_INT8_FP8) return layout(B, H, N, d).total;
  if (mode == SAGE_MODE_INT8_FP8_QTOKEN) return layout(B, H, N, d, true).total;
  return 0;
}

size_t sage_prepass_scratch_bytes(int B, int H, int N, int d) {
  if (check_shape(B, H, N, d) != SAGE_OK) return 0;
  return prepass_scratch_bytes(B * H, N, d);
}

int sage_quantize_qk(const void* q, const void* k, const void* v, int B, int H, int N, int d, int8_t* q_i8,
                     float* q_scale, int8_t* k_i8, float* k_scale, float* k_mean, uint8_t* v_f8t, float* v_scale,
                     void* scratch, size_t scratch_bytes, void* stream) {
  return sage_quantize_qk_ex(q, k, v, B, H, N, d, SAGE_BLK_Q, q_i8, q_scale, k_i8, k_scale, k_mean, v_f8t, v_scale,
                             scratch, scratch_bytes, stream);
}

int sage_quantize_qk_ex(const void* q, const void* k, const void* v, int B, int H, int N, int d, int q_granularity,
                        int8_t* q_i8, float* q_scale, int8_t* k_i8, float* k_scale, float* k_mean, uint8_t* v_f8t,
                        float* v_scale, void* scratch, size_t scratch_bytes, void* stream) {
  if (q_granularity != SAGE_BLK_Q && q_granularity != 1) return SAGE_EINVAL;
  int rc = check_shape(B, H, N, d);
  if (rc != SAGE_OK) return rc;
  const void* ptrs[] = {q, k, v, q_i8, q_scale, k_i8, k_scale, k_mean, v_f8t, v_scale, scratch};
  for (const void* p : ptrs)
    if (!p || !aligned16(p)) return SAGE_EINVAL;
  if (scratch_bytes < prepass_scratch_bytes(B * H, N, d)) return SAGE_EWORKSPACE;
  if ((rc = check_device()) != SAGE_OK) return rc;
  const PrepassScratch s = prepass_scratch_carve(scratch, B * H, N, d);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return debug_collect(st, launch_status(launch_prepass(q, k, v, B * H, N, d, q_i8, q_scale, k_i8, k_scale, k_mean,
                                                        v_f8t, v_scale, s, st, q_granularity == 1)));
}

int sage_attn_quantized(const int8_t* q_i8, const float* q_scale, const int8_t* k_i8, const float* k_scale,
                        const uint8_t* v_f8t, const float* v_scale, void* o, int B, int H, int N, int d, void* status,
                        void* stream) {
  return sage_attn_quantized_ex(q_i8, q_scale, k_i8, k_scale, v_f8t, v_scale, o, B, H, N, d, SAGE_BLK_Q, status,
                                stream);
}

int sage_attn_quantized_ex(const int8_t* q_i8, const float* q_scale, const int8_t* k_i8, const float* k_scale,
                           const uint8_t* v_f8t, const float* v_scale, void* o, int B, int H, int N, int d,
                           int q_granularity, void* status, void* stream) {
  if (q_granularity != SAGE_BLK_Q && q_granularity != 1) return SAGE_EINVAL;
  int rc = check_shape(B, H, N, d);
  if (rc != SAGE_OK) return rc;
  const void* ptrs[] = {q_i8, q_scale, k_i8, k_scale, v_f8t, v_scale, o, status};
  for (const void* p : ptrs)
    if (!p || !aligned16(p)) return SAGE_EINVAL;
  if ((rc = check_device()) != SAGE_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return debug_collect(st, launch_status(launch_attn_i8f8(q_i8, q_scale, k_i8, k_scale, v_f8t, v_scale, o, B * H, N,
                                                          d, static_cast<uint32_t*>(status), kDefaultTimeoutCycles, 0,
                                                          st, q_granularity == 1)));
}

namespace sage {
namespace {
// The INT8/FP8 path (prepass + attention) over a workspace laid out by layout();
// q, k, v rows found through in_map, output rows written through o_map.
int run_quantized(const void* q, const void* k, const void* v, void* o, int B, int H, int N, int d, bool qtok,
                  char* ws, cudaStream_t st, RowMap in_map, RowMap o_map) {
  uint32_t* status = reinterpret_cast<uint32_t*>(ws);
  const Layout L = layout(B, H, N, d, qtok);
  auto q_i8 = reinterpret_cast<int8_t*>(ws + L.q_i8);
  auto k_i8 = reinterpret_cast<int8_t*>(ws + L.k_i8);
  auto v_f8t = reinterpret_cast<uint8_t*>(ws + L.v_f8t);
  auto q_scale = reinterpret_cast<float*>(ws + L.q_scale);
  auto k_scale = reinterpret_cast<float*>(ws + L.k_scale);
  auto k_mean = reinterpret_cast<float*>(ws + L.k_mean);
  auto v_scale = reinterpret_cast<float*>(ws + L.v_scale);
  const PrepassScratch s = prepass_scratch_carve(ws + L.scratch, B * H, N, d);
  cudaError_t e =
      launch_prepass(q, k, v, B * H, N, d, q_i8, q_scale, k_i8, k_scale, k_mean, v_f8t, v_scale, s, st, qtok, in_map);
  if (e != cudaSuccess) return launch_status(e);
  return debug_collect(st, launch_status(launch_attn_i8f8(q_i8, q_scale, k_i8, k_scale, v_f8t, v_scale, o, B * H, N,
                                                          d, status, kDefaultTimeoutCycles, 0, st, qtok, o_map)));
}
}  // namespace
}  // namespace sage

int sage_attn_fwd(const void* q, const void* k, const void* v, void* o, int B, int H, int N, int d, int mode,
                  void* workspace, size_t workspace_bytes, void* stream) {
  int rc = check_shape(B, H, N, d);
  if (rc != SAGE_OK) return rc;
  if (mode != SAGE_MODE_BF16 && mode != SAGE_MODE_INT8_FP8 && mode != SAGE_MODE_INT8_FP8_QTOKEN) return SAGE_EINVAL;
  const void* ptrs[] = {q, k, v, o, workspace};
  for (const void* p : ptrs)
    if (!p || !aligned16(p)) return SAGE_EINVAL;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return SAGE_EINVAL;
  if (workspace_bytes < sage_workspace_bytes(B, H, N, d, mode)) return SAGE_EWORKSPACE;
  if ((rc = check_device()) != SAGE_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  uint32_t* status = reinterpret_cast<uint32_t*>(ws);
  if (mode == SAGE_MODE_BF16)
    return debug_collect(st, launch_status(launch_attn_bf16(q, k, v, o, B * H, N, d, status, kDefaultTimeoutCycles,
                                                            st)));
  const RowMap plain{0, 0, 0, 0};
  return run_quantized(q, k, v, o, B, H, N, d, mode == SAGE_MODE_INT8_FP8_QTOKEN, ws, st, plain, plain);
}

size_t sage_seqpar_workspace_bytes(int P, int B, int Nl, int Hl, int d, int mode) {
  if (P < 1 || Nl < 1 || (long long)P * Nl > (1LL << 30)) return 0;
  const int N = P * Nl;
  if (check_shape(B, Hl, N, d) != SAGE_OK) return 0;
  if (mode == SAGE_MODE_BF16) return 256 + 3 * align_up((size_t)B * Hl * N * d * 2, 256);
  return sage_workspace_bytes(B, Hl, N, d, mode);
}

int sage_attn_fwd_seqpar(const void* q, const void* k, const void* v, void* o, int P, int B, int Nl, int Hl, int d,
                         int mode, void* workspace, size_t workspace_bytes, void* stream) {
  if (P < 1 || Nl < 1 || (long long)P * Nl > (1LL << 30)) return SAGE_EINVAL;
  const int N = P * Nl;
  int rc = check_shape(B, Hl, N, d);
  if (rc != SAGE_OK) return rc;
  if (mode != SAGE_MODE_BF16 && mode != SAGE_MODE_INT8_FP8 && mode != SAGE_MODE_INT8_FP8_QTOKEN) return SAGE_EINVAL;
  const void* ptrs[] = {q, k, v, o, workspace};
  for (const void* p : ptrs)
    if (!p || !aligned16(p)) return SAGE_EINVAL;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return SAGE_EINVAL;
  if (workspace_bytes < sage_seqpar_workspace_bytes(P, B, Nl, Hl, d, mode)) return SAGE_EWORKSPACE;
  if ((rc = check_device()) != SAGE_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  const RowMap chunks{P, B, Nl, Hl};
  if (mode != SAGE_MODE_BF16)
    return run_quantized(q, k, v, o, B, Hl, N, d, mode == SAGE_MODE_INT8_FP8_QTOKEN, ws, st, chunks, chunks);
  // BF16: the kernel's TMA tiles need the plain layout, so q, k, v are gathered first; O is
  // written straight into the chunk layout
  uint32_t* status = reinterpret_cast<uint32_t*>(ws);
  const size_t region = align_up((size_t)B * Hl * N * d * 2, 256);
  char* g[3] = {ws + 256, ws + 256 + region, ws + 256 + 2 * region};
  const void* src[3] = {q, k, v};
  for (int i = 0; i < 3; ++i) {
    const cudaError_t e = launch_ulysses_permute(src[i], g[i], B, Nl, P * Hl, d, P, SAGE_ULYSSES_GATHER, 0, 0, st);
    if (e != cudaSuccess) return launch_status(e);
  }
  return debug_collect(st, launch_status(launch_attn_bf16(g[0], g[1], g[2], o, B * Hl, N, d, status,
                                                          kDefaultTimeoutCycles, st, chunks)));
}

int sage_host_chunk_heads(int B, int H, int N, int d) {
  if (check_shape(B, H, N, d) != SAGE_OK) return 0;
  int sms = 148, dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      sms <= 0) {
    cudaGetLastError();
    sms = 148;
  }
  // the smallest chunk whose attention launch (one CTA per 256 query rows of a head) fills 4 waves
  const long long ctas_per_head = (N + 255) / 256;
  long long chunk = (4LL * sms + ctas_per_head - 1) / ctas_per_head;
  const long long BH = (long long)B * H;
  if (chunk < 1) chunk = 1;
  if (chunk > BH) chunk = BH;
  return (int)chunk;
}

size_t sage_host_workspace_bytes(int B, int H, int N, int d, int mode, int chunk_heads) {
  if (check_shape(B, H, N, d) != SAGE_OK) return 0;
  if (mode != SAGE_MODE_BF16 && mode != SAGE_MODE_INT8_FP8 && mode != SAGE_MODE_INT8_FP8_QTOKEN) return 0;
  const int BH = B * H;
  if (chunk_heads <= 0) chunk_heads = sage_host_chunk_heads(B, H, N, d);
  if (chunk_heads > BH) chunk_heads = BH;
  const size_t one = align_up(sage_workspace_bytes(1, chunk_heads, N, d, mode), 256);
  return BH > 1 ? 2 * one : one;      // two chunks in flight, one workspace each
}

int sage_attn_fwd_host(const void* q_host, const void* k_host, const void* v_host, void* o_host, int B, int H, int N,
                       int d, int mode, void* q_dev, void* k_dev, void* v_dev, void* o_dev, void* workspace,
                       size_t workspace_bytes, int chunk_heads, void* stream) {
  int rc = check_shape(B, H, N, d);
  if (rc != SAGE_OK) return rc;
  if (mode != SAGE_MODE_BF16 && mode != SAGE_MODE_INT8_FP8 && mode != SAGE_MODE_INT8_FP8_QTOKEN) return SAGE_EINVAL;
  const void* ptrs[] = {q_host, k_host, v_host, o_host, q_dev, k_dev, v_dev, o_dev, workspace};
  for (const void* p : ptrs)
    if (!p || !aligned16(p)) return SAGE_EINVAL;
  // each chunk workspace is handed to sage_attn_fwd, which wants 256-byte alignment
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return SAGE_EINVAL;
  const int BH = B * H;
  if (chunk_heads <= 0) chunk_heads = sage_host_chunk_heads(B, H, N, d);
  if (chunk_heads > BH) chunk_heads = BH;
  if (workspace_bytes < sage_host_workspace_bytes(B, H, N, d, mode, chunk_heads)) return SAGE_EWORKSPACE;
  // The two chunk workspaces split the buffer in halves whatever the mode, so
  // their status words sit at the same places for every call on one buffer
  // (a layer stack alternates modes on the same workspace).
  const int n_ws = BH > 1 ? 2 : 1;
  const size_t ws_one = n_ws == 2 ? (workspace_bytes / 2) & ~size_t(255) : workspace_bytes;
  if ((rc = check_device()) != SAGE_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxHostDevices) return SAGE_ELAUNCH;
  HostPipe& pipe = g_pipes[dev];
  std::lock_guard<std::mutex> lock(pipe.mu);
  if (!pipe_ready(pipe)) return SAGE_ELAUNCH;
  cudaStream_t s_in = pipe.s_in, s_out = pipe.s_out;
  cudaEvent_t ev_start = pipe.ev_start, ev_in = pipe.ev_in, ev_done = pipe.ev_done;
  // Chunks alternate between the caller's stream and a second compute stream,
  // each with its own half of the workspace, so that chunk i+1's prepass and
  // the start of its attention fill the SMs that chunk i's last wave leaves
  // idle.  Inputs of chunk i land (s_in) -> its prepass and attention run
  // (compute stream i % 2) -> its output leaves (s_out).  Nothing starts
  // before earlier work on the caller's stream.
  cudaStream_t s_comp[2] = {st, pipe.s_alt};
  cudaEventRecord(ev_start, st);
  cudaStreamWaitEvent(s_in, ev_start, 0);
  cudaStreamWaitEvent(pipe.s_alt, ev_start, 0);
  const size_t head_bytes = (size_t)N * d * 2;
  const char* qh = static_cast<const char*>(q_host);
  const char* kh = static_cast<const char*>(k_host);
  const char* vh = static_cast<const char*>(v_host);
  char* oh = static_cast<char*>(o_host);
  char* qd = static_cast<char*>(q_dev);
  char* kd = static_cast<char*>(k_dev);
  char* vd = static_cast<char*>(v_dev);
  char* od = static_cast<char*>(o_dev);
  char* ws = static_cast<char*>(workspace);
  // The first and the last chunk take half as many heads: the first upload and
  // the last download are the parts of the pipeline nothing overlaps.
  const int half = std::max(1, chunk_heads / 2);
  const int first = std::min(half, BH);
  const int last = std::min(half, BH - first);
  rc = SAGE_OK;
  int i = 0;
  for (int h0 = 0; h0 < BH && rc == SAGE_OK; ++i) {
    int hc = h0 == 0 ? first : std::min(chunk_heads, BH - last - h0);
    if (hc <= 0) hc = BH - h0;                       // the last chunk
    const size_t off = (size_t)h0 * head_bytes, bytes = (size_t)hc * head_bytes;
    cudaStream_t sc = s_comp[i % n_ws];
    char* wsi = ws + (size_t)(i % n_ws) * ws_one;
    if (cudaMemcpyAsync(qd + off, qh + off, bytes, cudaMemcpyHostToDevice, s_in) != cudaSuccess ||
        cudaMemcpyAsync(kd + off, kh + off, bytes, cudaMemcpyHostToDevice, s_in) != cudaSuccess ||
        cudaMemcpyAsync(vd + off, vh + off, bytes, cudaMemcpyHostToDevice, s_in) != cudaSuccess ||
        cudaEventRecord(ev_in, s_in) != cudaSuccess || cudaStreamWaitEvent(sc, ev_in, 0) != cudaSuccess) {
      rc = SAGE_ELAUNCH;
      break;
    }
    rc = sage_attn_fwd(qd + off, kd + off, vd + off, od + off, 1, hc, N, d, mode, wsi, ws_one, sc);
    if (rc != SAGE_OK) break;
    if (cudaEventRecord(ev_done, sc) != cudaSuccess || cudaStreamWaitEvent(s_out, ev_done, 0) != cudaSuccess ||
        cudaMemcpyAsync(oh + off, od + off, bytes, cudaMemcpyDeviceToHost, s_out) != cudaSuccess)
      rc = SAGE_ELAUNCH;
    h0 += hc;
  }
  // every chunk's compute precedes its output copy on s_out, so the caller's
  // stream resumes after the last output copy
  cudaEventRecord(ev_done, s_out);
  cudaStreamWaitEvent(st, ev_done, 0);
  if (cudaStreamSynchronize(s_out) != cudaSuccess || cudaStreamSynchronize(pipe.s_alt) != cudaSuccess ||
      cudaStreamSynchronize(st) != cudaSuccess)
    rc = SAGE_ELAUNCH;
  if (rc != SAGE_OK) return rc;
  for (int w = 0; w < n_ws; ++w) {
    const int r = sage_status(ws + (size_t)w * ws_one, stream);
    if (r != SAGE_OK) rc = r;
  }
  return rc;
}

int attn_layer_schedule(int num_layers, const int* full_precision_layers, int n_fp, int8_t* modes_out) {
  if (num_layers < 0 || n_fp < 0) return SAGE_EINVAL;
  if (n_fp > 0 && !full_precision_layers) return SAGE_EINVAL;
  if (num_layers > 0 && !modes_out) return SAGE_EINVAL;
  for (int i = 0; i < n_fp; ++i)
    if (full_precision_layers[i] < 0 || full_precision_layers[i] >= num_layers) return SAGE_EINVAL;
  for (int l = 0; l < num_layers; ++l) modes_out[l] = (int8_t)SAGE_MODE_INT8_FP8;
  for (int i = 0; i < n_fp; ++i) modes_out[full_precision_layers[i]] = (int8_t)SAGE_MODE_BF16;
  return SAGE_OK;
}

namespace {
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

int check_linear(const int8_t* xq, const float* sx, const int8_t* wq, const float* sw, const void* bias, void* y,
                 int y_dtype, int M, int N, int K, void* status) {
  if (M < 1 || N < 128 || K < 128 || N % 128 != 0 || K % 128 != 0) return SAGE_EINVAL;
  if (y_dtype != SAGE_DTYPE_BF16 && y_dtype != SAGE_DTYPE_F32) return SAGE_EINVAL;
  const void* p16[] = {xq, wq, y};
  for (const void* p : p16)
    if (!p || !aligned16(p)) return SAGE_EINVAL;
  if (bias && !aligned16(bias)) return SAGE_EINVAL;
  const void* p4[] = {sx, sw, status};
  for (const void* p : p4)
    if (!p || !aligned4(p)) return SAGE_EINVAL;
  return check_device();
}
}  // namespace

int sage_quantize_blocks_2d(const void* x, int R, int K, int8_t* codes, float* scales, void* stream) {
  if (R < 1 || K < 128 || K % 128 != 0 || (R + 127) / 128 > 65535) return SAGE_EINVAL;
  if (!x || !codes || !scales || !aligned16(x) || !aligned16(codes) || !aligned4(scales)) return SAGE_EINVAL;
  const int rc = check_device();
  if (rc != SAGE_OK) return rc;
  return launch_status(launch_quant_blocks_2d(x, R, K, codes, scales, static_cast<cudaStream_t>(stream)));
}

int sage_linear_w8a8(const int8_t* xq, const float* sx, const int8_t* wq, const float* sw, const void* bias, void* y,
                     int y_dtype, int M, int N, int K, void* status, void* stream) {
  const int rc = check_linear(xq, sx, wq, sw, bias, y, y_dtype, M, N, K, status);
  if (rc != SAGE_OK) return rc;
  return launch_status(launch_linear_w8a8(xq, sx, wq, sw, bias, y, y_dtype == SAGE_DTYPE_F32, M, N, K,
                                          static_cast<uint32_t*>(status), kDefaultTimeoutCycles, 0,
                                          static_cast<cudaStream_t>(stream)));
}

int sage_dbg_linear_forced_timeout(const int8_t* xq, const float* sx, const int8_t* wq, const float* sw,
                                   const void* bias, void* y, int y_dtype, int M, int N, int K, void* status,
                                   long long timeout_cycles, void* stream) {
  if (timeout_cycles < 1) return SAGE_EINVAL;
  const int rc = check_linear(xq, sx, wq, sw, bias, y, y_dtype, M, N, K, status);
  if (rc != SAGE_OK) return rc;
  return launch_status(launch_linear_w8a8(xq, sx, wq, sw, bias, y, y_dtype == SAGE_DTYPE_F32, M, N, K,
                                          static_cast<uint32_t*>(status), timeout_cycles, 1,
                                          static_cast<cudaStream_t>(stream)));
}

int sage_dequant_blocks_2d(const int8_t* codes, const float* scales, int R, int K, void* out, void* stream) {
  if (R < 1 || K < 128 || K % 128 != 0 || (R + 127) / 128 > 65535) return SAGE_EINVAL;
  if (!codes || !scales || !out || !aligned16(codes) || !aligned16(out) || !aligned4(scales)) return SAGE_EINVAL;
  const int rc = check_device();
  if (rc != SAGE_OK) return rc;
  return launch_status(launch_dequant_blocks_2d(codes, scales, R, K, out, static_cast<cudaStream_t>(stream)));
}

namespace {
int check_linear_bf16(const void* x, const void* w, const void* bias, void* y, int y_dtype, int M, int N, int K,
                      void* status) {
  if (M < 1 || N < 128 || K < 64 || N % 128 != 0 || K % 64 != 0) return SAGE_EINVAL;
  if (y_dtype != SAGE_DTYPE_BF16 && y_dtype != SAGE_DTYPE_F32) return SAGE_EINVAL;
  const void* p16[] = {x, w, y};
  for (const void* p : p16)
    if (!p || !aligned16(p)) return SAGE_EINVAL;
  if (bias && !aligned16(bias)) return SAGE_EINVAL;
  if (!status || !aligned4(status)) return SAGE_EINVAL;
  return SAGE_OK;
}
}  // namespace

int sage_linear_bf16(const void* x, const void* w, const void* bias, void* y, int y_dtype, int M, int N, int K,
                     void* status, void* stream) {
  int rc = check_linear_bf16(x, w, bias, y, y_dtype, M, N, K, status);
  if (rc != SAGE_OK) return rc;
  if ((rc = check_device()) != SAGE_OK) return rc;
  return launch_status(launch_linear_bf16(x, w, bias, y, y_dtype == SAGE_DTYPE_F32, M, N, K,
                                          static_cast<uint32_t*>(status), kDefaultTimeoutCycles, 0,
                                          static_cast<cudaStream_t>(stream)));
}

int sage_dbg_linear_bf16_forced_timeout(const void* x, const void* w, const void* bias, void* y, int y_dtype, int M,
                                        int N, int K, void* status, long long timeout_cycles, void* stream) {
  if (timeout_cycles < 1) return SAGE_EINVAL;
  int rc = check_linear_bf16(x, w, bias, y, y_dtype, M, N, K, status);
  if (rc != SAGE_OK) return rc;
  if ((rc = check_device()) != SAGE_OK) return rc;
  return launch_status(launch_linear_bf16(x, w, bias, y, y_dtype == SAGE_DTYPE_F32, M, N, K,
                                          static_cast<uint32_t*>(status), timeout_cycles, 1,
                                          static_cast<cudaStream_t>(stream)));
}

size_t sage_linear_w8a16_workspace_bytes(int N, int K) {
  if (N < 1 || K < 1) return 0;
  return align_up((size_t)N * K * 2, 256);
}

int sage_linear_w8a16(const void* x, const int8_t* wq, const float* sw, const void* bias, void* y, int y_dtype, int M,
                      int N, int K, void* workspace, size_t workspace_bytes, void* status, void* stream) {
  if (K % 128 != 0 || (N + 127) / 128 > 65535) return SAGE_EINVAL;
  int rc = check_linear_bf16(x, workspace, bias, y, y_dtype, M, N, K, status);
  if (rc != SAGE_OK) return rc;
  if (!wq || !sw || !aligned16(wq) || !aligned4(sw)) return SAGE_EINVAL;
  if (workspace_bytes < sage_linear_w8a16_workspace_bytes(N, K)) return SAGE_EWORKSPACE;
  if ((rc = check_device()) != SAGE_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  rc = launch_status(launch_dequant_blocks_2d(wq, sw, N, K, workspace, st));
  if (rc != SAGE_OK) return rc;
  return launch_status(launch_linear_bf16(x, workspace, bias, y, y_dtype == SAGE_DTYPE_F32, M, N, K,
                                          static_cast<uint32_t*>(status), kDefaultTimeoutCycles, 0, st));
}

int sage_ulysses_permute(const void* src, void* dst, int B, int Nl, int H, int d, int P, int op,
                         long long chunk_rows, long long base_rows, void* stream) {
  if (B < 1 || Nl < 1 || H < 1 || P < 1 || H % P != 0 || (d != 64 && d != 128)) return SAGE_EINVAL;
  if (op < SAGE_ULYSSES_SEND || op > SAGE_ULYSSES_SCATTER || chunk_rows < 0 || base_rows < 0) return SAGE_EINVAL;
  if (!src || !dst || !aligned16(src) || !aligned16(dst) || src == dst) return SAGE_EINVAL;
  const long long rows = (long long)B * Nl * H;
  const long long dense = (long long)B * (H / P) * Nl;
  if (chunk_rows != 0 && chunk_rows < dense) return SAGE_EINVAL;
  if (rows * (d / 8) >= (1LL << 40)) return SAGE_EINVAL;
  const int rc = check_device();
  if (rc != SAGE_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return debug_collect(st, launch_status(launch_ulysses_permute(src, dst, B, Nl, H, d, P, op, chunk_rows, base_rows,
                                                                st)));
}

int sage_dbg_mma_peak(int kind, int n, int iters, long long* cycles, int grid, void* status, void* stream) {
  if (kind < SAGE_MMA_BF16 || kind > SAGE_MMA_I8 || (n != 128 && n != 256) || iters < 1 || grid < 1) return SAGE_EINVAL;
  if (!cycles || !status || (reinterpret_cast<uintptr_t>(cycles) & 7u) || (reinterpret_cast<uintptr_t>(status) & 3u))
    return SAGE_EINVAL;
  const int rc = check_device();
  if (rc != SAGE_OK) return rc;
  // SAGE_MMA_* follow the kind numbering of the kernels (f16, f8f6f4, i8)
  return launch_status(launch_mma_peak(kind, n, iters, cycles, static_cast<uint32_t*>(status), grid,
                                       static_cast<cudaStream_t>(stream)));
}

int sage_status(void* workspace, void* stream) {
  if (!workspace) return SAGE_EINVAL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint32_t word = 0;
  if (cudaMemcpyAsync(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost, st) != cudaSuccess) return SAGE_ELAUNCH;
  if (cudaMemsetAsync(workspace, 0, sizeof(word), st) != cudaSuccess) return SAGE_ELAUNCH;
  if (cudaStreamSynchronize(st) != cudaSuccess) return SAGE_ELAUNCH;
  if (word & kStatusTimeout) return SAGE_ETIMEOUT;
  return word ? SAGE_ELAUNCH : SAGE_OK;
}

const char* sage_strerror(int code) {
  switch (code) {
    case SAGE_OK: return "ok";
    case SAGE_EINVAL: return "invalid argument (size, null or misaligned pointer, mode)";
    case SAGE_EUNSUPPORTED: return "unsupported (head dim must be 64 or 128; device must be sm_100)";
    case SAGE_ELAUNCH: return "CUDA launch or runtime error";
    case SAGE_EWORKSPACE: return "workspace too small";
    case SAGE_ETIMEOUT: return "a bounded device-side wait ran out";
    case SAGE_EBOUNDS: return "a device-side bounds check failed (debug build)";
    default: return "unknown status";
  }
}

int sage_device_check(void) { return check_device(); }

int sage_debug_build(void) {
#ifdef SAGE_DEBUG
  return 1;
#else
  return 0;
#endif
}

int sage_debug_last_failure(int* site, long long* index) {
  if (!site || !index) return SAGE_EINVAL;
#ifdef SAGE_DEBUG
  std::lock_guard<std::mutex> lock(g_debug_mu);
  *site = (int)(g_debug_first >> 48);
  *index = (long long)(g_debug_first & 0xFFFFFFFFFFFFull);
  return SAGE_OK;
#else
  *site = 0;
  *index = 0;
  return SAGE_EUNSUPPORTED;
#endif
}

int sage_dbg_bounds_selftest(void* stream) {
#ifdef SAGE_DEBUG
  int rc = check_device();
  if (rc != SAGE_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return debug_collect(st, launch_status(launch_debug_selftest(st)));
#else
  (void)stream;
  return SAGE_EUNSUPPORTED;
#endif
}

int sage_dbg_qk_tiles(const int8_t* q_i8, const int8_t* k_i8, int B, int H, int N, int d, const int* tile_list, int n,
                      int32_t* out, void* stream) {
  int rc = check_shape(B, H, N, d);
  if (rc != SAGE_OK) return rc;
  if (n < 1 || n > 65535 || !q_i8 || !k_i8 || !tile_list || !out || !aligned16(q_i8) || !aligned16(k_i8))
    return SAGE_EINVAL;
  if ((rc = check_device()) != SAGE_OK) return rc;
  return launch_status(
      launch_dbg_qk_tiles(q_i8, k_i8, B * H, H, N, d, tile_list, n, out, static_cast<cudaStream_t>(stream)));
}

int sage_dbg_pv_tile(const void* p, const void* vt, int d, int mode, float* out, void* stream) {
  if (d != 64 && d != 128) return SAGE_EUNSUPPORTED;
  if (mode != SAGE_MODE_BF16 && mode != SAGE_MODE_INT8_FP8) return SAGE_EINVAL;
  if (!p || !vt || !out || !aligned16(p) || !aligned16(vt)) return SAGE_EINVAL;
  int rc = check_device();
  if (rc != SAGE_OK) return rc;
  return launch_status(launch_dbg_pv_tile(p, vt, d, mode, out, static_cast<cudaStream_t>(stream)));
}

int sage_dbg_qk_bf16_tile(const void* q, const void* k, int d, float* out, void* stream) {
  if (d != 64 && d != 128) return SAGE_EUNSUPPORTED;
  if (!q || !k || !out || !aligned16(q) || !aligned16(k)) return SAGE_EINVAL;
  int rc = check_device();
  if (rc != SAGE_OK) return rc;
  return launch_status(launch_dbg_qk_bf16_tile(q, k, d, out, static_cast<cudaStream_t>(stream)));
}

int sage_dbg_attn_forced_timeout(const int8_t* q_i8, const float* q_scale, const int8_t* k_i8, const float* k_scale,
                                 const uint8_t* v_f8t, const float* v_scale, void* o, int B, int H, int N, int d,
                                 void* status, long long timeout_cycles, void* stream) {
  int rc = check_shape(B, H, N, d);
  if (rc != SAGE_OK) return rc;
  const void* ptrs[] = {q_i8, q_scale, k_i8, k_scale, v_f8t, v_scale, o, status};
  for (const void* p : ptrs)
    if (!p || !aligned16(p)) return SAGE_EINVAL;
  if (timeout_cycles < 1000 || timeout_cycles > kDefaultTimeoutCycles) return SAGE_EINVAL;
  if ((rc = check_device()) != SAGE_OK) return rc;
  return launch_status(launch_attn_i8f8(q_i8, q_scale, k_i8, k_scale, v_f8t, v_scale, o, B * H, N, d,
                                        static_cast<uint32_t*>(status), timeout_cycles, 1,
                                        static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
