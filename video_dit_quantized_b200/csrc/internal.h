// internal.h -- declarations shared by the library's translation units (not
// part of the C ABI).
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <cstddef>
#include <cstdint>

namespace sage {

constexpr int kTile = 128;

// Bits OR-ed into the device status word.
constexpr uint32_t kStatusTimeout = 1u;

// ---- debug build (-DSAGE_DEBUG): device-side bounds checks ----------------
// In a debug build every global access of the prepass, the attention
// epilogue and scale loads, and the Ulysses permutations whose index is
// computed checks the index against the extent of its buffer first.  A failed
// check skips the access (nothing traps) and records itself in this
// translation unit's debug word, with the site and index of the first
// failure; the entry points of a debug build synchronise their stream and
// return SAGE_EBOUNDS when any word is set.  A release build compiles every
// check to `true`.  TMA loads need no check: the tensor maps bound them.
#ifdef SAGE_DEBUG
namespace dbg {
static __device__ unsigned int g_word;            // one pair per translation unit
static __device__ unsigned long long g_first;     // site << 48 | index of the first failure
}  // namespace dbg
__device__ __forceinline__ bool dcheck(long long idx, long long extent, unsigned site) {
  if (idx >= 0 && idx < extent) return true;
  atomicOr(&dbg::g_word, 1u);
  atomicCAS(&dbg::g_first, 0ull, ((unsigned long long)site << 48) | ((unsigned long long)idx & 0xFFFFFFFFFFFFull));
  return false;
}
#define SAGE_DCHECK(idx, extent, site) ::sage::dcheck((long long)(idx), (long long)(extent), (unsigned)(site))
// Reads and clears this translation unit's words (host; after the work has
// finished).  Returns the word; *first gets the first failure if it is 0.
static inline unsigned debug_take_tu(unsigned long long* first) {
  unsigned w = 0;
  unsigned long long f = 0;
  const unsigned zw = 0;
  const unsigned long long zf = 0;
  if (cudaMemcpyFromSymbol(&w, dbg::g_word, sizeof(w)) != cudaSuccess ||
      cudaMemcpyFromSymbol(&f, dbg::g_first, sizeof(f)) != cudaSuccess)
    return 1u;
  cudaMemcpyToSymbol(dbg::g_word, &zw, sizeof(zw));
  cudaMemcpyToSymbol(dbg::g_first, &zf, sizeof(zf));
  if (w && first && *first == 0) *first = f;
  return w;
}
#else
#define SAGE_DCHECK(idx, extent, site) true
#endif
// Debug sites (the site field of a recorded failure).
enum DebugSite : unsigned {
  kSiteStatsIn = 1, kSiteStatsQ8, kSiteStatsQScale, kSiteStatsPartials,
  kSiteFinIn, kSiteFinOut,
  kSiteQuantIn, kSiteQuantPartials, kSiteQuantK8, kSiteQuantKScale, kSiteQuantV8,
  kSiteAttnQScale = 20, kSiteAttnKScale, kSiteAttnVScale, kSiteAttnOut,
  kSiteUlyssesSrc = 30, kSiteUlyssesDst,
  kSiteSelftest = 99
};
// Per translation unit: reads and clears its debug words (0 in a release build).
unsigned debug_take_prepass(unsigned long long* first);
unsigned debug_take_attention(unsigned long long* first);
unsigned debug_take_ulysses(unsigned long long* first);
// A kernel that fails one check on purpose (the index equals the extent; no
// memory is touched): the debug path's self-test.
cudaError_t launch_debug_selftest(cudaStream_t stream);
// Debug build: synchronises `st` and returns SAGE_EBOUNDS if a check failed
// (rc when rc is already an error).  Release build: rc.
int debug_collect(cudaStream_t st, int rc);

inline int num_tiles(int N) { return (N + kTile - 1) / kTile; }
inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Where token n of head bh sits, in rows of d values.  P == 0: the plain
// [BH, N, d] layout, row bh * N + n.  P >= 1: the sequence-parallel chunk
// layout [P][B][Nl][Hl][d] (chunk p holds tokens p*Nl .. p*Nl + Nl - 1 of the
// B x Hl heads, token-major), row ((p*B + b)*Nl + n % Nl)*Hl + h for
// bh = b*Hl + h, p = n / Nl.
struct RowMap {
  int P, B, Nl, Hl;
  __host__ __device__ long long row(int bh, int n, int N) const {
    if (P == 0) return (long long)bh * N + n;
    const int b = bh / Hl, h = bh - b * Hl, p = n / Nl, nl = n - p * Nl;
    return (((long long)p * B + b) * Nl + nl) * Hl + h;
  }
};

// Prepass scratch: per (bh, key block, channel) fp64 partial sums, fp32
// block min / max of K and block absmax of V; per (bh, channel) V absmax.
struct PrepassScratch {
  double* k_psum;
  float* k_pmin;
  float* k_pmax;
  float* v_pamax;
  float* v_amax;
};
size_t prepass_scratch_bytes(int BH, int N, int d);
PrepassScratch prepass_scratch_carve(void* base, int BH, int N, int d);

// q_per_token: q_scale is [BH, Npad] (one scale per token) instead of [BH, nT].
// in_map: where token n of head bh sits in q, k and v.
cudaError_t launch_prepass(const void* q, const void* k, const void* v, int BH, int N, int d, int8_t* q_i8,
                           float* q_scale, int8_t* k_i8, float* k_scale, float* k_mean, uint8_t* v_f8t,
                           float* v_scale, const PrepassScratch& scratch, cudaStream_t stream,
                           bool q_per_token = false, RowMap in_map = RowMap{0, 0, 0, 0});

// Quantized attention (INT8 QK^T, FP8 PV).  status: device uint32 word.
cudaError_t launch_attn_i8f8(const int8_t* q_i8, const float* q_scale, const int8_t* k_i8, const float* k_scale,
                             const uint8_t* v_f8t, const float* v_scale, void* o, int BH, int N, int d,
                             uint32_t* status, long long timeout_cycles, int dbg_flags, cudaStream_t stream,
                             bool q_per_token = false, RowMap o_map = RowMap{0, 0, 0, 0});

// BF16 attention.
cudaError_t launch_attn_bf16(const void* q, const void* k, const void* v, void* o, int BH, int N, int d,
                             uint32_t* status, long long timeout_cycles, cudaStream_t stream,
                             RowMap o_map = RowMap{0, 0, 0, 0});

// 8-bit linear layers with 128 x 128 block scales.
cudaError_t launch_quant_blocks_2d(const void* x, int R, int K, int8_t* codes, float* scales, cudaStream_t stream);
cudaError_t launch_linear_w8a8(const int8_t* xq, const float* sx, const int8_t* wq, const float* sw, const void* bias,
                               void* y, int y_f32, int M, int N, int K, uint32_t* status, long long timeout_cycles,
                               int dbg_flags, cudaStream_t stream);
cudaError_t launch_dequant_blocks_2d(const int8_t* codes, const float* scales, int R, int K, void* out,
                                     cudaStream_t stream);
cudaError_t launch_linear_bf16(const void* x, const void* w, const void* bias, void* y, int y_f32, int M, int N,
                               int K, uint32_t* status, long long timeout_cycles, int dbg_flags, cudaStream_t stream);

// Ulysses layout permutations (op 0..3, see ulysses.cu).
cudaError_t launch_ulysses_permute(const void* src, void* dst, int B, int Nl, int H, int d, int P, int op,
                                   long long chunk_rows, long long base_rows, cudaStream_t stream);

// Tensor-core throughput probe (kind: kKindF16 / kKindF8F6F4 / kKindI8 of sm100.cuh; n 128 or 256).
cudaError_t launch_mma_peak(int kind, int n, int iters, long long* cycles, uint32_t* status, int grid,
                            cudaStream_t stream);

// Diagnostics.
cudaError_t launch_dbg_qk_tiles(const int8_t* q_i8, const int8_t* k_i8, int BH, int H, int N, int d,
                                const int* tile_list, int n, int32_t* out, cudaStream_t stream);
cudaError_t launch_dbg_pv_tile(const void* p, const void* vt, int d, int mode, float* out, cudaStream_t stream);
cudaError_t launch_dbg_qk_bf16_tile(const void* q, const void* k, int d, float* out, cudaStream_t stream);

// Tensor-map encoding through the driver entry point (no libcuda link).
bool encode_tmap_2d(void* map, CUtensorMapDataType dtype, const void* base, uint64_t inner, uint64_t outer,
                    uint64_t outer_stride_bytes, uint32_t box_inner, uint32_t box_outer,
                    CUtensorMapSwizzle swizzle);
bool encode_tmap_3d(void* map, CUtensorMapDataType dtype, const void* base, uint64_t d0, uint64_t d1,
                    uint64_t d2, uint64_t stride1_bytes, uint64_t stride2_bytes, uint32_t box0, uint32_t box1,
                    uint32_t box2, CUtensorMapSwizzle swizzle);

// Unique id of the current CUDA context (0 if it cannot be read); a new id
// after cudaDeviceReset tells cached per-device handles to be made again.
unsigned long long current_context_id();

// Default wait limit of the bounded device waits, in SM clocks (~1-2 s).
constexpr long long kDefaultTimeoutCycles = 2000000000LL;

}  // namespace sage
