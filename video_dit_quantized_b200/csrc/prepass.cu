// prepass.cu -- the quantization prepass of the SageAttention-style scheme
// (page 1 of the TMAP write-up, "Attention performance optimisation":
// SageAttention operator; zero-channel fix under "operator details").
//
// Three HBM-bound kernels, one CTA per (128-token block, head) where a block
// is involved (the inputs are read through a RowMap: the plain [B,H,N,d]
// layout, or the sequence-parallel exchange layout [P][B][Nl][Hl][d]):
//   stats     : Q block -> absmax -> INT8 codes + q_scale (single pass);
//               K block -> per-channel fp64 partial sums (ascending tokens),
//               fp32 min / max;  V block -> per-channel absmax.
//   finalize  : per head, k_mean = fp32(sum of partials in ascending block
//               order / N) and v_scale = amax / 448.
//   quant_kv  : K block -> k_scale from (min, max, mean), smoothed INT8 codes;
//               V block -> e4m3 codes of V * (448 / amax), written transposed.
// All roundings are explicit (__f*_rn, cvt.rni, cvt.rn.satfinite) so that the
// results are bit-for-bit those of the scheme's definition.
#include <cuda_bf16.h>
#include <cstdint>

#include "internal.h"
#include "sm100.cuh"

namespace sage {

namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ void unpack8(const uint4& u, float (&x)[8]) {
  x[0] = bf16_lo(u.x); x[1] = bf16_hi(u.x);
  x[2] = bf16_lo(u.y); x[3] = bf16_hi(u.y);
  x[4] = bf16_lo(u.z); x[5] = bf16_hi(u.z);
  x[6] = bf16_lo(u.w); x[7] = bf16_hi(u.w);
}

__device__ __forceinline__ int quant_i8(float x, float inv) {
  int c = __float2int_rn(__fmul_rn(x, inv));
  return max(-127, min(127, c));
}

__device__ __forceinline__ uint2 pack_i8x8(const int (&c)[8]) {
  uint2 r;
  r.x = (uint32_t)(c[0] & 0xFF) | ((uint32_t)(c[1] & 0xFF) << 8) | ((uint32_t)(c[2] & 0xFF) << 16) |
        ((uint32_t)(c[3] & 0xFF) << 24);
  r.y = (uint32_t)(c[4] & 0xFF) | ((uint32_t)(c[5] & 0xFF) << 8) | ((uint32_t)(c[6] & 0xFF) << 16) |
        ((uint32_t)(c[7] & 0xFF) << 24);
  return r;
}

__device__ __forceinline__ float block_max(float v, float* red) {
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  float r = red[0];
  for (int i = 1; i < kThreads / 32; ++i) r = fmaxf(r, red[i]);
  return r;
}

// grid (nK, BH), or (nK * BH) with the head fastest when CHUNKED.  TOKQ: Q gets one scale per token (q_scale [BH, Npad]) instead
// of one per 128-token block (q_scale [BH, nK]).
template <int D, bool TOKQ, bool CHUNKED>
__global__ void __launch_bounds__(kThreads, 3) prepass_stats_kernel(const uint4* __restrict__ q,
                                                                 const uint4* __restrict__ k,
                                                                 const uint4* __restrict__ v, int N, int Npad,
                                                                 int8_t* __restrict__ q_i8,
                                                                 float* __restrict__ q_scale, PrepassScratch scr,
                                                                 RowMap in_map) {
  constexpr int V8 = D / 8;                        // uint4 per token row
  constexpr int PER_T = kTile * V8 / kThreads;     // uint4 per thread per block
  static_assert(kThreads % V8 == 0, "a thread must always see the same 8 channels");
  __shared__ __align__(16) uint4 ks[kTile * V8];
  __shared__ int vamax_s[D];                       // non-negative floats as int bits
  __shared__ float red[kThreads / 32];

  // chunked layout: a 1-D grid, head fastest, so that the CTAs resident at one
  // time read the same token tile of every local head, one contiguous range
  const int BHc = CHUNKED ? in_map.B * in_map.Hl : 1;
  const int kb = CHUNKED ? (int)(blockIdx.x / BHc) : (int)blockIdx.x;
  const int bh = CHUNKED ? (int)(blockIdx.x % BHc) : (int)blockIdx.y;
  const int nK = CHUNKED ? (int)(gridDim.x / BHc) : (int)gridDim.x;
  const int n0 = kb * kTile;
  const int nr = min(kTile, N - n0);
  const size_t in_base = ((size_t)bh * N + n0) * V8;  // plain layout, in uint4
  // buffer extents, for the checks of a debug build
  const long long BHt = CHUNKED ? BHc : (int)gridDim.y;
  const long long in_ext = BHt * N * V8, i8_ext = BHt * Npad * D / 8, part_ext = BHt * nK * D;
  (void)in_ext; (void)i8_ext; (void)part_ext;

  if (threadIdx.x < D) vamax_s[threadIdx.x] = 0;

  // ---- Q: absmax over the block, then INT8 codes (one read) ----
  uint4 qv[PER_T];
  float amax = 0.f;
  float va[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};   // V absmax of this thread's 8 channels
#pragma unroll
  for (int i = 0; i < PER_T; ++i) {
    const int e = threadIdx.x + i * kThreads;       // uint4 index within block
    const int row = e / V8;
    qv[i] = make_uint4(0, 0, 0, 0);
    if (row < nr) {
      const size_t at = CHUNKED ? (size_t)in_map.row(bh, n0 + row, N) * V8 + (e % V8) : in_base + e;
      if (SAGE_DCHECK(at, in_ext, kSiteStatsIn)) {
        qv[i] = q[at];
        ks[e] = k[at];
        float y[8];
        unpack8(v[at], y);
#pragma unroll
        for (int u = 0; u < 8; ++u) va[u] = fmaxf(va[u], fabsf(y[u]));
      }
    }
    float x[8];
    unpack8(qv[i], x);
#pragma unroll
    for (int u = 0; u < 8; ++u) amax = fmaxf(amax, fabsf(x[u]));
  }
  amax = block_max(amax, red);   // also orders the vamax_s initialisation and the K staging (and is
                                 // the block absmax of Q for the per-block scale)
  {
    const int c0 = (threadIdx.x % V8) * 8;
#pragma unroll
    for (int u = 0; u < 8; ++u) atomicMax(&vamax_s[c0 + u], __float_as_int(va[u]));
  }
  uint2* qo = reinterpret_cast<uint2*>(q_i8 + ((size_t)bh * Npad + n0) * D);
  if constexpr (!TOKQ) {
    const float qinv = amax > 0.f ? __fdiv_rn(127.0f, amax) : 0.f;
    if (threadIdx.x == 0 && SAGE_DCHECK((size_t)bh * nK + kb, BHt * nK, kSiteStatsQScale))
      q_scale[(size_t)bh * nK + kb] = amax > 0.f ? __fdiv_rn(amax, 127.0f) : 0.f;
#pragma unroll
    for (int i = 0; i < PER_T; ++i) {
      const int e = threadIdx.x + i * kThreads;
      float x[8];
      unpack8(qv[i], x);
      int c[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) c[u] = qinv > 0.f ? quant_i8(x[u], qinv) : 0;
      if (SAGE_DCHECK(((size_t)bh * Npad + n0) * D / 8 + e, i8_ext, kSiteStatsQ8))
        qo[e] = pack_i8x8(c);   // rows >= nr hold zeros (qv was zeroed)
    }
  } else {
    // the V8 consecutive lanes that hold one token reduce its absmax
#pragma unroll
    for (int i = 0; i < PER_T; ++i) {
      const int e = threadIdx.x + i * kThreads;
      float x[8];
      unpack8(qv[i], x);
      float ra = 0.f;
#pragma unroll
      for (int u = 0; u < 8; ++u) ra = fmaxf(ra, fabsf(x[u]));
#pragma unroll
      for (int o = V8 / 2; o > 0; o >>= 1) ra = fmaxf(ra, __shfl_xor_sync(0xffffffffu, ra, o));
      const float rinv = ra > 0.f ? __fdiv_rn(127.0f, ra) : 0.f;
      if (e % V8 == 0 && SAGE_DCHECK((size_t)bh * Npad + n0 + e / V8, BHt * Npad, kSiteStatsQScale))
        q_scale[(size_t)bh * Npad + n0 + e / V8] = ra > 0.f ? __fdiv_rn(ra, 127.0f) : 0.f;
      int c[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) c[u] = rinv > 0.f ? quant_i8(x[u], rinv) : 0;
      if (SAGE_DCHECK(((size_t)bh * Npad + n0) * D / 8 + e, i8_ext, kSiteStatsQ8))
        qo[e] = pack_i8x8(c);   // rows >= nr: zero codes and scale 0
    }
  }
  __syncthreads();

  // ---- K column statistics (thread per channel, ascending tokens) ----
  const __nv_bfloat16* kh = reinterpret_cast<const __nv_bfloat16*>(ks);
  const size_t pidx = ((size_t)bh * nK + kb) * D;
  if (threadIdx.x < D) {
    const int c = threadIdx.x;
    double s = 0.0;
    float mn = __bfloat162float(kh[c]), mx = mn;
    for (int n = 0; n < nr; ++n) {
      const float x = __bfloat162float(kh[n * D + c]);
      s = __dadd_rn(s, (double)x);
      mn = fminf(mn, x);
      mx = fmaxf(mx, x);
    }
    if (SAGE_DCHECK(pidx + c, part_ext, kSiteStatsPartials)) {
      scr.k_psum[pidx + c] = s;
      scr.k_pmin[pidx + c] = mn;
      scr.k_pmax[pidx + c] = mx;
      scr.v_pamax[pidx + c] = __int_as_float(vamax_s[c]);
    }
  }
}

// grid (BH, D / 32), block 64.  Warp 0 adds the K partial sums of 32
// channels in ascending block order (the fp64 order of the K mean), warp 1
// takes the V absmax of the same channels.  Each lane walks its channel's
// column of partials (a warp reads 32 consecutive channels of one block per
// load, 256 or 128 contiguous bytes) with the next kFinBatch blocks' loads in
// flight while it adds the current ones, so the chain of additions, not the
// load latency, sets the time.
constexpr int kFinBatch = 32;
template <int D>
__global__ void __launch_bounds__(64) prepass_finalize_kernel(int N, int nK, PrepassScratch scr,
                                                              float* __restrict__ k_mean,
                                                              float* __restrict__ v_scale) {
  const int bh = blockIdx.x;
  const int c = blockIdx.y * 32 + (threadIdx.x & 31);
  const size_t col = (size_t)bh * nK * D + c;       // partial (bh, block 0, c); block t is t * D further
  const long long part_ext = (long long)gridDim.x * nK * D, out_ext = (long long)gridDim.x * D;
  (void)part_ext; (void)out_ext;
  if (threadIdx.x < 32) {
    const double* gs = scr.k_psum + col;
    double total = 0.0;
    double A[kFinBatch], B[kFinBatch];
    auto load = [&](double(&r)[kFinBatch], int t0) {
#pragma unroll
      for (int i = 0; i < kFinBatch; ++i)
        r[i] = t0 + i < nK && SAGE_DCHECK(col + (size_t)(t0 + i) * D, part_ext, kSiteFinIn) ? gs[(size_t)(t0 + i) * D]
                                                                                           : 0.0;
    };
    auto add = [&](const double(&r)[kFinBatch], int t0) {
#pragma unroll
      for (int i = 0; i < kFinBatch; ++i)
        if (t0 + i < nK) total = __dadd_rn(total, r[i]);
    };
    load(A, 0);
    for (int t0 = 0; t0 < nK; t0 += 2 * kFinBatch) {
      load(B, t0 + kFinBatch);
      add(A, t0);
      load(A, t0 + 2 * kFinBatch);
      add(B, t0 + kFinBatch);
    }
    if (SAGE_DCHECK((size_t)bh * D + c, out_ext, kSiteFinOut))
      k_mean[(size_t)bh * D + c] = __double2float_rn(__ddiv_rn(total, (double)N));
  } else {
    const float* ga = scr.v_pamax + col;
    float a = 0.f;
    float A[kFinBatch], B[kFinBatch];
    auto load = [&](float(&r)[kFinBatch], int t0) {
#pragma unroll
      for (int i = 0; i < kFinBatch; ++i)
        r[i] = t0 + i < nK && SAGE_DCHECK(col + (size_t)(t0 + i) * D, part_ext, kSiteFinIn) ? ga[(size_t)(t0 + i) * D]
                                                                                           : 0.f;
    };
    auto take = [&](const float(&r)[kFinBatch]) {
#pragma unroll
      for (int i = 0; i < kFinBatch; ++i) a = fmaxf(a, r[i]);   // absmax partials are >= 0; padding adds 0
    };
    load(A, 0);
    for (int t0 = 0; t0 < nK; t0 += 2 * kFinBatch) {
      load(B, t0 + kFinBatch);
      take(A);
      load(A, t0 + 2 * kFinBatch);
      take(B);
    }
    if (SAGE_DCHECK((size_t)bh * D + c, out_ext, kSiteFinOut)) {
      v_scale[(size_t)bh * D + c] = a > 0.f ? __fdiv_rn(a, 448.0f) : 0.f;
      scr.v_amax[(size_t)bh * D + c] = a;
    }
  }
}

// grid (nK, BH), or (nK * BH) with the head fastest when CHUNKED
template <int D, bool CHUNKED>
__global__ void __launch_bounds__(kThreads) prepass_quant_kv_kernel(const uint4* __restrict__ k,
                                                                    const uint4* __restrict__ v, int N, int Npad,
                                                                    const float* __restrict__ k_mean,
                                                                    int8_t* __restrict__ k_i8,
                                                                    float* __restrict__ k_scale,
                                                                    uint8_t* __restrict__ v_f8t, PrepassScratch scr,
                                                                    RowMap in_map) {
  constexpr int V8 = D / 8;
  constexpr int PER_T = kTile * V8 / kThreads;
  __shared__ float mean_s[D];
  __shared__ float vinv_s[D];
  __shared__ __align__(16) uint4 vs[kTile * V8];
  __shared__ float red[kThreads / 32];

  // chunked layout: a 1-D grid, head fastest, so that the CTAs resident at one
  // time read the same token tile of every local head, one contiguous range
  const int BHc = CHUNKED ? in_map.B * in_map.Hl : 1;
  const int kb = CHUNKED ? (int)(blockIdx.x / BHc) : (int)blockIdx.x;
  const int bh = CHUNKED ? (int)(blockIdx.x % BHc) : (int)blockIdx.y;
  const int nK = CHUNKED ? (int)(gridDim.x / BHc) : (int)gridDim.x;
  const int n0 = kb * kTile;
  const int nr = min(kTile, N - n0);
  const size_t in_base = ((size_t)bh * N + n0) * V8;  // plain layout, in uint4
  const size_t pidx = ((size_t)bh * nK + kb) * D;
  // buffer extents, for the checks of a debug build
  const long long BHt = CHUNKED ? BHc : (int)gridDim.y;
  const long long in_ext = BHt * N * V8, i8_ext = BHt * Npad * D / 8, part_ext = BHt * nK * D, ch_ext = BHt * D;
  (void)in_ext; (void)i8_ext; (void)part_ext; (void)ch_ext;

  // the block's K and V rows go in flight first; the scales below only need
  // the per-head and per-block statistics
  uint4 kr[PER_T], vr[PER_T];
#pragma unroll
  for (int i = 0; i < PER_T; ++i) {
    const int e = threadIdx.x + i * kThreads;
    const int row = e / V8;
    kr[i] = vr[i] = make_uint4(0, 0, 0, 0);
    if (row < nr) {
      const size_t at = CHUNKED ? (size_t)in_map.row(bh, n0 + row, N) * V8 + (e % V8) : in_base + e;
      if (SAGE_DCHECK(at, in_ext, kSiteQuantIn)) {
        kr[i] = k[at];
        vr[i] = v[at];
      }
    }
  }

  // k_scale of this block from the partial min / max: fp32 subtraction is
  // monotone, so max|fl(x - m)| over the block is attained at its min or max.
  float kam = 0.f;
  if (threadIdx.x < D) {
    const int c = threadIdx.x;
    float m = 0.f, a = 0.f;
    if (SAGE_DCHECK((size_t)bh * D + c, ch_ext, kSiteQuantPartials)) {
      m = k_mean[(size_t)bh * D + c];
      a = scr.v_amax[(size_t)bh * D + c];
    }
    mean_s[c] = m;
    if (SAGE_DCHECK(pidx + c, part_ext, kSiteQuantPartials))
      kam = fmaxf(fabsf(__fsub_rn(scr.k_pmax[pidx + c], m)), fabsf(__fsub_rn(scr.k_pmin[pidx + c], m)));
    vinv_s[c] = a > 0.f ? __fdiv_rn(448.0f, a) : 0.f;
  }
  kam = block_max(kam, red);   // contains __syncthreads
  const float kinv = kam > 0.f ? __fdiv_rn(127.0f, kam) : 0.f;
  if (threadIdx.x == 0 && SAGE_DCHECK((size_t)bh * nK + kb, BHt * nK, kSiteQuantKScale))
    k_scale[(size_t)bh * nK + kb] = kam > 0.f ? __fdiv_rn(kam, 127.0f) : 0.f;

  // ---- K: smoothed INT8 codes ----
  uint2* ko = reinterpret_cast<uint2*>(k_i8 + ((size_t)bh * Npad + n0) * D);
#pragma unroll
  for (int i = 0; i < PER_T; ++i) {
    const int e = threadIdx.x + i * kThreads;
    const int row = e / V8, c0 = (e % V8) * 8;
    int c[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    if (row < nr && kinv > 0.f) {
      float x[8];
      unpack8(kr[i], x);
#pragma unroll
      for (int u = 0; u < 8; ++u) c[u] = quant_i8(__fsub_rn(x[u], mean_s[c0 + u]), kinv);
    }
    if (SAGE_DCHECK(((size_t)bh * Npad + n0) * D / 8 + e, i8_ext, kSiteQuantK8)) ko[e] = pack_i8x8(c);
  }

  // ---- V: stage the block (padding rows +0), then e4m3 codes written channel-major ----
#pragma unroll
  for (int i = 0; i < PER_T; ++i) vs[threadIdx.x + i * kThreads] = vr[i];
  __syncthreads();
  const __nv_bfloat16* vh = reinterpret_cast<const __nv_bfloat16*>(vs);
  constexpr int PAIRS = D * (kTile / 16);   // (channel, 16-token chunk)
#pragma unroll
  for (int i = 0; i < PAIRS / kThreads; ++i) {
    const int p = threadIdx.x + i * kThreads;
    const int c = p % D, chunk = p / D;
    const float inv = vinv_s[c];
    uint32_t w[4];
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      float x[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int n = chunk * 16 + g * 4 + u;
        x[u] = __fmul_rn(__bfloat162float(vh[n * D + c]), inv);
      }
      w[g] = inv > 0.f ? pack_e4m3x4(x[0], x[1], x[2], x[3]) : 0u;
    }
    // padding tokens (n >= nr) were staged as +0 and encode to 0x00
    const size_t off = ((size_t)bh * D + c) * Npad + (size_t)n0 + chunk * 16;   // bytes, a multiple of 16
    if (SAGE_DCHECK(off / 16, BHt * D * Npad / 16, kSiteQuantV8))
      *reinterpret_cast<uint4*>(v_f8t + off) = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

template <int D>
cudaError_t launch_prepass_d(const void* q, const void* k, const void* v, int BH, int N, int8_t* q_i8,
                             float* q_scale, int8_t* k_i8, float* k_scale, float* k_mean, uint8_t* v_f8t,
                             float* v_scale, const PrepassScratch& scr, bool q_per_token, cudaStream_t stream,
                             RowMap in_map) {
  const int nK = num_tiles(N), Npad = nK * kTile;
  const bool chunked = in_map.P != 0;
  if (chunked && in_map.B * in_map.Hl != BH) return cudaErrorInvalidValue;
  const dim3 grid = chunked ? dim3((unsigned)nK * BH) : dim3(nK, BH);
  const uint4* q4 = static_cast<const uint4*>(q);
  const uint4* k4 = static_cast<const uint4*>(k);
  const uint4* v4 = static_cast<const uint4*>(v);
  if (q_per_token && chunked)
    prepass_stats_kernel<D, true, true><<<grid, kThreads, 0, stream>>>(q4, k4, v4, N, Npad, q_i8, q_scale, scr, in_map);
  else if (q_per_token)
    prepass_stats_kernel<D, true, false><<<grid, kThreads, 0, stream>>>(q4, k4, v4, N, Npad, q_i8, q_scale, scr, in_map);
  else if (chunked)
    prepass_stats_kernel<D, false, true><<<grid, kThreads, 0, stream>>>(q4, k4, v4, N, Npad, q_i8, q_scale, scr, in_map);
  else
    prepass_stats_kernel<D, false, false><<<grid, kThreads, 0, stream>>>(q4, k4, v4, N, Npad, q_i8, q_scale, scr, in_map);
  prepass_finalize_kernel<D><<<dim3(BH, D / 32), 64, 0, stream>>>(N, nK, scr, k_mean, v_scale);
  if (chunked)
    prepass_quant_kv_kernel<D, true><<<grid, kThreads, 0, stream>>>(k4, v4, N, Npad, k_mean, k_i8, k_scale, v_f8t, scr,
                                                                    in_map);
  else
    prepass_quant_kv_kernel<D, false><<<grid, kThreads, 0, stream>>>(k4, v4, N, Npad, k_mean, k_i8, k_scale, v_f8t, scr,
                                                                     in_map);
  return cudaGetLastError();
}

__global__ void debug_selftest_kernel() {
  // one check that fails (index == extent); nothing is read or written
  (void)SAGE_DCHECK(1, 1, kSiteSelftest);
}

}  // namespace

unsigned debug_take_prepass(unsigned long long* first) {
#ifdef SAGE_DEBUG
  return debug_take_tu(first);
#else
  (void)first;
  return 0;
#endif
}

cudaError_t launch_debug_selftest(cudaStream_t stream) {
  debug_selftest_kernel<<<1, 1, 0, stream>>>();
  return cudaGetLastError();
}

size_t prepass_scratch_bytes(int BH, int N, int d) {
  const size_t n = (size_t)BH * num_tiles(N) * d;
  return align_up(n * 8, 256) + 3 * align_up(n * 4, 256) + align_up((size_t)BH * d * 4, 256);
}

PrepassScratch prepass_scratch_carve(void* base, int BH, int N, int d) {
  const size_t n = (size_t)BH * num_tiles(N) * d;
  char* p = static_cast<char*>(base);
  PrepassScratch s;
  s.k_psum = reinterpret_cast<double*>(p);
  p += align_up(n * 8, 256);
  s.k_pmin = reinterpret_cast<float*>(p);
  p += align_up(n * 4, 256);
  s.k_pmax = reinterpret_cast<float*>(p);
  p += align_up(n * 4, 256);
  s.v_pamax = reinterpret_cast<float*>(p);
  p += align_up(n * 4, 256);
  s.v_amax = reinterpret_cast<float*>(p);
  return s;
}

cudaError_t launch_prepass(const void* q, const void* k, const void* v, int BH, int N, int d, int8_t* q_i8,
                           float* q_scale, int8_t* k_i8, float* k_scale, float* k_mean, uint8_t* v_f8t,
                           float* v_scale, const PrepassScratch& scratch, cudaStream_t stream, bool q_per_token,
                           RowMap in_map) {
  if (d == 128)
    return launch_prepass_d<128>(q, k, v, BH, N, q_i8, q_scale, k_i8, k_scale, k_mean, v_f8t, v_scale, scratch,
                                 q_per_token, stream, in_map);
  if (d == 64)
    return launch_prepass_d<64>(q, k, v, BH, N, q_i8, q_scale, k_i8, k_scale, k_mean, v_f8t, v_scale, scratch,
                                q_per_token, stream, in_map);
  return cudaErrorInvalidValue;
}

}  // namespace sage
