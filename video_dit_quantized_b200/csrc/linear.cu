// linear.cu -- 8-bit linear layers with 128 x 128 block scales.
//
// TMAP write-up, "FFN performance optimisation / linear-layer quantization":
// the DiT's linear layers run with 8-bit weights and activations (W8A8), each
// operand quantized per 128 x 128 block.  Two kernels:
//
//   quant_blocks_2d_kernel   bf16 [R, K] -> int8 codes [R, K] and one fp32
//                            scale per 128 x 128 block (absmax / 127, RNE,
//                            zero guard), one CTA per block.
//   linear_w8a8_kernel       Y[m, n] = sum over K blocks kb of
//                            (sx[m/128, kb] * sw[n/128, kb]) * S_kb[m, n]
//                            (+ bias[n]), S_kb the exact int32 product of one
//                            128-wide K block; fp32 sum, one FMA per block.
//
//   dequant_blocks_2d_kernel codes + block scales -> bf16(scale * code), the
//                            weights a W8A16 layer multiplies (8-bit storage,
//                            16-bit compute).
//   linear_bf16_kernel       Y = X W^T (+ bias) with bf16 X and W: the W8A16
//                            layers (W dequantized first) and plain bf16 ones.
//
// linear_w8a8_kernel is persistent, one CTA per SM, 12 warps:
//   warps 0, 2    TMA producers (one thread each): the X code tile
//                 [128 x 128] and the W code tile [256 x 128] (int8, 128-byte
//                 swizzle) of each K block into a 4-stage ring
//   warp 1        MMA issuer: four tcgen05.mma kind::i8 (M=128, N=256, K=32)
//                 per K block into one of two 256-column TMEM accumulators
//   warps 4..11   block-scale epilogue: each thread owns one output row and
//                 128 columns (warpgroup 0: columns 0..127 of the tile,
//                 warpgroup 1: 128..255) and keeps their fp32 sums in
//                 registers across the K loop.
//
// The per-block promotion (one int32 -> fp32 conversion and one FMA per
// output element and K block) is as much work per block as the MMAs, so the
// epilogue, not the tensor core, bounds this kernel: it converts with cvt
// (exact, |S_kb| <= 128 * 127 * 127 < 2^22), sums with packed fp32 FMAs, and
// hands each accumulator back to the MMA issuer as soon as the block's last
// 32 columns are in registers.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "internal.h"
#include "sm100.cuh"

namespace sage {

namespace {

// ------------------------------------------------------------ quantizer ----
// One CTA per 128 x 128 block, 256 threads; thread t covers row t / 2, columns
// 64 * (t % 2) .. +63 of the block.  Rows at or beyond R are not touched.
__global__ void __launch_bounds__(256) quant_blocks_2d_kernel(const __nv_bfloat16* __restrict__ x, int R, int K,
                                                              int8_t* __restrict__ codes, float* __restrict__ scales) {
  const int kb = blockIdx.x, rb = blockIdx.y, nk = gridDim.x;
  const int r = rb * 128 + (threadIdx.x >> 1);
  const int c0 = kb * 128 + (threadIdx.x & 1) * 64;
  const bool live = r < R;
  uint4 raw[8];
  float amax = 0.f;
  if (live) {
    const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)r * K + c0);
#pragma unroll
    for (int i = 0; i < 8; ++i) raw[i] = src[i];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint32_t w[4] = {raw[i].x, raw[i].y, raw[i].z, raw[i].w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        amax = fmaxf(amax, fabsf(__uint_as_float(w[j] << 16)));
        amax = fmaxf(amax, fabsf(__uint_as_float(w[j] & 0xFFFF0000u)));
      }
    }
  }
  // |x| >= 0, so the float order is the unsigned order of the bit patterns
  __shared__ uint32_t wmax[8];
  const uint32_t m = __reduce_max_sync(0xFFFFFFFFu, __float_as_uint(amax));
  if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = m;
  __syncthreads();
  uint32_t bm = wmax[0];
#pragma unroll
  for (int i = 1; i < 8; ++i) bm = max(bm, wmax[i]);
  const float bmax = __uint_as_float(bm);
  if (threadIdx.x == 0) scales[(size_t)rb * nk + kb] = bmax == 0.f ? 0.f : __fdiv_rn(bmax, 127.f);
  if (!live) return;
  uint4* dst = reinterpret_cast<uint4*>(codes + (size_t)r * K + c0);
  if (bmax == 0.f) {
#pragma unroll
    for (int i = 0; i < 4; ++i) dst[i] = make_uint4(0, 0, 0, 0);
    return;
  }
  const float inv = __fdiv_rn(127.f, bmax);
  uint32_t out[16];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint32_t w[4] = {raw[i].x, raw[i].y, raw[i].z, raw[i].w};
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      uint32_t pk = 0;
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        const uint32_t bits = w[2 * j + (h >> 1)];
        const float v = __uint_as_float((h & 1) ? (bits & 0xFFFF0000u) : (bits << 16));
        int q = __float2int_rn(__fmul_rn(v, inv));
        q = max(-127, min(127, q));
        pk |= (uint32_t)(q & 0xFF) << (8 * h);
      }
      out[2 * i + j] = pk;
    }
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) dst[i] = make_uint4(out[4 * i], out[4 * i + 1], out[4 * i + 2], out[4 * i + 3]);
}

// ---------------------------------------------------------- dequantizer ----
// One CTA per 128 x 128 block, 256 threads; thread t covers row t / 2, columns
// 64 * (t % 2) .. +63: out = bf16_rne(fl(scale * code)).
__global__ void __launch_bounds__(256) dequant_blocks_2d_kernel(const int8_t* __restrict__ codes,
                                                                const float* __restrict__ scales, int R, int K,
                                                                __nv_bfloat16* __restrict__ out) {
  const int kb = blockIdx.x, rb = blockIdx.y, nk = gridDim.x;
  const int r = rb * 128 + (threadIdx.x >> 1);
  if (r >= R) return;
  const int c0 = kb * 128 + (threadIdx.x & 1) * 64;
  const float sc = scales[(size_t)rb * nk + kb];
  const uint4* src = reinterpret_cast<const uint4*>(codes + (size_t)r * K + c0);
  uint4* dst = reinterpret_cast<uint4*>(out + (size_t)r * K + c0);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint4 q = src[i];
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
    uint32_t o[8];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float v0 = __fmul_rn(sc, (float)(int8_t)(w[j] & 0xFF));
      const float v1 = __fmul_rn(sc, (float)(int8_t)((w[j] >> 8) & 0xFF));
      const float v2 = __fmul_rn(sc, (float)(int8_t)((w[j] >> 16) & 0xFF));
      const float v3 = __fmul_rn(sc, (float)(int8_t)(w[j] >> 24));
      o[2 * j] = pack_bf16x2(v0, v1);
      o[2 * j + 1] = pack_bf16x2(v2, v3);
    }
    dst[2 * i] = make_uint4(o[0], o[1], o[2], o[3]);
    dst[2 * i + 1] = make_uint4(o[4], o[5], o[6], o[7]);
  }
}

// ------------------------------------------------------------ tile order ---
// Persistent CTAs walk the output tiles in groups of `group_m` row bands:
// inside a group the row band changes fastest, then the column band.  With
// group_m = 16 the ~148 tiles in flight span 16 row bands of X and ~9 column
// bands of W, so both stay in L2 even when W is larger than L2 (W is then
// re-read once per group); group_m = 1 is the plain column-fastest order,
// better when all of W stays in L2 anyway.
__device__ __forceinline__ void tile_coords(int t, int n_tiles_m, int n_tiles_n, int group_m, int& mt, int& nt) {
  const int per_group = group_m * n_tiles_n;
  const int grp = t / per_group;
  const int m0 = grp * group_m;
  const int rows = min(group_m, n_tiles_m - m0);
  const int r = t - grp * per_group;
  mt = m0 + r % rows;
  nt = r / rows;
}

// ------------------------------------------------------------ W8A8 GEMM ----
constexpr int kThreads = 384;
constexpr int kLaunchRegs = 168;                 // 65536 / 384, rounded down to a multiple of 8
constexpr int BM = 128, BN = 256, BK = 128;
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK, B_BYTES = BN * BK, STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int OFF_BAR = STAGES * STAGE_BYTES;
constexpr int SMEM_BYTES = OFF_BAR + 256 + 1024;
constexpr int REGS_LOW = 40, REGS_HIGH = 232;
constexpr uint32_t kTmemCols = 512;              // two 256-column accumulators
constexpr uint32_t IDESC = make_idesc(kFmtS32Acc, kFmtS8, kFmtS8, 0, BM, BN);
static_assert(128 * REGS_LOW + 256 * REGS_HIGH <= kThreads * kLaunchRegs, "register split exceeds the launch budget");
static_assert(SMEM_BYTES <= 232448, "shared memory budget");

struct LinParams {
  const float* sx;          // [ceil(M/128), nk]
  const float* sw;          // [N/128, nk]
  const __nv_bfloat16* bias;  // [N] or null
  void* y;                  // [M, N] bf16 or fp32
  uint32_t* status;
  int M, N, nk, n_tiles_m, n_tiles_n, n_tiles, group_m;
  int y_f32;
  long long timeout;
  int dbg_flags;            // bit 0: the MMA thread first waits on a barrier nobody arrives on
};

__global__ void __launch_bounds__(kThreads, 1)
    linear_w8a8_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                       const LinParams prm) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint64_t* full = bars;                    // [STAGES] operand tiles landed (two producers)
  uint64_t* empty = bars + STAGES;          // [STAGES] operand tiles consumed by the MMAs
  uint64_t* tfull = bars + 2 * STAGES;      // [2] accumulator holds a finished K block
  uint64_t* tempty = tfull + 2;             // [2] accumulator read and re-biased (8 warp arrivals)
  uint64_t* mma_done = tempty + 2;
  uint64_t* never = mma_done + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(never + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nk = prm.nk;
  const long long limit = prm.timeout;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 2);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 8);
    }
    mbar_init(mma_done, 1);
    mbar_init(never, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp < 4) {
    regs_release<REGS_LOW>();
    if ((warp == 0 || warp == 2) && lane == 0) {
      // ---------------------------------------------------------- producers
      // warp 0 loads the X tiles, warp 2 the W tiles: one thread issues TMA
      // boxes at about half the rate the MMAs consume them
      const bool is_x = warp == 0;
      const CUtensorMap* map = is_x ? &tmX : &tmW;
      const uint32_t bytes = is_x ? A_BYTES : B_BYTES;
      tma_prefetch_desc(map);
      long long g = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < prm.n_tiles; t += gridDim.x) {
        int mt, nt;
        tile_coords(t, prm.n_tiles_m, prm.n_tiles_n, prm.group_m, mt, nt);
        const int row0 = is_x ? mt * BM : nt * BN;
        for (int kb = 0; kb < nk; ++kb, ++g) {
          const int s = (int)(g % STAGES);
          if (g >= STAGES && !mbar_wait(&empty[s], (uint32_t)((g / STAGES) - 1) & 1u, abort_flag, limit)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[s], bytes);
          tma_load_2d(smem + s * STAGE_BYTES + (is_x ? 0 : A_BYTES), map, &full[s], kb * BK, row0);
        }
      }
      // drain: every load issued must land before the CTA exits
      volatile int no_abort = 0;
      for (long long j = g - STAGES < 0 ? 0 : g - STAGES; j < g; ++j)
        mbar_wait(&full[j % STAGES], (uint32_t)(j / STAGES) & 1u, &no_abort, limit);
    } else if (warp == 1 && lane == 0) {
      // ---------------------------------------------------------- MMA issuer
      bool ok = true;
      if (prm.dbg_flags & 1) ok = mbar_wait(never, 0, abort_flag, limit);
      long long g = 0;
      for (int t = blockIdx.x; ok && t < prm.n_tiles; t += gridDim.x) {
        for (int kb = 0; kb < nk; ++kb, ++g) {
          const int s = (int)(g % STAGES);
          const int b = (int)(g & 1);
          if (!mbar_wait(&full[s], (uint32_t)(g / STAGES) & 1u, abort_flag, limit)) {
            ok = false;
            break;
          }
          const uint32_t a_s = smem_u32(smem + s * STAGE_BYTES);
          const uint32_t b_s = a_s + A_BYTES;
          if (!mbar_wait(&tempty[b], (uint32_t)(g >> 1) & 1u, abort_flag, limit)) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int k = 0; k < BK / 32; ++k) {
            const uint64_t ad = make_sdesc(a_s + k * 32, 16, 1024, kLayoutSW128);
            const uint64_t bd = make_sdesc(b_s + k * 32, 16, 1024, kLayoutSW128);
            mma_ss<kKindI8>(tmem + (uint32_t)b * BN, ad, bd, IDESC, k > 0 ? 1u : 0u);
          }
          mma_commit(&tfull[b]);
          mma_commit(&empty[s]);
        }
      }
      // drain: every MMA issued must complete before TMEM is released
      mma_commit(mma_done);
      volatile int no_abort = 0;
      mbar_wait(mma_done, 0, &no_abort, limit);
    }
  } else {
    regs_claim<REGS_HIGH>();
    // ------------------------------------------------------------ epilogue
    const int wg = (warp - 4) >> 2;               // column half of the tile
    const int quarter = warp & 3;                 // TMEM lane quadrant
    const int row = quarter * 32 + lane;
    const uint32_t t_lane = tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)wg * 128;
    // both accumulators start out free
    if (lane == 0) {
      mbar_arrive(&tempty[0]);
      mbar_arrive(&tempty[1]);
    }
    bool ok = true;
    long long g = 0;
    for (int t = blockIdx.x; ok && t < prm.n_tiles; t += gridDim.x) {
      int mt, nt;
      tile_coords(t, prm.n_tiles_m, prm.n_tiles_n, prm.group_m, mt, nt);
      const int nb = nt * 2 + wg;                       // 128-column scale block of this warpgroup
      const bool cols_live = nb * 128 < prm.N;
      const float* sxr = prm.sx + (size_t)mt * nk;
      const float* swr = prm.sw + (size_t)(cols_live ? nb : 0) * nk;
      float acc[128];
#pragma unroll
      for (int i = 0; i < 128; ++i) acc[i] = 0.f;
      // block scales in windows of 32 K blocks: lane l holds fl(sx * sw) of block w0 + l;
      // the next window's raw scales are loaded one window ahead (multiplied at the switch)
      auto load_window = [&](int w0, float& a, float& c) {
        const int kb = w0 + lane;
        const bool live = cols_live && kb < nk;
        a = live ? sxr[kb] : 0.f;
        c = live ? swr[kb] : 0.f;
      };
      float xa, wa, xn = 0.f, wn = 0.f;
      load_window(0, xa, wa);
      if (nk > 32) load_window(32, xn, wn);
      float sc_win = __fmul_rn(xa, wa);
      for (int kb = 0; kb < nk; ++kb, ++g) {
        const int b = (int)(g & 1);
        if ((kb & 31) == 0 && kb > 0) {
          sc_win = __fmul_rn(xn, wn);
          if (kb + 32 < nk) load_window(kb + 32, xn, wn);
        }
        const float sc = __shfl_sync(0xFFFFFFFFu, sc_win, kb & 31);
        if (!mbar_wait(&tfull[b], (uint32_t)(g >> 1) & 1u, abort_flag, limit)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t tb = t_lane + b * BN;
        uint32_t ra[32], rb[32];
        tmem_ld32(tb, ra);
        tmem_wait_ld_regs(ra);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t(&cur)[32] = (c & 1) ? rb : ra;
          uint32_t(&nxt)[32] = (c & 1) ? ra : rb;
          if (c < 3) {
            tmem_ld32(tb + (c + 1) * 32, nxt);                // in flight while chunk c is summed
          } else {
            // the whole block is in registers: hand the accumulator back before the last chunk's sums
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[b]);
          }
#pragma unroll
          for (int j = 0; j < 32; j += 2) {
            // |S| < 2^22: the conversion is exact
            const float f0 = __int2float_rn((int)cur[j]), f1 = __int2float_rn((int)cur[j + 1]);
            uint64_t d;
            asm("fma.rn.f32x2 %0, %1, %2, %3;"
                : "=l"(d)
                : "l"(f2_pack(f0, f1)), "l"(f2_pack(sc, sc)), "l"(f2_pack(acc[c * 32 + j], acc[c * 32 + j + 1])));
            const float2 o = f2_unpack(d);
            acc[c * 32 + j] = o.x;
            acc[c * 32 + j + 1] = o.y;
          }
          if (c < 3) tmem_wait_ld_regs(nxt);
        }
      }
      if (!ok) break;
      // bias, rounding, store: this thread's row, 128 consecutive columns
      const int gm = mt * BM + row;
      if (cols_live && gm < prm.M) {
        const int n0 = nb * 128;
        if (prm.bias) {
          const uint4* bp = reinterpret_cast<const uint4*>(prm.bias + n0);
#pragma unroll
          for (int v = 0; v < 16; ++v) {
            const uint4 bb = bp[v];
            const uint32_t w[4] = {bb.x, bb.y, bb.z, bb.w};
#pragma unroll
            for (int h = 0; h < 4; ++h) {
              acc[8 * v + 2 * h] = __fadd_rn(acc[8 * v + 2 * h], __uint_as_float(w[h] << 16));
              acc[8 * v + 2 * h + 1] = __fadd_rn(acc[8 * v + 2 * h + 1], __uint_as_float(w[h] & 0xFFFF0000u));
            }
          }
        }
        if (prm.y_f32) {
          uint4* dst = reinterpret_cast<uint4*>(static_cast<float*>(prm.y) + (size_t)gm * prm.N + n0);
#pragma unroll
          for (int v = 0; v < 32; ++v)
            dst[v] = make_uint4(__float_as_uint(acc[4 * v]), __float_as_uint(acc[4 * v + 1]),
                                __float_as_uint(acc[4 * v + 2]), __float_as_uint(acc[4 * v + 3]));
        } else {
          uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(prm.y) + (size_t)gm * prm.N + n0);
#pragma unroll
          for (int v = 0; v < 16; ++v)
            dst[v] = make_uint4(pack_bf16x2(acc[8 * v], acc[8 * v + 1]), pack_bf16x2(acc[8 * v + 2], acc[8 * v + 3]),
                                pack_bf16x2(acc[8 * v + 4], acc[8 * v + 5]),
                                pack_bf16x2(acc[8 * v + 6], acc[8 * v + 7]));
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
  if (threadIdx.x == 0 && *abort_flag) atomicOr(prm.status, kStatusTimeout);
}

// ------------------------------------------------------------ bf16 GEMM ----
// Persistent, one CTA per SM, 12 warps: warps 0 and 2 load the X [128 x 64]
// and W [256 x 64] bf16 tiles of every 64-deep K step (128-byte swizzle) into
// a 4-stage ring; warp 1 issues four kind::f16 MMAs (M=128, N=256, K=16) per
// step and accumulates the whole K of a tile in one of two 256-column TMEM
// accumulators (tiles alternate); warps 4..11 read a finished tile once (one
// row and 128 columns per thread), add the bias and store.
namespace bf16g {
constexpr int BM = 128, BN = 256, BK = 64;                       // BK: one 128-byte bf16 row
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK * 2, B_BYTES = BN * BK * 2, STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int OFF_BAR = STAGES * STAGE_BYTES;
constexpr int SMEM_BYTES = OFF_BAR + 256 + 1024;
constexpr uint32_t IDESC = make_idesc(kFmtF32Acc, kFmtBF16, kFmtBF16, 0, BM, BN);
static_assert(SMEM_BYTES <= 232448, "shared memory budget");
}  // namespace bf16g

struct Bf16Params {
  const __nv_bfloat16* bias;  // [N] or null
  void* y;                    // [M, N] bf16 or fp32
  uint32_t* status;
  int M, N, nks, n_tiles_m, n_tiles_n, n_tiles, group_m;
  int y_f32;
  long long timeout;
  int dbg_flags;              // bit 0: the MMA thread first waits on a barrier nobody arrives on
};

__global__ void __launch_bounds__(kThreads, 1)
    linear_bf16_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                       const Bf16Params prm) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + bf16g::OFF_BAR);
  uint64_t* full = bars;                    // [bf16g::STAGES] operand tiles landed (two producers)
  uint64_t* empty = bars + bf16g::STAGES;          // [bf16g::STAGES] operand tiles consumed by the MMAs
  uint64_t* tfull = bars + 2 * bf16g::STAGES;      // [2] accumulator holds a finished tile
  uint64_t* tempty = tfull + 2;             // [2] accumulator read (8 warp arrivals)
  uint64_t* mma_done = tempty + 2;
  uint64_t* never = mma_done + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(never + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nks = prm.nks;
  const long long limit = prm.timeout;

  if (threadIdx.x == 0) {
    for (int s = 0; s < bf16g::STAGES; ++s) {
      mbar_init(&full[s], 2);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 8);
    }
    mbar_init(mma_done, 1);
    mbar_init(never, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if ((warp == 0 || warp == 2) && lane == 0) {
    // ------------------------------------------------------------ producers
    const bool is_x = warp == 0;
    const CUtensorMap* map = is_x ? &tmX : &tmW;
    const uint32_t bytes = is_x ? bf16g::A_BYTES : bf16g::B_BYTES;
    tma_prefetch_desc(map);
    long long g = 0;
    bool ok = true;
    for (int t = blockIdx.x; ok && t < prm.n_tiles; t += gridDim.x) {
      int mt, nt;
      tile_coords(t, prm.n_tiles_m, prm.n_tiles_n, prm.group_m, mt, nt);
      const int row0 = is_x ? mt * bf16g::BM : nt * bf16g::BN;
      for (int ks = 0; ks < nks; ++ks, ++g) {
        const int s = (int)(g % bf16g::STAGES);
        if (g >= bf16g::STAGES && !mbar_wait(&empty[s], (uint32_t)((g / bf16g::STAGES) - 1) & 1u, abort_flag, limit)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&full[s], bytes);
        tma_load_2d(smem + s * bf16g::STAGE_BYTES + (is_x ? 0 : bf16g::A_BYTES), map, &full[s], ks * bf16g::BK, row0);
      }
    }
    volatile int no_abort = 0;
    for (long long j = g - bf16g::STAGES < 0 ? 0 : g - bf16g::STAGES; j < g; ++j)
      mbar_wait(&full[j % bf16g::STAGES], (uint32_t)(j / bf16g::STAGES) & 1u, &no_abort, limit);
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------------ MMA issuer
    bool ok = true;
    if (prm.dbg_flags & 1) ok = mbar_wait(never, 0, abort_flag, limit);
    long long g = 0;
    int i = 0;
    for (int t = blockIdx.x; ok && t < prm.n_tiles; t += gridDim.x, ++i) {
      const int b = i & 1;
      if (!mbar_wait(&tempty[b], (uint32_t)(i >> 1) & 1u, abort_flag, limit)) {
        ok = false;
        break;
      }
      for (int ks = 0; ks < nks; ++ks, ++g) {
        const int s = (int)(g % bf16g::STAGES);
        if (!mbar_wait(&full[s], (uint32_t)(g / bf16g::STAGES) & 1u, abort_flag, limit)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a_s = smem_u32(smem + s * bf16g::STAGE_BYTES);
        const uint32_t b_s = a_s + bf16g::A_BYTES;
#pragma unroll
        for (int k = 0; k < bf16g::BK / 16; ++k) {
          const uint64_t ad = make_sdesc(a_s + k * 32, 16, 1024, kLayoutSW128);
          const uint64_t bd = make_sdesc(b_s + k * 32, 16, 1024, kLayoutSW128);
          mma_ss<kKindF16>(tmem + (uint32_t)b * bf16g::BN, ad, bd, bf16g::IDESC, (ks > 0 || k > 0) ? 1u : 0u);
        }
        mma_commit(&empty[s]);
      }
      if (!ok) break;
      mma_commit(&tfull[b]);
    }
    mma_commit(mma_done);
    volatile int no_abort = 0;
    mbar_wait(mma_done, 0, &no_abort, limit);
  } else if (warp >= 4) {
    // ------------------------------------------------------------ epilogue
    const int wg = (warp - 4) >> 2;
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t t_lane = tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)wg * 128;
    if (lane == 0) {
      mbar_arrive(&tempty[0]);
      mbar_arrive(&tempty[1]);
    }
    int i = 0;
    for (int t = blockIdx.x; t < prm.n_tiles; t += gridDim.x, ++i) {
      const int b = i & 1;
      int mt, nt;
      tile_coords(t, prm.n_tiles_m, prm.n_tiles_n, prm.group_m, mt, nt);
      const int n0 = nt * bf16g::BN + wg * 128;
      const int gm = mt * bf16g::BM + row;
      const bool live = n0 < prm.N && gm < prm.M;
      if (!mbar_wait(&tfull[b], (uint32_t)(i >> 1) & 1u, abort_flag, limit)) break;
      tc_fence_after();
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t r[32];
        tmem_ld32(t_lane + b * bf16g::BN + c * 32, r);
        tmem_wait_ld_regs(r);
        if (c == 3) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&tempty[b]);
        }
        if (!live) continue;
        float v[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
        if (prm.bias) {
          const uint4* bp = reinterpret_cast<const uint4*>(prm.bias + n0 + c * 32);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const uint4 bb = bp[q];
            const uint32_t w[4] = {bb.x, bb.y, bb.z, bb.w};
#pragma unroll
            for (int h = 0; h < 4; ++h) {
              v[8 * q + 2 * h] = __fadd_rn(v[8 * q + 2 * h], __uint_as_float(w[h] << 16));
              v[8 * q + 2 * h + 1] = __fadd_rn(v[8 * q + 2 * h + 1], __uint_as_float(w[h] & 0xFFFF0000u));
            }
          }
        }
        if (prm.y_f32) {
          uint4* dst = reinterpret_cast<uint4*>(static_cast<float*>(prm.y) + (size_t)gm * prm.N + n0 + c * 32);
#pragma unroll
          for (int q = 0; q < 8; ++q)
            dst[q] = make_uint4(__float_as_uint(v[4 * q]), __float_as_uint(v[4 * q + 1]), __float_as_uint(v[4 * q + 2]),
                                __float_as_uint(v[4 * q + 3]));
        } else {
          uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(prm.y) + (size_t)gm * prm.N + n0 + c * 32);
#pragma unroll
          for (int q = 0; q < 4; ++q)
            dst[q] = make_uint4(pack_bf16x2(v[8 * q], v[8 * q + 1]), pack_bf16x2(v[8 * q + 2], v[8 * q + 3]),
                                pack_bf16x2(v[8 * q + 4], v[8 * q + 5]), pack_bf16x2(v[8 * q + 6], v[8 * q + 7]));
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
  if (threadIdx.x == 0 && *abort_flag) atomicOr(prm.status, kStatusTimeout);
}

}  // namespace

cudaError_t launch_quant_blocks_2d(const void* x, int R, int K, int8_t* codes, float* scales, cudaStream_t stream) {
  const dim3 grid(K / 128, (R + 127) / 128);
  quant_blocks_2d_kernel<<<grid, 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(x), R, K, codes, scales);
  return cudaGetLastError();
}

cudaError_t launch_linear_w8a8(const int8_t* xq, const float* sx, const int8_t* wq, const float* sw, const void* bias,
                               void* y, int y_f32, int M, int N, int K, uint32_t* status, long long timeout_cycles,
                               int dbg_flags, cudaStream_t stream) {
  CUtensorMap tmX, tmW;
  if (!encode_tmap_2d(&tmX, CU_TENSOR_MAP_DATA_TYPE_UINT8, xq, (uint64_t)K, (uint64_t)M, (uint64_t)K, BK, BM,
                      CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tmap_2d(&tmW, CU_TENSOR_MAP_DATA_TYPE_UINT8, wq, (uint64_t)K, (uint64_t)N, (uint64_t)K, BK, BN,
                      CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  cudaFuncAttributes fa;
  if ((e = cudaFuncGetAttributes(&fa, linear_w8a8_kernel)) != cudaSuccess) return e;
  if (fa.numRegs * kThreads < 128 * REGS_LOW + 256 * REGS_HIGH) return cudaErrorInvalidConfiguration;
  // set on every launch (per device, thread-safe; allowed during stream capture)
  if ((e = cudaFuncSetAttribute(linear_w8a8_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES)) !=
      cudaSuccess)
    return e;
  int sms = 0;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  LinParams prm;
  prm.sx = sx;
  prm.sw = sw;
  prm.bias = static_cast<const __nv_bfloat16*>(bias);
  prm.y = y;
  prm.status = status;
  prm.M = M;
  prm.N = N;
  prm.nk = K / BK;
  prm.n_tiles_m = (M + BM - 1) / BM;
  prm.n_tiles_n = (N + BN - 1) / BN;
  prm.n_tiles = prm.n_tiles_m * prm.n_tiles_n;
  prm.group_m = 1;                              // int8 W of a DiT layer (<= 71 MB) stays in L2
  prm.y_f32 = y_f32;
  prm.timeout = timeout_cycles;
  prm.dbg_flags = dbg_flags;
  const int grid = prm.n_tiles < sms ? prm.n_tiles : sms;
  linear_w8a8_kernel<<<grid, kThreads, SMEM_BYTES, stream>>>(tmX, tmW, prm);
  return cudaGetLastError();
}

}  // namespace sage

namespace sage {

cudaError_t launch_dequant_blocks_2d(const int8_t* codes, const float* scales, int R, int K, void* out,
                                     cudaStream_t stream) {
  const dim3 grid(K / 128, (R + 127) / 128);
  dequant_blocks_2d_kernel<<<grid, 256, 0, stream>>>(codes, scales, R, K, static_cast<__nv_bfloat16*>(out));
  return cudaGetLastError();
}

cudaError_t launch_linear_bf16(const void* x, const void* w, const void* bias, void* y, int y_f32, int M, int N,
                               int K, uint32_t* status, long long timeout_cycles, int dbg_flags, cudaStream_t stream) {
  CUtensorMap tmX, tmW;
  if (!encode_tmap_2d(&tmX, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x, (uint64_t)K, (uint64_t)M, (uint64_t)K * 2, bf16g::BK, bf16g::BM,
                      CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tmap_2d(&tmW, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, w, (uint64_t)K, (uint64_t)N, (uint64_t)K * 2, bf16g::BK, bf16g::BN,
                      CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if ((e = cudaFuncSetAttribute(linear_bf16_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bf16g::SMEM_BYTES)) !=
      cudaSuccess)
    return e;
  int sms = 0;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  Bf16Params prm;
  prm.bias = static_cast<const __nv_bfloat16*>(bias);
  prm.y = y;
  prm.status = status;
  prm.M = M;
  prm.N = N;
  prm.nks = K / bf16g::BK;
  prm.n_tiles_m = (M + bf16g::BM - 1) / bf16g::BM;
  prm.n_tiles_n = (N + bf16g::BN - 1) / bf16g::BN;
  prm.n_tiles = prm.n_tiles_m * prm.n_tiles_n;
  prm.group_m = 16;                             // grouped order (see tile_coords)
  prm.y_f32 = y_f32;
  prm.timeout = timeout_cycles;
  prm.dbg_flags = dbg_flags;
  const int grid = prm.n_tiles < sms ? prm.n_tiles : sms;
  linear_bf16_kernel<<<grid, kThreads, bf16g::SMEM_BYTES, stream>>>(tmX, tmW, prm);
  return cudaGetLastError();
}

}  // namespace sage
