// attention.cu -- sm_100a attention kernels for video-DiT self-attention.
//
// The op: full-sequence, non-causal O = softmax(Q K^T / sqrt(d)) V, profiled
// on page 1 of the TMAP write-up ("Attention performance optimisation /
// Background") and replaced there by the SageAttention operator ("attention
// quantization"), with some layers kept at original precision ("keeping
// video quality").  Two instantiations of one pipeline:
//   QUANT = true : S = Q_i8 K_i8^T (tcgen05 kind::i8, exact int32), dequant
//                  with q_scale * k_scale * log2(e)/sqrt(d), P8 = e4m3(p*448)
//                  kept in tensor memory, O += P8 V8 (kind::f8f6f4, fp32).
//   QUANT = false: S = Q K^T and O += P V with kind::f16 (bf16 in, fp32 acc),
//                  P rounded to bf16 in tensor memory.
//
// One CTA = two 128-row Q tiles of one (b, h) and every 128-key tile of that
// head.  Warp roles (12 warps):
//   warp 0      TMA producer: Q tiles once, then K/V tiles through a ring of
//               STAGES shared-memory slots (mbarrier full / empty pairs);
//   warp 1      TMEM allocator and the single MMA-issuing thread;
//   warps 4-7   softmax for Q tile 0, warps 8-11 for Q tile 1: one thread
//               per query row (TMEM lane), online softmax in registers, P
//               written back over its S columns, O rescaled in place, and the
//               epilogue (normalise, round to bf16, store).
// TMEM (512 columns): S0 [0,128), S1 [128,256), O0 [256,256+D), O1 after it.
// Per key tile j the MMA thread issues PV_t(j) and then QK_t(j+1) into the
// same S_t columns; tcgen05 operations from one thread execute in order, and
// the commit after QK_t(j+1) also covers PV_t(j), so when the softmax warps
// see S_t(j+1) the accumulator O_t is stable and may be rescaled.
//
// Every wait is bounded (clock64 limit); a wait that runs out raises a
// CTA-wide abort flag, every role leaves its loop, in-flight TMA loads and
// MMAs are drained with bounded waits, TMEM is freed and the status word gets
// kStatusTimeout.  No __trap, no unbounded spin.
#include <cuda_bf16.h>
#include <climits>
#include <cstdint>

#include "internal.h"
#include "sm100.cuh"

namespace sage {

namespace {

constexpr int kWarps = 12;
constexpr int kThreads = kWarps * 32;
constexpr uint32_t kTmemCols = 512;

// log2(e) / sqrt(d), formed in double and rounded once to fp32
__host__ __device__ constexpr float softmax_c(int d) {
  return d == 128 ? (float)(1.4426950408889634073599246810019 / 11.313708498984760390413509793678)
                  : (float)(1.4426950408889634073599246810019 / 8.0);
}

template <int D, bool QUANT>
struct Cfg {
  static constexpr int ELEM = QUANT ? 1 : 2;
  static constexpr int TILE_BYTES = 128 * D * ELEM;               // one Q, K or V tile
  static constexpr int STAGES = QUANT ? (D == 128 ? 4 : 8) : (D == 128 ? 2 : 3);
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = 2 * TILE_BYTES;
  static constexpr int OFF_V = OFF_K + STAGES * TILE_BYTES;
  static constexpr int OFF_BAR = OFF_V + STAGES * TILE_BYTES;
  static constexpr int SMEM_BYTES = OFF_BAR + 512 + 1024;          // barriers + 1 KB alignment slack
  // Q/K operand rows in shared memory (bytes) and their swizzle
  static constexpr int QK_ROW = QUANT ? D : 128;                   // bf16: one 64-element atom
  static constexpr uint32_t QK_LAYOUT = (QUANT && D == 64) ? kLayoutSW64 : kLayoutSW128;
  static constexpr uint32_t QK_SBO = 8 * QK_ROW;
  static constexpr int QK_KSTEPS = QUANT ? D / 32 : D / 16;
  static constexpr int PV_KSTEPS = QUANT ? 128 / 32 : 128 / 16;
  static constexpr int P_COLS = QUANT ? 32 : 64;                   // TMEM columns of P per row
  static constexpr uint32_t IDESC_QK =
      QUANT ? make_idesc(kFmtS32Acc, kFmtS8, kFmtS8, 0, 128, 128) : make_idesc(kFmtF32Acc, kFmtBF16, kFmtBF16, 0, 128, 128);
  static constexpr uint32_t IDESC_PV =
      QUANT ? make_idesc(kFmtF32Acc, kFmtE4M3, kFmtE4M3, 0, 128, D) : make_idesc(kFmtF32Acc, kFmtBF16, kFmtBF16, 1, 128, D);
  static constexpr int KIND_QK = QUANT ? kKindI8 : kKindF16;
  static constexpr int KIND_PV = QUANT ? kKindF8F6F4 : kKindF16;
};

// S[tmem] = Q[smem] K[smem]^T for one 128x128 tile (K-major operands).
template <int D, bool QUANT>
__device__ __forceinline__ void issue_qk(uint32_t d_tmem, uint32_t q_smem, uint32_t k_smem) {
  using C = Cfg<D, QUANT>;
#pragma unroll
  for (int s = 0; s < C::QK_KSTEPS; ++s) {
    // 32-byte K step; bf16 tiles hold 64-element (128-byte) atoms of 16 KB each
    const uint32_t off = QUANT ? s * 32 : (s / 4) * 16384 + (s % 4) * 32;
    const uint64_t a = make_sdesc(q_smem + off, 16, C::QK_SBO, C::QK_LAYOUT);
    const uint64_t b = make_sdesc(k_smem + off, 16, C::QK_SBO, C::QK_LAYOUT);
    mma_ss<C::KIND_QK>(d_tmem, a, b, C::IDESC_QK, s > 0 ? 1u : 0u);
  }
}

// O[tmem] (+)= P[tmem] V[smem] for one 128-key tile.
//  QUANT: V^T tile [D rows][128 keys] e4m3, K-major, 128-byte swizzle.
//  bf16 : V tile [128 keys][D] as 64-channel atoms (16 KB each), MN-major.
template <int D, bool QUANT>
__device__ __forceinline__ void issue_pv(uint32_t d_tmem, uint32_t p_tmem, uint32_t v_smem, uint32_t accumulate) {
  using C = Cfg<D, QUANT>;
#pragma unroll
  for (int s = 0; s < C::PV_KSTEPS; ++s) {
    uint64_t b;
    if constexpr (QUANT)
      b = make_sdesc(v_smem + s * 32, 16, 1024, kLayoutSW128);
    else
      b = make_sdesc(v_smem + s * 2048, 16384, 1024, kLayoutSW128);
    mma_ts<C::KIND_PV>(d_tmem, p_tmem + s * 8, b, C::IDESC_PV, (s > 0 || accumulate) ? 1u : 0u);
  }
}

struct Params {
  // QUANT operands
  const float* q_scale;   // [BH, nT]
  const float* k_scale;   // [BH, nT]
  const float* v_scale;   // [BH, D]
  __nv_bfloat16* o;       // [BH, N, D]
  uint32_t* status;
  int N, nT, Npad;
  long long timeout;
  int dbg_flags;          // bit 0: MMA thread first waits on a barrier nobody arrives on
};

template <int D, bool QUANT>
__global__ void __launch_bounds__(kThreads, 1)
    attn_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const Params prm) {
  using C = Cfg<D, QUANT>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* q_full = bars + 0;
  uint64_t* kv_full = bars + 1;                       // [STAGES]
  uint64_t* kv_empty = bars + 1 + C::STAGES;          // [STAGES]
  uint64_t* s_full = bars + 1 + 2 * C::STAGES;        // [2]
  uint64_t* p_full = s_full + 2;                      // [2]
  uint64_t* o_final = p_full + 2;                     // [2]
  uint64_t* mma_done = o_final + 2;
  uint64_t* never = mma_done + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(never + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.y;
  const int N = prm.N, nT = prm.nT;
  const int qt0 = 2 * blockIdx.x;
  const long long limit = prm.timeout;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&s_full[t], 1);
      mbar_init(&p_full[t], 128);
      mbar_init(&o_final[t], 1);
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

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      mbar_arrive_expect_tx(q_full, 2 * C::TILE_BYTES);
      for (int t = 0; t < 2; ++t) {
        uint8_t* dst = smem + C::OFF_Q + t * C::TILE_BYTES;
        if constexpr (QUANT) {
          tma_load_2d(dst, &tmQ, q_full, 0, bh * prm.Npad + (qt0 + t) * 128);
        } else {
#pragma unroll
          for (int a = 0; a < D / 64; ++a) tma_load_3d(dst + a * 16384, &tmQ, q_full, a * 64, (qt0 + t) * 128, bh);
        }
      }
      int issued = 0;
      for (int j = 0; j < nT; ++j) {
        const int s = j % C::STAGES;
        if (j >= C::STAGES && !mbar_wait(&kv_empty[s], ((j / C::STAGES) - 1) & 1, abort_flag, limit)) break;
        mbar_arrive_expect_tx(&kv_full[s], 2 * C::TILE_BYTES);
        uint8_t* kd = smem + C::OFF_K + s * C::TILE_BYTES;
        uint8_t* vd = smem + C::OFF_V + s * C::TILE_BYTES;
        if constexpr (QUANT) {
          tma_load_2d(kd, &tmK, &kv_full[s], 0, bh * prm.Npad + j * 128);
          tma_load_2d(vd, &tmV, &kv_full[s], j * 128, bh * D);
        } else {
#pragma unroll
          for (int a = 0; a < D / 64; ++a) {
            tma_load_3d(kd + a * 16384, &tmK, &kv_full[s], a * 64, j * 128, bh);
            tma_load_3d(vd + a * 16384, &tmV, &kv_full[s], a * 64, j * 128, bh);
          }
        }
        issued = j + 1;
      }
      // drain: every load this thread issued must land before the CTA exits
      volatile int no_abort = 0;
      mbar_wait(q_full, 0, &no_abort, limit);
      for (int j = issued - C::STAGES < 0 ? 0 : issued - C::STAGES; j < issued; ++j)
        mbar_wait(&kv_full[j % C::STAGES], (j / C::STAGES) & 1, &no_abort, limit);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t q_s = smem_u32(smem + C::OFF_Q);
      const uint32_t k_s = smem_u32(smem + C::OFF_K);
      const uint32_t v_s = smem_u32(smem + C::OFF_V);
      bool ok = true;
      if (prm.dbg_flags & 1) ok = mbar_wait(never, 0, abort_flag, limit);
      ok = ok && mbar_wait(q_full, 0, abort_flag, limit) && mbar_wait(&kv_full[0], 0, abort_flag, limit);
      if (ok) {
        tc_fence_after();
        for (int t = 0; t < 2; ++t) {
          issue_qk<D, QUANT>(tmem + t * 128, q_s + t * C::TILE_BYTES, k_s);
          mma_commit(&s_full[t]);
        }
        for (int j = 0; j < nT && ok; ++j) {
          const int s = j % C::STAGES;
          for (int t = 0; t < 2; ++t) {
            if (!mbar_wait(&p_full[t], j & 1, abort_flag, limit)) { ok = false; break; }
            tc_fence_after();
            issue_pv<D, QUANT>(tmem + 256 + t * D, tmem + t * 128, v_s + s * C::TILE_BYTES, j > 0 ? 1u : 0u);
            if (j + 1 < nT) {
              const int s1 = (j + 1) % C::STAGES;
              if (t == 0 && !mbar_wait(&kv_full[s1], ((j + 1) / C::STAGES) & 1, abort_flag, limit)) {
                ok = false;
                break;
              }
              issue_qk<D, QUANT>(tmem + t * 128, q_s + t * C::TILE_BYTES, k_s + s1 * C::TILE_BYTES);
              mma_commit(&s_full[t]);
            } else {
              mma_commit(&o_final[t]);
            }
          }
          if (ok) mma_commit(&kv_empty[s]);
        }
      }
      // drain: every MMA issued must complete before TMEM is released
      mma_commit(mma_done);
      volatile int no_abort = 0;
      mbar_wait(mma_done, 0, &no_abort, limit);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax
    const int t = (warp - 4) >> 2;
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const uint32_t tS = tmem + lane_off + t * 128;
    const uint32_t tO = tmem + lane_off + 256 + t * D;
    const int qt = qt0 + t;
    const float c = softmax_c(D);
    float qs = 1.0f;
    if constexpr (QUANT) qs = qt < nT ? prm.q_scale[(size_t)bh * nT + qt] : 0.f;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < nT; ++j) {
      if (!mbar_wait(&s_full[t], j & 1, abort_flag, limit)) { ok = false; break; }
      tc_fence_after();
      const int valid = min(128, N - j * 128);
      float sc = c;
      if constexpr (QUANT) sc = __fmul_rn(__fmul_rn(qs, prm.k_scale[(size_t)bh * nT + j]), c);
      // pass 1: row max of the raw scores (monotone in s since sc >= 0)
      float mt;
      if constexpr (QUANT) {
        int mx = INT_MIN;
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          uint32_t r[32];
          tmem_ld32(tS + ch * 32, r);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (ch * 32 + i < valid) mx = max(mx, (int)r[i]);
        }
        mt = __fmul_rn((float)mx, sc);
      } else {
        float mx = -INFINITY;
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          uint32_t r[32];
          tmem_ld32(tS + ch * 32, r);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (ch * 32 + i < valid) mx = fmaxf(mx, __uint_as_float(r[i]));
        }
        mt = __fmul_rn(mx, sc);
      }
      const float m_new = fmaxf(m, mt);
      const float alpha = (m == -INFINITY) ? 0.f : ex2_approx(__fsub_rn(m, m_new));
      // rescale O_t (complete: the commit that signalled S_t(j) covers PV_t(j-1))
      if (j > 0 && __any_sync(0xffffffffu, m_new > m)) {
#pragma unroll
        for (int ch = 0; ch < D / 32; ++ch) {
          uint32_t r[32];
          tmem_ld32(tO + ch * 32, r);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__fmul_rn(__uint_as_float(r[i]), alpha));
          tmem_st32(tO + ch * 32, r);
        }
        tmem_wait_st();
      }
      // pass 2: p = 2^(s - m_new), row sum, P written over the S columns
      float psum = 0.f;
      uint32_t pk[2 * 32];
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) {
        uint32_t r[32];
        tmem_ld32(tS + ch * 32, r);
        tmem_wait_ld();
        float p[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float s = QUANT ? __fmul_rn((float)(int)r[i], sc) : __fmul_rn(__uint_as_float(r[i]), sc);
          p[i] = (ch * 32 + i < valid) ? ex2_approx(__fsub_rn(s, m_new)) : 0.f;
          psum = __fadd_rn(psum, p[i]);
        }
        if constexpr (QUANT) {
#pragma unroll
          for (int g = 0; g < 8; ++g)
            pk[ch * 8 + g] = pack_e4m3x4(__fmul_rn(p[4 * g], 448.f), __fmul_rn(p[4 * g + 1], 448.f),
                                         __fmul_rn(p[4 * g + 2], 448.f), __fmul_rn(p[4 * g + 3], 448.f));
        } else {
#pragma unroll
          for (int g = 0; g < 16; ++g) pk[ch * 16 + g] = pack_bf16x2(p[2 * g], p[2 * g + 1]);
        }
      }
      {
        uint32_t (&lo)[32] = *reinterpret_cast<uint32_t(*)[32]>(&pk[0]);
        tmem_st32(tS, lo);
        if constexpr (!QUANT) {
          uint32_t (&hi)[32] = *reinterpret_cast<uint32_t(*)[32]>(&pk[32]);
          tmem_st32(tS + 32, hi);
        }
      }
      tmem_wait_st();
      l = __fadd_rn(__fmul_rn(l, alpha), psum);
      m = m_new;
      tc_fence_before();
      mbar_arrive(&p_full[t]);
    }
    // ---------------------------------------------------------- epilogue
    if (ok && mbar_wait(&o_final[t], 0, abort_flag, limit)) {
      tc_fence_after();
      const int gq = qt * 128 + row;
      const float denom = QUANT ? __fmul_rn(448.f, l) : l;
      __nv_bfloat16* orow = prm.o + ((size_t)bh * N + gq) * D;
#pragma unroll
      for (int ch = 0; ch < D / 32; ++ch) {
        uint32_t r[32];
        tmem_ld32(tO + ch * 32, r);
        tmem_wait_ld();
        uint32_t w[16];
#pragma unroll
        for (int g = 0; g < 16; ++g) {
          float a0 = __uint_as_float(r[2 * g]), a1 = __uint_as_float(r[2 * g + 1]);
          if constexpr (QUANT) {
            a0 = __fmul_rn(a0, prm.v_scale[(size_t)bh * D + ch * 32 + 2 * g]);
            a1 = __fmul_rn(a1, prm.v_scale[(size_t)bh * D + ch * 32 + 2 * g + 1]);
          }
          w[g] = pack_bf16x2(__fdiv_rn(a0, denom), __fdiv_rn(a1, denom));
        }
        if (qt < nT && gq < N) {
          uint4* dst = reinterpret_cast<uint4*>(orow + ch * 32);
#pragma unroll
          for (int v = 0; v < 4; ++v) dst[v] = make_uint4(w[4 * v], w[4 * v + 1], w[4 * v + 2], w[4 * v + 3]);
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

// ---------------------------------------------------------------- diagnostics
// One (b, h, qb, kb) int32 QK^T tile per CTA, 128 threads, through issue_qk.
template <int D>
__global__ void __launch_bounds__(128, 1)
    dbg_qk_tiles_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                        const int* tiles, int H, int Npad, int32_t* out) {
  using C = Cfg<D, true>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + 2 * C::TILE_BYTES);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2);
  __shared__ int abort_s;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int* tl = tiles + 4 * blockIdx.x;
  const int bh = tl[0] * H + tl[1], qb = tl[2], kb = tl[3];
  if (threadIdx.x == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    abort_s = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (threadIdx.x == 0) {
    mbar_arrive_expect_tx(&bars[0], 2 * C::TILE_BYTES);
    tma_load_2d(smem, &tmQ, &bars[0], 0, bh * Npad + qb * 128);
    tma_load_2d(smem + C::TILE_BYTES, &tmK, &bars[0], 0, bh * Npad + kb * 128);
    if (mbar_wait(&bars[0], 0, &abort_s, kDefaultTimeoutCycles)) {
      tc_fence_after();
      issue_qk<D, true>(tmem, smem_u32(smem), smem_u32(smem + C::TILE_BYTES));
    }
    mma_commit(&bars[1]);
  }
  __syncthreads();
  const bool ok = mbar_wait(&bars[1], 0, &abort_s, kDefaultTimeoutCycles);
  tc_fence_after();
  const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
  int32_t* orow = out + ((size_t)blockIdx.x * 128 + warp * 32 + lane) * 128;
#pragma unroll
  for (int ch = 0; ch < 4; ++ch) {
    uint32_t r[32];
    tmem_ld32(tmem + lane_off + ch * 32, r);
    tmem_wait_ld();
    for (int i = 0; i < 32; ++i) orow[ch * 32 + i] = ok && !abort_s ? (int32_t)r[i] : INT_MIN;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, 128);
}

// One 128-row P.V product: P from global into TMEM (tcgen05.st), V via TMA.
template <int D, bool QUANT>
__global__ void __launch_bounds__(128, 1)
    dbg_pv_kernel(const __grid_constant__ CUtensorMap tmV, const uint8_t* p, float* out) {
  using C = Cfg<D, QUANT>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::TILE_BYTES);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2);
  __shared__ int abort_s;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    abort_s = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
  const int row = warp * 32 + lane;
  // P row -> TMEM columns [0, P_COLS) (P occupies the start of an S region)
  const uint32_t* prow = reinterpret_cast<const uint32_t*>(p + (size_t)row * 128 * (QUANT ? 1 : 2));
  for (int h = 0; h < C::P_COLS / 32; ++h) {
    uint32_t r[32];
    for (int i = 0; i < 32; ++i) r[i] = prow[h * 32 + i];
    tmem_st32(tmem + lane_off + h * 32, r);
  }
  tmem_wait_st();
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) {
    tc_fence_after();
    mbar_arrive_expect_tx(&bars[0], C::TILE_BYTES);
    if constexpr (QUANT) {
      tma_load_2d(smem, &tmV, &bars[0], 0, 0);
    } else {
      for (int a = 0; a < D / 64; ++a) tma_load_2d(smem + a * 16384, &tmV, &bars[0], a * 64, 0);
    }
    if (mbar_wait(&bars[0], 0, &abort_s, kDefaultTimeoutCycles))
      issue_pv<D, QUANT>(tmem + 128, tmem, smem_u32(smem), 0u);
    mma_commit(&bars[1]);
  }
  __syncthreads();
  const bool ok = mbar_wait(&bars[1], 0, &abort_s, kDefaultTimeoutCycles);
  tc_fence_after();
  for (int ch = 0; ch < D / 32; ++ch) {
    uint32_t r[32];
    tmem_ld32(tmem + lane_off + 128 + ch * 32, r);
    tmem_wait_ld();
    for (int i = 0; i < 32; ++i) out[(size_t)row * D + ch * 32 + i] = ok && !abort_s ? __uint_as_float(r[i]) : NAN;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, 256);
}

// One 128x128 bf16 QK^T tile.
template <int D>
__global__ void __launch_bounds__(128, 1)
    dbg_qk_bf16_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK, float* out) {
  using C = Cfg<D, false>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + 2 * C::TILE_BYTES);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2);
  __shared__ int abort_s;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    abort_s = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (threadIdx.x == 0) {
    mbar_arrive_expect_tx(&bars[0], 2 * C::TILE_BYTES);
    for (int a = 0; a < D / 64; ++a) {
      tma_load_2d(smem + a * 16384, &tmQ, &bars[0], a * 64, 0);
      tma_load_2d(smem + C::TILE_BYTES + a * 16384, &tmK, &bars[0], a * 64, 0);
    }
    if (mbar_wait(&bars[0], 0, &abort_s, kDefaultTimeoutCycles)) {
      tc_fence_after();
      issue_qk<D, false>(tmem, smem_u32(smem), smem_u32(smem + C::TILE_BYTES));
    }
    mma_commit(&bars[1]);
  }
  __syncthreads();
  const bool ok = mbar_wait(&bars[1], 0, &abort_s, kDefaultTimeoutCycles);
  tc_fence_after();
  const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
  const int row = warp * 32 + lane;
  for (int ch = 0; ch < 4; ++ch) {
    uint32_t r[32];
    tmem_ld32(tmem + lane_off + ch * 32, r);
    tmem_wait_ld();
    for (int i = 0; i < 32; ++i) out[(size_t)row * 128 + ch * 32 + i] = ok && !abort_s ? __uint_as_float(r[i]) : NAN;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, 128);
}

template <int D, bool QUANT>
cudaError_t launch_attn_d(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const Params& prm,
                          int BH, cudaStream_t stream) {
  using C = Cfg<D, QUANT>;
  auto kern = attn_kernel<D, QUANT>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  dim3 grid((prm.nT + 1) / 2, BH);
  kern<<<grid, kThreads, C::SMEM_BYTES, stream>>>(tq, tk, tv, prm);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_i8f8(const int8_t* q_i8, const float* q_scale, const int8_t* k_i8, const float* k_scale,
                             const uint8_t* v_f8t, const float* v_scale, void* o, int BH, int N, int d,
                             uint32_t* status, long long timeout_cycles, int dbg_flags, cudaStream_t stream) {
  const int nT = num_tiles(N), Npad = nT * kTile;
  alignas(64) CUtensorMap tq, tk, tv;
  const CUtensorMapSwizzle qk_sw = d == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  if (!encode_tmap_2d(&tq, CU_TENSOR_MAP_DATA_TYPE_UINT8, q_i8, d, (uint64_t)BH * Npad, d, d, 128, qk_sw) ||
      !encode_tmap_2d(&tk, CU_TENSOR_MAP_DATA_TYPE_UINT8, k_i8, d, (uint64_t)BH * Npad, d, d, 128, qk_sw) ||
      !encode_tmap_2d(&tv, CU_TENSOR_MAP_DATA_TYPE_UINT8, v_f8t, Npad, (uint64_t)BH * d, Npad, 128, d,
                      CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  Params prm{q_scale, k_scale, v_scale, static_cast<__nv_bfloat16*>(o), status, N, nT, Npad, timeout_cycles, dbg_flags};
  if (d == 128) return launch_attn_d<128, true>(tq, tk, tv, prm, BH, stream);
  if (d == 64) return launch_attn_d<64, true>(tq, tk, tv, prm, BH, stream);
  return cudaErrorInvalidValue;
}

cudaError_t launch_attn_bf16(const void* q, const void* k, const void* v, void* o, int BH, int N, int d,
                             uint32_t* status, long long timeout_cycles, cudaStream_t stream) {
  const int nT = num_tiles(N);
  alignas(64) CUtensorMap tq, tk, tv;
  const uint64_t s1 = (uint64_t)d * 2, s2 = (uint64_t)N * d * 2;
  if (!encode_tmap_3d(&tq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, q, d, N, BH, s1, s2, 64, 128, 1,
                      CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tmap_3d(&tk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, k, d, N, BH, s1, s2, 64, 128, 1,
                      CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tmap_3d(&tv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, v, d, N, BH, s1, s2, 64, 128, 1,
                      CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  Params prm{nullptr, nullptr, nullptr, static_cast<__nv_bfloat16*>(o), status, N, nT, nT * kTile, timeout_cycles, 0};
  if (d == 128) return launch_attn_d<128, false>(tq, tk, tv, prm, BH, stream);
  if (d == 64) return launch_attn_d<64, false>(tq, tk, tv, prm, BH, stream);
  return cudaErrorInvalidValue;
}

cudaError_t launch_dbg_qk_tiles(const int8_t* q_i8, const int8_t* k_i8, int BH, int H, int N, int d,
                                const int* tile_list, int n, int32_t* out, cudaStream_t stream) {
  const int Npad = num_tiles(N) * kTile;
  alignas(64) CUtensorMap tq, tk;
  const CUtensorMapSwizzle sw = d == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  if (!encode_tmap_2d(&tq, CU_TENSOR_MAP_DATA_TYPE_UINT8, q_i8, d, (uint64_t)BH * Npad, d, d, 128, sw) ||
      !encode_tmap_2d(&tk, CU_TENSOR_MAP_DATA_TYPE_UINT8, k_i8, d, (uint64_t)BH * Npad, d, d, 128, sw))
    return cudaErrorInvalidValue;
  const int smem = 2 * 128 * d + 64 + 1024;
  if (d == 128) {
    cudaFuncSetAttribute(dbg_qk_tiles_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    dbg_qk_tiles_kernel<128><<<n, 128, smem, stream>>>(tq, tk, tile_list, H, Npad, out);
  } else {
    cudaFuncSetAttribute(dbg_qk_tiles_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    dbg_qk_tiles_kernel<64><<<n, 128, smem, stream>>>(tq, tk, tile_list, H, Npad, out);
  }
  return cudaGetLastError();
}

cudaError_t launch_dbg_pv_tile(const void* p, const void* vt, int d, int mode, float* out, cudaStream_t stream) {
  alignas(64) CUtensorMap tv;
  const bool quant = mode == 1;
  bool okm;
  if (quant)
    okm = encode_tmap_2d(&tv, CU_TENSOR_MAP_DATA_TYPE_UINT8, vt, 128, d, 128, 128, d, CU_TENSOR_MAP_SWIZZLE_128B);
  else
    okm = encode_tmap_2d(&tv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, vt, d, 128, (uint64_t)d * 2, 64, 128,
                         CU_TENSOR_MAP_SWIZZLE_128B);
  if (!okm) return cudaErrorInvalidValue;
  const int smem = 128 * d * (quant ? 1 : 2) + 64 + 1024;
  const uint8_t* pp = static_cast<const uint8_t*>(p);
#define SAGE_DBG_PV(DD, QQ)                                                                         \
  do {                                                                                              \
    cudaFuncSetAttribute(dbg_pv_kernel<DD, QQ>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem); \
    dbg_pv_kernel<DD, QQ><<<1, 128, smem, stream>>>(tv, pp, out);                                   \
  } while (0)
  if (d == 128 && quant) SAGE_DBG_PV(128, true);
  else if (d == 64 && quant) SAGE_DBG_PV(64, true);
  else if (d == 128) SAGE_DBG_PV(128, false);
  else SAGE_DBG_PV(64, false);
#undef SAGE_DBG_PV
  return cudaGetLastError();
}

cudaError_t launch_dbg_qk_bf16_tile(const void* q, const void* k, int d, float* out, cudaStream_t stream) {
  alignas(64) CUtensorMap tq, tk;
  if (!encode_tmap_2d(&tq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, q, d, 128, (uint64_t)d * 2, 64, 128,
                      CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tmap_2d(&tk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, k, d, 128, (uint64_t)d * 2, 64, 128,
                      CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  const int smem = 2 * 128 * d * 2 + 64 + 1024;
  if (d == 128) {
    cudaFuncSetAttribute(dbg_qk_bf16_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    dbg_qk_bf16_kernel<128><<<1, 128, smem, stream>>>(tq, tk, out);
  } else {
    cudaFuncSetAttribute(dbg_qk_bf16_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    dbg_qk_bf16_kernel<64><<<1, 128, smem, stream>>>(tq, tk, out);
  }
  return cudaGetLastError();
}

}  // namespace sage
