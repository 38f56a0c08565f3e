// attention.cu -- sm_100a attention kernels for video-DiT self-attention.
//
// The op: full-sequence, non-causal O = softmax(Q K^T / sqrt(d)) V, profiled
// on page 1 of the TMAP write-up ("Attention performance optimisation /
// Background") and replaced there by the SageAttention operator ("attention
// quantization"), with some layers kept at original precision ("keeping
// video quality").  Two kernels with one warp-specialised pipeline:
//   attn_i8f8_kernel: S = Q_i8 K_i8^T (tcgen05 kind::i8, exact int32),
//                  dequant with q_scale * k_scale * log2(e)/sqrt(d),
//                  P8 = e4m3(p*448) staged in shared memory, O += P8 V8
//                  (kind::f8f6f4, fp32).
//   attn_bf16_kernel: S = Q K^T and O += P V with kind::f16 (bf16 in, fp32
//                  acc), P rounded to bf16 and kept in tensor memory over S.
//
// One CTA = two 128-row Q tiles of one (b, h) and every 128-key tile of that
// head.  Warp roles (12 warps, registers re-split with setmaxnreg):
//   warp 0      TMA producer: Q tiles once, then K/V tiles through a ring of
//               STAGES shared-memory slots (mbarrier full / empty pairs);
//   warp 1      TMEM allocator and the single MMA-issuing thread;
//   warps 4-7   softmax for Q tile 0, warps 8-11 for Q tile 1: one thread
//               per query row (TMEM lane), online softmax in registers, O
//               rescaled in place in TMEM, and the epilogue.  The two
//               warpgroups take turns on the exponential phase (an mbarrier
//               token), so one's compare phase overlaps the other's ex2s.
// TMEM (512 columns): S0 [0,128), S1 [128,256), O0 [256,256+D), O1 after it.
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
// Register split: the kernel is compiled for kLaunchRegs per thread (384 threads,
// one CTA per SM); warpgroup 0 (producer, MMA, idle warps) drops to Cfg::REGS_LOW
// and the two softmax warpgroups rise to Cfg::REGS_HIGH, within 384 * 168.
constexpr int kLaunchRegs = 168;

// log2(e) / sqrt(d), formed in double and rounded once to fp32
__host__ __device__ constexpr float softmax_c(int d) {
  return d == 128 ? (float)(1.4426950408889634073599246810019 / 11.313708498984760390413509793678)
                  : (float)(1.4426950408889634073599246810019 / 8.0);
}

template <int D, bool QUANT>
struct Cfg {
  static constexpr int ELEM = QUANT ? 1 : 2;
  static constexpr int TILE_BYTES = 128 * D * ELEM;               // one Q, K or V tile
  static constexpr int P_BYTES = QUANT ? 128 * 128 : 0;           // one e4m3 P tile in smem
  static constexpr int STAGES = QUANT ? (D == 128 ? 4 : 8) : (D == 128 ? 2 : 3);
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = 2 * TILE_BYTES;
  static constexpr int OFF_V = OFF_K + STAGES * TILE_BYTES;
  static constexpr int OFF_P = OFF_V + STAGES * TILE_BYTES;
  static constexpr int OFF_BAR = OFF_P + 2 * P_BYTES;
  static constexpr int SMEM_BYTES = OFF_BAR + 512 + 1024;          // barriers + 1 KB alignment slack
  // Q/K operand rows in shared memory (bytes) and their swizzle
  static constexpr int QK_ROW = QUANT ? D : 128;                   // bf16: one 64-element atom
  static constexpr uint32_t QK_LAYOUT = (QUANT && D == 64) ? kLayoutSW64 : kLayoutSW128;
  static constexpr uint32_t QK_SBO = 8 * QK_ROW;
  static constexpr int QK_KSTEPS = QUANT ? D / 32 : D / 16;
  static constexpr int PV_KSTEPS = QUANT ? 128 / 32 : 128 / 16;
  static constexpr uint32_t IDESC_QK =
      QUANT ? make_idesc(kFmtS32Acc, kFmtS8, kFmtS8, 0, 128, 128) : make_idesc(kFmtF32Acc, kFmtBF16, kFmtBF16, 0, 128, 128);
  static constexpr uint32_t IDESC_PV =
      QUANT ? make_idesc(kFmtF32Acc, kFmtE4M3, kFmtE4M3, 0, 128, D) : make_idesc(kFmtF32Acc, kFmtBF16, kFmtBF16, 1, 128, D);
  static constexpr int KIND_QK = QUANT ? kKindI8 : kKindF16;
  static constexpr int REGS_LOW = QUANT ? 96 : 80;
  static constexpr int REGS_HIGH = QUANT ? 200 : 208;
  static_assert(128 * REGS_LOW + 256 * REGS_HIGH <= kThreads * kLaunchRegs, "register split exceeds the launch budget");
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
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

// QUANT: O[tmem] (+)= P8[smem] V8[smem] for one 128-key tile.  P tile [128 rows]
// [128 keys] e4m3 and V^T tile [D rows][128 keys] e4m3, both K-major with the
// 128-byte swizzle; 32-byte K steps.
template <int D>
__device__ __forceinline__ void issue_pv_quant(uint32_t d_tmem, uint32_t p_smem, uint32_t v_smem, uint32_t accumulate) {
  using C = Cfg<D, true>;
#pragma unroll
  for (int s = 0; s < C::PV_KSTEPS; ++s) {
    const uint64_t a = make_sdesc(p_smem + s * 32, 16, 1024, kLayoutSW128);
    const uint64_t b = make_sdesc(v_smem + s * 32, 16, 1024, kLayoutSW128);
    mma_ss<kKindF8F6F4>(d_tmem, a, b, C::IDESC_PV, (s > 0 || accumulate) ? 1u : 0u);
  }
}

// BF16: O[tmem] (+)= P[tmem] V[smem]; V tile [128 keys][D] stored as 64-channel
// atoms (16 KB each), MN-major; P bf16 in TMEM (64 columns).
template <int D>
__device__ __forceinline__ void issue_pv_bf16(uint32_t d_tmem, uint32_t p_tmem, uint32_t v_smem, uint32_t accumulate) {
  using C = Cfg<D, false>;
#pragma unroll
  for (int s = 0; s < C::PV_KSTEPS; ++s) {
    const uint64_t b = make_sdesc(v_smem + s * 2048, 16384, 1024, kLayoutSW128);
    mma_ts<kKindF16>(d_tmem, p_tmem + s * 8, b, C::IDESC_PV, (s > 0 || accumulate) ? 1u : 0u);
  }
}

// One thread's 128-byte P row into a [128 x 128 B] tile with the 128-byte
// swizzle (16-byte chunk c of row r sits at chunk position c ^ (r % 8)); the
// tile base is 1024-byte aligned.
__device__ __forceinline__ void store_p_row(uint8_t* tile, int row, const uint32_t (&pk)[32]) {
  uint8_t* rp = tile + row * 128;
#pragma unroll
  for (int c = 0; c < 8; ++c)
    *reinterpret_cast<uint4*>(rp + ((c ^ (row & 7)) << 4)) = make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
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
  int q_per_token;        // QUANT: q_scale is [BH, Npad] (one scale per query token), else [BH, nT]
  RowMap o_map;           // where output row (bh, n) goes
};

// BF16 mode: S = Q K^T and O += P V with kind::f16 (bf16 in, fp32 acc), P
// rounded to bf16 and written over S in tensor memory.  P_t(j) overwrites
// S_t(j), so QK_t(j+1) follows PV_t(j) in issue order; tcgen05 operations from
// one thread execute in order and the commit after QK_t(j+1) also covers
// PV_t(j), so S_t(j+1) implies O_t stable.
template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    attn_bf16_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const Params prm) {
  using C = Cfg<D, false>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* q_full = bars + 0;
  uint64_t* kv_full = bars + 1;                       // [STAGES]
  uint64_t* kv_empty = bars + 1 + C::STAGES;          // [STAGES]
  uint64_t* s_full = bars + 1 + 2 * C::STAGES;        // [2] S_t written (MMA commit)
  uint64_t* p_full = s_full + 2;                      // [2] P_t written, O_t rescaled
  uint64_t* o_ready = p_full + 2;                     // [2] the last PV_t done
  uint64_t* tok = o_ready + 2;                        // [2] exp-phase token of softmax warpgroup t
  uint64_t* mma_done = tok + 2;
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
      mbar_init(&o_ready[t], 1);
      mbar_init(&tok[t], 128);
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
    regs_release<C::REGS_LOW>();
    if (warp == 0 && lane == 0) {
      // ---------------------------------------------------------- producer
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      mbar_arrive_expect_tx(q_full, 2 * C::TILE_BYTES);
      for (int t = 0; t < 2; ++t) {
        uint8_t* dst = smem + C::OFF_Q + t * C::TILE_BYTES;
#pragma unroll
        for (int a = 0; a < D / 64; ++a) tma_load_3d(dst + a * 16384, &tmQ, q_full, a * 64, (qt0 + t) * 128, bh);
      }
      int issued = 0;
      for (int j = 0; j < nT; ++j) {
        const int s = j % C::STAGES;
        if (j >= C::STAGES && !mbar_wait(&kv_empty[s], ((j / C::STAGES) - 1) & 1, abort_flag, limit)) break;
        mbar_arrive_expect_tx(&kv_full[s], 2 * C::TILE_BYTES);
        uint8_t* kd = smem + C::OFF_K + s * C::TILE_BYTES;
        uint8_t* vd = smem + C::OFF_V + s * C::TILE_BYTES;
#pragma unroll
        for (int a = 0; a < D / 64; ++a) {
          tma_load_3d(kd + a * 16384, &tmK, &kv_full[s], a * 64, j * 128, bh);
          tma_load_3d(vd + a * 16384, &tmV, &kv_full[s], a * 64, j * 128, bh);
        }
        issued = j + 1;
      }
      // drain: every load this thread issued must land before the CTA exits
      volatile int no_abort = 0;
      mbar_wait(q_full, 0, &no_abort, limit);
      for (int j = issued - C::STAGES < 0 ? 0 : issued - C::STAGES; j < issued; ++j)
        mbar_wait(&kv_full[j % C::STAGES], (j / C::STAGES) & 1, &no_abort, limit);
    } else if (warp == 1 && lane == 0) {
      // ---------------------------------------------------------- MMA issuer
      const uint32_t q_s = smem_u32(smem + C::OFF_Q);
      const uint32_t k_s = smem_u32(smem + C::OFF_K);
      const uint32_t v_s = smem_u32(smem + C::OFF_V);
      bool ok = true;
      if (prm.dbg_flags & 1) ok = mbar_wait(never, 0, abort_flag, limit);
      ok = ok && mbar_wait(q_full, 0, abort_flag, limit) && mbar_wait(&kv_full[0], 0, abort_flag, limit);
      if (ok) {
        tc_fence_after();
        for (int t = 0; t < 2; ++t) {
          issue_qk<D, false>(tmem + t * 128, q_s + t * C::TILE_BYTES, k_s);
          mma_commit(&s_full[t]);
        }
        for (int j = 0; j < nT && ok; ++j) {
          const int s = j % C::STAGES;
          for (int t = 0; t < 2; ++t) {
            if (!mbar_wait(&p_full[t], j & 1, abort_flag, limit)) { ok = false; break; }
            tc_fence_after();
            issue_pv_bf16<D>(tmem + 256 + t * D, tmem + t * 128, v_s + s * C::TILE_BYTES, j > 0 ? 1u : 0u);
            if (j + 1 < nT) {
              const int s1 = (j + 1) % C::STAGES;
              if (t == 0 && !mbar_wait(&kv_full[s1], ((j + 1) / C::STAGES) & 1, abort_flag, limit)) {
                ok = false;
                break;
              }
              issue_qk<D, false>(tmem + t * 128, q_s + t * C::TILE_BYTES, k_s + s1 * C::TILE_BYTES);
              mma_commit(&s_full[t]);
            } else {
              mma_commit(&o_ready[t]);
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
  } else {
    regs_claim<C::REGS_HIGH>();
    // ------------------------------------------------------------ softmax
    const int t = (warp - 4) >> 2;
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const uint32_t tS = tmem + lane_off + t * 128;
    const uint32_t tO = tmem + lane_off + 256 + t * D;
    const int qt = qt0 + t;
    const float sc = softmax_c(D);
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < nT; ++j) {
      if (!mbar_wait(&s_full[t], j & 1, abort_flag, limit)) { ok = false; break; }
      tc_fence_after();
      const int valid = min(128, N - j * 128);
      // the whole S row in registers (one wait for four loads)
      uint32_t sr[128];
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) tmem_ld32(tS + ch * 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[ch * 32]));
      tmem_wait_ld();
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) regs_after_wait(*reinterpret_cast<uint32_t(*)[32]>(&sr[ch * 32]));
      float f[128];
#pragma unroll
      for (int i = 0; i < 128; ++i) f[i] = __uint_as_float(sr[i]);
      const bool full = valid == 128;
      // row max of the raw scores (s is monotone in f since sc > 0)
      float mx;
      if (full) {
        float a0 = f[0], a1 = f[1], a2 = f[2], a3 = f[3];
#pragma unroll
        for (int i = 4; i + 8 <= 128; i += 8) {   // columns 4 .. 123
          a0 = fmax3(a0, f[i], f[i + 1]);
          a1 = fmax3(a1, f[i + 2], f[i + 3]);
          a2 = fmax3(a2, f[i + 4], f[i + 5]);
          a3 = fmax3(a3, f[i + 6], f[i + 7]);
        }
        mx = fmaxf(fmax3(a0, a1, f[124]), fmax3(a2, a3, fmax3(f[125], f[126], f[127])));
      } else {
        mx = -INFINITY;
#pragma unroll
        for (int i = 0; i < 128; ++i) mx = fmaxf(mx, i < valid ? f[i] : -INFINITY);
      }
      const float m_new = fmaxf(m, __fmul_rn(mx, sc));
      const float alpha = (m == -INFINITY) ? 0.f : ex2_approx(__fsub_rn(m, m_new));
      const float bias = __fsub_rn(0.f, m_new);         // x = f * sc + bias = s - m_new
      // The two warpgroups take turns on the exponential phase (the SFU-bound
      // part), so each one's compare phase overlaps the other's exponentials:
      // warpgroup 0 goes first, then they alternate.
      if (t == 1 || j > 0) {
        if (!mbar_wait(&tok[t], (t == 0 ? (j - 1) : j) & 1, abort_flag, limit)) { ok = false; break; }
      }
      // p = 2^x, row sum (two packed accumulators), P packed as bf16 for the PV MMA
      float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
      uint32_t pk[64];
      if (full) {
#pragma unroll
        for (int g = 0; g < 32; ++g) {
          const float2 x01 = ffma2(f[4 * g], f[4 * g + 1], sc, bias);
          const float2 x23 = ffma2(f[4 * g + 2], f[4 * g + 3], sc, bias);
          const float p0 = ex2_approx(x01.x), p1 = ex2_approx(x01.y), p2 = ex2_approx(x23.x), p3 = ex2_approx(x23.y);
          acc0 = fadd2(acc0, make_float2(p0, p1));
          acc1 = fadd2(acc1, make_float2(p2, p3));
          pk[2 * g] = pack_bf16x2(p0, p1);
          pk[2 * g + 1] = pack_bf16x2(p2, p3);
        }
      } else {
#pragma unroll
        for (int g = 0; g < 32; ++g) {
          const float2 x01 = ffma2(f[4 * g], f[4 * g + 1], sc, bias);
          const float2 x23 = ffma2(f[4 * g + 2], f[4 * g + 3], sc, bias);
          const float p0 = 4 * g + 0 < valid ? ex2_approx(x01.x) : 0.f;
          const float p1 = 4 * g + 1 < valid ? ex2_approx(x01.y) : 0.f;
          const float p2 = 4 * g + 2 < valid ? ex2_approx(x23.x) : 0.f;
          const float p3 = 4 * g + 3 < valid ? ex2_approx(x23.y) : 0.f;
          acc0 = fadd2(acc0, make_float2(p0, p1));
          acc1 = fadd2(acc1, make_float2(p2, p3));
          pk[2 * g] = pack_bf16x2(p0, p1);
          pk[2 * g + 1] = pack_bf16x2(p2, p3);
        }
      }
      mbar_arrive(&tok[1 - t]);     // hand the exponential phase to the other warpgroup
      const bool grew = j > 0 && __any_sync(0xffffffffu, m_new > m);
      tmem_st32(tS, *reinterpret_cast<uint32_t(*)[32]>(&pk[0]));
      tmem_st32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&pk[32]));
      // rescale O_t by alpha where the max grew (O_t is complete: the commit
      // after QK_t(j) covers PV_t(j-1))
      if (grew) {
#pragma unroll
        for (int ch = 0; ch < D / 32; ++ch) {
          uint32_t r[32];
          tmem_ld32(tO + ch * 32, r);
          tmem_wait_ld_regs(r);
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            const float2 v = fmul2(make_float2(__uint_as_float(r[i]), __uint_as_float(r[i + 1])), alpha);
            r[i] = __float_as_uint(v.x);
            r[i + 1] = __float_as_uint(v.y);
          }
          tmem_st32(tO + ch * 32, r);
        }
      }
      tmem_wait_st();
      const float2 acc = fadd2(acc0, acc1);
      l = __fadd_rn(__fmul_rn(l, alpha), __fadd_rn(acc.x, acc.y));
      m = m_new;
      tc_fence_before();
      mbar_arrive(&p_full[t]);
    }
    // ---------------------------------------------------------- epilogue
    if (ok && mbar_wait(&o_ready[t], 0, abort_flag, limit)) {
      tc_fence_after();
      const int gq = qt * 128 + row;
      __nv_bfloat16* orow = prm.o + prm.o_map.row(bh, gq, N) * D;
#pragma unroll
      for (int ch = 0; ch < D / 32; ++ch) {
        uint32_t r[32];
        tmem_ld32(tO + ch * 32, r);
        tmem_wait_ld_regs(r);
        uint32_t w[16];
#pragma unroll
        for (int g = 0; g < 16; ++g) w[g] = pack_bf16x2(__fdiv_rn(__uint_as_float(r[2 * g]), l), __fdiv_rn(__uint_as_float(r[2 * g + 1]), l));
        if (qt < nT && gq < N) {
          uint4* dst = reinterpret_cast<uint4*>(orow + ch * 32);
#pragma unroll
          for (int v = 0; v < 4; ++v)
            if (SAGE_DCHECK((prm.o_map.row(bh, gq, N) * D + ch * 32) / 8 + v, (long long)gridDim.y * N * D / 8,
                            kSiteAttnOut))
              dst[v] = make_uint4(w[4 * v], w[4 * v + 1], w[4 * v + 2], w[4 * v + 3]);
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

// ---------------------------------------------------------------- INT8/FP8 kernel
// The INT8/FP8 kernel: the same CTA shape, warp roles and tensor-memory map as
// the BF16 kernel (12 warps; warpgroups 1 and 2 own Q tiles 0 and 1, one query
// row per thread, and take turns on the exponential phase), with the P tile in
// shared memory and an event-driven MMA thread:
//   S = Q_i8 K_i8^T (tcgen05 kind::i8, exact int32), dequantized with
//   q_scale * k_scale * log2(e)/sqrt(d); P8 = e4m3(p * 448) written to a
//   128-byte-swizzled shared-memory tile; O += P8 V8 (kind::f8f6f4 from shared
//   memory, fp32 in tensor memory).  As soon as a softmax warpgroup has S_t(j)
//   in registers it releases the S columns (s_free), so QK_t(j+1) runs while
//   the exponentials of step j do; PV_t(j) is issued on p_full, and its
//   commit (o_ready) tells the warpgroup that O_t is stable and the P buffer
//   free again.
//   SAGE_Q12_POLY_GROUPS of every 16 groups of four scores can take 2^x on the
//   FMA pipe (exp2_fma2) instead of the SFU; 0 by default: in this schedule the
//   exponential phase is bound by its instruction stream, and the longer FMA
//   sequence made it slower.
#ifndef SAGE_Q12_POLY_GROUPS
#define SAGE_Q12_POLY_GROUPS 0
#endif

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    attn_i8f8_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const Params prm) {
  using C = Cfg<D, true>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* q_full = bars + 0;
  uint64_t* kv_full = bars + 1;                       // [STAGES]
  uint64_t* kv_empty = bars + 1 + C::STAGES;          // [STAGES]
  uint64_t* s_full = bars + 1 + 2 * C::STAGES;        // [2] S_t written (MMA commit)
  uint64_t* s_free = s_full + 2;                      // [2] S_t read into registers
  uint64_t* p_full = s_free + 2;                      // [2] P_t written, O_t rescaled
  uint64_t* o_ready = p_full + 2;                     // [2] PV_t done
  uint64_t* tok = o_ready + 2;                        // [2] exp-phase token of softmax warpgroup t
  uint64_t* mma_done = tok + 2;
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
      mbar_init(&s_free[t], 128);
      mbar_init(&p_full[t], 128);
      mbar_init(&o_ready[t], 1);
      mbar_init(&tok[t], 128);
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
    regs_release<C::REGS_LOW>();
    if (warp == 0 && lane == 0) {
      // ---------------------------------------------------------- producer
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      mbar_arrive_expect_tx(q_full, 2 * C::TILE_BYTES);
      for (int t = 0; t < 2; ++t) tma_load_2d(smem + C::OFF_Q + t * C::TILE_BYTES, &tmQ, q_full, 0, bh * prm.Npad + (qt0 + t) * 128);
      int issued = 0;
      for (int j = 0; j < nT; ++j) {
        const int s = j % C::STAGES;
        if (j >= C::STAGES && !mbar_wait(&kv_empty[s], ((j / C::STAGES) - 1) & 1, abort_flag, limit)) break;
        mbar_arrive_expect_tx(&kv_full[s], 2 * C::TILE_BYTES);
        tma_load_2d(smem + C::OFF_K + s * C::TILE_BYTES, &tmK, &kv_full[s], 0, bh * prm.Npad + j * 128);
        tma_load_2d(smem + C::OFF_V + s * C::TILE_BYTES, &tmV, &kv_full[s], j * 128, bh * D);
        issued = j + 1;
      }
      // drain: every load this thread issued must land before the CTA exits
      volatile int no_abort = 0;
      mbar_wait(q_full, 0, &no_abort, limit);
      for (int j = issued - C::STAGES < 0 ? 0 : issued - C::STAGES; j < issued; ++j)
        mbar_wait(&kv_full[j % C::STAGES], (j / C::STAGES) & 1, &no_abort, limit);
    } else if (warp == 1 && lane == 0) {
      // ---------------------------------------------------------- MMA issuer
      const uint32_t q_s = smem_u32(smem + C::OFF_Q);
      const uint32_t k_s = smem_u32(smem + C::OFF_K);
      const uint32_t v_s = smem_u32(smem + C::OFF_V);
      const uint32_t p_s = smem_u32(smem + C::OFF_P);
      bool ok = true;
      if (prm.dbg_flags & 1) ok = mbar_wait(never, 0, abort_flag, limit);
      ok = ok && mbar_wait(q_full, 0, abort_flag, limit) && mbar_wait(&kv_full[0], 0, abort_flag, limit);
      if (ok) {
        tc_fence_after();
        for (int t = 0; t < 2; ++t) {
          issue_qk<D, true>(tmem + t * 128, q_s + t * C::TILE_BYTES, k_s);
          mma_commit(&s_full[t]);
        }
        // Event driven: each tile runs QK(1), PV(0), QK(2), PV(1), ... as its
        // barriers allow, so one slow tile never holds back the other.
        //   QK_t(j+1) needs s_free_t(j) (S_t(j) read out) and K_{j+1} loaded;
        //   PV_t(j)   needs p_full_t(j) (P_t(j) stored, O_t rescaled).
        int qk_next[2] = {1, 1}, pv_next[2] = {0, 0};
        long long last = clock64();
        while (ok && (pv_next[0] < nT || pv_next[1] < nT)) {
          bool progressed = false;
#pragma unroll
          for (int t = 0; t < 2; ++t) {
            const int jq = qk_next[t];
            if (jq < nT && mbar_test(&s_free[t], (jq - 1) & 1) &&
                mbar_test(&kv_full[jq % C::STAGES], (jq / C::STAGES) & 1)) {
              tc_fence_after();
              issue_qk<D, true>(tmem + t * 128, q_s + t * C::TILE_BYTES, k_s + (jq % C::STAGES) * C::TILE_BYTES);
              mma_commit(&s_full[t]);
              qk_next[t] = jq + 1;
              progressed = true;
            }
            const int jp = pv_next[t];
            if (jp < qk_next[t] && jp < nT && mbar_test(&p_full[t], jp & 1)) {
              tc_fence_after();
              issue_pv_quant<D>(tmem + 256 + t * D, p_s + t * C::P_BYTES, v_s + (jp % C::STAGES) * C::TILE_BYTES,
                                jp > 0 ? 1u : 0u);
              mma_commit(&o_ready[t]);
              pv_next[t] = jp + 1;
              // the K/V stage of step jp is free once both tiles' PV(jp) are issued
              if (pv_next[1 - t] > jp) mma_commit(&kv_empty[jp % C::STAGES]);
              progressed = true;
            }
          }
          if (progressed) {
            last = clock64();
          } else if (*abort_flag || clock64() - last > limit) {
            *abort_flag = 1;
            ok = false;
          } else {
            __nanosleep(20);   // leave the issue slots to the softmax warps on this SMSP
          }
        }
      }
      // drain: every MMA issued must complete before TMEM is released
      mma_commit(mma_done);
      volatile int no_abort = 0;
      mbar_wait(mma_done, 0, &no_abort, limit);
    }
  } else {
    regs_claim<C::REGS_HIGH>();
    // ------------------------------------------------------------ softmax
    const int t = (warp - 4) >> 2;
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const uint32_t tS = tmem + lane_off + t * 128;
    const uint32_t tO = tmem + lane_off + 256 + t * D;
    uint8_t* p_row = smem + C::OFF_P + t * C::P_BYTES + row * 128;   // this row of the swizzled P tile
    const int qt = qt0 + t;
    const float c = softmax_c(D);
    float qs;
    if (qt < nT)
    {
      const size_t qi = prm.q_per_token ? (size_t)bh * prm.Npad + qt * 128 + row : (size_t)bh * nT + qt;
      const long long qe = (long long)gridDim.y * (prm.q_per_token ? prm.Npad : nT);
      qs = SAGE_DCHECK(qi, qe, kSiteAttnQScale) ? prm.q_scale[qi] : 0.f;
      (void)qe;
    }
    else
      qs = 0.f;
    // p is produced already multiplied by the P scale 448 (2^(s - m + log2 448)),
    // so l accumulates 448 * sum(p) and the epilogue divides by it directly.
    constexpr float kLog2PScale = 8.807354922057604f;
    // int32 S + 0x4B400000 read as a float is 12582912 + S exactly (|S| <= 127*127*128 < 2^22)
    constexpr uint32_t kMagicBits = 0x4B400000u;
    constexpr float kMagic = 12582912.0f;
    const long long ks_ext = (long long)gridDim.y * nT;
    (void)ks_ext;
    float ks_next = SAGE_DCHECK((size_t)bh * nT, ks_ext, kSiteAttnKScale) ? prm.k_scale[(size_t)bh * nT] : 0.f;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    uint32_t sr[128];
    for (int j = 0; j < nT && ok; ++j) {
      const float sc = __fmul_rn(__fmul_rn(qs, ks_next), c);
      if (j + 1 < nT && SAGE_DCHECK((size_t)bh * nT + j + 1, ks_ext, kSiteAttnKScale))
        ks_next = prm.k_scale[(size_t)bh * nT + j + 1];   // prefetch the next tile's scale
      if (!mbar_wait(&s_full[t], j & 1, abort_flag, limit)) { ok = false; break; }
      tc_fence_after();
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) tmem_ld32(tS + ch * 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[ch * 32]));
      tmem_wait_ld();
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) regs_after_wait(*reinterpret_cast<uint32_t(*)[32]>(&sr[ch * 32]));
      tc_fence_before();
      mbar_arrive(&s_free[t]);     // the S columns may now take QK_t(j+1)
      const int valid = min(128, N - j * 128);
      const bool full = valid == 128;
      // scores as 12582912 + S (exact) until after the max
      float f[128];
#pragma unroll
      for (int i = 0; i < 128; ++i) f[i] = __uint_as_float(sr[i] + kMagicBits);
      float mx;
      if (full) {
        float a0 = f[0], a1 = f[1], a2 = f[2], a3 = f[3];
#pragma unroll
        for (int i = 4; i + 8 <= 128; i += 8) {   // columns 4 .. 123
          a0 = fmax3(a0, f[i], f[i + 1]);
          a1 = fmax3(a1, f[i + 2], f[i + 3]);
          a2 = fmax3(a2, f[i + 4], f[i + 5]);
          a3 = fmax3(a3, f[i + 6], f[i + 7]);
        }
        mx = fmaxf(fmax3(a0, a1, f[124]), fmax3(a2, a3, fmax3(f[125], f[126], f[127])));
      } else {
        mx = -INFINITY;
#pragma unroll
        for (int i = 0; i < 128; ++i) mx = fmaxf(mx, i < valid ? f[i] : -INFINITY);
      }
      mx = __fsub_rn(mx, kMagic);                       // exact: the integer max as a float
#pragma unroll
      for (int i = 0; i < 128; i += 2) {                // exact: back to S as a float
        const float2 v = fadd2(make_float2(f[i], f[i + 1]), make_float2(-kMagic, -kMagic));
        f[i] = v.x;
        f[i + 1] = v.y;
      }
      const float m_new = fmaxf(m, __fmul_rn(mx, sc));
      const float alpha = (m == -INFINITY) ? 0.f : ex2_approx(__fsub_rn(m, m_new));
      const float bias = __fsub_rn(kLog2PScale, m_new);  // x = s * sc + bias = s - m_new + log2 448
      // the two warpgroups take turns on the exponential phase: warpgroup 0
      // first, then they alternate
      if (t == 1 || j > 0) {
        if (!mbar_wait(&tok[t], (t == 0 ? (j - 1) : j) & 1, abort_flag, limit)) { ok = false; break; }
      }
      float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
      uint32_t pk[32];
      // one group of four scores: 2^x (SFU, or FMA pipe for the polynomial groups), row sum, e4m3 pack;
      // MASK zeroes the keys >= N of the last tile.  Two copies of the loop, so the full tiles carry no
      // masking at all.
      auto group = [&](int g, bool mask) {
        const float2 x01 = ffma2(f[4 * g], f[4 * g + 1], sc, bias);
        const float2 x23 = ffma2(f[4 * g + 2], f[4 * g + 3], sc, bias);
        float p0, p1, p2, p3;
        if (g % 16 >= 16 - SAGE_Q12_POLY_GROUPS) {
          const float2 e01 = exp2_fma2(x01), e23 = exp2_fma2(x23);
          p0 = e01.x; p1 = e01.y; p2 = e23.x; p3 = e23.y;
        } else {
          p0 = ex2_approx(x01.x); p1 = ex2_approx(x01.y); p2 = ex2_approx(x23.x); p3 = ex2_approx(x23.y);
        }
        if (mask) {
          p0 = 4 * g + 0 < valid ? p0 : 0.f;
          p1 = 4 * g + 1 < valid ? p1 : 0.f;
          p2 = 4 * g + 2 < valid ? p2 : 0.f;
          p3 = 4 * g + 3 < valid ? p3 : 0.f;
        }
        acc0 = fadd2(acc0, make_float2(p0, p1));
        acc1 = fadd2(acc1, make_float2(p2, p3));
        pk[g] = pack_e4m3x4(p0, p1, p2, p3);
      };
      if (full) {
#pragma unroll
        for (int g = 0; g < 32; ++g) group(g, false);
      } else {
#pragma unroll
        for (int g = 0; g < 32; ++g) group(g, true);
      }
      mbar_arrive(&tok[1 - t]);     // hand the exponential phase to the other warpgroup
      const bool grew = j > 0 && __any_sync(0xffffffffu, m_new > m);
      if (j > 0) {
        if (!mbar_wait(&o_ready[t], (j - 1) & 1, abort_flag, limit)) { ok = false; break; }
        tc_fence_after();
      }
#pragma unroll
      for (int cc = 0; cc < 8; ++cc)
        *reinterpret_cast<uint4*>(p_row + ((cc ^ (row & 7)) << 4)) = make_uint4(pk[4 * cc], pk[4 * cc + 1], pk[4 * cc + 2], pk[4 * cc + 3]);
      fence_proxy_async_smem();    // generic-proxy writes -> visible to the MMA
      // rescale O_t by alpha where the max grew (PV_t(j-1) is done)
      if (grew) {
#pragma unroll
        for (int ch = 0; ch < D / 32; ++ch) {
          uint32_t r[32];
          tmem_ld32(tO + ch * 32, r);
          tmem_wait_ld_regs(r);
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            const float2 v = fmul2(make_float2(__uint_as_float(r[i]), __uint_as_float(r[i + 1])), alpha);
            r[i] = __float_as_uint(v.x);
            r[i + 1] = __float_as_uint(v.y);
          }
          tmem_st32(tO + ch * 32, r);
        }
        tmem_wait_st();
      }
      const float2 acc = fadd2(acc0, acc1);
      l = __fadd_rn(__fmul_rn(l, alpha), __fadd_rn(acc.x, acc.y));
      m = m_new;
      tc_fence_before();
      mbar_arrive(&p_full[t]);
    }
    // ---------------------------------------------------------- epilogue
    if (ok && mbar_wait(&o_ready[t], (uint32_t)((nT - 1) & 1), abort_flag, limit)) {
      tc_fence_after();
      const int gq = qt * 128 + row;
      __nv_bfloat16* orow = prm.o + prm.o_map.row(bh, gq, N) * D;
      const float* vs = prm.v_scale + (size_t)bh * D;
      const bool vs_ok = SAGE_DCHECK((size_t)bh * D + D - 1, (long long)gridDim.y * D, kSiteAttnVScale);
#pragma unroll
      for (int ch = 0; ch < D / 32; ++ch) {
        uint32_t r[32];
        tmem_ld32(tO + ch * 32, r);
        tmem_wait_ld_regs(r);
        uint32_t w[16];
#pragma unroll
        for (int g = 0; g < 16; ++g) {
          const float a0 = __fmul_rn(__uint_as_float(r[2 * g]), vs_ok ? vs[ch * 32 + 2 * g] : 0.f);
          const float a1 = __fmul_rn(__uint_as_float(r[2 * g + 1]), vs_ok ? vs[ch * 32 + 2 * g + 1] : 0.f);
          w[g] = pack_bf16x2(__fdiv_rn(a0, l), __fdiv_rn(a1, l));   // l holds 448 * sum(p)
        }
        if (qt < nT && gq < N) {
          uint4* dst = reinterpret_cast<uint4*>(orow + ch * 32);
#pragma unroll
          for (int v = 0; v < 4; ++v)
            if (SAGE_DCHECK((prm.o_map.row(bh, gq, N) * D + ch * 32) / 8 + v, (long long)gridDim.y * N * D / 8,
                            kSiteAttnOut))
              dst[v] = make_uint4(w[4 * v], w[4 * v + 1], w[4 * v + 2], w[4 * v + 3]);
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

template <int D>
cudaError_t launch_attn_i8f8_d(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const Params& prm,
                            int BH, cudaStream_t stream) {
  using C = Cfg<D, true>;
  auto kern = attn_i8f8_kernel<D>;
  // the setmaxnreg split must fit in the registers the block is launched with,
  // or the increase would wait forever
  cudaFuncAttributes fa;
  cudaError_t e = cudaFuncGetAttributes(&fa, kern);
  if (e != cudaSuccess) return e;
  if (fa.numRegs * kThreads < 128 * C::REGS_LOW + 256 * C::REGS_HIGH) return cudaErrorInvalidConfiguration;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  dim3 grid((prm.nT + 1) / 2, BH);
  kern<<<grid, kThreads, C::SMEM_BYTES, stream>>>(tq, tk, tv, prm);
  return cudaGetLastError();
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

// One 128-row P.V product through the attention kernels' operand paths: QUANT
// writes P rows into a swizzled shared-memory tile (store_p_row) and issues the
// SS kind::f8f6f4 MMA; BF16 writes P into TMEM (tcgen05.st) and issues the TS
// kind::f16 MMA with an MN-major V.  V arrives by TMA.
template <int D, bool QUANT>
__global__ void __launch_bounds__(128, 1)
    dbg_pv_kernel(const __grid_constant__ CUtensorMap tmV, const uint8_t* p, float* out) {
  using C = Cfg<D, QUANT>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* p_tile = smem + C::TILE_BYTES;                           // QUANT only: [128 x 128 B]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::TILE_BYTES + (QUANT ? 128 * 128 : 0));
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
  const uint32_t* prow = reinterpret_cast<const uint32_t*>(p + (size_t)row * 128 * (QUANT ? 1 : 2));
  if constexpr (QUANT) {
    uint32_t r[32];
    for (int i = 0; i < 32; ++i) r[i] = prow[i];
    store_p_row(p_tile, row, r);
    fence_proxy_async_smem();
  } else {
    for (int h = 0; h < 2; ++h) {
      uint32_t r[32];
      for (int i = 0; i < 32; ++i) r[i] = prow[h * 32 + i];
      tmem_st32(tmem + lane_off + h * 32, r);
    }
    tmem_wait_st();
  }
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
    if (mbar_wait(&bars[0], 0, &abort_s, kDefaultTimeoutCycles)) {
      if constexpr (QUANT)
        issue_pv_quant<D>(tmem + 128, smem_u32(p_tile), smem_u32(smem), 0u);
      else
        issue_pv_bf16<D>(tmem + 128, tmem, smem_u32(smem), 0u);
    }
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

template <int D>
cudaError_t launch_attn_bf16_d(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const Params& prm,
                               int BH, cudaStream_t stream) {
  using C = Cfg<D, false>;
  auto kern = attn_bf16_kernel<D>;
  // the setmaxnreg split must fit in the registers the block is launched with,
  // or the increase would wait forever
  cudaFuncAttributes fa;
  cudaError_t e = cudaFuncGetAttributes(&fa, kern);
  if (e != cudaSuccess) return e;
  if (fa.numRegs * kThreads < 128 * C::REGS_LOW + 256 * C::REGS_HIGH) return cudaErrorInvalidConfiguration;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  dim3 grid((prm.nT + 1) / 2, BH);
  kern<<<grid, kThreads, C::SMEM_BYTES, stream>>>(tq, tk, tv, prm);
  return cudaGetLastError();
}

}  // namespace

unsigned debug_take_attention(unsigned long long* first) {
#ifdef SAGE_DEBUG
  return debug_take_tu(first);
#else
  (void)first;
  return 0;
#endif
}

cudaError_t launch_attn_i8f8(const int8_t* q_i8, const float* q_scale, const int8_t* k_i8, const float* k_scale,
                             const uint8_t* v_f8t, const float* v_scale, void* o, int BH, int N, int d,
                             uint32_t* status, long long timeout_cycles, int dbg_flags, cudaStream_t stream,
                             bool q_per_token, RowMap o_map) {
  const int nT = num_tiles(N), Npad = nT * kTile;
  alignas(64) CUtensorMap tq, tk, tv;
  const CUtensorMapSwizzle qk_sw = d == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  if (!encode_tmap_2d(&tq, CU_TENSOR_MAP_DATA_TYPE_UINT8, q_i8, d, (uint64_t)BH * Npad, d, d, 128, qk_sw) ||
      !encode_tmap_2d(&tk, CU_TENSOR_MAP_DATA_TYPE_UINT8, k_i8, d, (uint64_t)BH * Npad, d, d, 128, qk_sw) ||
      !encode_tmap_2d(&tv, CU_TENSOR_MAP_DATA_TYPE_UINT8, v_f8t, Npad, (uint64_t)BH * d, Npad, 128, d,
                      CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  Params prm{q_scale, k_scale, v_scale, static_cast<__nv_bfloat16*>(o), status, N, nT, Npad, timeout_cycles, dbg_flags,
             q_per_token ? 1 : 0, o_map};
  if (d == 128) return launch_attn_i8f8_d<128>(tq, tk, tv, prm, BH, stream);
  if (d == 64) return launch_attn_i8f8_d<64>(tq, tk, tv, prm, BH, stream);
  return cudaErrorInvalidValue;
}

cudaError_t launch_attn_bf16(const void* q, const void* k, const void* v, void* o, int BH, int N, int d,
                             uint32_t* status, long long timeout_cycles, cudaStream_t stream, RowMap o_map) {
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
  Params prm{nullptr, nullptr, nullptr, static_cast<__nv_bfloat16*>(o), status, N, nT, nT * kTile, timeout_cycles, 0, 0,
             o_map};
  if (d == 128) return launch_attn_bf16_d<128>(tq, tk, tv, prm, BH, stream);
  if (d == 64) return launch_attn_bf16_d<64>(tq, tk, tv, prm, BH, stream);
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
  const int smem = 128 * d * (quant ? 1 : 2) + (quant ? 128 * 128 : 0) + 64 + 1024;
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
