// ulysses.cu -- layout copies around the DeepSpeed-Ulysses all-to-all.
//
// TMAP write-up, "Optimising multi-GPU parallelism" (DeepSpeed-Ulysses
// sequence parallelism): each GPU holds a 1/P slice of the sequence for all H
// heads; an all-to-all hands every GPU the whole sequence for H/P heads,
// attention runs per head, and a second all-to-all returns the output to the
// sequence slices.  The collectives themselves are NCCL's; these kernels only
// move rows of d contiguous bf16 values between the layouts (Hl = H / P,
// N = P * Nl).  The exchange buffers are [P][B][Nl][Hl][d]: chunk r holds the
// sending rank's tokens for heads r*Hl .. r*Hl + Hl - 1, token-major, so one
// token's heads of one chunk are Hl consecutive rows.
//
//   op 0  send:     x [B, Nl, H, d]          -> s [P][B][Nl][Hl][d]
//   op 1  recv O:   r [P][B][Nl][Hl][d]      -> y [B, Nl, H, d]
//   op 2  gather:   r [P][B][Nl][Hl][d]      -> y [B, Hl, N, d]  (the plain attention layout)
//   op 3  scatter:  y [B, Hl, N, d]          -> s [P][B][Nl][Hl][d]
//
// sage_attn_fwd_seqpar reads and writes the [P] layout directly in INT8/FP8
// mode; ops 2 and 3 serve the BF16 mode and tests.  The [P] side may be
// strided (chunk_rows rows between consecutive chunks, first chunk at row
// base_rows), so that several tensors can share one exchange buffer.
#include <cuda_runtime.h>

#include <cstdint>

#include "internal.h"

namespace sage {

namespace {

struct UlyGeom {
  long long B, Nl, H, Hl, P, N;
  long long chunk_rows, base_rows;  // of the [P] side
  long long src_rows, dst_rows;     // extents of the two buffers, in rows (checks of a debug build)
};

// Row of the [P] side holding (chunk r, b, token n of the chunk, head hl).
__device__ __forceinline__ long long p_row(const UlyGeom& g, long long r, long long b, long long n, long long hl) {
  return g.base_rows + r * g.chunk_rows + (b * g.Nl + n) * g.Hl + hl;
}

// Source row of destination row i (i enumerates the destination densely).
__device__ __forceinline__ long long src_row(long long i, int op, const UlyGeom& g) {
  if (op == 0 || op == 3) {  // dst (r, b, n, hl) in the [P] buffer
    const long long inner = g.B * g.Nl * g.Hl;
    const long long r = i / inner, q = i - r * inner;
    const long long b = q / (g.Nl * g.Hl), n = (q / g.Hl) % g.Nl, hl = q % g.Hl;
    if (op == 0) return (b * g.Nl + n) * g.H + r * g.Hl + hl;     // x (b, n, r*Hl + hl)
    return (b * g.Hl + hl) * g.N + r * g.Nl + n;                  // y (b, hl, r*Nl + n)
  }
  if (op == 1) {  // dst (b, n, h) <- [P] buffer (h / Hl, b, n, h % Hl)
    const long long b = i / (g.Nl * g.H), n = (i / g.H) % g.Nl, h = i % g.H;
    const long long r = h / g.Hl;
    return p_row(g, r, b, n, h - r * g.Hl);
  }
  // op 2: dst (b, hl, tok) <- [P] buffer (tok / Nl, b, tok % Nl, hl)
  const long long b = i / (g.Hl * g.N), hl = (i / g.N) % g.Hl, tok = i % g.N;
  const long long r = tok / g.Nl;
  return p_row(g, r, b, tok - r * g.Nl, hl);
}

// Destination row of the i-th row of the dense destination enumeration.
__device__ __forceinline__ long long dst_row(long long i, int op, const UlyGeom& g) {
  if (op == 0 || op == 3) {  // the destination is the [P] buffer
    const long long inner = g.B * g.Nl * g.Hl;
    const long long r = i / inner;
    return g.base_rows + r * g.chunk_rows + (i - r * inner);
  }
  return i;
}

// One row is VPR 16-byte vectors; each thread copies one vector.
template <int VPR>
__global__ void __launch_bounds__(256) permute_rows_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst,
                                                           long long rows, int op, UlyGeom g) {
  const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long i = t / VPR;
  if (i >= rows) return;
  const int v = (int)(t % VPR);
  const long long si = src_row(i, op, g) * VPR + v, di = dst_row(i, op, g) * VPR + v;
  if (SAGE_DCHECK(si, g.src_rows * VPR, kSiteUlyssesSrc) && SAGE_DCHECK(di, g.dst_rows * VPR, kSiteUlyssesDst))
    dst[di] = src[si];
}

}  // namespace

unsigned debug_take_ulysses(unsigned long long* first) {
#ifdef SAGE_DEBUG
  return debug_take_tu(first);
#else
  (void)first;
  return 0;
#endif
}

cudaError_t launch_ulysses_permute(const void* src, void* dst, int B, int Nl, int H, int d, int P, int op,
                                   long long chunk_rows, long long base_rows, cudaStream_t stream) {
  UlyGeom g;
  g.B = B;
  g.Nl = Nl;
  g.H = H;
  g.P = P;
  g.Hl = H / P;
  g.N = (long long)P * Nl;
  g.chunk_rows = chunk_rows > 0 ? chunk_rows : (long long)B * g.Hl * Nl;
  g.base_rows = base_rows;
  const long long rows = (long long)B * Nl * H;
  // the [P] side spans base_rows + (P - 1) * chunk_rows + one chunk; the other side is dense
  const long long p_rows = g.base_rows + (g.P - 1) * g.chunk_rows + (long long)B * g.Hl * Nl;
  const bool p_is_dst = op == 0 || op == 3;
  g.src_rows = p_is_dst ? rows : p_rows;
  g.dst_rows = p_is_dst ? p_rows : rows;
  const int vpr = d * 2 / 16;
  const long long threads = rows * vpr;
  const unsigned grid = (unsigned)((threads + 255) / 256);
  if (vpr == 16)
    permute_rows_kernel<16><<<grid, 256, 0, stream>>>(static_cast<const uint4*>(src), static_cast<uint4*>(dst), rows,
                                                      op, g);
  else
    permute_rows_kernel<8><<<grid, 256, 0, stream>>>(static_cast<const uint4*>(src), static_cast<uint4*>(dst), rows, op,
                                                     g);
  return cudaGetLastError();
}

}  // namespace sage
