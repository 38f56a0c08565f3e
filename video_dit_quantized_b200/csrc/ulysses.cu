// ulysses.cu -- layout permutations around the DeepSpeed-Ulysses all-to-all.
//
// TMAP write-up, "Optimising multi-GPU parallelism" (DeepSpeed-Ulysses
// sequence parallelism): each GPU holds a 1/P slice of the sequence for all H
// heads; an all-to-all hands every GPU the whole sequence for H/P heads,
// attention runs per head, and a second all-to-all returns the output to the
// sequence slices.  The collectives
// themselves are NCCL's; these kernels only move rows of d contiguous bf16
// values between the four layouts (Hl = H / P, N = P * Nl):
//
//   op 0  send Q/K/V:  x [B, Nl, H, d]          -> s [P][B, Hl, Nl, d]
//   op 1  recv Q/K/V:  r [P][B, Hl, Nl, d]      -> y [B, Hl, N, d]  (the attention layout)
//   op 2  send O:      o [B, Hl, N, d]          -> s [P][B, Hl, Nl, d]
//   op 3  recv O:      r [P][B, Hl, Nl, d]      -> y [B, Nl, H, d]
//
// The [P] side may be strided (chunk_rows rows between consecutive chunks,
// first chunk at row base_rows) so that Q, K and V share one send buffer
// [P][3][B, Hl, Nl, d] and one all-to-all.
#include <cuda_runtime.h>

#include <cstdint>

#include "internal.h"

namespace sage {

namespace {

struct UlyGeom {
  long long B, Nl, H, Hl, P, N;
  long long chunk_rows, base_rows;  // of the [P] side
};

// Source row of destination row i.
__device__ __forceinline__ long long src_row(long long i, int op, const UlyGeom& g) {
  if (op == 0) {  // dst (r, b, hl, n) in the [P] buffer <- x (b, n, r*Hl + hl)
    const long long inner = g.B * g.Hl * g.Nl;
    const long long r = i / inner, q = i - r * inner;
    const long long b = q / (g.Hl * g.Nl), hl = (q / g.Nl) % g.Hl, n = q % g.Nl;
    return (b * g.Nl + n) * g.H + r * g.Hl + hl;
  }
  if (op == 1) {  // dst (b, hl, tok) <- [P] buffer (tok / Nl, b, hl, tok % Nl)
    const long long b = i / (g.Hl * g.N), hl = (i / g.N) % g.Hl, tok = i % g.N;
    const long long r = tok / g.Nl, n = tok - r * g.Nl;
    return g.base_rows + r * g.chunk_rows + (b * g.Hl + hl) * g.Nl + n;
  }
  if (op == 2) {  // dst (r, b, hl, n) in the [P] buffer <- o (b, hl, r*Nl + n)
    const long long inner = g.B * g.Hl * g.Nl;
    const long long r = i / inner, q = i - r * inner;
    const long long b = q / (g.Hl * g.Nl), hl = (q / g.Nl) % g.Hl, n = q % g.Nl;
    return (b * g.Hl + hl) * g.N + r * g.Nl + n;
  }
  // op 3: dst (b, n, h) <- [P] buffer (h / Hl, b, h % Hl, n)
  const long long b = i / (g.Nl * g.H), n = (i / g.H) % g.Nl, h = i % g.H;
  const long long r = h / g.Hl, hl = h - r * g.Hl;
  return g.base_rows + r * g.chunk_rows + (b * g.Hl + hl) * g.Nl + n;
}

// Destination row of the i-th row of the dense destination enumeration.
__device__ __forceinline__ long long dst_row(long long i, int op, const UlyGeom& g) {
  if (op == 0 || op == 2) {  // the destination is the [P] buffer
    const long long inner = g.B * g.Hl * g.Nl;
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
  dst[dst_row(i, op, g) * VPR + v] = src[src_row(i, op, g) * VPR + v];
}

}  // namespace

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
