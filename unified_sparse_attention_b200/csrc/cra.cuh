// cra.cuh -- cumulative residual attention of a sparse prefill mask.
//
// LServe + SampleAttention blog post, "CRA - The Accuracy Proxy" and Fig. 4:
// for every query, the share of its (causal, unmasked) softmax probability mass
// that the sparse mask keeps; CRA takes the minimum over the queries.  With the
// log-sum-exp of both passes in hand (the prefill kernel writes them), the share
// of row i is  r_i = exp(lse_sparse(i) - lse_causal(i))  (the two normalisers
// share the row's scores), and the minimum is a reduction per (sequence, head).
#pragma once

#include "common.cuh"

namespace lserve {

constexpr int kCraThreads = 256;
constexpr int kCraChunk = 2048;   // rows per block

// Grid (sequence b x query head h = blockIdx.x, chunk of kCraChunk rows = blockIdx.y):
// retained[b, h, i] = r_i (if retained is not null) and cra[b, h] = min_i r_i.  A row that
// keeps nothing (lse_sparse = -inf) retains 0.  The chunks' minima meet in cra[b, h] by an
// integer atomic minimum on the float bits (every r_i is >= 0, where the bit patterns order
// as the values do); cra must hold an upper bound beforehand (the host sets 0x7f7f7f7f).
__global__ void __launch_bounds__(kCraThreads) cra_reduce_kernel(const float* __restrict__ lse_sparse,
                                                                 const float* __restrict__ lse_full, int S,
                                                                 float* __restrict__ retained,
                                                                 float* __restrict__ cra) {
  __shared__ float s_min[kCraThreads / 32];
  const long base = static_cast<long>(blockIdx.x) * S;
  const int i0 = blockIdx.y * kCraChunk, i1 = min(S, i0 + kCraChunk);
  float mn = __int_as_float(0x7f800000);   // +inf
  for (int i = i0 + threadIdx.x; i < i1; i += blockDim.x) {
    const float ls = lse_sparse[base + i], lf = lse_full[base + i];
    const float r = ls == kNegInf ? 0.f : expf(ls - lf);
    if (retained) retained[base + i] = r;
    mn = fminf(mn, r);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
  if ((threadIdx.x & 31) == 0) s_min[threadIdx.x >> 5] = mn;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 1; w < kCraThreads / 32; ++w) mn = fminf(mn, s_min[w]);
    atomicMin(reinterpret_cast<int*>(cra) + blockIdx.x, __float_as_int(mn));
  }
}

}  // namespace lserve
