// page_stats.cuh -- per-logical-page key min/max summaries.
//
// LServe + SampleAttention blog post, "LServe - Decode Phase": every page is
// scored cheaply from a summary vector kept per page.  The summary is the
// channelwise min and max of the keys of each 16-token logical page (Quest,
// listed under "Builds on" on the mlsanity LServe page).
//
// One warp per (sequence, physical page, dense KV head): the 64 x d page is
// read with 16-byte coalesced loads (one row = d/8 lanes), min/max are taken
// with bf16x2 min/max (exact), and the partial results of the rows a warp
// covers per load are folded with shuffles.  Pure HBM streaming: 2 bytes read
// per key element, 2*2*d bytes written per logical page.
#pragma once

#include "common.cuh"

namespace lserve {

template <int D>
__global__ void __launch_bounds__(256) page_stats_kernel(const bf16* __restrict__ k_pages,
                                                         const int32_t* __restrict__ page_table, int maxP,
                                                         const int32_t* __restrict__ seq_lens, int first_lp,
                                                         const uint8_t* __restrict__ head_kind, int Hkv,
                                                         int num_pages, bf16* __restrict__ stats) {
  constexpr int LPR = D / 8;        // lanes per key row (8 channels per lane)
  constexpr int RPL = 32 / LPR;     // rows per warp-wide load
  constexpr int LOADS = kLogical / RPL;
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int b = blockIdx.y;
  const long unit = static_cast<long>(blockIdx.x) * (blockDim.x >> 5) + warp;
  const int i = static_cast<int>(unit / Hkv);   // page index within the sequence
  const int g = static_cast<int>(unit % Hkv);
  if (i >= maxP) return;
  const int L = seq_lens[b];
  const int n_pages = (L + kPage - 1) / kPage;
  if (i >= n_pages || head_kind[g] != LSERVE_HEAD_DENSE) return;
  if ((i + 1) * kNL <= first_lp) return;
  const int p = page_table[static_cast<long>(b) * maxP + i];
  if (p < 0 || p >= num_pages) {
    if (lane == 0) report(LSERVE_ERR_DEVICE_BOUNDS);
    return;
  }
  const int r0 = lane / LPR;        // first row this lane reads within a load
  const int c8 = (lane % LPR) * 8;  // first channel of this lane
  const bf16* page = k_pages + (static_cast<long>(p) * Hkv + g) * kPage * D;
  bf16* out = stats + (static_cast<long>(p) * Hkv + g) * kNL * 2 * D;
  const __nv_bfloat162 pinf = __floats2bfloat162_rn(__builtin_inff(), __builtin_inff());
  const __nv_bfloat162 ninf = __floats2bfloat162_rn(-__builtin_inff(), -__builtin_inff());

#pragma unroll
  for (int l = 0; l < kNL; ++l) {
    if (i * kNL + l < first_lp) continue;
    uint4 raw[LOADS];
#pragma unroll
    for (int m = 0; m < LOADS; ++m) {
      const int row = l * kLogical + r0 + m * RPL;
      raw[m] = (i * kPage + row < L) ? __ldg(reinterpret_cast<const uint4*>(page + row * D + c8))
                                     : make_uint4(0, 0, 0, 0);
    }
    __nv_bfloat162 mn[4] = {pinf, pinf, pinf, pinf};
    __nv_bfloat162 mx[4] = {ninf, ninf, ninf, ninf};
#pragma unroll
    for (int m = 0; m < LOADS; ++m) {
      const int row = l * kLogical + r0 + m * RPL;
      if (i * kPage + row < L) {
        const __nv_bfloat162* v = reinterpret_cast<const __nv_bfloat162*>(&raw[m]);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          mn[e] = __hmin2(mn[e], v[e]);
          mx[e] = __hmax2(mx[e], v[e]);
        }
      }
    }
    // fold the RPL row groups of the warp
#pragma unroll
    for (int off = LPR; off < 32; off <<= 1) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        uint32_t a = __shfl_xor_sync(0xffffffffu, *reinterpret_cast<uint32_t*>(&mn[e]), off);
        uint32_t c = __shfl_xor_sync(0xffffffffu, *reinterpret_cast<uint32_t*>(&mx[e]), off);
        mn[e] = __hmin2(mn[e], *reinterpret_cast<__nv_bfloat162*>(&a));
        mx[e] = __hmax2(mx[e], *reinterpret_cast<__nv_bfloat162*>(&c));
      }
    }
    if (r0 == 0) {
      *reinterpret_cast<uint4*>(out + (l * 2 + 0) * D + c8) = *reinterpret_cast<uint4*>(mn);
      *reinterpret_cast<uint4*>(out + (l * 2 + 1) * D + c8) = *reinterpret_cast<uint4*>(mx);
    }
  }
}

}  // namespace lserve
