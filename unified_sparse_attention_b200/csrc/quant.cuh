// quant.cuh -- INT4 KV pages.
//
// LServe + SampleAttention blog post, "LServe - Decode Phase" and Fig. 2: INT4
// KV quantization cuts the bytes of every page the decode step reads.  The
// pages name no scheme; this one (asymmetric INT4) takes one step s and offset
// lo per (page, KV head, channel) for keys, over the page's valid tokens, and
// per (page, KV head, token) for values, over the d channels.  In float32:
//   s = (hi - lo) / 15,  code = clamp(rint((x - lo) / s), 0, 15)  (0 when s == 0),
//   dequantised value = fma(code, s, lo)  (float32; never formed in bf16).
// Layouts (a byte holds two codes, the one with the even nibble index n in its
// low four bits; nibble n of a 32-bit word lies in byte n / 2, little-endian):
//   kq   uint8 [NP, Hkv, 64, d/2]: a key row is four chunks of d/8 bytes; word w
//        of chunk t holds nibbles n = j + 4 e of the channel pairs r = 4 w + j,
//        pair r being channels 16 (r / 2) + 8 (r % 2) + 2 t + e
//   vq   uint8 [NP, Hkv, 64 * d/2]: four slices of 16 tokens, each 32 chunks of
//        d/4 bytes; word m of chunk 4 g + t holds nibbles n = j + 4 e of channel
//        16 m + g + 8 (j % 2), token 16 slice + 2 t + 8 (j / 2) + e
//   kpar fp32 [NP, Hkv, 2, d]: s then lo, each four chunks of d/4 channels,
//        entry i of chunk t being channel 16 (i / 4) + 8 ((i / 2) % 2) + 2 t + i % 2
//   vpar fp32 [NP, Hkv, 64, 2]: (s, lo) per token
// These orders give each lane of the decode step its share of a page as a few
// contiguous words (the operand layout of its tensor-core fragments).
// The page summaries of dense heads are taken over the dequantised keys -- the
// values the decode step attends to -- with the minimum rounded down and the
// maximum rounded up to bf16, so the bound stays a bound.
#pragma once

#include "common.cuh"

namespace lserve {

__device__ __forceinline__ uint32_t int4_code(float x, float lo, float s) {
  if (!(s > 0.f)) return 0u;
  const float c = rintf(__fdiv_rn(x - lo, s));
  return static_cast<uint32_t>(fminf(fmaxf(c, 0.f), 15.f));
}

// Channel of entry i of the lane-t chunk of a key row / parameter row.
template <int D>
__device__ __forceinline__ int kq_channel(int t, int i) {
  return 16 * (i >> 2) + 8 * ((i >> 1) & 1) + 2 * t + (i & 1);
}

// One block of 128 threads per (page index i, sequence b, KV head g): the
// page's valid K and V rows are staged in shared memory once, then parameters,
// codes and summaries are computed from there.  Pages with index below
// first_page are left as they are.
template <int D>
__global__ void __launch_bounds__(128) quant_int4_kernel(
    const bf16* __restrict__ k_pages, const bf16* __restrict__ v_pages, const int32_t* __restrict__ page_table,
    int maxP, const int32_t* __restrict__ seq_lens, int first_page, const uint8_t* __restrict__ head_kind,
    int Hkv, int num_pages, uint8_t* __restrict__ kq, float* __restrict__ kpar, uint8_t* __restrict__ vq,
    float* __restrict__ vpar, bf16* __restrict__ stats) {
  __shared__ __align__(16) bf16 sk[kPage * D], sv[kPage * D];
  __shared__ float s_ks[D], s_klo[D], s_vs[kPage], s_vlo[kPage];
  const int i = blockIdx.x, b = blockIdx.y, g = blockIdx.z;
  const int L = max(0, seq_lens[b]);
  const int n = min(maxP, L > 0 ? (L - 1) / kPage + 1 : 0);
  if (i >= n || i < first_page) return;
  const int p = page_table[static_cast<long>(b) * maxP + i];
  if (p < 0 || p >= num_pages) {
    if (threadIdx.x == 0) report(LSERVE_ERR_DEVICE_BOUNDS);
    return;
  }
  const int nv = min(kPage, L - i * kPage);   // valid token rows of the page (>= 1)
  const long ph = static_cast<long>(p) * Hkv + g;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const float inf = __int_as_float(0x7f800000);

  // ---- stage the valid rows (16-byte loads; rows past nv are never read)
  {
    const uint4* kg = reinterpret_cast<const uint4*>(k_pages + ph * kPage * D);
    const uint4* vg = reinterpret_cast<const uint4*>(v_pages + ph * kPage * D);
    for (int x = tid; x < nv * D / 8; x += 128) {
      reinterpret_cast<uint4*>(sk)[x] = kg[x];
      reinterpret_cast<uint4*>(sv)[x] = vg[x];
    }
  }
  __syncthreads();
  // ---- key step and offset per channel, over the valid rows
  if (tid < D) {
    float lo = inf, hi = -inf;
    for (int r = 0; r < nv; ++r) {
      const float x = __bfloat162float(sk[r * D + tid]);
      lo = fminf(lo, x);
      hi = fmaxf(hi, x);
    }
    s_ks[tid] = __fdiv_rn(hi - lo, 15.f);
    s_klo[tid] = lo;
  }
  // ---- value step and offset per token row: one warp per row, lanes over channels
  for (int r = warp; r < kPage; r += 4) {
    float lo = inf, hi = -inf;
    if (r < nv)
      for (int c = lane; c < D; c += 32) {
        const float x = __bfloat162float(sv[r * D + c]);
        lo = fminf(lo, x);
        hi = fmaxf(hi, x);
      }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
      hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
    }
    if (lane == 0) {
      s_vs[r] = r < nv ? __fdiv_rn(hi - lo, 15.f) : 0.f;
      s_vlo[r] = r < nv ? lo : 0.f;
    }
  }
  __syncthreads();
  // ---- parameters out, in the decode step's order
  for (int x = tid; x < D; x += 128) {
    const int c = kq_channel<D>(x / (D / 4), x % (D / 4));
    kpar[ph * 2 * D + x] = s_ks[c];
    kpar[ph * 2 * D + D + x] = s_klo[c];
  }
  if (tid < kPage) {
    vpar[(ph * kPage + tid) * 2] = s_vs[tid];
    vpar[(ph * kPage + tid) * 2 + 1] = s_vlo[tid];
  }
  // ---- key codes: word (row r, chunk t, word w); rows past nv get code 0
  {
    constexpr int WR = D / 8, WC = D / 32;   // words per row, per chunk
    uint32_t* kqw = reinterpret_cast<uint32_t*>(kq + ph * kPage * (D / 2));
    for (int x = tid; x < kPage * WR; x += 128) {
      const int r = x / WR, t = (x % WR) / WC, w = x % WC;
      uint32_t word = 0u;
      if (r < nv) {
#pragma unroll
        for (int nb = 0; nb < 8; ++nb) {
          const int c = kq_channel<D>(t, 2 * (4 * w + (nb & 3)) + (nb >> 2));
          word |= int4_code(__bfloat162float(sk[r * D + c]), s_klo[c], s_ks[c]) << (4 * nb);
        }
      }
      kqw[x] = word;
    }
  }
  // ---- value codes: word (slice, chunk 4 g8 + t, word m)
  {
    constexpr int WM = D / 16;   // words per chunk
    uint32_t* vqw = reinterpret_cast<uint32_t*>(vq + ph * kPage * (D / 2));
    for (int x = tid; x < kPage * D / 8; x += 128) {
      const int m = x % WM, ch = (x / WM) % 32, sl = x / (WM * 32);
      const int g8 = ch >> 2, t = ch & 3;
      uint32_t word = 0u;
#pragma unroll
      for (int nb = 0; nb < 8; ++nb) {
        const int j = nb & 3, e = nb >> 2;
        const int c = 16 * m + g8 + 8 * (j & 1);
        const int u = 16 * sl + 2 * t + 8 * (j >> 1) + e;
        if (u < nv) word |= int4_code(__bfloat162float(sv[u * D + c]), s_vlo[u], s_vs[u]) << (4 * nb);
      }
      vqw[x] = word;
    }
  }
  // ---- summaries of the dequantised keys (dense heads); a logical page
  // without a valid token gets +inf / -inf
  if (tid < D && head_kind[g] == LSERVE_HEAD_DENSE) {
    const float s = s_ks[tid], lo = s_klo[tid];
#pragma unroll
    for (int l = 0; l < kNL; ++l) {
      float mn = inf, mx = -inf;
      for (int r = l * kLogical; r < min(nv, (l + 1) * kLogical); ++r) {
        const uint32_t code = int4_code(__bfloat162float(sk[r * D + tid]), lo, s);
        const float dq = fmaf(static_cast<float>(code), s, lo);
        mn = fminf(mn, dq);
        mx = fmaxf(mx, dq);
      }
      bf16* sp = stats + (ph * kNL + l) * 2 * D;
      sp[tid] = __float2bfloat16_rd(mn);
      sp[D + tid] = __float2bfloat16_ru(mx);
    }
  }
}

}  // namespace lserve
