// quant.cuh -- INT4 KV pages.
//
// LServe + SampleAttention blog post, "LServe - Decode Phase" and Fig. 2: INT4
// KV quantization cuts the bytes of every page the decode step reads.  The
// pages name no scheme; this one (asymmetric INT4) takes one step s and offset
// lo per (page, KV head, channel) for keys, over the page's valid tokens, and
// per (page, KV head, token) for values, over the d channels.  In float32:
//   s = (hi - lo) / 15,  code = clamp(rint((x - lo) / s), 0, 15)  (0 when s == 0),
//   dequantised value = bf16(fma(code, s, lo))  (nearest even).
// Layouts: kq, vq uint8 [NP, Hkv, 64, d/2] (channel 2j in the low nibble of byte
// j), kpar fp32 [NP, Hkv, 2, d] (s; lo), vpar fp32 [NP, Hkv, 2, 64] (s; lo).
// The page summaries of dense heads are taken over the dequantised keys -- the
// values the decode step attends to -- so the bound stays a bound.
#pragma once

#include "common.cuh"

namespace lserve {

__device__ __forceinline__ uint32_t int4_code(float x, float lo, float s) {
  if (!(s > 0.f)) return 0u;
  const float c = rintf(__fdiv_rn(x - lo, s));
  return static_cast<uint32_t>(fminf(fmaxf(c, 0.f), 15.f));
}

// One block of 128 threads per (page index i, sequence b, KV head g): threads
// 0 .. D/2-1 take the keys' channel pairs, threads 64 .. 127 the values' token
// rows.  Pages with index below first_page are left as they are.
template <int D>
__global__ void __launch_bounds__(128) quant_int4_kernel(
    const bf16* __restrict__ k_pages, const bf16* __restrict__ v_pages, const int32_t* __restrict__ page_table,
    int maxP, const int32_t* __restrict__ seq_lens, int first_page, const uint8_t* __restrict__ head_kind,
    int Hkv, int num_pages, uint8_t* __restrict__ kq, float* __restrict__ kpar, uint8_t* __restrict__ vq,
    float* __restrict__ vpar, bf16* __restrict__ stats) {
  const int i = blockIdx.x, b = blockIdx.y, g = blockIdx.z;
  const int L = max(0, seq_lens[b]);
  const int n = min(maxP, L > 0 ? (L - 1) / kPage + 1 : 0);
  if (i >= n || i < first_page) return;
  const int p = page_table[static_cast<long>(b) * maxP + i];
  if (p < 0 || p >= num_pages) {
    if (threadIdx.x == 0) report(LSERVE_ERR_DEVICE_BOUNDS);
    return;
  }
  const int nv = min(kPage, L - i * kPage);   // valid token rows of the page
  const long ph = static_cast<long>(p) * Hkv + g;
  const int tid = threadIdx.x;
  const float inf = __int_as_float(0x7f800000);
  if (tid < D / 2) {
    // ---- keys: channels 2j, 2j + 1 over the valid rows
    const int j = tid;
    const bf16* kp = k_pages + ph * kPage * D + 2 * j;
    float lo0 = inf, hi0 = -inf, lo1 = inf, hi1 = -inf;
    for (int r = 0; r < nv; ++r) {
      const __nv_bfloat162 x = *reinterpret_cast<const __nv_bfloat162*>(kp + r * D);
      lo0 = fminf(lo0, __low2float(x));
      hi0 = fmaxf(hi0, __low2float(x));
      lo1 = fminf(lo1, __high2float(x));
      hi1 = fmaxf(hi1, __high2float(x));
    }
    const float s0 = __fdiv_rn(hi0 - lo0, 15.f), s1 = __fdiv_rn(hi1 - lo1, 15.f);
    float* kpp = kpar + ph * 2 * D;
    kpp[2 * j] = s0;
    kpp[2 * j + 1] = s1;
    kpp[D + 2 * j] = lo0;
    kpp[D + 2 * j + 1] = lo1;
    const bool dense = head_kind[g] == LSERVE_HEAD_DENSE;
    float mn0[kNL], mx0[kNL], mn1[kNL], mx1[kNL];
#pragma unroll
    for (int l = 0; l < kNL; ++l) mn0[l] = mn1[l] = inf, mx0[l] = mx1[l] = -inf;
    uint8_t* kqp = kq + ph * kPage * (D / 2) + j;
#pragma unroll 4
    for (int r = 0; r < kPage; ++r) {
      uint32_t byte = 0u;
      if (r < nv) {
        const __nv_bfloat162 x = *reinterpret_cast<const __nv_bfloat162*>(kp + r * D);
        const uint32_t c0 = int4_code(__low2float(x), lo0, s0), c1 = int4_code(__high2float(x), lo1, s1);
        byte = c0 | (c1 << 4);
        const float d0 = __bfloat162float(__float2bfloat16_rn(fmaf(static_cast<float>(c0), s0, lo0)));
        const float d1 = __bfloat162float(__float2bfloat16_rn(fmaf(static_cast<float>(c1), s1, lo1)));
        const int l = r / kLogical;
#pragma unroll
        for (int ll = 0; ll < kNL; ++ll)
          if (ll == l) {
            mn0[ll] = fminf(mn0[ll], d0);
            mx0[ll] = fmaxf(mx0[ll], d0);
            mn1[ll] = fminf(mn1[ll], d1);
            mx1[ll] = fmaxf(mx1[ll], d1);
          }
      }
      kqp[r * (D / 2)] = static_cast<uint8_t>(byte);
    }
    if (dense) {   // summaries of the dequantised keys (logical pages without a valid token: +inf / -inf)
#pragma unroll
      for (int l = 0; l < kNL; ++l) {
        bf16* sp = stats + (ph * kNL + l) * 2 * D;
        *reinterpret_cast<__nv_bfloat162*>(sp + 2 * j) = __floats2bfloat162_rn(mn0[l], mn1[l]);
        *reinterpret_cast<__nv_bfloat162*>(sp + D + 2 * j) = __floats2bfloat162_rn(mx0[l], mx1[l]);
      }
    }
  } else if (tid >= 64 && tid < 64 + kPage) {
    // ---- values: token row t over the d channels
    const int t = tid - 64;
    const bf16* vp = v_pages + (ph * kPage + t) * D;
    float* vpp = vpar + ph * 2 * kPage;
    uint8_t* vqp = vq + (ph * kPage + t) * (D / 2);
    if (t >= nv) {
      vpp[t] = 0.f;
      vpp[kPage + t] = 0.f;
      for (int c = 0; c < D / 2; c += 16) *reinterpret_cast<uint4*>(vqp + c) = make_uint4(0u, 0u, 0u, 0u);
      return;
    }
    float lo = inf, hi = -inf;
    for (int c = 0; c < D; c += 2) {
      const __nv_bfloat162 x = *reinterpret_cast<const __nv_bfloat162*>(vp + c);
      lo = fminf(lo, fminf(__low2float(x), __high2float(x)));
      hi = fmaxf(hi, fmaxf(__low2float(x), __high2float(x)));
    }
    const float s = __fdiv_rn(hi - lo, 15.f);
    vpp[t] = s;
    vpp[kPage + t] = lo;
    for (int c = 0; c < D; c += 32) {   // 16 bytes = 32 channels at a time
      uint32_t w[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        uint32_t word = 0u;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const __nv_bfloat162 x = *reinterpret_cast<const __nv_bfloat162*>(vp + c + 8 * e + 2 * q);
          const uint32_t byte = int4_code(__low2float(x), lo, s) | (int4_code(__high2float(x), lo, s) << 4);
          word |= byte << (8 * q);
        }
        w[e] = word;
      }
      *reinterpret_cast<uint4*>(vqp + c / 2) = make_uint4(w[0], w[1], w[2], w[3]);
    }
  }
}

}  // namespace lserve
