// decode.cuh -- split-KV sparse paged decode attention + log-sum-exp merge.
//
// LServe + SampleAttention blog post, "LServe - Decode Phase" and Fig. 2:
// token-level attention only inside the selected pages.  Streaming heads attend
// to their sink + local tokens (mlsanity LServe page, Abstract: streaming heads
// in both the prefilling and the decoding stages).
//
// paged_decode_kernel: one CTA per (sequence b, KV head g, split s); a split
// covers `pages_per_split` consecutive entries of the (b, g) selection.  The CTA
// streams each selected K and V page (64 x d bf16, contiguous in the pool)
// into a 3-stage shared-memory ring with TMA (128-byte swizzle, completion on
// an mbarrier; thread 0 is the producer).  Each of the 4 warps owns 16 tokens
// of every page and keeps its own online-softmax state for the G query heads of
// the group: q.k and p.v run on mma.sync m16n8k16 with the G heads as the M
// rows (zero-padded to 16), so the kernel spends its issue slots on moving
// bytes, not on dot-product reductions.  At the end the 4 warp states are
// merged through shared memory into one (o, lse) partial per head and split.
//
// Bytes per selected page: 2 * 64 * d * 2 (K and V); the kernel is HBM-bound.
// Tokens outside the attended set (past seq_len; outside the Lambda set of a
// streaming head) are masked exactly: their logits become -inf by selection
// (not arithmetic) and their V rows are zeroed in the MMA operand, so even NaN
// garbage there cannot reach the result.
//
// The last split CTA of each (b, KV head) to finish (a counter per unit, zeroed
// by the top-k kernel and reset by that CTA) merges the partials by log-sum-exp:
// out = sum_s w_s o_s with w_s = 2^(lse_s - lse), lse = log2 sum_s 2^lse_s.
#pragma once

#include "common.cuh"

namespace lserve {

constexpr int kDecodeStages = 3;
constexpr int kDecodeThreads = 128;

template <int D>
struct DecodeCfg {
  static constexpr int kBoxes = D / 64;                 // 64-channel TMA boxes per row
  static constexpr int kBoxBytes = 64 * 128;            // 64 rows x 128 bytes
  static constexpr int kKVBytes = kBoxes * kBoxBytes;   // one K (or V) page
  static constexpr int kStageBytes = 2 * kKVBytes;
  static constexpr int kSmemBytes = kDecodeStages * kStageBytes + 1024;   // + alignment slack
};

template <int D>
__global__ void __launch_bounds__(kDecodeThreads) paged_decode_kernel(
    const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
    const bf16* __restrict__ q, const int32_t* __restrict__ page_table, int maxP,
    const int32_t* __restrict__ seq_lens, const uint8_t* __restrict__ head_kind,
    const int32_t* __restrict__ sel, const int32_t* __restrict__ sel_n, int kcap, int pages_per_split,
    int nsplit, int Hkv, int G, int num_pages, int sink, int local, float scale_log2,
    unsigned long long timeout_ns, float* __restrict__ part_o, float* __restrict__ part_lse,
    int32_t* __restrict__ done_count, bf16* __restrict__ out, float* __restrict__ lse_out) {
  using Cfg = DecodeCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[kDecodeStages];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  const int unit = blockIdx.y;   // b * Hkv + g
  const int split = blockIdx.x;
  const int b = unit / Hkv, g = unit % Hkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  pdl_wait();   // the selection comes from the previous kernel
  const int n_sel = min(sel_n[unit], kcap);
  const int p_begin = split * pages_per_split;
  if (n_sel == 0 && split == 0) {   // nothing to attend to: out = 0, lse = -inf
    for (int idx = tid; idx < G * D; idx += kDecodeThreads) {
      const long bh = static_cast<long>(b) * Hkv * G + static_cast<long>(g) * G + idx / D;
      out[bh * D + idx % D] = __float2bfloat16_rn(0.f);
      if (lse_out && idx % D == 0) lse_out[bh] = kNegInf;
    }
    return;
  }
  if (p_begin >= n_sel) return;
  const int n_my = min(pages_per_split, n_sel - p_begin);
  const int L = seq_lens[b];
  const bool streaming = head_kind[g] != LSERVE_HEAD_DENSE;
  const int32_t* my_sel = sel + static_cast<long>(unit) * kcap + p_begin;

  if (tid == 0) {
    prefetch_tensormap(&tmK);
    prefetch_tensormap(&tmV);
    for (int s = 0; s < kDecodeStages; ++s) mbar_init(&full_bar[s], 1);
    fence_barrier_init();
  }
  __syncthreads();

  // physical page of selection entry `it`, or -1 when out of range
  auto phys_page = [&](int it) -> int {
    const int pidx = my_sel[it];
    if (pidx < 0 || pidx >= maxP) return -1;
    const int p = page_table[static_cast<long>(b) * maxP + pidx];
    return (p >= 0 && p < num_pages) ? p : -1;
  };
  auto issue = [&](int it) {
    const int st = it % kDecodeStages;
    int p = phys_page(it);
    if (p < 0) {
      report(LSERVE_ERR_DEVICE_BOUNDS);
      p = 0;   // load a harmless in-range page; every token of it is masked below
    }
    uint8_t* kdst = smem + st * Cfg::kStageBytes;
    uint8_t* vdst = kdst + Cfg::kKVBytes;
    mbar_arrive_expect_tx(&full_bar[st], Cfg::kStageBytes);
    const int row = (p * Hkv + g) * kPage;
#pragma unroll
    for (int x = 0; x < Cfg::kBoxes; ++x) {
      tma_load_2d(kdst + x * Cfg::kBoxBytes, &tmK, &full_bar[st], x * 64, row);
      tma_load_2d(vdst + x * Cfg::kBoxBytes, &tmV, &full_bar[st], x * 64, row);
    }
  };
  if (tid == 0)
    for (int it = 0; it < min(kDecodeStages, n_my); ++it) issue(it);

  // Q as the A operand: rows = the G query heads of the group (zero-padded to 16)
  constexpr int KS = D / 16;
  uint32_t qa[KS][4];
  {
    const int r = lane >> 2, c = 2 * (lane & 3);
    const bf16* qb = q + (static_cast<long>(b) * Hkv * G + static_cast<long>(g) * G) * D;
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
      qa[ks][0] = r < G ? __ldg(reinterpret_cast<const uint32_t*>(qb + r * D + ks * 16 + c)) : 0u;
      qa[ks][2] = r < G ? __ldg(reinterpret_cast<const uint32_t*>(qb + r * D + ks * 16 + 8 + c)) : 0u;
      qa[ks][1] = r + 8 < G ? __ldg(reinterpret_cast<const uint32_t*>(qb + (r + 8) * D + ks * 16 + c)) : 0u;
      qa[ks][3] = r + 8 < G ? __ldg(reinterpret_cast<const uint32_t*>(qb + (r + 8) * D + ks * 16 + 8 + c)) : 0u;
    }
  }

  float acc[D / 8][4];
#pragma unroll
  for (int n = 0; n < D / 8; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
  float m_run[2] = {kNegInf, kNegInf}, l_run[2] = {0.f, 0.f};
  const int mi = lane >> 3, rr = lane & 7;

  bool timed_out = false;
  for (int it = 0; it < n_my; ++it) {
    const int st = it % kDecodeStages;
    const uint32_t parity = (it / kDecodeStages) & 1;
    if (!mbar_wait_bounded(&full_bar[st], parity, timeout_ns)) timed_out = true;
    const uint8_t* ks_base = smem + st * Cfg::kStageBytes;
    const uint8_t* vs_base = ks_base + Cfg::kKVBytes;
    const int pidx = my_sel[it];
    const bool page_ok = phys_page(it) >= 0;
    const int t_warp = pidx * kPage + warp * 16;   // first token of this warp's slice

    // ---- S = Q K^T for this warp's 16 tokens (two n-tiles of 8)
    float s[2][4];
#pragma unroll
    for (int n = 0; n < 2; ++n) s[n][0] = s[n][1] = s[n][2] = s[n][3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
      const int box = ks >> 2, chunk = (ks & 3) * 2 + (mi & 1);
      const int row = warp * 16 + (mi >> 1) * 8 + rr;
      uint32_t b0, b1, b2, b3;
      ldmatrix_x4(smem_u32(ks_base + box * Cfg::kBoxBytes + swz128(row, chunk)), b0, b1, b2, b3);
      mma_bf16_16816(s[0], qa[ks], b0, b1);
      mma_bf16_16816(s[1], qa[ks], b2, b3);
    }
    // ---- mask + online softmax (rows lane/4 and lane/4 + 8)
    const int tc = 2 * (lane & 3);
    auto valid = [&](int t) -> bool {
      return page_ok && t < L && (!streaming || t < sink || t >= L - local);
    };
    bool all_valid = true;
    float mloc[2] = {kNegInf, kNegInf};
#pragma unroll
    for (int n = 0; n < 2; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int t = t_warp + n * 8 + tc + (e & 1);
        const bool ok = valid(t);
        all_valid &= ok;
        s[n][e] = ok ? s[n][e] * scale_log2 : kNegInf;
        mloc[e >> 1] = fmaxf(mloc[e >> 1], s[n][e]);
      }
    float corr[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      mloc[h] = fmaxf(mloc[h], __shfl_xor_sync(0xffffffffu, mloc[h], 1));
      mloc[h] = fmaxf(mloc[h], __shfl_xor_sync(0xffffffffu, mloc[h], 2));
      const float m_new = fmaxf(m_run[h], mloc[h]);
      const float m_use = m_new == kNegInf ? 0.f : m_new;
      corr[h] = fast_exp2(m_run[h] - m_use);
      m_run[h] = m_new;
      mloc[h] = m_use;
    }
    float psum[2] = {0.f, 0.f};
#pragma unroll
    for (int n = 0; n < 2; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        s[n][e] = fast_exp2(s[n][e] - mloc[e >> 1]);
        psum[e >> 1] += s[n][e];
      }
    l_run[0] = l_run[0] * corr[0] + psum[0];
    l_run[1] = l_run[1] * corr[1] + psum[1];
#pragma unroll
    for (int n = 0; n < D / 8; ++n) {
      acc[n][0] *= corr[0];
      acc[n][1] *= corr[0];
      acc[n][2] *= corr[1];
      acc[n][3] *= corr[1];
    }
    // ---- O += P V
    uint32_t pa[4];
    pa[0] = pack_bf16x2(s[0][0], s[0][1]);
    pa[1] = pack_bf16x2(s[0][2], s[0][3]);
    pa[2] = pack_bf16x2(s[1][0], s[1][1]);
    pa[3] = pack_bf16x2(s[1][2], s[1][3]);
    const bool warp_all_valid = __all_sync(0xffffffffu, all_valid);
    uint32_t vm0 = 0xffffffffu, vm1 = 0xffffffffu;   // zero V of masked tokens (may hold NaN)
    if (!warp_all_valid) {
      const int t0 = t_warp + tc;
      vm0 = (valid(t0) ? 0x0000ffffu : 0u) | (valid(t0 + 1) ? 0xffff0000u : 0u);
      vm1 = (valid(t0 + 8) ? 0x0000ffffu : 0u) | (valid(t0 + 9) ? 0xffff0000u : 0u);
    }
#pragma unroll
    for (int np = 0; np < D / 16; ++np) {
      const int ch = np * 16 + (mi >> 1) * 8;   // first channel of this lane's matrix
      const int row = warp * 16 + (mi & 1) * 8 + rr;
      uint32_t b0, b1, b2, b3;
      ldmatrix_x4_trans(smem_u32(vs_base + (ch >> 6) * Cfg::kBoxBytes + swz128(row, (ch & 63) >> 3)), b0, b1,
                        b2, b3);
      b0 &= vm0;
      b1 &= vm1;
      b2 &= vm0;
      b3 &= vm1;
      mma_bf16_16816(acc[2 * np], pa, b0, b1);
      mma_bf16_16816(acc[2 * np + 1], pa, b2, b3);
    }
    // ---- release the stage and refill it
    if (__syncthreads_or(timed_out)) {
      timed_out = true;
      break;
    }
    if (tid == 0 && it + kDecodeStages < n_my) issue(it + kDecodeStages);
  }
  if (timed_out) {
    // let every load this CTA issued land before the CTA (and its smem) goes away
    if (tid == 0) {
      for (int it = 0; it < n_my; ++it) {
        const int st = it % kDecodeStages;
        mbar_wait_bounded(&full_bar[st], (it / kDecodeStages) & 1, timeout_ns);
      }
    }
    __syncthreads();
    return;
  }

  // ---- merge the 4 warps' states through shared memory (the ring is idle now)
  float* o_w = reinterpret_cast<float*>(smem);           // [4][16][D]
  float* m_w = o_w + 4 * 16 * D;                          // [4][16]
  float* l_w = m_w + 4 * 16;                              // [4][16]
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    l_run[h] += __shfl_xor_sync(0xffffffffu, l_run[h], 1);
    l_run[h] += __shfl_xor_sync(0xffffffffu, l_run[h], 2);
  }
  {
    const int r = lane >> 2, c = 2 * (lane & 3);
    if ((lane & 3) == 0) {
      m_w[warp * 16 + r] = m_run[0];
      m_w[warp * 16 + r + 8] = m_run[1];
      l_w[warp * 16 + r] = l_run[0];
      l_w[warp * 16 + r + 8] = l_run[1];
    }
#pragma unroll
    for (int n = 0; n < D / 8; ++n) {
      if (r < G) *reinterpret_cast<float2*>(&o_w[(warp * 16 + r) * D + n * 8 + c]) = make_float2(acc[n][0], acc[n][1]);
      if (r + 8 < G)
        *reinterpret_cast<float2*>(&o_w[(warp * 16 + r + 8) * D + n * 8 + c]) = make_float2(acc[n][2], acc[n][3]);
    }
  }
  __syncthreads();
  const long part = static_cast<long>(unit) * nsplit + split;
  for (int idx = tid; idx < G * D; idx += kDecodeThreads) {
    const int h = idx / D, c = idx % D;
    float m = kNegInf;
#pragma unroll
    for (int w = 0; w < 4; ++w) m = fmaxf(m, m_w[w * 16 + h]);
    float o = 0.f, l = 0.f;
    if (m != kNegInf) {
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const float sc = fast_exp2(m_w[w * 16 + h] - m);
        o += sc * o_w[(w * 16 + h) * D + c];
        l += sc * l_w[w * 16 + h];
      }
    }
    const bool has = m != kNegInf && l > 0.f;
    part_o[(part * G + h) * D + c] = has ? o / l : 0.f;
    if (c == 0) part_lse[part * G + h] = has ? m + __log2f(l) : kNegInf;
  }
  // ---- the last split of this (sequence, KV head) to finish merges all splits:
  // out = sum_s w_s o_s with w_s = 2^(lse_s - lse), lse = log2 sum_s 2^lse_s
  __shared__ int s_last;
  __threadfence();
  __syncthreads();
  const int ns = (n_sel + pages_per_split - 1) / pages_per_split;
  if (tid == 0) s_last = atomicAdd(&done_count[unit], 1) == ns - 1;
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  // per query head: m = max_s lse_s, lse = m + log2 sum_s 2^(lse_s - m); warp w owns heads w, w + 4, ...
  __shared__ float s_lse[16];
  const long base = static_cast<long>(unit) * nsplit;
  for (int hh = warp; hh < G; hh += 4) {
    float m = kNegInf;
    for (int sp = lane; sp < ns; sp += 32) m = fmaxf(m, __ldcg(&part_lse[(base + sp) * G + hh]));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float l = 0.f;
    if (m != kNegInf)
      for (int sp = lane; sp < ns; sp += 32) l += fast_exp2(__ldcg(&part_lse[(base + sp) * G + hh]) - m);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
    if (lane == 0) s_lse[hh] = (m != kNegInf && l > 0.f) ? m + __log2f(l) : kNegInf;
  }
  __syncthreads();
  // out = sum_s 2^(lse_s - lse) o_s, four channels per thread; the split loads are independent
  for (int idx = tid * 4; idx < G * D; idx += kDecodeThreads * 4) {
    const int hh = idx / D, c = idx % D;
    const float lse_h = s_lse[hh];
    float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
    if (lse_h != kNegInf) {
#pragma unroll 4
      for (int sp = 0; sp < ns; ++sp) {
        const float w = fast_exp2(__ldcg(&part_lse[(base + sp) * G + hh]) - lse_h);
        const float4 x = __ldcg(reinterpret_cast<const float4*>(&part_o[((base + sp) * G + hh) * D + c]));
        o.x += w * x.x;
        o.y += w * x.y;
        o.z += w * x.z;
        o.w += w * x.w;
      }
    }
    const long bh = static_cast<long>(b) * Hkv * G + static_cast<long>(g) * G + hh;
    __nv_bfloat162* dst = reinterpret_cast<__nv_bfloat162*>(out + bh * D + c);
    dst[0] = __floats2bfloat162_rn(o.x, o.y);
    dst[1] = __floats2bfloat162_rn(o.z, o.w);
    if (lse_out && c == 0) lse_out[bh] = lse_h == kNegInf ? kNegInf : lse_h * 0.6931471805599453f;
  }
  if (tid == 0) done_count[unit] = 0;   // ready for the next call
}

}  // namespace lserve
