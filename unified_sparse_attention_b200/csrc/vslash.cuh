// vslash.cuh -- vertical-slash block masks for dense heads, built from sampled queries.
//
// LServe + SampleAttention blog post, "SampleAttention - Column Pattern" and
// "Slash Pattern" (Fig. 3): a few key positions take attention from nearly all
// queries (columns) and attention gathers at fixed relative offsets (slashes);
// "CRA - The Accuracy Proxy" (Fig. 4): columns and slashes are added until the
// minimum, over queries, of the kept share of the causal softmax mass reaches
// a threshold tau.  At the prefill's 64 x 64 tile grain (the reading of the
// estimator, which the post leaves to its paper):
//   sampled queries  the last row of query tiles nQT-1, nQT-1-stride, ..., each
//                    for the G query heads of the KV head
//   tile masses      r[s, h, kt] = the row's causal softmax weights summed over
//                    the keys of tile kt
//   candidates       column kt scores sum_{s,h} r[s,h,kt]; slash delta scores
//                    sum_{s,h} r[s,h,qt(s)-delta]
//   greedy           the diagonal slash first, then by score (desc; columns
//                    before slashes, then lower index on equal scores), until the
//                    minimum retained mass over (s, h) reaches tau
//   mask             tile (qt, kt <= qt) kept iff a taken column or slash covers it
//
// vslash_mass_kernel    one CTA per (sampled row, sequence, dense KV head): two
//                       passes over the row's keys (16-byte loads, fp32 FMAs),
//                       the row's log-sum-exp per query head, then per-tile sums;
//                       every reduction runs in a fixed order (deterministic)
// vslash_greedy_kernel  one CTA per (sequence, KV head): scores, ranks of the
//                       candidates, the greedy over the sampled rows' retained
//                       masses (shared memory), the mask
#pragma once

#include "common.cuh"

namespace lserve {

constexpr int kVsThreads = 256;          // tile-mass kernel: 8 warps
constexpr int kVsWarps = kVsThreads / 32;
constexpr int kVsGreedyThreads = 1024;
constexpr int kVsMaxG = 8;
constexpr int kVsMaxEntries = 16384;     // sampled rows x G of one (sequence, KV head)
constexpr int kVsMaxTiles = 8192;        // query (and key) tiles

__host__ __device__ __forceinline__ int vs_rows(int nQT, int stride) { return (nQT - 1) / stride + 1; }
__host__ __device__ __forceinline__ int vs_tile(int s, int n_rows, int nQT, int stride) {
  return nQT - 1 - (n_rows - 1 - s) * stride;
}
// greedy kernel's shared memory: retained masses, candidate scores and order, taken flags
__host__ __device__ __forceinline__ size_t vs_greedy_smem(int n_entries, int nKT) {
  return static_cast<size_t>(n_entries) * 4 + static_cast<size_t>(nKT) * (4 + 4 + 1 + 1) +
         static_cast<size_t>(2 * nKT) * 4 + 64;
}

// base-2 logits of one key row against the G pre-scaled query rows in shared memory
template <int D>
__device__ __forceinline__ void vs_logits(const bf16* krow, const float* qs, int G, float (&x)[kVsMaxG]) {
#pragma unroll
  for (int h = 0; h < kVsMaxG; ++h) x[h] = 0.f;
#pragma unroll 4
  for (int c8 = 0; c8 < D; c8 += 8) {
    const uint4 raw = *reinterpret_cast<const uint4*>(krow + c8);
    const uint32_t w4[4] = {raw.x, raw.y, raw.z, raw.w};
    float kf[8];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      kf[2 * e] = bf16_lo(w4[e]);
      kf[2 * e + 1] = bf16_hi(w4[e]);
    }
#pragma unroll
    for (int h = 0; h < kVsMaxG; ++h) {
      if (h < G) {
        const float* qh = qs + h * D + c8;
#pragma unroll
        for (int e = 0; e < 8; ++e) x[h] = fmaf(kf[e], qh[e], x[h]);
      }
    }
  }
}

template <int D>
__global__ void __launch_bounds__(kVsThreads) vslash_mass_kernel(
    const bf16* __restrict__ q, const bf16* __restrict__ k, const uint8_t* __restrict__ head_kind, int S, int Hkv,
    int G, int nQT, int stride, int n_rows, float scale_log2, float* __restrict__ r_out) {
  __shared__ float qs[kVsMaxG * D];
  __shared__ float red_m[kVsWarps][kVsMaxG], red_l[kVsWarps][kVsMaxG], lse[kVsMaxG];
  const int s = blockIdx.x, bg = blockIdx.y, g = bg % Hkv, b = bg / Hkv;
  if (head_kind[g] != LSERVE_HEAD_DENSE) return;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int qt = vs_tile(s, n_rows, nQT, stride);
  const int i = qt * kTile + kTile - 1;   // the sampled query row
  const int Hq = Hkv * G;
  for (int e = tid; e < G * D; e += kVsThreads) {
    const int h = e / D, c = e % D;
    qs[e] = __bfloat162float(q[(static_cast<long>(b) * S + i) * Hq * D + static_cast<long>(g * G + h) * D + c]) *
            scale_log2;
  }
  __syncthreads();
  const bf16* kb = k + (static_cast<long>(b) * S * Hkv + g) * D;   // key j at kb + j * Hkv * D
  // pass 1: per-lane running (max, sum) of 2^x for each head; warp w takes tiles w, w+8, ...
  float m[kVsMaxG], l[kVsMaxG];
#pragma unroll
  for (int h = 0; h < kVsMaxG; ++h) {
    m[h] = kNegInf;
    l[h] = 0.f;
  }
  for (int kt = warp; kt <= qt; kt += kVsWarps) {
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int j = kt * kTile + half * 32 + lane;   // j <= i: every key of a tile <= qt is causal for the last row
      float x[kVsMaxG];
      vs_logits<D>(kb + static_cast<long>(j) * Hkv * D, qs, G, x);
#pragma unroll
      for (int h = 0; h < kVsMaxG; ++h) {
        if (h < G) {
          const float mn = fmaxf(m[h], x[h]);
          l[h] = l[h] * exp2f(m[h] - mn) + exp2f(x[h] - mn);
          m[h] = mn;
        }
      }
    }
  }
  // warp reduction (butterfly, fixed order), then warps combined in order by thread h
#pragma unroll
  for (int h = 0; h < kVsMaxG; ++h) {
    if (h >= G) break;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float mo = __shfl_xor_sync(0xffffffffu, m[h], o), lo = __shfl_xor_sync(0xffffffffu, l[h], o);
      const float mn = fmaxf(m[h], mo);
      l[h] = (mn == kNegInf) ? 0.f : l[h] * exp2f(m[h] - mn) + lo * exp2f(mo - mn);
      m[h] = mn;
    }
    if (lane == 0) {
      red_m[warp][h] = m[h];
      red_l[warp][h] = l[h];
    }
  }
  __syncthreads();
  if (tid < G) {
    float mm = kNegInf, ll = 0.f;
    for (int w = 0; w < kVsWarps; ++w) {
      const float mo = red_m[w][tid], lo = red_l[w][tid];
      const float mn = fmaxf(mm, mo);
      ll = (mn == kNegInf) ? 0.f : ll * exp2f(mm - mn) + lo * exp2f(mo - mn);
      mm = mn;
    }
    lse[tid] = mm + log2f(ll);
  }
  __syncthreads();
  // pass 2: the tile masses
  float* rs = r_out + (static_cast<long>(bg) * n_rows + s) * G * nQT;   // [h][kt]
  for (int kt = warp; kt <= qt; kt += kVsWarps) {
    float acc[kVsMaxG];
#pragma unroll
    for (int h = 0; h < kVsMaxG; ++h) acc[h] = 0.f;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int j = kt * kTile + half * 32 + lane;
      float x[kVsMaxG];
      vs_logits<D>(kb + static_cast<long>(j) * Hkv * D, qs, G, x);
#pragma unroll
      for (int h = 0; h < kVsMaxG; ++h)
        if (h < G) acc[h] += exp2f(x[h] - lse[h]);
    }
#pragma unroll
    for (int h = 0; h < kVsMaxG; ++h) {
      if (h >= G) break;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc[h] += __shfl_xor_sync(0xffffffffu, acc[h], o);
      if (lane == 0) rs[static_cast<long>(h) * nQT + kt] = acc[h];
    }
  }
  for (int e = tid; e < G * (nQT - qt - 1); e += kVsThreads) {
    const int h = e / (nQT - qt - 1), kt = qt + 1 + e % (nQT - qt - 1);
    rs[static_cast<long>(h) * nQT + kt] = 0.f;
  }
}

// candidate c: c < nKT is column c; otherwise slash c - nKT + 1 (slash 0 is taken first, apart)
__device__ __forceinline__ bool vs_before(float sa, int ca, float sb, int cb, int nKT) {
  if (sa != sb) return sa > sb;
  const int ka = ca >= nKT, kb = cb >= nKT;   // columns before slashes
  if (ka != kb) return ka < kb;
  return ca < cb;                             // then the lower index
}

__global__ void __launch_bounds__(kVsGreedyThreads) vslash_greedy_kernel(
    const float* __restrict__ r_in, const uint8_t* __restrict__ head_kind, int Hkv, int G, int nQT, int stride,
    int n_rows, float tau, uint8_t* __restrict__ mask, float* __restrict__ cra_out, int32_t* __restrict__ ncol_out,
    int32_t* __restrict__ nsla_out) {
  extern __shared__ __align__(16) uint8_t vs_smem[];
  __shared__ float red[kVsGreedyThreads / 32];
  __shared__ float s_cra;
  __shared__ int s_ncol, s_nsla;
  const int bg = blockIdx.x, g = bg % Hkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nKT = nQT;
  uint8_t* mrow = mask + static_cast<long>(bg) * nQT * nQT;
  if (head_kind[g] != LSERVE_HEAD_DENSE) {   // streaming head: no mask (it uses the Lambda support)
    for (long e = tid; e < static_cast<long>(nQT) * nQT; e += kVsGreedyThreads) mrow[e] = 0;
    if (tid == 0) {
      if (cra_out) cra_out[bg] = 0.f;
      if (ncol_out) ncol_out[bg] = 0;
      if (nsla_out) nsla_out[bg] = 0;
    }
    return;
  }
  const int n_ent = n_rows * G;
  float* retained = reinterpret_cast<float*>(vs_smem);
  float* col = retained + n_ent;
  float* sla = col + nKT;
  int* order = reinterpret_cast<int*>(sla + nKT);
  uint8_t* col_taken = reinterpret_cast<uint8_t*>(order + 2 * nKT);
  uint8_t* sla_taken = col_taken + nKT;
  const float* r = r_in + static_cast<long>(bg) * n_rows * G * nQT;   // [s][h][kt]
  auto R = [&](int s, int h, int kt) { return r[(static_cast<long>(s) * G + h) * nQT + kt]; };
  // candidate scores, each summed in (s, h) order
  for (int t = tid; t < nKT; t += kVsGreedyThreads) {
    float c = 0.f, d = 0.f;
    for (int s = 0; s < n_rows; ++s) {
      const int qt = vs_tile(s, n_rows, nQT, stride);
      for (int h = 0; h < G; ++h) {
        if (qt >= t) {
          c += R(s, h, t);
          d += R(s, h, qt - t);
        }
      }
    }
    col[t] = c == c ? c : kNegInf;   // NaN (from NaN inputs) ranks last: the order stays total
    sla[t] = d == d ? d : kNegInf;
    col_taken[t] = 0;
    sla_taken[t] = t == 0;
  }
  __syncthreads();
  // ranks: position of candidate c among all but slash 0
  const int nc = 2 * nKT - 1;
  auto score = [&](int c) { return c < nKT ? col[c] : sla[c - nKT + 1]; };
  for (int c = tid; c < nc; c += kVsGreedyThreads) {
    const float sc = score(c);
    int rank = 0;
    for (int c2 = 0; c2 < nc; ++c2) rank += vs_before(score(c2), c2, sc, c, nKT) ? 1 : 0;
    order[rank] = c;
  }
  // retained mass of every sampled (row, head) with the diagonal slash taken
  for (int e = tid; e < n_ent; e += kVsGreedyThreads) {
    const int s = e / G, h = e % G;
    retained[e] = R(s, h, vs_tile(s, n_rows, nQT, stride));
  }
  if (tid == 0) {
    s_ncol = 0;
    s_nsla = 1;
  }
  __syncthreads();
  auto block_min = [&](float v) -> float {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fminf(v, __shfl_xor_sync(0xffffffffu, v, o));
    if (lane == 0) red[warp] = v;
    __syncthreads();
    if (warp == 0) {
      float u = lane < kVsGreedyThreads / 32 ? red[lane] : 1e30f;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) u = fminf(u, __shfl_xor_sync(0xffffffffu, u, o));
      if (lane == 0) s_cra = u;
    }
    __syncthreads();
    return s_cra;
  };
  float mn = 1e30f;
  for (int e = tid; e < n_ent; e += kVsGreedyThreads) mn = fminf(mn, retained[e]);
  float cra = block_min(mn);
  for (int t = 0; t < nc && !(cra >= tau); ++t) {
    const int c = order[t];
    const bool is_col = c < nKT;
    const int idx = is_col ? c : c - nKT + 1;
    mn = 1e30f;
    for (int e = tid; e < n_ent; e += kVsGreedyThreads) {
      const int s = e / G, h = e % G;
      const int qt = vs_tile(s, n_rows, nQT, stride);
      if (is_col) {
        if (qt >= idx && !sla_taken[qt - idx]) retained[e] += R(s, h, idx);
      } else {
        if (qt >= idx && !col_taken[qt - idx]) retained[e] += R(s, h, qt - idx);
      }
      mn = fminf(mn, retained[e]);
    }
    __syncthreads();   // every thread has read the taken flags of this candidate's tiles
    if (tid == 0) {
      if (is_col) {
        col_taken[idx] = 1;
        ++s_ncol;
      } else {
        sla_taken[idx] = 1;
        ++s_nsla;
      }
    }
    cra = block_min(mn);   // its barriers publish the flags too
  }
  for (long e = tid; e < static_cast<long>(nQT) * nQT; e += kVsGreedyThreads) {
    const int qt = static_cast<int>(e / nQT), kt = static_cast<int>(e % nQT);
    mrow[e] = (kt <= qt && (col_taken[kt] || sla_taken[qt - kt])) ? 1 : 0;
  }
  if (tid == 0) {
    if (cra_out) cra_out[bg] = cra;
    if (ncol_out) ncol_out[bg] = s_ncol;
    if (nsla_out) nsla_out[bg] = s_nsla;
  }
}

}  // namespace lserve
