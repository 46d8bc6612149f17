// select.cuh -- query-aware hierarchical page selection for decode.
//
// LServe + SampleAttention blog post, "LServe - Decode Phase" and Fig. 2: score
// every page from its summary, keep the top-k, then attend inside those pages
// only; mlsanity LServe page, Abstract: a hierarchical KV page selection policy
// by query-centric similarity, with a constant number of pages kept.
//
// Bound scoring (HBM-bound stream over the summaries)
//   bound of query head h on logical page l:  sum_c max(q_hc * kmax_c, q_hc * kmin_c)
//   group score: max over the G query heads of the KV head; page score: max over
//   the page's logical pages that hold a valid token.
//   score_pages_kernel (G = 1): one warp per physical page: lane = (logical
//     page l = lane/8, 16 (d=128) or 8 (d=64) channels), four 16-byte loads per
//     lane, fp32 products (exact for bf16 operands) and a 3-step shuffle sum.
//   score_pages_mma_kernel (G >= 2): the same bound as a contraction on the
//     tensor cores (see there); per-lane products would cost G x as much issue.
//
// topk_unit  (latency-bound, one CTA per (sequence, KV head); the kernel that
//   runs it is in decode.cuh)
//   k = min(budget/64, n_pages) pages by radix select (8-bit digits below the
//   bits all keys share) on the order-preserving uint32 image of the fp32
//   scores, ties to the lower page index, emitted in ascending page order by a
//   block-wide scan.  Streaming heads get their fixed sink + local page list.
#pragma once

#include "common.cuh"

namespace lserve {

// ------------------------------------------------------------------ scoring
// Per-lane fp32 products (one query head per KV head).  The work -- every
// (sequence, dense KV head, page) -- is one flat list, v = (b * ndense + i_g) *
// maxP + page, cut into gridDim.x equal contiguous shares (one wave of CTAs,
// so that no SM is left with an extra CTA's worth of pages at the end); a warp
// takes every nwarps-th (page, head) of its CTA's share and scores its four
// logical pages with 16-byte loads.
template <int D, int G>
__global__ void __launch_bounds__(256, 5) score_pages_kernel(
    const bf16* __restrict__ q, const bf16* __restrict__ stats, const int32_t* __restrict__ page_table, int B,
    int maxP, const int32_t* __restrict__ seq_lens, const uint8_t* __restrict__ head_kind, int Hkv, int num_pages,
    float* __restrict__ scores) {
  constexpr int CPL = D / 8;   // channels per lane
  __shared__ int s_dense[256];
  __shared__ int s_ndense;
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int nwarps = blockDim.x >> 5;
  if (threadIdx.x == 0) {
    int n = 0;
    for (int g = 0; g < Hkv; ++g)
      if (head_kind[g] == LSERVE_HEAD_DENSE) s_dense[n++] = g;
    s_ndense = n;
  }
  __syncthreads();
  const long long V = static_cast<long long>(B) * s_ndense * maxP;
  const long long v0 = V * blockIdx.x / gridDim.x, v1 = V * (blockIdx.x + 1) / gridDim.x;
  const int l = lane >> 3;           // logical page of this lane
  const int c0 = (lane & 7) * CPL;   // first channel of this lane
  const float ninf = kNegInf;

  int cur_bg = -1, L = 0, n_pages = 0;
  float qf[G][CPL];
  int bgi = static_cast<int>((v0 + warp) / maxP);                   // b * ndense + i_g
  int i = static_cast<int>(v0 + warp - static_cast<long long>(bgi) * maxP);   // page
  auto advance = [&] {
    i += nwarps;
    while (i >= maxP) {
      i -= maxP;
      ++bgi;
    }
  };
  for (long long v = v0 + warp; v < v1; v += nwarps, advance()) {
    const int b = bgi / s_ndense, g = s_dense[bgi % s_ndense];
    if (bgi != cur_bg) {
      cur_bg = bgi;
      L = seq_lens[b];
      n_pages = L > 0 ? min(maxP, (L - 1) / kPage + 1) : 0;
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const bf16* qp = q + (static_cast<long>(b) * Hkv * G + g * G + h) * D + c0;
#pragma unroll
        for (int c = 0; c < CPL; c += 8) {
          uint4 u = __ldg(reinterpret_cast<const uint4*>(qp + c));
          const uint32_t* w = reinterpret_cast<const uint32_t*>(&u);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            qf[h][c + 2 * e] = bf16_lo(w[e]);
            qf[h][c + 2 * e + 1] = bf16_hi(w[e]);
          }
        }
      }
    }
    if (i >= n_pages) continue;   // past the sequence: no score
    const int p = page_table[static_cast<long>(b) * maxP + i];
    float s = ninf;
    if (p >= 0 && p < num_pages) {
      const bf16* sp = stats + ((static_cast<long>(p) * Hkv + g) * kNL + l) * 2 * D + c0;
      uint4 mn[CPL / 8], mx[CPL / 8];
#pragma unroll
      for (int c = 0; c < CPL / 8; ++c) {
        mn[c] = __ldg(reinterpret_cast<const uint4*>(sp + c * 8));
        mx[c] = __ldg(reinterpret_cast<const uint4*>(sp + D + c * 8));
      }
      float best = ninf;
#pragma unroll
      for (int h = 0; h < G; ++h) {
        float acc = 0.f;
#pragma unroll
        for (int c = 0; c < CPL / 8; ++c) {
          const uint32_t* a = reinterpret_cast<const uint32_t*>(&mn[c]);
          const uint32_t* z = reinterpret_cast<const uint32_t*>(&mx[c]);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float q0 = qf[h][c * 8 + 2 * e], q1 = qf[h][c * 8 + 2 * e + 1];
            acc += fmaxf(q0 * bf16_lo(z[e]), q0 * bf16_lo(a[e]));
            acc += fmaxf(q1 * bf16_hi(z[e]), q1 * bf16_hi(a[e]));
          }
        }
        acc += __shfl_xor_sync(0xffffffffu, acc, 1);
        acc += __shfl_xor_sync(0xffffffffu, acc, 2);
        acc += __shfl_xor_sync(0xffffffffu, acc, 4);
        best = fmaxf(best, acc);
      }
      // logical pages without a valid token do not count
      s = (i * kPage + l * kLogical < L) ? best : ninf;
    } else if (lane == 0) {
      report(LSERVE_ERR_DEVICE_BOUNDS);
    }
    s = fmaxf(s, __shfl_xor_sync(0xffffffffu, s, 8));
    s = fmaxf(s, __shfl_xor_sync(0xffffffffu, s, 16));
    if (lane == 0) scores[(static_cast<long>(b) * Hkv + g) * maxP + i] = s;
  }
}

// Bound scoring on the tensor cores.  max(q_c kmax_c, q_c kmin_c) is q_c kmax_c
// when q_c >= 0 and q_c kmin_c otherwise, so the bound of query head h on a
// logical page is  q-_h . kmin + q+_h . kmax  (q- = min(q, 0), q+ = max(q, 0)):
// one contraction of the summary row [kmin | kmax] (2d bf16, as stored) with
// [q- | q+].  One warp takes 4 physical pages = 16 logical pages of one dense
// KV head as the M = 16 rows of m16n8k16 tiles, K = 2d, and the group's G <= 8
// query heads as N = 8 (q- and q+ are exact bf16 values; products are exact
// and sums are fp32).  The K order inside the tiles is permuted so that every
// lane reads 16 contiguous bytes of a row per 32 channels (channels 32 j + 8 t
// .. + 7 of lane t of a quad feed k-steps 2 j and 2 j + 1); the q fragments use
// the same order.  The group max is over the valid heads of each row, the page
// max over the rows of a page that hold a valid token (quad shuffles).
constexpr int kScoreThreads = 256;
constexpr int kScoreCtasPerSm = 2;

template <int D>
__global__ void __launch_bounds__(kScoreThreads, kScoreCtasPerSm) score_pages_mma_kernel(
    const bf16* __restrict__ q, const bf16* __restrict__ stats, const int32_t* __restrict__ page_table, int B,
    int maxP, const int32_t* __restrict__ seq_lens, const uint8_t* __restrict__ head_kind, int Hkv, int G,
    int num_pages, float* __restrict__ scores) {
  constexpr int NJ = 2 * D / 32;   // 32-channel groups of [kmin | kmax]
  __shared__ int s_dense[256];
  __shared__ int s_ndense;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  if (threadIdx.x == 0) {
    int n = 0;
    for (int g = 0; g < Hkv; ++g)
      if (head_kind[g] == LSERVE_HEAD_DENSE) s_dense[n++] = g;
    s_ndense = n;
  }
  __syncthreads();
  // items (b, dense head, group of 4 pages) in that order; each warp takes an
  // equal contiguous run of them (the grid is one wave)
  const int ngrp = (maxP + 3) / 4;
  const long long items = static_cast<long long>(B) * s_ndense * ngrp;
  const long long total_warps = static_cast<long long>(gridDim.x) * nwarps;
  const long long per = (items + total_warps - 1) / total_warps;
  const long long it0 = (static_cast<long long>(blockIdx.x) * nwarps + warp) * per;
  const long long it1 = min(items, it0 + per);
  const int r = lane >> 2, t = lane & 3;   // fragment row (and row + 8), lane of the quad
  const float ninf = kNegInf;
  const uint64_t pol = l2_evict_first();

  struct Item {
    int b, g, ib, n_pages, L;
    int p[2];   // physical pages of rows r and r + 8 (-1: none)
  };
  auto locate = [&](long long it) -> Item {
    Item m;
    m.b = static_cast<int>(it / (static_cast<long long>(s_ndense) * ngrp));
    const int rem = static_cast<int>(it % (static_cast<long long>(s_ndense) * ngrp));
    m.g = s_dense[rem / ngrp];
    m.ib = (rem % ngrp) * 4;
    m.L = seq_lens[m.b];
    m.n_pages = min(maxP, (max(m.L, 0) + kPage - 1) / kPage);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int i = m.ib + (r + 8 * h) / 4;
      int pg = -1;
      if (i < m.n_pages) {
        pg = page_table[static_cast<long>(m.b) * maxP + i];
        if (pg < 0 || pg >= num_pages) {
          if (((r + 8 * h) & 3) == 0 && t == 0) report(LSERVE_ERR_DEVICE_BOUNDS);
          pg = -1;
        }
      }
      m.p[h] = pg;
    }
    return m;
  };

  int cur_b = -1, cur_g = -1;
  uint32_t qb[NJ][4];   // per 32-channel group: b0, b1 of k-step 2j, then of 2j + 1 (query head r)
  Item nx = it0 < it1 ? locate(it0) : Item{};
  for (long long it = it0; it < it1; ++it) {
    const Item m = nx;
    if (m.ib >= m.n_pages) {   // past the end of this sequence
      if (it + 1 < it1) nx = locate(it + 1);
      continue;
    }
    // the summaries of rows r and r + 8 (logical page (row % 4) of page ib + row / 4)
    uint4 a[NJ][2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int row = r + 8 * h;
      const bf16* srow =
          m.p[h] >= 0 ? stats + ((static_cast<long>(m.p[h]) * Hkv + m.g) * kNL + (row & 3)) * 2 * D + 8 * t
                      : nullptr;
#pragma unroll
      for (int j = 0; j < NJ; ++j)
        a[j][h] = srow ? ld_once_u4(srow + 32 * j, pol) : make_uint4(0u, 0u, 0u, 0u);
    }
    if (it + 1 < it1) nx = locate(it + 1);   // the next item's pages load meanwhile
    if (m.b != cur_b || m.g != cur_g) {
      cur_b = m.b;
      cur_g = m.g;
      const bf16* qh = q + (static_cast<long>(m.b) * Hkv * G + static_cast<long>(m.g) * G + r) * D;
#pragma unroll
      for (int j = 0; j < NJ; ++j) {
        const bool plus = 32 * j >= D;   // kmax half: q+, kmin half: q-
        uint4 w = make_uint4(0u, 0u, 0u, 0u);
        if (r < G) w = __ldg(reinterpret_cast<const uint4*>(qh + (32 * j) % D + 8 * t));
        auto half = [&](uint32_t x) -> uint32_t {
          uint32_t o = 0u;
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const uint32_t hb = (x >> (16 * e)) & 0xffffu;
            if (((hb & 0x8000u) != 0) != plus) o |= hb << (16 * e);
          }
          return o;
        };
        qb[j][0] = half(w.x);
        qb[j][1] = half(w.y);
        qb[j][2] = half(w.z);
        qb[j][3] = half(w.w);
      }
    }
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int j = 0; j < NJ; ++j) {
      const uint32_t fa[4] = {a[j][0].x, a[j][1].x, a[j][0].y, a[j][1].y};   // k-step 2j
      const uint32_t fb[4] = {a[j][0].z, a[j][1].z, a[j][0].w, a[j][1].w};   // k-step 2j + 1
      mma_bf16_16816(acc, fa, qb[j][0], qb[j][1]);
      mma_bf16_16816(acc, fb, qb[j][2], qb[j][3]);
    }
    // element e: row r + 8 (e >> 1), head 2 t + (e & 1)
    float sc[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      float mx = ninf;
#pragma unroll
      for (int e = 0; e < 2; ++e)
        if (2 * t + e < G) mx = fmaxf(mx, acc[2 * h + e]);
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      const int row = r + 8 * h;
      const int i = m.ib + row / 4;
      // logical pages without a valid token (and missing pages) do not count
      sc[h] = (m.p[h] >= 0 && i * kPage + (row & 3) * kLogical < m.L) ? mx : ninf;
      sc[h] = fmaxf(sc[h], __shfl_xor_sync(0xffffffffu, sc[h], 4));
      sc[h] = fmaxf(sc[h], __shfl_xor_sync(0xffffffffu, sc[h], 8));
    }
    // lanes 0 and 16 hold pages r / 4 and r / 4 + 2 of the group
    if ((lane & 15) == 0) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int i = m.ib + (r + 8 * h) / 4;
        if (i < m.n_pages) scores[(static_cast<long>(m.b) * Hkv + m.g) * maxP + i] = sc[h];
      }
    }
  }
}

// -------------------------------------------------------------------- top-k
__device__ __forceinline__ uint32_t order_key(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Block-wide exclusive scan of one int per thread; returns the prefix, writes
// the block total to *total.  Needs blockDim.x/32 ints of scratch.
__device__ __forceinline__ int block_exclusive_scan(int v, int* scratch, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) scratch[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = lane < nw ? scratch[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    if (lane < nw) scratch[lane] = w;
  }
  __syncthreads();
  const int before = (warp > 0 ? scratch[warp - 1] : 0) + x - v;
  *total = scratch[nw - 1];
  __syncthreads();
  return before;
}

constexpr int kTopkThreads = 512;
constexpr int kTopkSmemKeys = 16384;   // scores cached in shared memory up to this many pages

// Pages of a sequence of L tokens.
__device__ __forceinline__ int seq_pages(int L) { return L > 0 ? (L - 1) / kPage + 1 : 0; }

// Streaming head over the n pages of a sequence of L tokens: the pages holding
// a token of [0, sink) or [L - local, L) are [0, a) and [bb, bb + cnt - a);
// returns cnt.
__device__ __forceinline__ int streaming_pages(int L, int n, int sink, int local, int& a, int& bb) {
  const int w0 = local > 0 ? max(0, L - local) / kPage : n;   // first window page
  const int w1 = local > 0 ? seq_pages(L) : n;                 // one past the last
  a = min(seq_pages(min(sink, L)), n);
  bb = max(w0, a);
  return L > 0 ? a + max(0, min(w1, n) - bb) : 0;
}

// Pages the selection keeps for one unit (sequence of L tokens, one KV head):
// a dense head min(budget, pages), a streaming head its sink and window pages,
// at most kcap.  topk_unit() writes exactly this many.
__device__ __forceinline__ int unit_selected(int L, int maxP, bool dense, int budget_pages, int sink, int local,
                                             int kcap) {
  L = max(0, L);
  const int n = min(seq_pages(L), maxP);
  if (dense) return min(budget_pages, n);
  int a, bb;
  return min(streaming_pages(L, n, sink, local, a, bb), kcap);
}

// Block-wide exclusive scan of one 64-bit value per thread (two packed 32-bit
// counts); returns the prefix.  Needs blockDim.x/32 values of scratch.
__device__ __forceinline__ unsigned long long block_exclusive_scan64(unsigned long long v,
                                                                     unsigned long long* scratch) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  unsigned long long x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned long long y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) scratch[warp] = x;
  __syncthreads();
  unsigned long long before = x - v;
  for (int w = 0; w < warp; ++w) before += scratch[w];   // broadcast reads, no second barrier
  return before;
}

// Top-k pages of one unit (b, g) = `unit`, by one block.  The scores come from
// the scoring kernel, which may still be running when the block starts: they
// are read only after the caller's dependency wait, with L2 loads through a
// pointer that is not restrict-qualified (no load of them can move above it).
// Dense head: k = min(budget, pages) pages with the largest scores, ties to
// the lower index, written in ascending order.  Radix select over the order-
// preserving integer keys: the digits start below the bits that all keys
// share, a pass costs two barriers (the histogram of the next pass is cleared
// while this one fills), and the search ends once the k-th key's bin is
// taken whole; one scan of (above, equal) counts places the output.
// Returns the number of pages selected (the same value in every thread).
__device__ __forceinline__ int topk_unit(const float* scores, int unit, int maxP, int L, bool dense,
                                          int budget_pages, int sink, int local, int32_t* sel, int32_t* sel_n,
                                          int kcap, const int32_t* sel_in = nullptr,
                                          const int32_t* sel_n_in = nullptr) {
  extern __shared__ uint32_t s_keys[];
  __shared__ __align__(16) int s_hist[2][256];
  __shared__ unsigned long long s_scan[32];
  __shared__ uint32_t s_mm[2][32];
  __shared__ int s_step[3];   // prefix, remaining, count of the k-th key's bin
  L = max(0, L);
  int n = seq_pages(L);
  if (n > maxP) {   // sequence longer than its page-table row
    if (threadIdx.x == 0) report(LSERVE_ERR_DEVICE_BOUNDS);
    n = maxP;
  }
  int32_t* row = sel + static_cast<long>(unit) * kcap;
  const int tid = threadIdx.x, nt = blockDim.x;

  if (!dense) {
    int a, bb;
    int cnt = streaming_pages(L, n, sink, local, a, bb);
    if (cnt > kcap) {
      if (tid == 0) report(LSERVE_ERR_DEVICE_BOUNDS);
      cnt = kcap;
    }
    for (int j = tid; j < kcap; j += nt) {
      int v = -1;
      if (j < a) v = j;
      else if (j < cnt) v = bb + (j - a);
      row[j] = v;
    }
    if (tid == 0 && sel_n) sel_n[unit] = cnt;
    return cnt;
  }

  if (sel_in) {   // a selection kept from an earlier step: its row as it stands
    const int m = min(max(sel_n_in[unit], 0), kcap);
    const int32_t* src = sel_in + static_cast<long>(unit) * kcap;
    for (int j = tid; j < kcap; j += nt) row[j] = j < m ? src[j] : -1;
    if (tid == 0 && sel_n) sel_n[unit] = m;
    return m;
  }
  const int k = min(budget_pages, n);
  if (k >= n) {
    for (int j = tid; j < kcap; j += nt) row[j] = j < n ? j : -1;
    if (tid == 0 && sel_n) sel_n[unit] = n;
    return n;
  }
  const float* srow = scores + static_cast<long>(unit) * maxP;
  const bool cached = n <= kTopkSmemKeys;
  auto key_at = [&](int j) -> uint32_t { return cached ? s_keys[j] : order_key(__ldcg(srow + j)); };

  // keys (cached), their min and max, both histograms cleared
  uint32_t kmin = 0xffffffffu, kmax = 0u;
  for (int j0 = 0; j0 < n; j0 += 4 * nt) {   // four independent loads in flight per thread
    float f[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int j = j0 + r * nt + tid;
      f[r] = j < n ? __ldcg(srow + j) : 0.f;
    }
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int j = j0 + r * nt + tid;
      if (j < n) {
        const uint32_t kk = order_key(f[r]);
        if (cached) s_keys[j] = kk;
        kmin = min(kmin, kk);
        kmax = max(kmax, kk);
      }
    }
  }
  for (int j = tid; j < 2 * 256; j += nt) (&s_hist[0][0])[j] = 0;
  kmin = __reduce_min_sync(0xffffffffu, kmin);
  kmax = __reduce_max_sync(0xffffffffu, kmax);
  if ((tid & 31) == 0) {
    s_mm[0][tid >> 5] = kmin;
    s_mm[1][tid >> 5] = kmax;
  }
  __syncthreads();
  for (int w = 0; w < (nt >> 5); ++w) {   // every thread reduces the per-warp values itself
    kmin = min(kmin, s_mm[0][w]);
    kmax = max(kmax, s_mm[1][w]);
  }
  // The bits above the highest one in which the keys differ are common to all
  // of them (scores of similar magnitude share sign and exponent): the radix
  // digits start below them, so that no pass piles every key into one bin.
  int shift = (kmin ^ kmax) ? 32 - __clz(kmin ^ kmax) : 0;   // low bits still to resolve
  uint32_t mask = shift >= 32 ? 0u : ~((1u << shift) - 1u);    // bits fixed so far
  uint32_t prefix = kmax & mask;                                // their value for the k-th key
  int remaining = k;                                            // keys still to take at prefix
  int pass = 0;
  // 8-bit digits (the first may be narrower); a pass ends the search when the
  // k-th key's bin is taken whole -- the lower bits need not be resolved
#pragma unroll 1
  while (shift > 0) {
    const int w = min(8, shift);
    shift -= w;
    int* hist = s_hist[pass & 1];
    for (int j = tid; j < n; j += nt) {
      const uint32_t kk = key_at(j);
      if ((kk & mask) == prefix) atomicAdd(&hist[(kk >> shift) & ((1u << w) - 1u)], 1);
    }
    // the other histogram was last read before the previous pass's final barrier
    for (int j = tid; j < 256; j += nt) s_hist[(pass + 1) & 1][j] = 0;
    __syncthreads();
    if (tid < 32) {
      // lane t owns digits 8t..8t+7; find the digit holding the remaining-th largest
      const int4 h0 = *reinterpret_cast<const int4*>(hist + tid * 8);
      const int4 h1 = *reinterpret_cast<const int4*>(hist + tid * 8 + 4);
      const int c[8] = {h0.x, h0.y, h0.z, h0.w, h1.x, h1.y, h1.z, h1.w};
      const int sum = ((c[0] + c[1]) + (c[2] + c[3])) + ((c[4] + c[5]) + (c[6] + c[7]));
      int suf = sum;   // inclusive suffix sum over lanes (sum of lanes >= tid)
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_down_sync(0xffffffffu, suf, o);
        if (tid + o < 32) suf += y;
      }
      const int above = suf - sum;   // keys with a higher digit
      if (above < remaining && remaining <= suf) {   // exactly one lane
        int acc = above, digit = tid * 8, cnt = 0;
#pragma unroll
        for (int e = 7; e >= 0; --e) {
          if (cnt == 0 && acc + c[e] >= remaining) {
            digit = tid * 8 + e;
            cnt = c[e];
          } else if (cnt == 0) {
            acc += c[e];
          }
        }
        s_step[0] = static_cast<int>(prefix | (static_cast<uint32_t>(digit) << shift));
        s_step[1] = remaining - acc;
        s_step[2] = cnt;
      }
    }
    __syncthreads();
    prefix = static_cast<uint32_t>(s_step[0]);
    mask |= ((1u << w) - 1u) << shift;
    remaining = s_step[1];
    ++pass;
    if (s_step[2] == remaining) break;   // the whole bin is taken
  }
  // keys compare on the fixed bits: above T is taken, at T the lowest indices
  const uint32_t T = prefix;
  const int take_eq = remaining;

  // ascending emission: each thread owns a contiguous run of indices; one scan
  // of the packed counts (equal << 32 | above) gives every thread its place
  const int per = (n + nt - 1) / nt;
  const int j0 = min(n, tid * per), j1 = min(n, j0 + per);
  unsigned int n_eq = 0, n_gt = 0;
  for (int j = j0; j < j1; ++j) {
    const uint32_t kk = key_at(j) & mask;
    n_eq += kk == T;
    n_gt += kk > T;
  }
  const unsigned long long before =
      block_exclusive_scan64((static_cast<unsigned long long>(n_eq) << 32) | n_gt, s_scan);
  int e = static_cast<int>(before >> 32);
  int pos = static_cast<int>(before & 0xffffffffu) + min(e, take_eq);
  for (int j = j0; j < j1; ++j) {
    const uint32_t kk = key_at(j) & mask;
    bool take = kk > T;
    if (kk == T) take = (e++ < take_eq);
    if (take && pos < kcap) row[pos++] = j;
  }
  for (int j = k + tid; j < kcap; j += nt) row[j] = -1;
  if (tid == 0 && sel_n) sel_n[unit] = k;
  return k;
}

}  // namespace lserve
