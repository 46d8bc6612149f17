// tile_lists.cuh -- device-built kept-tile lists for block-sparse prefill.
//
// LServe + SampleAttention blog post, "LServe - Prefill Phase", Fig. 1: every KV
// block is fully computed or fully skipped at the kernel's tile granularity;
// dense heads walk the causal tiles (optionally thinned by a block mask),
// streaming heads only the tiles that meet the Lambda support.
//
// Row r = (b * Hkv + g) * nQT + qt owns the ascending list of kept KV tiles kt:
//   dense      kt <= qt  and (no mask or block_mask[b, g, qt, kt] != 0)
//   streaming  kt <= qt  and (64 kt < sink  or  max(64 qt - 64 kt - 63, 0) < local)
// Built in three launches, all on device, no host round trip:
//   tile_count_kernel  one warp per row: count kept tiles (4 mask bytes per lane
//                      per step), histogram of row lengths per (b, kvh)
//   tile_scan_kernel   one CTA: CSR offsets (exclusive scan of the counts) and the
//                      start of every row-length bucket in the work order
//   tile_fill_kernel   one warp per row: ballot-ordered compaction of kt into the
//                      CSR, and the row's slot in the work order
// Work order: (b, kvh) groups one after another, longest rows first inside a
// group.  Concurrent CTAs then share one KV head's K/V, which stays in L2 even
// when the whole K/V of a long sequence does not.
//
// Closed-form rows (TileListParams::closed_form, the tcgen05 prefill): the list
// of a streaming head's row (Lambda at tile level: the sink tiles, then the
// window of the row's query tiles) and of a dense head's row without a block
// mask (every causal tile) is two runs of consecutive tiles, which the attention
// kernel computes itself (row_runs).  Such rows get no CSR entries; their length
// still orders the work.
#pragma once

#include "common.cuh"

namespace lserve {

struct TileListParams {
  int B, Hkv, nQT, sink, local;
  const uint8_t* head_kind;
  const uint8_t* block_mask;   // [B, Hkv, nQT, nQT] or null
  int qg = 1;                  // query tiles per row (a row keeps the union of their lists)
  int nRow = 0;                // rows per (b, kvh) = ceil(nQT / qg)
  int closed_form = 0;         // rows with a closed-form list get no CSR entries
};

// counts[r] of a closed-form row: its length with this flag set (the CSR holds
// nothing for it; the work order uses the length)
constexpr int kClosedRow = 1 << 30;
__device__ __forceinline__ int csr_count(int v) { return (v & kClosedRow) ? 0 : v; }
__device__ __forceinline__ int row_length(int v) { return v & ~kClosedRow; }

// The kept list of row r as two runs, tiles [0, a) then [w, w + n - a), when it
// has that form: a streaming head's row (tiles holding a sink token, 64 kt <
// sink, then the union of the windows of its query tiles qt_lo..qt_hi: tile kt
// meets the window of qt when max(64 (qt - kt) - 63, 0) < local, i.e. qt - kt <
// nw with nw = (local + 62) / 64 + 1 for local > 0 and nw = 0 for local = 0),
// or a dense head's row without a block mask (all tiles kt <= qt_hi).  Returns
// false for a block-masked dense row.  Entry j of the list is j < a ? j : w + j - a.
struct RowRuns {
  int a, w, n;
};
__device__ __forceinline__ bool row_runs(const TileListParams& P, int r, RowRuns* rr) {
  const int qgi = r % P.nRow;
  const int g = (r / P.nRow) % P.Hkv;
  const int qt_lo = qgi * P.qg;
  const int qt_hi = min(P.nQT - 1, qt_lo + P.qg - 1);
  if (P.head_kind[g] == LSERVE_HEAD_DENSE) {
    if (P.block_mask) return false;
    rr->a = rr->w = rr->n = qt_hi + 1;
    return true;
  }
  const int a = min((P.sink + kTile - 1) / kTile, qt_hi + 1);
  int w0 = qt_hi + 1;   // no window
  if (P.local > 0) w0 = max(0, qt_lo - ((P.local + kTile - 2) / kTile + 1) + 1);
  const int w = max(w0, a);
  rr->a = a;
  rr->w = w;
  rr->n = a + (qt_hi + 1 - w);
  return true;
}

__device__ __forceinline__ bool tile_keep(const TileListParams& P, bool streaming, const uint8_t* mrow, int qt,
                                          int kt) {
  if (kt > qt) return false;
  if (streaming) {
    const int mind = max(kTile * (qt - kt) - (kTile - 1), 0);
    return kTile * kt < P.sink || mind < P.local;
  }
  return mrow == nullptr || mrow[kt] != 0;
}

// Is every element of a kept tile (qt, kt) attended?  Then no element mask is
// needed: a tile below the diagonal of a dense head, or one of a streaming head
// that lies wholly inside the sink or wholly inside the window of every row of qt.
__device__ __forceinline__ bool tile_is_full(bool streaming, int qt, int kt, int sink, int local) {
  if (kt >= qt) return false;   // diagonal (or beyond): causal mask needed
  if (!streaming) return true;
  return kTile * kt + kTile <= sink || kTile * qt + (kTile - 1) - kTile * kt < local;
}

// Calls f(base, kt0, keep[4]) for kt = 0..(last query tile of the row) in
// ascending order, 32 lanes x 4 tiles per step.  A row of qg query tiles keeps
// the union of their tiles.
template <typename F>
__device__ __forceinline__ void tile_row_walk(const TileListParams& P, int r, F&& f) {
  const int qgi = r % P.nRow;
  const int bg = r / P.nRow;
  const int g = bg % P.Hkv;
  const int qt_lo = qgi * P.qg;
  const int qt_hi = min(P.nQT - 1, qt_lo + P.qg - 1);
  const bool streaming = P.head_kind[g] != LSERVE_HEAD_DENSE;
  const uint8_t* mbase = (!streaming && P.block_mask) ? P.block_mask + static_cast<long>(bg) * P.nQT * P.nQT
                                                      : nullptr;
  const int lane = threadIdx.x & 31;
  for (int base = 0; base <= qt_hi; base += 128) {
    const int kt0 = base + lane * 4;
    bool k4[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      bool keep = false;
      for (int qt = qt_lo; qt <= qt_hi; ++qt)
        keep |= tile_keep(P, streaming, mbase ? mbase + static_cast<long>(qt) * P.nQT : nullptr, qt, kt0 + e);
      k4[e] = keep;
    }
    f(base, kt0, k4);
  }
}

__global__ void __launch_bounds__(256) tile_count_kernel(TileListParams P, int* __restrict__ counts,
                                                         int* __restrict__ hist) {
  const int r = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int R = P.B * P.Hkv * P.nRow;
  if (r >= R) return;
  RowRuns rr;
  if (P.closed_form && row_runs(P, r, &rr)) {
    if ((threadIdx.x & 31) == 0) {
      counts[r] = rr.n | kClosedRow;
      atomicAdd(&hist[(r / P.nRow) * (P.nQT + 1) + rr.n], 1);
    }
    return;
  }
  int cnt = 0;
  tile_row_walk(P, r, [&](int, int, const bool (&k4)[4]) { cnt += k4[0] + k4[1] + k4[2] + k4[3]; });
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
  if ((threadIdx.x & 31) == 0) {
    counts[r] = cnt;
    atomicAdd(&hist[(r / P.nRow) * (P.nQT + 1) + cnt], 1);
  }
}

// One CTA of 1024 threads.  offsets[r] = sum_{r' < r} counts[r']; for group g
// (rows g*nRow .. g*nRow + nRow - 1), bucket[g][c] = g*nRow + number of rows of
// the group with more than c kept tiles (start of bucket c of that group).
__global__ void __launch_bounds__(1024) tile_scan_kernel(const int* __restrict__ counts, int R,
                                                         int* __restrict__ offsets, const int* __restrict__ hist,
                                                         int nbucket, int* __restrict__ bucket, int nRow,
                                                         long long max_nnz, int* __restrict__ overflow) {
  __shared__ int s_warp[32];
  __shared__ long long s_carry;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) s_carry = 0;
  __syncthreads();
  for (int base = 0; base < R; base += 1024) {
    const int r = base + tid;
    const int v = r < R ? csr_count(counts[r]) : 0;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) s_warp[warp] = x;
    __syncthreads();
    if (warp == 0) {
      int w = s_warp[lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        int y = __shfl_up_sync(0xffffffffu, w, o);
        if (lane >= o) w += y;
      }
      s_warp[lane] = w;
    }
    __syncthreads();
    const long long carry = s_carry;
    const long long excl = carry + (warp > 0 ? s_warp[warp - 1] : 0) + x - v;
    if (r < R) offsets[r] = static_cast<int>(excl);
    __syncthreads();
    if (tid == 1023) s_carry = carry + s_warp[31];
    __syncthreads();
  }
  if (tid == 0) {
    offsets[R] = static_cast<int>(s_carry);
    *overflow = s_carry > max_nnz;
    if (s_carry > max_nnz) report(LSERVE_ERR_DEVICE_BOUNDS);
  }
  // bucket[grp][c] = grp * nRow + (rows of the group with more than c kept
  // tiles): a suffix sum over c per group, one warp per group, 32 buckets a step
  for (int grp = warp; grp < R / nRow; grp += blockDim.x / 32) {
    int carry = grp * nRow;
    for (int c0 = nbucket - 1; c0 >= 0; c0 -= 32) {
      const int c = c0 - lane;   // lane 0 takes the largest c of the step
      const int hv = c >= 0 ? hist[grp * nbucket + c] : 0;
      int x = hv;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
      }
      if (c >= 0) bucket[grp * nbucket + c] = carry + x - hv;
      carry += __shfl_sync(0xffffffffu, x, 31);
    }
  }
}

__global__ void __launch_bounds__(256) tile_fill_kernel(TileListParams P, const int* __restrict__ offsets,
                                                        const int* __restrict__ counts, uint16_t* __restrict__ cols,
                                                        const int* __restrict__ bucket, int* __restrict__ fill,
                                                        int* __restrict__ order, const int* __restrict__ overflow) {
  const int r = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int R = P.B * P.Hkv * P.nRow;
  if (r >= R || *overflow) return;
  const int lane = threadIdx.x & 31;
  int pos = offsets[r];
  const int cr = counts[r];
  if (!(cr & kClosedRow)) tile_row_walk(P, r, [&](int, int kt0, const bool (&k4)[4]) {
    const int c = k4[0] + k4[1] + k4[2] + k4[3];
    int x = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    int w = pos + x - c;
#pragma unroll
    for (int e = 0; e < 4; ++e)
      if (k4[e]) cols[w++] = static_cast<uint16_t>(kt0 + e);
    pos += __shfl_sync(0xffffffffu, x, 31);
  });
  if (lane == 0 && order) {
    const int k = (r / P.nRow) * (P.nQT + 1) + row_length(cr);
    order[bucket[k] + atomicAdd(&fill[k], 1)] = r;
  }
}

}  // namespace lserve
