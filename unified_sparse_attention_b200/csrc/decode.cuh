// decode.cuh -- sparse paged decode attention over the selected pages: the
// selection step's kernel, the attention grid and the log-sum-exp merge.
//
// LServe + SampleAttention blog post, "LServe - Decode Phase" and Fig. 2:
// token-level attention only inside the selected pages.  Streaming heads attend
// to their sink + local tokens (mlsanity LServe page, Abstract: streaming heads
// in both the prefilling and the decoding stages).
//
// Work split.  Unit u = (sequence b, KV head g) has n_u selected pages; the
// pages of all units, laid end to end in unit order, form one flat list of
// T = sum_u n_u pages with unit u at [off_u, off_u + n_u).  The list is cut
// into Re = ranges_in_use(R, T) equal ranges of at least kMinRangePages pages.
// n_u follows from the sequence lengths alone, so one extra block of the top-k
// grid builds this plan (decode_partition) while the other blocks select.
//
// The top-k blocks also write the flat list itself, pre-resolved: entry f holds
// (unit, logical page, physical page, sequence length and flags), so that the
// attention kernel reads one 16-byte entry per page instead of chasing the
// plan, the selection and the page table.
//
// paged_decode_kernel: one wave of CTAs (SMs x 2) that claim ranges from a
// counter, so that SMs that run ahead take more.  Per CTA:
//   * a resolver warp claims ranges (CTA c's first is range c, later ones come
//     from the counter; the next claim in flight while one is
//     copied) and copies their entries of the flat list into a shared-memory
//     ring ahead of the loads, adding the range's own start and end; a range
//     that crosses unit boundaries is cut into segments, one per unit;
//   * an issuer warp streams each page's K and V (64 x d bf16 each, contiguous
//     in the pool) through a 3-stage ring with TMA (128-byte swizzle), and the
//     group's G query rows with a bulk copy at a segment start (full and empty
//     mbarriers per stage);
//   * four consumer warps each own 16 tokens of every page, copy their K/V
//     fragments to registers and release the stage at once, then keep an online
//     softmax for the G <= 8 query heads on mma.sync m16n8k16 tiles laid out
//     transposed: S^T = K Q^T (M = 16 tokens, N = 8 heads) and O^T += V^T P^T
//     with P^T from movmatrix, so the heads fill N exactly;
//   * at the end of a segment each consumer warp writes its own normalised
//     partial (o, lse) -- no cross-warp exchange, the ring keeps streaming.
// decode_merge_kernel (one CTA per unit) then combines a unit's partials:
// out = sum_i 2^(lse_i - lse) o_i, lse = log2 sum_i 2^lse_i.
//
// Partial slots.  Segment (range r, unit u) uses slot r + u: along the flat
// list both r and u never decrease and one of them grows at every segment
// boundary, so slots are distinct, and unit u's slots are the contiguous run
// r_first(u) + u .. r_last(u) + u.  Slots <= Re + units - 1.
//
// INT4 pages (paged_decode_kernel<D, true>, lserve_decode_int4; blog post,
// "LServe - Decode Phase" and Fig. 2: INT4 KV cuts the bytes of every page).
// A stage holds the page's K and V codes (d/2 bytes a row, in the order of the
// operand fragments, so a lane loads its share with 16-byte reads), the key
// steps/offsets per channel, the value steps/offsets per token (fp32) and the
// unit's q rows.  Each consumer warp takes whole pages (four 16-token tiles),
// so a page's step fold and softmax reductions are done once.  The codes go
// into fp16 MMAs as 1024 + code or 1024 + 16 code (one mask per code pair, the
// nibble lying in the mantissa of 1024, whose ulp is 1), the steps fold into
// the other operand (s q as fp16 hi + lo; s p as fp16), and the offsets into
// one fp32 term per head; the 1024 terms are taken out by MMAs of a constant
// 1024 operand with the same fp16 operands, so they cancel exactly.  Eight
// 12 KB stages, two CTAs per SM.  Bytes per selected page: 64 * d + 1.5 KB
// (d = 128).
//
// Bytes per selected page: 2 * 64 * d * 2 (K and V); the kernel is HBM-bound.
// Tokens outside the attended set (past seq_len; outside the Lambda set of a
// streaming head) are masked exactly: their logits become -inf by selection
// (not arithmetic) and their V rows are zeroed in the MMA operand, so even NaN
// garbage there cannot reach the result.  No CTA ever waits for another.
#pragma once

#include <climits>

#include "common.cuh"
#include "select.cuh"

namespace lserve {

constexpr int kDecodeStages = 3;     // bf16 pages: ring depth (three 34 KB stages at d = 128)
constexpr int kDecodeStagesQ4 = 8;   // INT4 pages: two pages in flight per consumer warp
constexpr int kDecodeWarps = 4;                           // consumer warps
constexpr int kIssuerWarp = kDecodeWarps;                  // issues the TMA loads
constexpr int kResolverWarp = kDecodeWarps + 1;            // claims ranges, resolves their pages
constexpr int kDecodeThreads = (kDecodeWarps + 2) * 32;
constexpr int kDecodeCtasPerSm = 2;     // bf16 pages: the three-stage ring's shared memory admits two
constexpr int kDecodeCtasPerSmQ4 = 2;   // INT4 pages: registers admit two
constexpr int kDecodeMaxG = 8;
constexpr int kRangesPerCta = 4;   // ranges of the flat page list per attention CTA
constexpr int kMetaRing = 64;      // resolved pages buffered ahead of the loads

constexpr int kSegStart = 1, kSegEnd = 2, kSegStreaming = 4;
// Wait for the loads still in flight when a CTA gives up: fixed, independent of
// the (possibly very short) limit of the ordinary waits, so that no copy can
// land in shared memory after the CTA has left.
constexpr unsigned long long kDrainTimeoutNs = 1000000000ull;

template <int D>
struct DecodeCfg {
  static constexpr int kBoxes = D / 64;                 // 64-channel TMA boxes per row
  static constexpr int kBoxBytes = 64 * 128;            // 64 rows x 128 bytes
  static constexpr int kKVBytes = kBoxes * kBoxBytes;   // one K (or V) page
  // stage = K page | V page | q rows of the group (rounded up to 1 KB)
  __host__ __device__ static int stage_bytes(int G) { return 2 * kKVBytes + ((G * D * 2 + 1023) / 1024) * 1024; }
  __host__ __device__ static int smem_bytes(int G) { return kDecodeStages * stage_bytes(G) + 1024; }   // + alignment slack
  // INT4 pages (lserve_decode_int4): stage = K codes | V codes | K steps, offsets |
  // V steps, offsets | q rows (layouts in quant.cuh); the consumers build their
  // tensor-core fragments from the code words directly
  static constexpr int kQ4Bytes = 64 * (D / 2);   // one page of codes
  static constexpr int kParKBytes = 2 * D * 4;    // fp32 step and offset per channel
  static constexpr int kParVBytes = 2 * 64 * 4;   // fp32 step and offset per token
  static constexpr int kQ4ParK = 2 * kQ4Bytes, kQ4ParV = kQ4ParK + kParKBytes, kQ4Q = kQ4ParV + kParVBytes;
  __host__ __device__ static int stage_bytes_q4(int G) { return ((kQ4Q + G * D * 2 + 1023) / 1024) * 1024; }
  __host__ __device__ static int smem_bytes_q4(int G) { return kDecodeStagesQ4 * stage_bytes_q4(G) + 1024; }
};

// Ranges the T selected pages are cut into: at most R (the workspace's
// capacity), each of at least kMinRangePages pages so that the per-range costs
// (resolving, a partial per warp, merging) stay small next to streaming the
// pages; one range when T is smaller.  Every kernel of the step computes it
// alike from T.
constexpr int kMinRangePages = 8;
__host__ __device__ __forceinline__ long long ranges_in_use(long long R, long long T) {
  const long long r = T / kMinRangePages;
  return r < 1 ? 1 : (r < R ? r : R);
}

// CTA owning flat position f: the largest c with floor(c T / P) <= f.  With
// P <= T no share is empty, so the owners of a range are every CTA between the
// owners of its ends.
__host__ __device__ __forceinline__ int flat_owner(long long f, long long T, long long P) {
  return static_cast<int>(((f + 1) * P + T - 1) / T - 1);
}

__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
               ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

// Pages selected for unit u: known from the sequence length alone
// (unit_selected(), the count topk_unit() writes), or a kept selection's size.
__device__ __forceinline__ int unit_count(int u, const int32_t* __restrict__ seq_lens,
                                          const uint8_t* __restrict__ head_kind, int Hkv, int maxP, int budget_pages,
                                          int sink, int local, int kcap, const int32_t* sel_n_in) {
  const bool dense = head_kind[u % Hkv] == LSERVE_HEAD_DENSE;
  return (dense && sel_n_in) ? min(max(sel_n_in[u], 0), kcap)
                             : unit_selected(seq_lens[u / Hkv], maxP, dense, budget_pages, sink, local, kcap);
}

// The plan of the attention grid, by one block (any multiple of 32 threads).
// The selection sizes are known before the selection (unit_count()), so this
// runs beside the top-k blocks instead of after them.  off[u] = pages selected
// before unit u, off[units] = T; the range counter zeroed for the attention
// kernel.  Units with nothing selected get their output here: out = 0,
// lse = -inf.
__device__ __forceinline__ void decode_partition(const int32_t* __restrict__ seq_lens,
                                                 const uint8_t* __restrict__ head_kind, int Hkv, int maxP,
                                                 int budget_pages, int sink, int local, int units, int kcap,
                                                 int G, int D, int32_t* off, int32_t* range_counter, bf16* out,
                                                 float* lse_out, const int32_t* sel_n_in) {
  __shared__ int s_warp[32];
  __shared__ int s_carry;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nt = blockDim.x, nw = nt >> 5;
  if (tid == 0) s_carry = 0;
  __syncthreads();
  for (int base = 0; base < units; base += nt) {
    const int u = base + tid;
    const int v = u < units ? unit_count(u, seq_lens, head_kind, Hkv, maxP, budget_pages, sink, local, kcap,
                                         sel_n_in)
                            : 0;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) s_warp[warp] = x;
    __syncthreads();
    if (warp == 0) {
      int w = lane < nw ? s_warp[lane] : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, w, o);
        if (lane >= o) w += y;
      }
      if (lane < nw) s_warp[lane] = w;
    }
    __syncthreads();
    const int carry = s_carry;
    if (u < units) off[u] = carry + (warp > 0 ? s_warp[warp - 1] : 0) + x - v;
    __syncthreads();
    if (tid == nt - 1) s_carry = carry + s_warp[nw - 1];
    __syncthreads();
  }
  const long long T = s_carry;
  if (tid == 0) {
    off[units] = static_cast<int>(T);
    *range_counter = 0;
  }
  __syncthreads();   // off[] of this block is visible to the block from here on
  for (int u = tid; u < units; u += nt) {
    if (off[u + 1] == off[u]) {   // nothing selected: out = 0, lse = -inf
      for (int idx = 0; idx < G * D; idx += 8)
        *reinterpret_cast<uint4*>(out + static_cast<long>(u) * G * D + idx) = make_uint4(0u, 0u, 0u, 0u);
      if (lse_out)
        for (int h = 0; h < G; ++h) lse_out[static_cast<long>(u) * G + h] = kNegInf;
    }
  }
}

// Selection step: blocks 0 .. units-1 select the pages of one unit each
// (topk_unit; with a kept selection sel_in / sel_n_in the dense units copy
// their rows instead) and write the unit's entries of the flat list; block
// `units` lays out the attention grid's work (decode_partition), which does not
// depend on the selected pages.
__global__ void __launch_bounds__(kTopkThreads, 2) topk_pages_kernel(
    const float* scores, int maxP, const int32_t* __restrict__ seq_lens, const uint8_t* __restrict__ head_kind,
    const int32_t* __restrict__ page_table, int num_pages, int Hkv, int budget_pages, int sink, int local,
    int32_t* sel, int32_t* sel_n, int kcap, int units, int G, int D, int32_t* off, int4* flat,
    int32_t* range_counter, bf16* out, float* lse_out, const int32_t* sel_in, const int32_t* sel_n_in) {
  __shared__ int s_part[kTopkThreads / 32];
  const int unit = blockIdx.x, tid = threadIdx.x;
  // sequence length, head kind and the unit's place in the flat list are inputs
  // of the step, not results of the scoring grid: computed before the wait
  const int L = unit < units ? seq_lens[unit / Hkv] : 0;
  const bool dense = unit < units && head_kind[unit % Hkv] == LSERVE_HEAD_DENSE;
  int start = 0;
  if (unit < units) {
    int part = 0;
    for (int v = tid; v < unit; v += blockDim.x)
      part += unit_count(v, seq_lens, head_kind, Hkv, maxP, budget_pages, sink, local, kcap, sel_n_in);
    part = __reduce_add_sync(0xffffffffu, part);
    if ((tid & 31) == 0) s_part[tid >> 5] = part;
    __syncthreads();
    for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) start += s_part[w];
  }
  pdl_wait();
  pdl_launch_dependents();   // the attention grid may get resident; it waits for this grid
  if (unit < units) {
    const int m = topk_unit(scores, unit, maxP, L, dense, budget_pages, sink, local, sel, sel_n, kcap, sel_in,
                            sel_n_in);
    __syncthreads();   // the unit's selection row, written by every thread, is complete
    const int32_t* row = sel + static_cast<long>(unit) * kcap;
    const int b = unit / Hkv;
    const int flags = dense ? 0 : kSegStreaming;
    for (int j = tid; j < m; j += blockDim.x) {
      const int pidx = row[j];
      int phys = -1;
      if (pidx >= 0 && pidx < maxP) {
        const int p = page_table[static_cast<long>(b) * maxP + pidx];
        if (p >= 0 && p < num_pages) phys = p;
      }
      if (phys < 0) report(LSERVE_ERR_DEVICE_BOUNDS);
      flat[start + j] = make_int4(unit, pidx, phys,
                                  (max(L, 0) << 3) | flags | (j == 0 ? kSegStart : 0) | (j == m - 1 ? kSegEnd : 0));
    }
  } else {
    decode_partition(seq_lens, head_kind, Hkv, maxP, budget_pages, sink, local, units, kcap, G, D, off,
                     range_counter, out, lse_out, sel_n_in);
  }
}

// Spin (with short sleeps) until cond() holds; false (and LSERVE_ERR_DEVICE_TIMEOUT
// recorded) once timeout_ns has passed.
template <typename F>
__device__ __forceinline__ bool spin_until(F&& cond, uint64_t timeout_ns) {
  if (cond()) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    for (int i = 0; i < 32; ++i) {
      if (cond()) return true;
      __nanosleep(32);
    }
    if (globaltimer_ns() - t0 > timeout_ns) {
      report(LSERVE_ERR_DEVICE_TIMEOUT);
      return false;
    }
  }
}

// fp16 operands from INT4 code words.  Code pair j of a word sits in nibbles j
// and j + 4 (bits 4j..4j+3 of each half-word); q4h_lo gives the pair in
// nibbles 0, 4 as 1024 + code and q4h_hi the pair in nibbles 1, 5 as
// 1024 + 16 code (fp16 1024 is 0x6400; its ulp is 1); the word shifted right
// by 8 gives pairs 2 and 3 the same way.
constexpr uint32_t kF16x2_1024 = 0x64006400u;
__device__ __forceinline__ uint32_t q4h_lo(uint32_t w) { return (w & 0x000F000Fu) | kF16x2_1024; }
__device__ __forceinline__ uint32_t q4h_hi(uint32_t w) { return (w & 0x00F000F0u) | kF16x2_1024; }

// fp16 pair {low half a, high half b}, rounded to nearest even
__device__ __forceinline__ uint32_t pack_f16x2(float a, float b) {
  uint32_t d;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(b), "f"(a));
  return d;
}
__device__ __forceinline__ float2 unpack_f16x2(uint32_t v) {
  float a, b;
  asm("{\n.reg .f16 l, h;\nmov.b32 {l, h}, %2;\ncvt.f32.f16 %0, l;\ncvt.f32.f16 %1, h;\n}" : "=f"(a), "=f"(b) : "r"(v));
  return make_float2(a, b);
}
// A compile-time int passed to a generic lambda.
template <int N>
struct IntConst {
  static constexpr int value = N;
};

// x = hi + lo with hi, lo fp16 pairs (about 22 significant bits together)
__device__ __forceinline__ void split_f16x2(float a, float b, uint32_t& hi, uint32_t& lo) {
  hi = pack_f16x2(a, b);
  const float2 h = unpack_f16x2(hi);
  lo = pack_f16x2(a - h.x, b - h.y);
}
// D = A(16x16, row) * B(16x8, col) + D, fp16 inputs, fp32 accumulators (no side
// effects, so that the compiler may interleave independent chains)
__device__ __forceinline__ void mma_f16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Q4 = false: bf16 pages (tmK, tmV over [NP * Hkv * 64, d] bf16).  Q4 = true:
// INT4 pages (tmK, tmV over [NP * Hkv * 64, d/2] bytes) with their steps and
// offsets kpar, vpar (layouts in quant.cuh).  The steps fold into the other
// operand, so the tensor cores multiply integer codes (exact in fp16, offset by
// 1024, with the multiplier m = 1 or 16 of their nibble position):
//   q.k_t = sum_c (1024 + m_c code_tc) (s_c q_c / m_c) + sum_c lo_c q_c - 1024 sum_c (s_c q_c / m_c)
//     with s q / m as two fp16 parts (hi + lo, two MMAs);
//   sum_t p_t v_tc = ((sum_t (1024 + m_c code_tc) (s_t p_t)) - 1024 sum_t (s_t p_t)) / m_c + sum_t lo_t p_t
//     with s p as one fp16 part (its rounding, 2^-11, is finer than the bf16 P of bf16 pages).
template <int D, bool Q4 = false>
__global__ void __launch_bounds__(kDecodeThreads, 2) paged_decode_kernel(
    const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
    const bf16* __restrict__ q, const int4* flat, const int32_t* off, int32_t* range_counter, int R,
    int kcap, int units, int Hkv, int G, int sink, int local, float scale_log2,
    unsigned long long timeout_ns, int debug_stall, float* __restrict__ part_o, float* __restrict__ part_lse,
    const float* __restrict__ kpar = nullptr, const float* __restrict__ vpar = nullptr) {
  using Cfg = DecodeCfg<D>;
  constexpr int NS = Q4 ? kDecodeStagesQ4 : kDecodeStages;   // ring depth
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[NS];    // stage loaded (issuer's expect_tx + bytes)
  __shared__ __align__(8) uint64_t empty_bar[NS];   // stage consumed (bf16: one arrive per consumer warp; INT4: one)
  __shared__ int4 s_meta[kMetaRing];   // {unit, logical page, physical page (-1: invalid), seq_len << 3 | flags}
  __shared__ int s_range[kMetaRing];   // range of each ring entry (its partial slot is range + unit)
  __shared__ int s_resolved;           // pages whose metadata is in the ring
  __shared__ int s_total;              // pages this CTA processes (INT_MAX until the ranges run out)
  __shared__ int s_issued;             // pages whose loads were issued
  __shared__ int s_abort;              // a bounded wait ran out or the plan was inconsistent
  __shared__ int s_seen[kDecodeWarps]; // INT4: pages whose metadata each consumer warp has read
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int stage_bytes = Q4 ? Cfg::stage_bytes_q4(G) : Cfg::stage_bytes(G);
  const int q_bytes = G * D * 2;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) {
    prefetch_tensormap(&tmK);
    prefetch_tensormap(&tmV);
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], Q4 ? 1 : kDecodeWarps);   // INT4: one warp consumes a page
    }
    fence_barrier_init();
    s_resolved = 0;
    s_total = INT_MAX;
    s_issued = 0;
    s_abort = 0;
    for (int w = 0; w < kDecodeWarps; ++w) s_seen[w] = 0;
  }
  __syncthreads();
  volatile int* v_resolved = &s_resolved;
  volatile int* v_total = &s_total;
  volatile int* v_issued = &s_issued;
  volatile int* v_abort = &s_abort;
  volatile int* v_seen = s_seen;
  // off / range_unit / the selection come from the previous kernels, which may
  // still be running: they are read only after this wait, with L2 loads through
  // pointers that are not restrict-qualified (no load of them can move above it).
  pdl_wait();
  const long long T = __ldcg(off + units);
  if (T <= 0 || T > static_cast<long long>(units) * kcap) {   // nothing selected anywhere, or a bad plan
    if (T != 0 && tid == 0) report(LSERVE_ERR_DEVICE_BOUNDS);
    return;
  }
  const long long Re = ranges_in_use(R, T);   // ranges that hold pages

  if (warp == kResolverWarp && debug_stall) {
    // failure-detection test: publish nothing, so that every other wait of the
    // CTA runs out (nothing is issued, so nothing is in flight when it leaves)
  } else if (warp == kResolverWarp) {
    // ---- claim ranges and copy their entries of the flat list into the ring,
    // adding each range's own start and end to the unit's; the next claim is in
    // flight while a range is copied, and a batch's entries are loaded before
    // the wait for room in the ring
    int gp = 0;   // pages in the ring so far
    bool ok = true, stopped = false;   // !ok: inconsistent entry; stopped: the CTA is giving up
    // the first range is this CTA's own (range blockIdx.x), so the first pages need no
    // atomic round trip; later ranges come from the counter, above the grid's own ones
    int r_next = blockIdx.x;
    while (ok && !stopped) {
      const int r = __shfl_sync(0xffffffffu, r_next, 0);
      if (r >= Re) break;
      if (lane == 0) r_next = static_cast<int>(gridDim.x) + atomicAdd(range_counter, 1);
      const int lo = static_cast<int>(r * T / Re), hi = static_cast<int>((r + 1) * T / Re);
      for (int f0 = lo; f0 < hi; f0 += 32) {
        const int f = f0 + lane, cnt = min(32, hi - f0);
        int4 e = make_int4(-1, 0, -1, 0);
        if (f < hi) e = __ldcg(flat + f);
        bool room = true;
        if (lane == 0)
          room = spin_until(
                     [&] {
                       if (*v_abort) return true;
                       const int need = gp + cnt - kMetaRing;   // entries of pages below it are reused
                       if (*v_issued < need + NS) return false;
                       if constexpr (Q4) {   // INT4 consumers read every page's entry, their own or not
                         for (int w = 0; w < kDecodeWarps; ++w)
                           if (v_seen[w] < need) return false;
                       }
                       return true;
                     },
                     timeout_ns) && !*v_abort;
        if (!__shfl_sync(0xffffffffu, room, 0)) {
          stopped = true;
          break;
        }
        const bool bad = f < hi && (e.x < 0 || e.x >= units);
        if (__any_sync(0xffffffffu, bad)) {
          ok = false;
          break;
        }
        if (f < hi) {
          e.w |= (f == lo ? kSegStart : 0) | (f == hi - 1 ? kSegEnd : 0);
          const int slot = (gp + lane) % kMetaRing;
          s_meta[slot] = e;
          s_range[slot] = r;
        }
        __syncwarp();
        __threadfence_block();
        gp += cnt;
        if (lane == 0) *v_resolved = gp;
      }
    }
    if (lane == 0) {
      if (!ok) report(LSERVE_ERR_DEVICE_BOUNDS);
      if (!ok || stopped) *v_abort = 1;
      __threadfence_block();
      *v_total = gp;
    }
  } else if (warp == kIssuerWarp) {
    // ---- issue each resolved page's loads once its stage is free
    if (lane == 0) {
      const uint64_t pol = l2_evict_first();   // every page is read once per step
      for (int gp = 0;; ++gp) {
        if (!spin_until([&] { return *v_resolved > gp || *v_total <= gp || *v_abort; }, timeout_ns)) {
          *v_abort = 1;
          break;
        }
        if (*v_resolved <= gp || *v_abort) break;   // no page gp: the ranges ran out
        __threadfence_block();
        const int st = gp % NS;
        if (gp >= NS && !mbar_wait_bounded(&empty_bar[st], ((gp / NS) - 1) & 1, timeout_ns)) {
          *v_abort = 1;
          break;
        }
        const int4 md = s_meta[gp % kMetaRing];
        const int g = md.x % Hkv;
        const int p = md.z >= 0 ? md.z : 0;   // an invalid page loads page 0; all its tokens are masked
        uint8_t* kdst = smem + st * stage_bytes;
        const bool with_q = Q4 || (md.w & kSegStart);   // INT4: every page carries q (its warp folds it)
        const int row = (p * Hkv + g) * kPage;
        if constexpr (Q4) {
          mbar_arrive_expect_tx(&full_bar[st], Cfg::kQ4Q + (with_q ? q_bytes : 0));
          tma_load_2d_hint(kdst, &tmK, &full_bar[st], 0, row, pol);
          tma_load_2d_hint(kdst + Cfg::kQ4Bytes, &tmV, &full_bar[st], 0, row, pol);
          const long ph = static_cast<long>(p) * Hkv + g;
          bulk_load(kdst + Cfg::kQ4ParK, kpar + ph * 2 * D, Cfg::kParKBytes, &full_bar[st]);
          bulk_load(kdst + Cfg::kQ4ParV, vpar + ph * 2 * kPage, Cfg::kParVBytes, &full_bar[st]);
          if (with_q) bulk_load(kdst + Cfg::kQ4Q, q + static_cast<long>(md.x) * G * D, q_bytes, &full_bar[st]);
        } else {
          uint8_t* vdst = kdst + Cfg::kKVBytes;
          mbar_arrive_expect_tx(&full_bar[st], 2 * Cfg::kKVBytes + (with_q ? q_bytes : 0));
#pragma unroll
          for (int x = 0; x < Cfg::kBoxes; ++x) {
            tma_load_2d_hint(kdst + x * Cfg::kBoxBytes, &tmK, &full_bar[st], x * 64, row, pol);
            tma_load_2d_hint(vdst + x * Cfg::kBoxBytes, &tmV, &full_bar[st], x * 64, row, pol);
          }
          if (with_q) bulk_load(vdst + Cfg::kKVBytes, q + static_cast<long>(md.x) * G * D, q_bytes, &full_bar[st]);
        }
        *v_issued = gp + 1;
      }
    }
    __syncwarp();
  } else if constexpr (Q4) {
    // ---- INT4 consumers: warp w takes the pages gp = w (mod 4) whole (four
    // 16-token tiles), so that a page's step fold, softmax reductions and
    // offsets' terms are computed once per page and its four tiles give the
    // tensor-core chains independent work.  Every warp reads every page's
    // metadata, keeps its own online softmax per segment and writes one partial
    // per segment (an empty one where it took no page of the segment).
    // Transposed fp16 tiles as for bf16 pages: S^T = K Q^T (M = 16 tokens, N =
    // 8 heads), O^T += V^T P^T (M = 16 channels, N = heads, K = 16 tokens); a
    // lane holds heads tc, tc + 1.
    constexpr int KS = D / 16;
    constexpr int WC = D / 32;   // key code words of one row in a lane's chunk
    const uint32_t kA1024[4] = {kF16x2_1024, kF16x2_1024, kF16x2_1024, kF16x2_1024};
    const int qr = lane >> 2, tq = lane & 3, tc = 2 * tq;
    float acc[D / 16][4];   // O^T: rows 16 mt + qr (code multiplier 1) and 16 mt + qr + 8 (multiplier 16)
    float voff[4];          // 1024 sum_t (s_t p_t): the codes' offset in every row of acc
    float m_run[2], l_run[2], vl_run[2];   // heads tc, tc + 1; vl = sum_t lo_t p_t (lane-partial)
    auto reset = [&]() {
#pragma unroll
      for (int mt = 0; mt < D / 16; ++mt) acc[mt][0] = acc[mt][1] = acc[mt][2] = acc[mt][3] = 0.f;
      voff[0] = voff[1] = voff[2] = voff[3] = 0.f;
      m_run[0] = m_run[1] = kNegInf;
      l_run[0] = l_run[1] = 0.f;
      vl_run[0] = vl_run[1] = 0.f;
    };
    reset();
    for (int gp = 0;; ++gp) {
      bool have = false;
      if (lane == 0) {
        const bool known = spin_until([&] { return *v_resolved > gp || *v_total <= gp || *v_abort; }, timeout_ns);
        if (!known) *v_abort = 1;
        have = known && *v_resolved > gp && !*v_abort;
      }
      if (!__shfl_sync(0xffffffffu, have, 0)) break;
      const int4 md = s_meta[gp % kMetaRing];
      const int vr = s_range[gp % kMetaRing];
      __syncwarp();
      __threadfence_block();
      if (lane == 0) v_seen[warp] = gp + 1;   // the resolver may reuse this ring entry from here on
      if (md.w & kSegStart) reset();
      if (gp % kDecodeWarps == warp) {
        const int st = gp % NS;
        const bool landed = mbar_wait_bounded(&full_bar[st], (gp / NS) & 1, timeout_ns);
        if (__any_sync(0xffffffffu, !landed || *v_abort != 0)) {
          if (lane == 0) *v_abort = 1;
          break;
        }
        const int pidx = md.y;
        const bool page_ok = md.z >= 0, streaming = md.w & kSegStreaming;
        const int L = md.w >> 3;
        const uint8_t* stg = smem + st * stage_bytes;
        const uint8_t* qs = stg + Cfg::kQ4Q;   // q rows of the unit, [G][D] bf16
        // ---- fold the key steps into q: B = s q of head qr at channels 16 ks + tc + {0, 1}
        // (b0) and + {8, 9} (b1, divided by 16: those codes carry the multiplier 16), each
        // as an fp16 pair hi + lo; kl = sum of lo_c q_c over this lane's channels
        uint32_t bh[KS][2], bl[KS][2];
        float kl = 0.f;
        const float* kps = reinterpret_cast<const float*>(stg + Cfg::kQ4ParK) + tq * (D / 4);
        // G = 1, 2, 4: only the lanes qr < G hold a non-zero B, so every lane group
        // qr = h + G r folds k-steps j R + r (R = 8 / G) of head h, and the head's
        // lanes take k-step ks from lane 4 (qr + G (ks % R)) + tq, slot ks / R
        auto fold_spread = [&](auto g_const) {
          constexpr int GG = decltype(g_const)::value, R = 8 / GG, NJ = (KS + R - 1) / R;
          const int h = qr % GG, r = qr / GG;
          uint32_t fh[NJ][2], fl[NJ][2];
#pragma unroll
          for (int j = 0; j < NJ; ++j) {
            const int ks = j * R + r;
            fh[j][0] = fh[j][1] = fl[j][0] = fl[j][1] = 0u;
            if (ks < KS) {
              const float4 s4 = *reinterpret_cast<const float4*>(kps + 4 * ks);
              const float4 l4 = *reinterpret_cast<const float4*>(kps + D + 4 * ks);
              const int c = 16 * ks + tc;
              const uint32_t qa = *reinterpret_cast<const uint32_t*>(qs + (h * D + c) * 2);
              const uint32_t qb = *reinterpret_cast<const uint32_t*>(qs + (h * D + c + 8) * 2);
              const float q0 = bf16_lo(qa), q1 = bf16_hi(qa), q2 = bf16_lo(qb), q3 = bf16_hi(qb);
              kl = fmaf(l4.x, q0, fmaf(l4.y, q1, fmaf(l4.z, q2, fmaf(l4.w, q3, kl))));
              split_f16x2(s4.x * q0, s4.y * q1, fh[j][0], fl[j][0]);
              split_f16x2((s4.z * 0.0625f) * q2, (s4.w * 0.0625f) * q3, fh[j][1], fl[j][1]);
            }
          }
#pragma unroll
          for (int ks = 0; ks < KS; ++ks) {
            const int src = 4 * (h + GG * (ks % R)) + tq;
            const uint32_t x0 = __shfl_sync(0xffffffffu, fh[ks / R][0], src);
            const uint32_t x1 = __shfl_sync(0xffffffffu, fh[ks / R][1], src);
            const uint32_t y0 = __shfl_sync(0xffffffffu, fl[ks / R][0], src);
            const uint32_t y1 = __shfl_sync(0xffffffffu, fl[ks / R][1], src);
            bh[ks][0] = qr < GG ? x0 : 0u;
            bh[ks][1] = qr < GG ? x1 : 0u;
            bl[ks][0] = qr < GG ? y0 : 0u;
            bl[ks][1] = qr < GG ? y1 : 0u;
          }
          // head h's lo_c q_c over every k-step, left on its own lanes (summed over tq below)
#pragma unroll
          for (int o = 4 * GG; o < 32; o <<= 1) kl += __shfl_xor_sync(0xffffffffu, kl, o);
          if (qr >= GG) kl = 0.f;
        };
        if (G == 1) {
          fold_spread(IntConst<1>{});
        } else if (G == 2) {
          fold_spread(IntConst<2>{});
        } else if (G == 4) {
          fold_spread(IntConst<4>{});
        } else {
#pragma unroll
          for (int ks = 0; ks < KS; ++ks) {
            const float4 s4 = *reinterpret_cast<const float4*>(kps + 4 * ks);
            const float4 l4 = *reinterpret_cast<const float4*>(kps + D + 4 * ks);
            const int c = 16 * ks + tc;
            uint32_t qa = 0u, qb = 0u;
            if (qr < G) {
              qa = *reinterpret_cast<const uint32_t*>(qs + (qr * D + c) * 2);
              qb = *reinterpret_cast<const uint32_t*>(qs + (qr * D + c + 8) * 2);
            }
            const float q0 = bf16_lo(qa), q1 = bf16_hi(qa), q2 = bf16_lo(qb), q3 = bf16_hi(qb);
            kl = fmaf(l4.x, q0, fmaf(l4.y, q1, fmaf(l4.z, q2, fmaf(l4.w, q3, kl))));
            split_f16x2(s4.x * q0, s4.y * q1, bh[ks][0], bl[ks][0]);
            split_f16x2((s4.z * 0.0625f) * q2, (s4.w * 0.0625f) * q3, bh[ks][1], bl[ks][1]);
          }
        }
        // the codes' offset: 1024 sum_c B (hi + lo) of heads tc, tc + 1, by the tensor
        // cores from the same operands, so that it cancels the MMAs' own term exactly
        float ko[4] = {0.f, 0.f, 0.f, 0.f}, kol[4] = {0.f, 0.f, 0.f, 0.f};   // two chains: hi and lo parts
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
          mma_f16_16816(ko, kA1024, bh[ks][0], bh[ks][1]);
          mma_f16_16816(kol, kA1024, bl[ks][0], bl[ks][1]);
        }
        ko[0] += kol[0];
        ko[1] += kol[1];
        kl += __shfl_xor_sync(0xffffffffu, kl, 1);
        kl += __shfl_xor_sync(0xffffffffu, kl, 2);
        const float kc[2] = {__shfl_sync(0xffffffffu, kl, 4 * tc) - ko[0],
                             __shfl_sync(0xffffffffu, kl, 4 * (tc + 1)) - ko[1]};
        // ---- S^T of the four tiles: A = 1024 + code (channels + 0, + 1) or 1024 + 16 code
        // (+ 8, + 9) of key rows 16 t + qr, + 8
        float sacc[4][4];
#pragma unroll
        for (int t = 0; t < 4; ++t) sacc[t][0] = sacc[t][1] = sacc[t][2] = sacc[t][3] = 0.f;
        // word wi of a row's chunk holds the code pairs of k-steps 2 wi (nibbles 0, 1, 4, 5)
        // and 2 wi + 1 (nibbles 2, 3, 6, 7); two tiles at a time, 16-byte reads
#pragma unroll
        for (int t0 = 0; t0 < 4; t0 += 2) {
          uint32_t kw[2][2][WC];
#pragma unroll
          for (int tt = 0; tt < 2; ++tt) {
#pragma unroll
            for (int r = 0; r < 2; ++r) {
              const uint8_t* kr = stg + (16 * (t0 + tt) + qr + 8 * r) * (D / 2) + tq * (D / 8);
              if constexpr (WC % 4 == 0) {
#pragma unroll
                for (int x = 0; x < WC; x += 4) {
                  const uint4 v = *reinterpret_cast<const uint4*>(kr + 4 * x);
                  kw[tt][r][x] = v.x, kw[tt][r][x + 1] = v.y, kw[tt][r][x + 2] = v.z, kw[tt][r][x + 3] = v.w;
                }
              } else {
#pragma unroll
                for (int x = 0; x < WC; x += 2) {
                  const uint2 v = *reinterpret_cast<const uint2*>(kr + 4 * x);
                  kw[tt][r][x] = v.x, kw[tt][r][x + 1] = v.y;
                }
              }
            }
          }
          float sl[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};   // lo parts: chains of their own
#pragma unroll
          for (int ks = 0; ks < KS; ++ks) {
#pragma unroll
            for (int tt = 0; tt < 2; ++tt) {
              const uint32_t w0 = (ks & 1) ? kw[tt][0][ks >> 1] >> 8 : kw[tt][0][ks >> 1];
              const uint32_t w1 = (ks & 1) ? kw[tt][1][ks >> 1] >> 8 : kw[tt][1][ks >> 1];
              const uint32_t a[4] = {q4h_lo(w0), q4h_lo(w1), q4h_hi(w0), q4h_hi(w1)};
              mma_f16_16816(sacc[t0 + tt], a, bh[ks][0], bh[ks][1]);
              mma_f16_16816(sl[tt], a, bl[ks][0], bl[ks][1]);
            }
          }
#pragma unroll
          for (int tt = 0; tt < 2; ++tt)
#pragma unroll
            for (int e = 0; e < 4; ++e) sacc[t0 + tt][e] += sl[tt][e];
        }
        // ---- mask + online softmax over the page.  Element (t, e): token 16 t + qr + 8 (e >> 1),
        // head tc + (e & 1)
        const int tok0 = pidx * kPage + qr;
        bool ok[4][2];
        float p[4][4];
        float mh[2] = {kNegInf, kNegInf};
#pragma unroll
        for (int t = 0; t < 4; ++t) {
#pragma unroll
          for (int r = 0; r < 2; ++r) {
            const int tk = tok0 + 16 * t + 8 * r;
            ok[t][r] = page_ok && tk < L && (!streaming || tk < sink || tk >= L - local);
          }
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            p[t][e] = ok[t][e >> 1] ? (sacc[t][e] + kc[e & 1]) * scale_log2 : kNegInf;
            mh[e & 1] = fmaxf(mh[e & 1], p[t][e]);
          }
        }
#pragma unroll
        for (int o = 4; o < 32; o <<= 1) {
          mh[0] = fmaxf(mh[0], __shfl_xor_sync(0xffffffffu, mh[0], o));
          mh[1] = fmaxf(mh[1], __shfl_xor_sync(0xffffffffu, mh[1], o));
        }
        float corr[2], m_use[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const float m_new = fmaxf(m_run[h], mh[h]);
          m_use[h] = m_new == kNegInf ? 0.f : m_new;
          corr[h] = fast_exp2(m_run[h] - m_use[h]);
          m_run[h] = m_new;
        }
        if (__any_sync(0xffffffffu, corr[0] != 1.f || corr[1] != 1.f)) {
#pragma unroll
          for (int mt = 0; mt < D / 16; ++mt) {
            acc[mt][0] *= corr[0];
            acc[mt][1] *= corr[1];
            acc[mt][2] *= corr[0];
            acc[mt][3] *= corr[1];
          }
          voff[0] *= corr[0];
          voff[1] *= corr[1];
          voff[2] *= corr[0];
          voff[3] *= corr[1];
        }
        // ---- per tile: P^T scaled by the value steps of its tokens (masked tokens: 0,
        // whatever the parameters of an unused row hold), as fp16, and the value offsets'
        // term; then O^T += (1024 + m code)^T (s P)^T and the offset 1024 sum_t (s P)^T
        const float2* vp2 = reinterpret_cast<const float2*>(stg + Cfg::kQ4ParV);
        float ls[2] = {0.f, 0.f}, vs[2] = {0.f, 0.f};
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          float sp[4];
#pragma unroll
          for (int r = 0; r < 2; ++r) {
            const float2 par = vp2[16 * t + qr + 8 * r];   // (s, lo) of the token
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const float pe = fast_exp2(p[t][2 * r + h] - m_use[h]);
              ls[h] += pe;
              sp[2 * r + h] = ok[t][r] ? pe * par.x : 0.f;
              vs[h] = ok[t][r] ? fmaf(pe, par.y, vs[h]) : vs[h];
            }
          }
          const uint32_t pb0 = movmatrix_trans(pack_f16x2(sp[0], sp[1]));   // tokens 0..7 of the tile
          const uint32_t pb1 = movmatrix_trans(pack_f16x2(sp[2], sp[3]));   // tokens 8..15
          uint32_t vw[D / 16];
          const uint8_t* vch = stg + Cfg::kQ4Bytes + (t * 32 + lane) * (D / 4);
#pragma unroll
          for (int x = 0; x < D / 16; x += 4) {
            const uint4 v = *reinterpret_cast<const uint4*>(vch + 4 * x);
            vw[x] = v.x, vw[x + 1] = v.y, vw[x + 2] = v.z, vw[x + 3] = v.w;
          }
#pragma unroll
          for (int mt = 0; mt < D / 16; ++mt) {
            const uint32_t w8 = vw[mt] >> 8;
            const uint32_t a[4] = {q4h_lo(vw[mt]), q4h_hi(vw[mt]), q4h_lo(w8), q4h_hi(w8)};
            mma_f16_16816(acc[mt], a, pb0, pb1);
          }
          mma_f16_16816(voff, kA1024, pb0, pb1);
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          l_run[h] = l_run[h] * corr[h] + ls[h];
          vl_run[h] = vl_run[h] * corr[h] + vs[h];
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty_bar[st]);   // every read of this stage is done
      }
      // ---- end of a segment: this warp's partial (empty if it took none of its pages)
      if (md.w & kSegEnd) {
        const int u = md.x;
        const bool slots_ok = vr >= 0 && vr < Re;   // slot vr + u < Re + units
        float lh[2] = {l_run[0], l_run[1]};
        float vh[2] = {vl_run[0], vl_run[1]};
#pragma unroll
        for (int o = 4; o < 32; o <<= 1) {
          lh[0] += __shfl_xor_sync(0xffffffffu, lh[0], o);
          lh[1] += __shfl_xor_sync(0xffffffffu, lh[1], o);
          vh[0] += __shfl_xor_sync(0xffffffffu, vh[0], o);
          vh[1] += __shfl_xor_sync(0xffffffffu, vh[1], o);
        }
        // an operand past the fp16 range (|s q| or |s p| > 65504) leaves a non-finite value
        // in the sums or the accumulators (masked tokens never contribute): reported here,
        // once per segment, not silent
        {
          float probe = (lh[0] + lh[1]) + (vh[0] + vh[1]) + (voff[0] + voff[1]);
#pragma unroll
          for (int mt = 0; mt < D / 16; ++mt) probe += (acc[mt][0] + acc[mt][1]) + (acc[mt][2] + acc[mt][3]);
          if (!(fabsf(probe) <= 3.0e38f)) report(LSERVE_ERR_DEVICE_BOUNDS);
        }
        const long pbase = (static_cast<long>(vr + u) * kDecodeWarps + warp) * G;
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
          const int h = tc + h2;
          if (h < G && slots_ok) {
            const bool has = m_run[h2] != kNegInf && lh[h2] > 0.f;
            const float inv = has ? 1.f / lh[h2] : 0.f;
            float* po = part_o + (pbase + h) * D + qr;
#pragma unroll
            for (int mt = 0; mt < D / 16; ++mt) {
              po[mt * 16] = (acc[mt][h2] - voff[h2] + vh[h2]) * inv;
              po[mt * 16 + 8] = fmaf(acc[mt][2 + h2] - voff[2 + h2], 0.0625f, vh[h2]) * inv;
            }
            if (qr == 0) part_lse[pbase + h] = has ? m_run[h2] + __log2f(lh[h2]) : kNegInf;
          }
        }
        if (!slots_ok && lane == 0) report(LSERVE_ERR_DEVICE_BOUNDS);
      }
    }
  } else {
    // ---- consumers.  Transposed tiles: S^T = K Q^T (M = the warp's 16 tokens,
    // N = 8 query heads, K = channels) and O^T += V^T P^T (M = channels, N =
    // heads, K = tokens), so the G <= 8 heads fill N exactly.  A lane holds
    // heads tc, tc + 1 of the tile.
    constexpr int KS = D / 16;
    uint32_t qb[KS][2];                   // Q^T as the B operand (heads >= G are zero)
    float acc[D / 16][4];                 // O^T: m-tile mt = channels 16 mt .. 16 mt + 15
    float m_run[2], l_run[2];             // online softmax of heads tc, tc + 1
    const int mi = lane >> 3, rr = lane & 7;
    const int qr = lane >> 2, tc = 2 * (lane & 3);
    for (int gp = 0;; ++gp) {
      bool have = false;
      if (lane == 0) {
        const bool known = spin_until([&] { return *v_resolved > gp || *v_total <= gp || *v_abort; }, timeout_ns);
        if (!known) *v_abort = 1;
        have = known && *v_resolved > gp && !*v_abort;
      }
      if (!__shfl_sync(0xffffffffu, have, 0)) break;
      const int st = gp % NS;
      const bool landed = mbar_wait_bounded(&full_bar[st], (gp / NS) & 1, timeout_ns);
      if (__any_sync(0xffffffffu, !landed || *v_abort != 0)) {
        if (lane == 0) *v_abort = 1;
        break;
      }
      const int4 md = s_meta[gp % kMetaRing];
      const int vr = s_range[gp % kMetaRing];
      const int u = md.x, pidx = md.y;
      const bool page_ok = md.z >= 0, streaming = md.w & kSegStreaming;
      const int L = md.w >> 3;
      const uint8_t* stg = smem + st * stage_bytes;
      const uint8_t* ks_base = stg;
      const uint8_t* vs_base = stg + Cfg::kKVBytes;
      if (md.w & kSegStart) {
        const uint8_t* qs = stg + 2 * Cfg::kKVBytes;   // [G][D] bf16, row-major
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {   // lane: head qr, channels 16 ks + tc, +1 and + 8, + 9
          const int c0 = ks * 16 + tc;
          qb[ks][0] = qr < G ? *reinterpret_cast<const uint32_t*>(qs + (qr * D + c0) * 2) : 0u;
          qb[ks][1] = qr < G ? *reinterpret_cast<const uint32_t*>(qs + (qr * D + c0 + 8) * 2) : 0u;
        }
#pragma unroll
        for (int mt = 0; mt < D / 16; ++mt) acc[mt][0] = acc[mt][1] = acc[mt][2] = acc[mt][3] = 0.f;
        m_run[0] = m_run[1] = kNegInf;
        l_run[0] = l_run[1] = 0.f;
      }
      const int t_warp = pidx * kPage + warp * 16;   // first token of this warp's slice

      // ---- S^T = K Q^T (16 tokens x 8 heads) into two accumulators (alternate k-steps)
      float sa[4] = {0.f, 0.f, 0.f, 0.f}, sb[4] = {0.f, 0.f, 0.f, 0.f};
      uint32_t vf[D / 16][4];             // V^T fragments
      {
        // ---- this warp's K and V fragments into registers, then the stage goes back
        // to the producer at once: the ring spends its time loading, not waiting for math
        uint32_t kf[KS][4];
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {   // K as the A operand of S^T: rows = tokens, k = channels
          const int box = ks >> 2, chunk = (ks & 3) * 2 + (lane >> 4);
          const int row = warp * 16 + (mi & 1) * 8 + rr;
          ldmatrix_x4(smem_u32(ks_base + box * Cfg::kBoxBytes + swz128(row, chunk)), kf[ks][0], kf[ks][1],
                      kf[ks][2], kf[ks][3]);
        }
#pragma unroll
        for (int mt = 0; mt < D / 16; ++mt) {   // V^T as the A operand of O^T: rows = channels, k = tokens
          const int ch = mt * 16 + (mi & 1) * 8;   // channels of this lane's 8x8 source block
          const int row = warp * 16 + (mi >> 1) * 8 + rr;
          ldmatrix_x4_trans(smem_u32(vs_base + (ch >> 6) * Cfg::kBoxBytes + swz128(row, (ch & 63) >> 3)),
                            vf[mt][0], vf[mt][1], vf[mt][2], vf[mt][3]);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty_bar[st]);   // release orders the shared-memory reads above
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
          if (ks & 1)
            mma_bf16_16816(sb, kf[ks], qb[ks][0], qb[ks][1]);
          else
            mma_bf16_16816(sa, kf[ks], qb[ks][0], qb[ks][1]);
        }
      }
      // ---- mask + online softmax.  Element e: token t_warp + qr + 8 (e >> 1), head tc + (e & 1)
      auto valid = [&](int t) -> bool {
        return page_ok && t < L && (!streaming || t < sink || t >= L - local);
      };
      const bool ok0 = valid(t_warp + qr), ok1 = valid(t_warp + qr + 8);
      float p[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) p[e] = ((e >> 1) ? ok1 : ok0) ? (sa[e] + sb[e]) * scale_log2 : kNegInf;
      // per-head max over the 16 tokens: the lanes with one lane % 4 hold one head pair
      float mh[2] = {fmaxf(p[0], p[2]), fmaxf(p[1], p[3])};
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) {
        mh[0] = fmaxf(mh[0], __shfl_xor_sync(0xffffffffu, mh[0], o));
        mh[1] = fmaxf(mh[1], __shfl_xor_sync(0xffffffffu, mh[1], o));
      }
      float corr[2], m_use[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const float m_new = fmaxf(m_run[h], mh[h]);
        m_use[h] = m_new == kNegInf ? 0.f : m_new;
        corr[h] = fast_exp2(m_run[h] - m_use[h]);
        m_run[h] = m_new;
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) p[e] = fast_exp2(p[e] - m_use[e & 1]);
      l_run[0] = l_run[0] * corr[0] + p[0] + p[2];   // lane-partial sums; reduced at the segment's end
      l_run[1] = l_run[1] * corr[1] + p[1] + p[3];
      if (__any_sync(0xffffffffu, corr[0] != 1.f || corr[1] != 1.f)) {
#pragma unroll
        for (int mt = 0; mt < D / 16; ++mt) {
          acc[mt][0] *= corr[0];
          acc[mt][1] *= corr[1];
          acc[mt][2] *= corr[0];
          acc[mt][3] *= corr[1];
        }
      }
      // ---- P^T as the B operand (k = tokens, n = heads): transpose the two 8x8 blocks
      const uint32_t pb0 = movmatrix_trans(pack_bf16x2(p[0], p[1]));   // tokens 0..7
      const uint32_t pb1 = movmatrix_trans(pack_bf16x2(p[2], p[3]));   // tokens 8..15
      // ---- O^T += V^T P^T.  V^T fragments hold tokens tc, tc + 1 (a0, a1) and tc + 8, + 9
      // (a2, a3) of the slice; rows of masked tokens are zeroed (the pool may hold NaN there)
      uint32_t vm0 = 0xffffffffu, vm1 = 0xffffffffu;
      if (!__all_sync(0xffffffffu, ok0 && ok1)) {
        const int t0 = t_warp + tc;
        vm0 = (valid(t0) ? 0x0000ffffu : 0u) | (valid(t0 + 1) ? 0xffff0000u : 0u);
        vm1 = (valid(t0 + 8) ? 0x0000ffffu : 0u) | (valid(t0 + 9) ? 0xffff0000u : 0u);
      }
#pragma unroll
      for (int mt = 0; mt < D / 16; ++mt) {
        vf[mt][0] &= vm0;
        vf[mt][1] &= vm0;
        vf[mt][2] &= vm1;
        vf[mt][3] &= vm1;
        mma_bf16_16816(acc[mt], vf[mt], pb0, pb1);
      }

      // ---- end of a segment: this warp's partial, and the merge if it completes the unit
      if (md.w & kSegEnd) {
        const bool slots_ok = vr >= 0 && vr < Re;   // slot vr + u < Re + units
        // (slot vr + u of every range of the unit is read by decode_merge_kernel)
        // l of heads tc, tc + 1: sum over the 8 lanes that share lane % 4
        float lh[2] = {l_run[0], l_run[1]};
#pragma unroll
        for (int o = 4; o < 32; o <<= 1) {
          lh[0] += __shfl_xor_sync(0xffffffffu, lh[0], o);
          lh[1] += __shfl_xor_sync(0xffffffffu, lh[1], o);
        }
        const long pbase = (static_cast<long>(vr + u) * kDecodeWarps + warp) * G;   // this warp's partial
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
          const int h = tc + h2;
          if (h < G && slots_ok) {
            const bool has = m_run[h2] != kNegInf && lh[h2] > 0.f;
            const float inv = has ? 1.f / lh[h2] : 0.f;
            float* po = part_o + (pbase + h) * D + qr;
#pragma unroll
            for (int mt = 0; mt < D / 16; ++mt) {
              po[mt * 16] = acc[mt][h2] * inv;
              po[mt * 16 + 8] = acc[mt][2 + h2] * inv;
            }
            if (qr == 0) part_lse[pbase + h] = has ? m_run[h2] + __log2f(lh[h2]) : kNegInf;
          }
        }
        if (!slots_ok && lane == 0) report(LSERVE_ERR_DEVICE_BOUNDS);
      }
    }
  }
  __syncthreads();
  if (*v_abort && warp == kIssuerWarp && lane == 0) {
    // let every load this CTA issued land before the CTA (and its smem) goes away;
    // the last NS issued pages sit in distinct stages, earlier ones have landed
    const int issued = *v_issued;
    for (int gp = max(0, issued - NS); gp < issued; ++gp)
      mbar_wait_bounded(&full_bar[gp % NS], (gp / NS) & 1, kDrainTimeoutNs);
  }
}

// One CTA per unit, after the attention grid: out = sum_i 2^(lse_i - lse) o_i,
// lse = log2 sum_i 2^lse_i over the unit's per-warp partials (slots c_first(u)
// + u .. c_last(u) + u, 4 warp partials each).  The threads split into groups
// over the partials; a thread keeps a running (max, sum, vector) of one float4
// of the output over its group's partials -- a single pass whose loads do not
// depend on one another -- and the groups are combined through shared memory.
constexpr int kMergeThreads = 1024;

__global__ void __launch_bounds__(kMergeThreads) decode_merge_kernel(const int32_t* off, int units, int R, int G, int D,
                                                                     const float* part_o, const float* part_lse,
                                                                     bf16* __restrict__ out,
                                                                     float* __restrict__ lse_out) {
  __shared__ float4 s_o[kMergeThreads];
  __shared__ float2 s_ml[kMergeThreads];
  // the plan and the partials come from the previous grids: read after the
  // wait, with L2 loads
  pdl_wait();
  const int u = blockIdx.x;
  const long long T = __ldcg(off + units);
  const long long a = __ldcg(off + u), e = __ldcg(off + u + 1);
  if (T <= 0 || e <= a) return;   // nothing selected: written by the partition block
  const long long Re = ranges_in_use(R, T);
  const int c_first = flat_owner(a, T, Re), c_last = flat_owner(e - 1, T, Re);
  if (c_first < 0 || c_last < c_first || c_last >= Re) {
    if (threadIdx.x == 0) report(LSERVE_ERR_DEVICE_BOUNDS);
    return;
  }
  const long first = static_cast<long>(c_first + u) * kDecodeWarps;   // first partial of the unit
  const int nparts = (c_last - c_first + 1) * kDecodeWarps;
  const int tid = threadIdx.x;
  const int n4 = G * D / 4;   // float4s of the unit's output (<= 256)
  const int groups = kMergeThreads / n4;
  const int pg = tid / n4, q4 = tid % n4, h = q4 * 4 / D;
  float m = kNegInf, l = 0.f;
  float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
  if (pg < groups) {
    const float4* po = reinterpret_cast<const float4*>(part_o) + first * n4 + q4;
    // eight partials per thread in flight at once: one L2 round trip for a unit
    // of up to 8 * groups partials
    for (int x0 = pg; x0 < nparts; x0 += 8 * groups) {
      float lx[8];
      float4 v[8];
#pragma unroll
      for (int s = 0; s < 8; ++s) {
        const int x = x0 + s * groups;
        lx[s] = kNegInf;
        if (x < nparts) {
          lx[s] = __ldcg(part_lse + (first + x) * G + h);
          v[s] = __ldcg(po + static_cast<long>(x) * n4);
        }
      }
#pragma unroll
      for (int s = 0; s < 8; ++s) {
        if (lx[s] == kNegInf) continue;   // no partial, or an empty one (its o is 0)
        const float mn = fmaxf(m, lx[s]);
        const float sc = fast_exp2(m - mn), w = fast_exp2(lx[s] - mn);
        m = mn;
        l = l * sc + w;
        o.x = o.x * sc + w * v[s].x;
        o.y = o.y * sc + w * v[s].y;
        o.z = o.z * sc + w * v[s].z;
        o.w = o.w * sc + w * v[s].w;
      }
    }
  }
  s_o[tid] = o;
  s_ml[tid] = make_float2(m, l);
  __syncthreads();
  if (tid < n4) {
    float mm = kNegInf;
    for (int gg = 0; gg < groups; ++gg) mm = fmaxf(mm, s_ml[gg * n4 + tid].x);
    float ll = 0.f;
    float4 oo = make_float4(0.f, 0.f, 0.f, 0.f);
    if (mm != kNegInf)
      for (int gg = 0; gg < groups; ++gg) {
        const float2 ml = s_ml[gg * n4 + tid];
        if (ml.x == kNegInf) continue;
        const float sc = fast_exp2(ml.x - mm);
        const float4 v = s_o[gg * n4 + tid];
        ll += ml.y * sc;
        oo.x += v.x * sc;
        oo.y += v.y * sc;
        oo.z += v.z * sc;
        oo.w += v.w * sc;
      }
    const bool has = mm != kNegInf && ll > 0.f;
    const float inv = has ? 1.f / ll : 0.f;
    const int c = tid * 4 % D;
    const long bh = static_cast<long>(u) * G + h;
    __nv_bfloat162* dst = reinterpret_cast<__nv_bfloat162*>(out + bh * D + c);
    dst[0] = __floats2bfloat162_rn(oo.x * inv, oo.y * inv);
    dst[1] = __floats2bfloat162_rn(oo.z * inv, oo.w * inv);
    if (lse_out && c == 0) lse_out[bh] = has ? (mm + __log2f(ll)) * 0.6931471805599453f : kNegInf;
  }
}

}  // namespace lserve
