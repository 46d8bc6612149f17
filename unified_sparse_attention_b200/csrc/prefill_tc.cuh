// prefill_tc.cuh -- block-sparse causal prefill attention on tcgen05 / TMEM.
//
// LServe + SampleAttention blog post, "LServe - Prefill Phase", Fig. 1: the KV
// loop of a flash-attention kernel walks only the kept 64x64 tiles (dense
// heads: causal tiles, optionally block-masked; streaming heads: tiles meeting
// the Lambda support of sink + local window); elements of kept boundary tiles
// are masked exactly.
//
// Work item: one M-tile of 128 query rows = two 64-row blocks that share one KV
// tile list.  With grouped-query attention the blocks are two query heads of
// the same KV head and query tile (G = 4: two items per tile row); with G = 1
// they are two adjacent query tiles of one head walking the union of their
// tile lists.
//
// Persistent CTAs, one per SM: the producer warp claims items from a global
// counter (in the device-built order: grouped by KV head, longest rows first)
// and hands each to the other roles through a two-slot ring in shared memory.
// Barrier phases (K/V rings, S/P/O handshakes) run on across items, so the next
// item's Q and K/V loads and its first S MMAs overlap this item's last steps and
// epilogue; q_empty frees the Q buffer once an item's last S MMA completed, and
// o_free lets the next item's first P.V overwrite the O accumulators once both
// softmax warpgroups have read them.
//
// Warp roles (384 threads, one CTA per SM; the third warpgroup hands registers
// to the two softmax warpgroups with setmaxnreg):
//   warp 8     TMA producer (one elected lane issues): Q once, then K and V of
//              every listed tile pair into shared-memory rings (128-byte
//              swizzle); K stages are released after the S MMAs, V stages after
//              the PV MMAs.
//   warp 9     allocates TMEM; runs the MMA loop converged, one elected lane
//              issues tcgen05.mma and tcgen05.commit:
//                S[x]  = Q [K_a;K_b]^T      (M=128, N=128, K=d; A and B from smem)
//                O[x] += P[x] [V_a;V_b]     (M=128, N=d, K=128; P from TMEM)
//              for step p on stream x = p & 1, in the order S(0) S(1) PV(0) S(2)
//              PV(1) S(3) ...
//   warps 0-7  two softmax warpgroups, one per stream (thread = query row): the
//              steps of a row are split between two independent online
//              softmaxes (own reference, sum and accumulator), which run out of
//              phase and keep both the exponential unit and the tensor core busy;
//              tcgen05.ld of S, exact element mask, base-2 exponentials in one
//              pass against a reference that moves only when the row sum shows
//              that it must: the first step of a stream takes the exact row max
//              (its largest weight is then exactly 1 in bf16); a row sum above
//              2^40 redoes a step against the exact row max; one above 2^12
//              moves the reference to the largest weight at the stream's next
//              step.  P is packed to bf16 over S with tcgen05.st.  The epilogue
//              merges the two streams by log-sum-exp; each warpgroup normalises
//              and stores half of the output columns.
// TMEM (512 columns): O[0] at 0, O[1] at 128, S[0] at 256, S[1] at 384; P[x]
// (bf16 pairs) is aliased over the first 64 columns of S[x].
#pragma once

#include "common.cuh"
#include "tile_lists.cuh"    // tile_keep, tile_is_full, row_runs

namespace lserve {
namespace tc {

// Arguments shared by every work item of one prefill launch.
struct PrefillArgs {
  const int32_t* row_offsets;   // CSR of the block-masked rows (closed-form rows have none)
  const uint16_t* cols;
  const int32_t* order;         // work order: row of each position
  const uint8_t* head_kind;
  bf16* out;                    // null: only the LSE is written (the CRA passes)
  float* lse;                   // nullable
  int G, Hkv, nQT, S, sink, local;
  float scale_log2;             // softmax scale times log2(e)
  unsigned long long timeout_ns;
  int lambda_tiles;             // streaming heads keep whole tiles (no element mask at the Lambda edges)
};

// ----------------------------------------------------------- tcgen05 wrappers
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void fence_before_sync() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void fence_after_sync() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void commit(uint64_t* bar) {   // call from a converged warp
  asm volatile(
      "{\n .reg .pred e;\n elect.sync _|e, 0xffffffff;\n"
      " @e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n}\n" ::"r"(
          smem_u32(bar))
      : "memory");
}
// The issuing warp runs converged with warp-uniform operands; one lane chosen
// by elect.sync issues the instructions.
// Four MMAs from one elected lane: the first takes `accumulate`, the others
// accumulate.  D[tmem] (+)= A[smem] * B[smem]  /  D[tmem] (+)= A[tmem] * B[smem]
__device__ __forceinline__ void mma_ss4(uint32_t d_tmem, uint64_t a0, uint64_t a1, uint64_t a2, uint64_t a3,
                                        uint64_t b0, uint64_t b1, uint64_t b2, uint64_t b3, uint32_t idesc,
                                        uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p, e, t;\n elect.sync _|e, 0xffffffff;\n setp.ne.b32 p, %9, 0;\n setp.eq.b32 t, %9, %9;\n"
      " @e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %5, %10, p;\n"
      " @e tcgen05.mma.cta_group::1.kind::f16 [%0], %2, %6, %10, t;\n"
      " @e tcgen05.mma.cta_group::1.kind::f16 [%0], %3, %7, %10, t;\n"
      " @e tcgen05.mma.cta_group::1.kind::f16 [%0], %4, %8, %10, t;\n}\n" ::"r"(d_tmem),
      "l"(a0), "l"(a1), "l"(a2), "l"(a3), "l"(b0), "l"(b1), "l"(b2), "l"(b3), "r"(accumulate), "r"(idesc)
      : "memory");
}
__device__ __forceinline__ void mma_ts4(uint32_t d_tmem, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                        uint64_t b0, uint64_t b1, uint64_t b2, uint64_t b3, uint32_t idesc,
                                        uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p, e, t;\n elect.sync _|e, 0xffffffff;\n setp.ne.b32 p, %9, 0;\n setp.eq.b32 t, %9, %9;\n"
      " @e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %5, %10, p;\n"
      " @e tcgen05.mma.cta_group::1.kind::f16 [%0], [%2], %6, %10, t;\n"
      " @e tcgen05.mma.cta_group::1.kind::f16 [%0], [%3], %7, %10, t;\n"
      " @e tcgen05.mma.cta_group::1.kind::f16 [%0], [%4], %8, %10, t;\n}\n" ::"r"(d_tmem),
      "r"(a0), "r"(a1), "r"(a2), "r"(a3), "l"(b0), "l"(b1), "l"(b2), "l"(b3), "r"(accumulate), "r"(idesc)
      : "memory");
}
__device__ __forceinline__ bool elect_one() {
  uint32_t e;
  asm volatile("{\n .reg .pred e;\n elect.sync _|e, 0xffffffff;\n selp.b32 %0, 1, 0, e;\n}\n" : "=r"(e));
  return e != 0;
}
// 32 consecutive 32-bit TMEM columns of this thread's lane
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]),
        "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]),
        "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
// 16 consecutive 32-bit TMEM columns of this thread's lane
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
      "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
      "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Shared-memory matrix descriptor, 128-byte swizzle (sm100 layout, version 1).
// lbo/sbo in bytes: K-major operands use sbo = 1024 (8-row groups) and an
// unused lbo; MN-major operands use lbo = distance between 64-element chunks
// along MN and sbo = 1024 (8-row groups along K).
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
  d |= static_cast<uint64_t>(1) << 46;   // descriptor version for sm100
  d |= static_cast<uint64_t>(2) << 61;   // SWIZZLE_128B
  return d;
}

// Instruction descriptor, kind::f16: bf16 A and B, fp32 D, A K-major.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(b_mn_major) << 16) |
         (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

// Bounded wait that also gives up at once when another thread already did.
__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, volatile int* abort,
                                              unsigned long long timeout_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  if (*abort) return false;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    for (int i = 0; i < 32; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (*abort) return false;
    if (globaltimer_ns() - t0 > timeout_ns) {
      report(LSERVE_ERR_DEVICE_TIMEOUT);
      *abort = 1;
      return false;
    }
  }
}

// 64-bit key masks over one tile (bit c <-> key offset c).
__device__ __forceinline__ uint64_t bits_upto(int d) {   // offsets 0..d
  return d < 0 ? 0ull : (d >= 63 ? ~0ull : (2ull << d) - 1ull);
}
__device__ __forceinline__ uint64_t bits_below(int h) {  // offsets 0..h-1
  return h <= 0 ? 0ull : (h >= 64 ? ~0ull : (1ull << h) - 1ull);
}
__device__ __forceinline__ uint64_t bits_from(int l) {   // offsets l..63
  return l <= 0 ? ~0ull : (l >= 64 ? 0ull : ~((1ull << l) - 1ull));
}

// A pipeline step covers two consecutive entries of the row's tile list (any two
// kept 64-key tiles; an odd tail repeats the last tile and masks the copy), so
// that S is a 128 x 128 tile and every barrier round trip and tcgen05.commit of
// the single issuing thread is amortised over 128 keys.
constexpr int kKStages = 3;   // K ring (tile pairs): freed once the S MMAs that read it complete
constexpr int kVStages = 2;   // V ring (tile pairs): freed once the PV MMAs that read it complete
constexpr int kItemReaders = 9;   // warps that read a claimed item index: the MMA warp and 8 softmax warps

template <int D>
struct Cfg {
  static constexpr int kBoxes = D / 64;
  static constexpr int kQTile = kBoxes * 16384;     // Q: [boxes][128 rows][128 B]
  static constexpr int kPair = kBoxes * 16384;      // one K (or V) tile pair: [boxes][128 keys][128 B]
  // at least ~half of the SM's shared memory, so that only one CTA (and one 512-column
  // TMEM allocation) is resident per SM
  static constexpr int kSmemUsed = kQTile + (kKStages + kVStages) * kPair + 1024;
  static constexpr int kSmem = kSmemUsed > 120 * 1024 ? kSmemUsed : 120 * 1024;
  // warps 0-7: two softmax warpgroups; warp 8: TMA producer; warp 9: MMA issue;
  // warps 10-11 complete the third warpgroup so that it can hand registers to
  // the softmax warpgroups (setmaxnreg acts on whole warpgroups)
  static constexpr int kThreads = 384;
  static constexpr int kWarpProducer = 8, kWarpMma = 9;
  // registers per thread after the split: the launch gives every thread the
  // kernel's count (168 at 384 threads, one CTA per SM); 128 x kRegsAux +
  // 256 x kRegsSoftmax must not exceed 384 x that count
  static constexpr int kRegsAux = 88, kRegsSoftmax = 200;
  static constexpr int kRegsNeeded = (128 * kRegsAux + 256 * kRegsSoftmax + kThreads - 1) / kThreads;
  // TMEM: O[x] (fp32, D columns) at 128 x; S[x] (fp32, 128 columns) at 256 + 128 x,
  // with P[x] (bf16 pairs, 64 columns) aliased over the first half of S[x]
  static constexpr int kColO = 0;
  static constexpr int kColS = 256;
  static constexpr int kTmemCols = 512;
};

struct TcArgs {
  PrefillArgs p;
  const uint8_t* block_mask;   // [B, Hkv, nQT, nQT] or null
  int QG;                      // query tiles per work item (1, or 2 for G = 1)
  int HG;                      // query heads per work item
  int nRow;                    // work rows per (b, kvh) = ceil(nQT / QG)
  int hsplit;                  // work items per row = G / HG
  int n_items;                 // work items in all = rows x hsplit
  int* work_counter;           // next unclaimed work item; zero at launch
  int debug_stall;             // failure-detection test hook: the producer hands out no item
};

// Wait for the loads and MMAs still in flight when a CTA gives up: fixed,
// independent of the (possibly very short) limit of the ordinary waits, so that
// nothing lands in shared memory or TMEM after the CTA has released them.
constexpr unsigned long long kPrefillDrainNs = 1000000000ull;

// One work item (128 query rows sharing a KV tile list), decoded from its index.
struct Item {
  int n, np;      // kept tiles; pipeline steps (tile pairs)
  int g, b, bg;   // KV head, sequence, b * Hkv + g
  int qgi, h0, tok0, QG, HG;
  bool streaming;
  const uint16_t* cols;   // CSR list, or null: the closed-form runs [0, ra), [rw, rw + n - ra)
  int ra, rw;
  __device__ int rb_head(int rb) const { return h0 + rb % HG; }
  __device__ int rb_qt(int rb) const { return qgi * QG + rb / HG; }
  // list entry of half h of step p (the odd tail repeats the last entry)
  __device__ int pair_tile(int p, int h) const {
    const int j = min(2 * p + h, n - 1);
    return cols ? cols[j] : (j < ra ? j : rw + (j - ra));
  }
};

__device__ __forceinline__ Item item_at(const TcArgs& T, int w) {
  const PrefillArgs& A = T.p;
  Item it;
  const int r = A.order[w / T.hsplit];
  const int hs = w % T.hsplit;
  it.qgi = r % T.nRow;
  it.bg = r / T.nRow;
  it.g = it.bg % A.Hkv;
  it.b = it.bg / A.Hkv;
  it.h0 = it.g * A.G + hs * T.HG;
  it.QG = T.QG;
  it.HG = T.HG;
  it.streaming = A.head_kind[it.g] != LSERVE_HEAD_DENSE;
  // the same rows as the list builder's closed-form ones (no CSR entries)
  TileListParams P{0, A.Hkv, A.nQT, A.sink, A.local, A.head_kind, T.block_mask, T.QG, T.nRow, 1};
  RowRuns rr;
  if (row_runs(P, r, &rr)) {
    it.n = rr.n;
    it.cols = nullptr;
    it.ra = rr.a;
    it.rw = rr.w;
  } else {
    const int beg = A.row_offsets[r];
    it.n = A.row_offsets[r + 1] - beg;
    it.cols = A.cols + beg;
    it.ra = it.rw = 0;
  }
  it.np = (it.n + 1) >> 1;
  it.tok0 = it.b * A.S;
  return it;
}

template <int D>
__global__ void __launch_bounds__(Cfg<D>::kThreads, 1)
    prefill_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, TcArgs T) {
  using C = Cfg<D>;
  const PrefillArgs& A = T.p;
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t q_full;
  __shared__ __align__(8) uint64_t k_full[kKStages], k_empty[kKStages], v_full[kVStages], v_empty[kVStages];
  __shared__ __align__(8) uint64_t s_full[2], p_full[2], o_done[2];
  // persistent CTA: the producer claims work items and passes them on through a
  // two-slot ring; q_empty frees the Q buffer (all S MMAs of an item done), o_free
  // frees the O accumulators (both warpgroups have read them in the epilogue)
  __shared__ __align__(8) uint64_t item_full[2], item_empty[2], q_empty, o_free, mma_drain;
  // ml_full[ii & 1]: both softmax warpgroups have published their (m, l) of item ii
  // (a bounded wait, unlike a named barrier, so that no protocol slip can hang a CTA)
  __shared__ __align__(8) uint64_t ml_full[2];
  __shared__ int s_item[2];
  __shared__ uint32_t s_tmem;
  __shared__ volatile int s_abort;
  __shared__ float s_ml[2][2][2][128];   // [item parity][warpgroup][m, l][row]: epilogue merge
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* q_s = smem;
  uint8_t* k_s = q_s + C::kQTile;
  uint8_t* v_s = k_s + kKStages * C::kPair;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int Hq = A.Hkv * A.G;
  // item index of ring slot `slot` (written before item_full completes)
  auto claimed = [&](int slot) { return *reinterpret_cast<volatile int*>(&s_item[slot]); };

  if (tid == 0) {
    mbar_init(&q_full, 1);
    for (int s = 0; s < kKStages; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
    }
    for (int s = 0; s < kVStages; ++s) {
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&s_full[x], 1);
      mbar_init(&p_full[x], 128);
      mbar_init(&o_done[x], 1);
      mbar_init(&item_full[x], 1);
      mbar_init(&item_empty[x], kItemReaders);
      mbar_init(&ml_full[x], 256);
    }
    mbar_init(&q_empty, 1);
    mbar_init(&o_free, 256);
    mbar_init(&mma_drain, 1);
    s_abort = 0;
    fence_barrier_init();
  }
  if (warp == C::kWarpMma) {
    tmem_alloc(&s_tmem, C::kTmemCols);
    tmem_relinquish();
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tmem = s_tmem;
  const unsigned long long tmo = A.timeout_ns;

  // Each warpgroup changes its register count at the top of its own branch
  // (code after a merge of the two would be held to the smaller count).
  if (warp >= C::kWarpProducer) {   // the third warpgroup gives registers to the softmax
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(C::kRegsAux));
   if (warp == C::kWarpProducer) {
    // ================================================================ producer
    // The whole warp walks the lists (warp-uniform coordinates); one elected lane
    // issues.  Work items are claimed from the global counter one at a time and
    // handed to the other roles through the item ring.  K and V stage indices and
    // phases run on across items (gk, gv: tile pairs issued so far).
    const bool leader = elect_one();
    if (leader) {
      prefetch_tensormap(&tmQ);
      prefetch_tensormap(&tmK);
      prefetch_tensormap(&tmV);
    }
    int gk = 0, gv = 0, nq = 0;   // K and V steps issued; items with tiles (Q loads)
    int kiss = 0, viss = 0;       // K and V stage loads actually issued (for the drain)
    bool live = !T.debug_stall;   // the test hook publishes nothing: every other wait runs out
    for (int ii = 0; live; ++ii) {
      const int slot = ii & 1;
      if (ii >= 2 && !wait_or_abort(&item_empty[slot], ((ii >> 1) - 1) & 1, &s_abort, tmo)) break;
      int w = 0;
      if (leader) {
        w = atomicAdd(T.work_counter, 1);
        s_item[slot] = w;
        mbar_arrive(&item_full[slot]);   // release: the index is visible to the waiters
      }
      w = __shfl_sync(0xffffffffu, w, __ffs(__ballot_sync(0xffffffffu, leader)) - 1);
      if (w >= T.n_items || s_abort) break;
      const Item it = item_at(T, w);
      const int n = it.n, np = it.np, g = it.g, tok0 = it.tok0;
      if (n == 0) continue;
      // the Q buffer is free once every S MMA of the previous item with tiles completed
      if (nq > 0 && !wait_or_abort(&q_empty, (nq - 1) & 1, &s_abort, tmo)) break;
      ++nq;
      int valid_rb = 0;
      for (int rb = 0; rb < 2; ++rb) valid_rb += it.rb_qt(rb) < A.nQT;
      if (leader) {
        mbar_arrive_expect_tx(&q_full, valid_rb * C::kBoxes * 8192);
        for (int rb = 0; rb < 2; ++rb) {
          if (it.rb_qt(rb) >= A.nQT) continue;
          for (int x = 0; x < C::kBoxes; ++x)
            tma_load_3d_hint(q_s + x * 16384 + rb * 8192, &tmQ, &q_full, x * 64, it.rb_head(rb),
                             tok0 + it.rb_qt(rb) * kTile, l2_evict_first());
        }
      }
      // K of step t+1 goes out before V of step t: S MMAs run ahead of PV MMAs
      for (int t = 0; t <= np && live; ++t) {
        if (t < np) {
          const int gt = gk + t, st = gt % kKStages;
          if (gt >= kKStages && !wait_or_abort(&k_empty[st], ((gt / kKStages) - 1) & 1, &s_abort, tmo)) {
            live = false;
            break;
          }
          const int ka = it.pair_tile(t, 0), kb = it.pair_tile(t, 1);
          kiss = gt + 1;
          if (leader) {
            mbar_arrive_expect_tx(&k_full[st], C::kPair);
            for (int x = 0; x < C::kBoxes; ++x) {
              uint8_t* dst = k_s + st * C::kPair + x * 16384;
              tma_load_3d(dst, &tmK, &k_full[st], x * 64, g, tok0 + ka * kTile);
              tma_load_3d(dst + 8192, &tmK, &k_full[st], x * 64, g, tok0 + kb * kTile);
            }
          }
        }
        if (t >= 1) {
          const int gu = gv + t - 1, st = gu % kVStages;
          if (gu >= kVStages && !wait_or_abort(&v_empty[st], ((gu / kVStages) - 1) & 1, &s_abort, tmo)) {
            live = false;
            break;
          }
          const int ka = it.pair_tile(t - 1, 0), kb = it.pair_tile(t - 1, 1);
          viss = gu + 1;
          if (leader) {
            mbar_arrive_expect_tx(&v_full[st], C::kPair);
            for (int x = 0; x < C::kBoxes; ++x) {
              uint8_t* dst = v_s + st * C::kPair + x * 16384;
              tma_load_3d(dst, &tmV, &v_full[st], x * 64, g, tok0 + ka * kTile);
              tma_load_3d(dst + 8192, &tmV, &v_full[st], x * 64, g, tok0 + kb * kTile);
            }
          }
        }
      }
      gk += np;
      gv += np;
    }
    if (s_abort) {   // let the copies still in flight land: the latest load of each stage, and Q
      for (int g0 = max(0, kiss - kKStages); g0 < kiss; ++g0)
        mbar_wait_bounded(&k_full[g0 % kKStages], (g0 / kKStages) & 1, kPrefillDrainNs);
      for (int g0 = max(0, viss - kVStages); g0 < viss; ++g0)
        mbar_wait_bounded(&v_full[g0 % kVStages], (g0 / kVStages) & 1, kPrefillDrainNs);
      if (nq > 0) mbar_wait_bounded(&q_full, (nq - 1) & 1, kPrefillDrainNs);
    }
  } else if (warp == C::kWarpMma) {
    // ================================================================== MMA
    // Step p of an item belongs to stream x = p & 1 (S[x], P[x], O[x]).  The whole
    // warp runs the loop (waits and descriptors warp-uniform); one elected lane
    // issues.  Tensor-core order within an item: S(0) S(1) PV(0) S(2) PV(1) S(3) ...
    // S(p+2) overwrites the S/P buffer that PV(p) reads; tcgen05.mma instructions
    // issued by one thread are pipelined in issue order, so S(p+2) is issued right
    // after PV(p) without waiting for its completion (checked: parity, and
    // bit-identical results over repeated runs).  The same order makes S(0), S(1)
    // of the next item safe right after the last PV of this one, so they run while
    // the softmax warpgroups finish this item's epilogue.
    constexpr uint32_t kIdS = idesc_bf16(128, 128, false);
    constexpr uint32_t kIdPV = idesc_bf16(128, D, true);
    const uint32_t qa = smem_u32(q_s), ka = smem_u32(k_s), va = smem_u32(v_s);
    int gk = 0, gv = 0, nq = 0;   // K and V steps consumed; items with tiles
    int cs[2] = {0, 0};           // steps of each stream over the previous items
    for (int ii = 0;; ++ii) {
      const int slot = ii & 1;
      if (!wait_or_abort(&item_full[slot], (ii >> 1) & 1, &s_abort, tmo)) break;
      const int w = claimed(slot);
      __syncwarp();
      if (lane == 0) mbar_arrive(&item_empty[slot]);
      if (w >= T.n_items) break;
      const Item it = item_at(T, w);
      const int np = it.np;
      if (it.n == 0) continue;
      auto issue_s = [&](int p) {   // S[p&1] = Q [K_a; K_b]^T
        const int gt = gk + p, st = gt % kKStages, x = p & 1;
        wait_or_abort(&k_full[st], (gt / kKStages) & 1, &s_abort, tmo);
        __syncwarp();   // converged for elect.sync / tcgen05
        fence_after_sync();
#pragma unroll
        for (int k4 = 0; k4 < D / 16; k4 += 4) {
          uint64_t ad[4], bd[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int ks = k4 + e;
            ad[e] = sdesc(qa + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024);
            bd[e] = sdesc(ka + st * C::kPair + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024);
          }
          mma_ss4(tmem + C::kColS + 128 * x, ad[0], ad[1], ad[2], ad[3], bd[0], bd[1], bd[2], bd[3], kIdS, k4 > 0);
        }
        commit(&s_full[x]);
        commit(&k_empty[st]);
        if (p == np - 1) commit(&q_empty);   // the item's last read of Q
      };
      wait_or_abort(&q_full, nq & 1, &s_abort, tmo);
      ++nq;
      issue_s(0);
      if (np > 1) {
        // stream 1 starts one exponential phase behind stream 0: S(1) goes out once P(0)
        // is ready, so that the two streams' exponentials alternate instead of sharing
        // the unit (the in-order issue that follows keeps them apart)
        wait_or_abort(&p_full[0], cs[0] & 1, &s_abort, tmo);
        issue_s(1);
      }
      for (int p = 0; p < np; ++p) {
        const int gu = gv + p, st = gu % kVStages, x = p & 1;
        wait_or_abort(&v_full[st], (gu / kVStages) & 1, &s_abort, tmo);
        wait_or_abort(&p_full[x], (cs[x] + (p >> 1)) & 1, &s_abort, tmo);
        // PV(0) overwrites O[0] (and PV(1) O[1]): the previous item's epilogue must
        // have read both accumulators
        if (p == 0 && ii > 0) wait_or_abort(&o_free, (ii - 1) & 1, &s_abort, tmo);
        __syncwarp();
        fence_after_sync();
#pragma unroll
        for (int k4 = 0; k4 < 8; k4 += 4) {
          uint64_t bd[4];
          uint32_t at[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            bd[e] = sdesc(va + st * C::kPair + (k4 + e) * 2048, 16384, 1024);
            at[e] = tmem + C::kColS + 128 * x + 8 * (k4 + e);
          }
          mma_ts4(tmem + C::kColO + 128 * x, at[0], at[1], at[2], at[3], bd[0], bd[1], bd[2], bd[3], kIdPV,
                  (p >= 2 || k4 > 0) ? 1u : 0u);
        }
        if (p + 2 >= np) commit(&o_done[x]);   // the stream's last P.V of the item (the epilogue waits)
        commit(&v_empty[st]);
        if (p + 2 < np) issue_s(p + 2);
      }
      gk += np;
      gv += np;
      cs[0] += (np + 1) >> 1;
      cs[1] += np >> 1;
      if (s_abort) break;
    }
    if (s_abort) {   // every MMA issued so far completes before TMEM is released
      commit(&mma_drain);
      mbar_wait_bounded(&mma_drain, 0, kPrefillDrainNs);
    }
   }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(C::kRegsSoftmax));
    // ============================================================== softmax
    // Warpgroup x runs an independent online softmax over the steps p = x, x+2, ...
    // with its own (m, l) and accumulator O[x]; the two are merged at the end.
    const int x = warp >> 2;
    const int quarter = warp & 3;           // TMEM lane quarter this warp may access
    const int row = quarter * 32 + lane;    // row within the M-tile
    const int rb = row >> 6;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t t_o = tmem + C::kColO + 128 * x + lane_off;
    const uint32_t t_s = tmem + C::kColS + 128 * x + lane_off;
    const float sc = A.scale_log2;
    TileListParams tp{0, A.Hkv, A.nQT, A.sink, A.local, nullptr, nullptr};
    int cs_own = 0;   // steps of this stream over the previous items (barrier phases)
    int n_last = 0;   // items in which this stream had steps (phases of o_done[x])
    for (int ii = 0;; ++ii) {
      const int slot = ii & 1;
      if (!wait_or_abort(&item_full[slot], (ii >> 1) & 1, &s_abort, tmo)) break;
      const int w = claimed(slot);
      __syncwarp();
      if (lane == 0) mbar_arrive(&item_empty[slot]);
      if (w >= T.n_items) break;
      const Item it = item_at(T, w);
      const int n = it.n, np = it.np, b = it.b, bg = it.bg;
      const bool streaming = it.streaming;
      const int h = it.rb_head(rb), qt = it.rb_qt(rb);
      const bool rb_valid = qt < A.nQT;
      const int i = qt * kTile + (row & 63);  // query position
      const int tok0 = it.tok0;
      const uint8_t* mrow = (!streaming && T.block_mask && rb_valid)
                                ? T.block_mask + (static_cast<long>(bg) * A.nQT + qt) * A.nQT
                                : nullptr;
      float m_run = kNegInf, l_run = 0.f;
      // keep mask of this row over one 64-key tile (bit c <-> key 64 kt + c)
      // (with tile-level Lambda a kept tile of a streaming head is masked like a dense one: causally only)
      const bool lam_edges = streaming && !A.lambda_tiles;
      auto tile_mask = [&](int kt) -> uint64_t {
        if (!rb_valid || !(T.QG == 1 || tile_keep(tp, streaming, mrow, qt, kt))) return 0ull;
        if (tile_is_full(lam_edges, qt, kt, A.sink, A.local)) return ~0ull;
        const int d0 = i - kt * kTile;   // offset of the query position inside the tile
        uint64_t k = bits_upto(d0);
        if (lam_edges) k &= bits_below(A.sink - kt * kTile) | bits_from(d0 - A.local + 1);
        return k;
      };
      // raw scores of one 64-key half, masked keys set to -inf
      auto load_half = [&](int half, uint64_t keep, uint32_t (&v)[64]) {
        tmem_ld32(t_s + 64 * half, *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
        tmem_ld32(t_s + 64 * half + 32, *reinterpret_cast<uint32_t(*)[32]>(&v[32]));
        tmem_wait_ld();
        if (!__all_sync(0xffffffffu, keep == ~0ull)) {
  #pragma unroll
          for (int c = 0; c < 64; ++c)
            if (!((keep >> c) & 1ull)) v[c] = 0xff800000u;   // -inf: exp2 gives exactly 0
        }
      };

      float rebase = 0.f;   // shift of the reference max decided at this stream's previous step
      // tile indices of this stream's next step, loaded one step ahead (hides the load latency)
      int nkt0 = 0, nkt1 = 0;
      if (x < np) {
        nkt0 = it.pair_tile(x, 0);
        nkt1 = it.pair_tile(x, 1);
      }
      for (int p = x; p < np; p += 2) {
        const int j = p >> 1;   // this stream's step index
        const int kt0 = nkt0, kt1 = nkt1;
        if (p + 2 < np) {
          nkt0 = it.pair_tile(p + 2, 0);
          nkt1 = it.pair_tile(p + 2, 1);
        }
        const uint64_t keep0 = tile_mask(kt0);
        const uint64_t keep1 = (2 * p + 1 < n) ? tile_mask(kt1) : 0ull;
        wait_or_abort(&s_full[x], (cs_own + j) & 1, &s_abort, tmo);
        __syncwarp();   // converged for the warp-collective tcgen05 loads
        fence_after_sync();
        uint32_t v[64];
        uint32_t pk0[32], pk1[32];
        float ps[4];
        // One 32-column chunk of S (already in registers): exponentials 2^(s*scale - m),
        // packed fp32 pairs for the scale/subtract and the running sums (half the
        // instructions: the softmax is issue-bound), bf16 pairs of P.
        auto exp_chunk = [&](uint32_t (&u)[32], uint64_t keep, int q, uint64_t sc2, uint64_t nm2, uint32_t* pk,
                             uint64_t (&ps2)[2]) {
          if (!__all_sync(0xffffffffu, keep == ~0ull)) {
  #pragma unroll
            for (int c = 0; c < 32; ++c)
              if (!((keep >> (32 * q + c)) & 1ull)) u[c] = 0xff800000u;   // -inf: exp2 gives 0
          }
  #pragma unroll
          for (int c = 0; c < 16; ++c) {
            float a0, a1;
            split_f32x2(fma_f32x2(f32x2(__uint_as_float(u[2 * c]), __uint_as_float(u[2 * c + 1])), sc2, nm2), a0, a1);
            const float p0 = fast_exp2(a0), p1 = fast_exp2(a1);
            ps2[c & 1] = add_f32x2(ps2[c & 1], f32x2(p0, p1));
            pk[c] = pack_bf16x2(p0, p1);
          }
        };
        auto exp_pass = [&](float m) -> float {   // returns the row sum of the exponentials
          const float m_use = m == kNegInf ? 0.f : m;
          const uint64_t sc2 = f32x2(sc, sc), nm2 = f32x2(-m_use, -m_use);
          uint64_t ps2[2] = {f32x2(0.f, 0.f), f32x2(0.f, 0.f)};
          // four 32-column chunks; the TMEM load of chunk c+1 is in flight while chunk c is processed
          uint32_t ua[32], ub[32];
          tmem_ld32(t_s, ua);
          tmem_wait_ld();
          tmem_ld32(t_s + 32, ub);
          exp_chunk(ua, keep0, 0, sc2, nm2, pk0, ps2);
          tmem_wait_ld();
          tmem_ld32(t_s + 64, ua);
          exp_chunk(ub, keep0, 1, sc2, nm2, pk0 + 16, ps2);
          tmem_wait_ld();
          tmem_ld32(t_s + 96, ub);
          exp_chunk(ua, keep1, 0, sc2, nm2, pk1, ps2);
          tmem_wait_ld();
          exp_chunk(ub, keep1, 1, sc2, nm2, pk1 + 16, ps2);
          split_f32x2(ps2[0], ps[0], ps[1]);
          split_f32x2(ps2[1], ps[2], ps[3]);
          return (ps[0] + ps[1]) + (ps[2] + ps[3]);
        };
        // O[x] and l are multiplied by f before this step's P is added
        float f = 1.f;
        if (rebase != 0.f) {
          f = fast_exp2(-rebase);
          m_run += rebase;
          rebase = 0.f;
        }
        // steady state: one pass against the current reference.  A warp with any row
        // still without a reference (the stream's first step), or whose pass shows a row
        // sum past 2^40 (a weight near the fp32/bf16 limit; inf/NaN too), takes the exact
        // row max and passes again.  Both decisions are warp votes, so the branches (which
        // hold warp-collective TMEM loads) are taken by the whole warp or not at all; one
        // copy of the pass serves both attempts.
        bool exact = !__all_sync(0xffffffffu, m_run != kNegInf);
        float rsum = 0.f;
  #pragma unroll 1
        while (true) {
          if (exact) {
            float mx[4] = {kNegInf, kNegInf, kNegInf, kNegInf};
  #pragma unroll 1
            for (int half = 0; half < 2; ++half) {
              load_half(half, half ? keep1 : keep0, v);
  #pragma unroll
              for (int c = 0; c < 64; c += 8) {
  #pragma unroll
                for (int e = 0; e < 4; ++e)
                  mx[e] = max3(mx[e], __uint_as_float(v[c + 2 * e]), __uint_as_float(v[c + 2 * e + 1]));
              }
            }
            const float mloc = max3(mx[0], mx[1], fmaxf(mx[2], mx[3])) * sc;
            const float m_new = fmaxf(m_run, mloc);
            if (m_run != kNegInf && m_new != m_run) f *= fast_exp2(m_run - m_new);
            m_run = m_new;
          }
          rsum = exp_pass(m_run);
          if (exact || !__any_sync(0xffffffffu, !(rsum <= 1099511627776.f))) break;   // 2^40
          exact = true;
        }
        // weights well above the reference (row sum beyond 2^12): move the reference to the
        // largest argument at this stream's next step (O must first absorb this step); the
        // largest weight is read back from the bf16 pairs of P
        if (m_run != kNegInf && rsum > 4096.f) {
          uint32_t mp = 0u;
  #pragma unroll
          for (int c = 0; c < 32; ++c) mp = max_bf16x2(mp, max_bf16x2(pk0[c], pk1[c]));
          const float wmax = fmaxf(bf16_lo(mp), bf16_hi(mp));
          if (wmax > 1.f) rebase = __log2f(wmax);
        }
        tmem_st32(t_s, pk0);        // P[x] over S[x] columns 0..63 (S is no longer needed)
        tmem_st32(t_s + 32, pk1);
        l_run = l_run * f + ((ps[0] + ps[1]) + (ps[2] + ps[3]));
        // O[x] holds this stream's steps < p, the latest being PV(p-2), and it is complete:
        // S(p) was issued after it, and the commit behind s_full tracks every earlier MMA of
        // the issuing thread.  PV(p) needs this step's P, so O[x] may be rescaled here.
        if (j > 0 && __any_sync(0xffffffffu, f != 1.f)) {
  #pragma unroll 1
          for (int c0 = 0; c0 < D; c0 += 32) {
            uint32_t ov[32];
            tmem_ld32(t_o + c0, ov);
            tmem_wait_ld();
  #pragma unroll
            for (int c = 0; c < 32; ++c) ov[c] = __float_as_uint(__uint_as_float(ov[c]) * f);
            tmem_st32(t_o + c0, ov);
          }
        }
        tmem_wait_st();
        fence_before_sync();
        mbar_arrive(&p_full[x]);
      }
      // a pending shift is never needed for the result: (m, l, O) stay consistent
      // ---- epilogue: merge the two streams (log-sum-exp), each warpgroup stores half of O
      const int nx = (np > x) ? (np - x + 1) >> 1 : 0;   // steps of this stream
      if (nx > 0) {   // o_done[x] completes once per item in which this stream has steps
        wait_or_abort(&o_done[x], n_last & 1, &s_abort, tmo);   // PV of its last step
        ++n_last;
        fence_after_sync();
      }
      s_ml[ii & 1][x][0][row] = m_run;
      s_ml[ii & 1][x][1][row] = l_run;
      // the other warpgroup observed its stream's last P.V before it arrived; the
      // fences order that observation before this warpgroup's reads of O[x^1].  The
      // next phase of ml_full[ii & 1] (item ii + 2) needs this thread's arrival, so
      // the parity wait is unambiguous.
      fence_before_sync();
      mbar_arrive(&ml_full[ii & 1]);
      wait_or_abort(&ml_full[ii & 1], (ii >> 1) & 1, &s_abort, tmo);
      __syncwarp();   // converged for the warp-collective tcgen05 loads below
      fence_after_sync();
      const float m_o = s_ml[ii & 1][x ^ 1][0][row], l_o = s_ml[ii & 1][x ^ 1][1][row];
      const int nx_o = (np > (x ^ 1)) ? (np - (x ^ 1) + 1) >> 1 : 0;
      const float m_all = fmaxf(m_run, m_o);
      const float m_ref = m_all == kNegInf ? 0.f : m_all;
      const float w_own = nx > 0 ? fast_exp2(m_run - m_ref) : 0.f;
      const float w_oth = nx_o > 0 ? fast_exp2(m_o - m_ref) : 0.f;
      const float l_tot = l_run * w_own + l_o * w_oth;
      if (rb_valid) {
        const int c_lo = x * (D / 2);   // this warpgroup's half of the output columns
        const bool has = n > 0 && m_all != kNegInf && l_tot > 0.f;
        const float inv = has ? 1.f / l_tot : 0.f;
        const uint32_t t_own = tmem + C::kColO + 128 * x + lane_off + c_lo;
        const uint32_t t_oth = tmem + C::kColO + 128 * (x ^ 1) + lane_off + c_lo;
        bf16* orow = A.out ? A.out + (static_cast<long>(tok0 + i) * Hq + h) * D + c_lo : nullptr;
  #pragma unroll 1
        for (int c0 = 0; orow && c0 < D / 2; c0 += 16) {   // no output: only the LSE (CRA passes)
          uint32_t oa[16], ob[16];
          if (nx > 0) tmem_ld16(t_own + c0, oa);
          if (nx_o > 0) tmem_ld16(t_oth + c0, ob);
          tmem_wait_ld();
          uint32_t pk[8];
  #pragma unroll
          for (int c = 0; c < 8; ++c) {
            float a0 = 0.f, a1 = 0.f;
            if (nx > 0) {
              a0 = __uint_as_float(oa[2 * c]) * w_own;
              a1 = __uint_as_float(oa[2 * c + 1]) * w_own;
            }
            if (nx_o > 0) {
              a0 = fmaf(__uint_as_float(ob[2 * c]), w_oth, a0);
              a1 = fmaf(__uint_as_float(ob[2 * c + 1]), w_oth, a1);
            }
            pk[c] = pack_bf16x2(a0 * inv, a1 * inv);
          }
          // Q and O are touched once per item: streaming stores (and evict-first Q
          // loads) leave L2 to the K/V tiles that other query tiles read again
          __stcs(reinterpret_cast<uint4*>(orow + c0), make_uint4(pk[0], pk[1], pk[2], pk[3]));
          __stcs(reinterpret_cast<uint4*>(orow + c0 + 8), make_uint4(pk[4], pk[5], pk[6], pk[7]));
        }
        if (A.lse && x == 0)
          A.lse[(static_cast<long>(b) * Hq + h) * A.S + i] =
              has ? (m_all + __log2f(l_tot)) * 0.6931471805599453f : kNegInf;
      }
      // both accumulators have been read: the MMA warp may let the next item's PV(0)
      // overwrite them
      fence_before_sync();
      mbar_arrive(&o_free);
      cs_own += nx;
      if (s_abort) break;
    }
  }
  fence_before_sync();
  __syncthreads();
  if (warp == C::kWarpMma) {
    fence_after_sync();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

}  // namespace tc
}  // namespace lserve
