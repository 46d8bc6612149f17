// prefill_tc.cuh -- block-sparse causal prefill attention on tcgen05 / TMEM.
//
// LServe + SampleAttention blog post, "LServe - Prefill Phase", Fig. 1: the KV
// loop of a flash-attention kernel walks only the kept 64x64 tiles (dense
// heads: causal tiles, optionally block-masked; streaming heads: tiles meeting
// the Lambda support of sink + local window); elements of kept boundary tiles
// are masked exactly.
//
// One CTA per work item: NM M-tiles of 128 query rows that share one KV tile
// list.  Each M-tile holds two 64-row blocks: with grouped-query attention the
// blocks are different query heads of the same KV head and query tile (G = 4:
// four heads, two M-tiles, every K/V tile feeds both); with G = 2 one M-tile of
// two heads; with G = 1 one M-tile of two adjacent query tiles walking the union
// of their tile lists.
//
// Warp roles (64 + 128 NM threads):
//   warp 0     TMA producer (one elected lane issues): Q once, then K and V of every listed tile into a
//              pair of 4-stage shared-memory rings (128-byte swizzle); K stages
//              are released after the S MMAs, V stages after the PV MMAs.
//   warp 1     allocates TMEM; runs the MMA loop converged, one elected lane issues tcgen05.mma:
//                S[m] = Q[m] K^T      (M=128, N=64, K=d; A and B from smem)
//                O[m] += P[m] V       (M=128, N=d, K=64; P from TMEM, V from smem)
//              and signals completion with tcgen05.commit -> mbarrier.
//   warps 2..  one warpgroup per M-tile: thread = query row.  tcgen05.ld of
//              its S row, exact element mask, base-2 online softmax with lazy
//              rescaling (O in TMEM is rescaled only when the running max grows
//              by more than 2^8), P packed to bf16 and written back over S with
//              tcgen05.st, then the epilogue normalises O and stores bf16 rows.
// TMEM columns: O[m] at m*d, S[m][buf] at NM*d + 64*(2m + buf) (double-buffered).
#pragma once

#include "common.cuh"
#include "prefill_mma.cuh"   // PrefillArgs, tile_is_full
#include "tile_lists.cuh"    // tile_keep

namespace lserve {
namespace tc {

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
// by elect.sync issues the instruction.
// D[tmem] (+)= A[smem] * B[smem]
__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p, e;\n elect.sync _|e, 0xffffffff;\n setp.ne.b32 p, %4, 0;\n"
      " @e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// D[tmem] (+)= A[tmem] * B[smem]
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p, e;\n elect.sync _|e, 0xffffffff;\n setp.ne.b32 p, %4, 0;\n"
      " @e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
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

constexpr int kKStages = 4;   // K ring: a stage is freed once the S MMAs that read it complete
constexpr int kVStages = 4;   // V ring: a stage is freed once the PV MMAs that read it complete

template <int D, int NM>
struct Cfg {
  static constexpr int kBoxes = D / 64;
  static constexpr int kQTile = kBoxes * 16384;      // one M-tile of Q: [boxes][128 rows][128 B]
  static constexpr int kKVTile = kBoxes * 8192;      // one K (or V) tile: [boxes][64 rows][128 B]
  static constexpr int kSmem = NM * kQTile + (kKStages + kVStages) * kKVTile + 1024;
  static constexpr int kThreads = 64 + 128 * NM;
  static constexpr int kTmemCols = (NM * D + NM * 128) <= 256 ? 256 : 512;
};

struct TcArgs {
  PrefillArgs p;
  const uint8_t* block_mask;   // [B, Hkv, nQT, nQT] or null
  int QG;                      // query tiles per work item (1, or 2 for G = 1)
  int HG;                      // query heads per work item
  int nRow;                    // work rows per (b, kvh) = ceil(nQT / QG)
  int hsplit;                  // work items per row = G / HG
};

template <int D, int NM>
__global__ void __launch_bounds__(Cfg<D, NM>::kThreads, 1)
    prefill_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, TcArgs T) {
  using C = Cfg<D, NM>;
  const PrefillArgs& A = T.p;
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t q_full;
  __shared__ __align__(8) uint64_t k_full[kKStages], k_empty[kKStages], v_full[kVStages], v_empty[kVStages];
  __shared__ __align__(8) uint64_t s_full[NM][2], p_full[NM][2], o_done[NM];
  __shared__ uint32_t s_tmem;
  __shared__ volatile int s_abort;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* q_s = smem;
  uint8_t* k_s = q_s + NM * C::kQTile;
  uint8_t* v_s = k_s + kKStages * C::kKVTile;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // ---- work item
  const int w = blockIdx.x;
  const int r = A.order[w / T.hsplit];
  const int hs = w % T.hsplit;
  const int qgi = r % T.nRow;
  const int bg = r / T.nRow;
  const int g = bg % A.Hkv, b = bg / A.Hkv;
  const int Hq = A.Hkv * A.G;
  const int h0 = g * A.G + hs * T.HG;
  const bool streaming = A.head_kind[g] != LSERVE_HEAD_DENSE;
  const int beg = A.row_offsets[r];
  const int n = A.row_offsets[r + 1] - beg;
  const uint16_t* cols = A.cols + beg;
  const int tok0 = b * A.S;
  auto rb_head = [&](int rb) { return h0 + rb % T.HG; };
  auto rb_qt = [&](int rb) { return qgi * T.QG + rb / T.HG; };

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
    for (int m = 0; m < NM; ++m) {
      mbar_init(&s_full[m][0], 1);
      mbar_init(&s_full[m][1], 1);
      mbar_init(&p_full[m][0], 128);
      mbar_init(&p_full[m][1], 128);
      mbar_init(&o_done[m], 1);
    }
    s_abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&s_tmem, C::kTmemCols);
    tmem_relinquish();
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tmem = s_tmem;
  const uint32_t t_o0 = tmem;                  // O[m] at column m*D
  const uint32_t t_s0 = tmem + NM * D;         // S[m][buf] at NM*D + 64*(2m+buf)
  const unsigned long long tmo = A.timeout_ns;

  if (warp == 0) {
    // ================================================================ producer
    // The whole warp walks the list (warp-uniform coordinates); one elected lane issues.
    const bool leader = elect_one();
    if (n > 0) {
      if (leader) {
        prefetch_tensormap(&tmQ);
        prefetch_tensormap(&tmK);
        prefetch_tensormap(&tmV);
      }
      int valid_rb = 0;
      for (int rb = 0; rb < 2 * NM; ++rb) valid_rb += rb_qt(rb) < A.nQT;
      if (leader) {
        mbar_arrive_expect_tx(&q_full, valid_rb * C::kBoxes * 8192);
        for (int rb = 0; rb < 2 * NM; ++rb) {
          if (rb_qt(rb) >= A.nQT) continue;
          uint8_t* dst = q_s + (rb >> 1) * C::kQTile + (rb & 1) * 8192;
          for (int x = 0; x < C::kBoxes; ++x)
            tma_load_3d(dst + x * 16384, &tmQ, &q_full, x * 64, rb_head(rb), tok0 + rb_qt(rb) * kTile);
        }
      }
      // K of tile t+1 goes out before V of tile t: S MMAs run one tile ahead of PV MMAs
      for (int t = 0; t <= n; ++t) {
        if (t < n) {
          const int st = t % kKStages;
          if (t >= kKStages && !wait_or_abort(&k_empty[st], ((t / kKStages) - 1) & 1, &s_abort, tmo)) break;
          const int kt = cols[t];
          if (leader) {
            mbar_arrive_expect_tx(&k_full[st], C::kKVTile);
            for (int x = 0; x < C::kBoxes; ++x)
              tma_load_3d(k_s + st * C::kKVTile + x * 8192, &tmK, &k_full[st], x * 64, g, tok0 + kt * kTile);
          }
        }
        if (t >= 1) {
          const int u = t - 1;
          const int st = u % kVStages;
          if (u >= kVStages && !wait_or_abort(&v_empty[st], ((u / kVStages) - 1) & 1, &s_abort, tmo)) break;
          const int kt = cols[u];
          if (leader) {
            mbar_arrive_expect_tx(&v_full[st], C::kKVTile);
            for (int x = 0; x < C::kBoxes; ++x)
              tma_load_3d(v_s + st * C::kKVTile + x * 8192, &tmV, &v_full[st], x * 64, g, tok0 + kt * kTile);
          }
        }
      }
    }
  } else if (warp == 1) {
    // ================================================================== MMA
    // The whole warp runs the loop (waits and descriptors warp-uniform); MMAs and
    // commits are issued by one elected lane.
    if (n > 0) {
      constexpr uint32_t kIdS = idesc_bf16(128, 64, false);
      constexpr uint32_t kIdPV = idesc_bf16(128, D, true);
      int o_seen[NM];
      for (int m = 0; m < NM; ++m) o_seen[m] = 0;
      auto wait_pv = [&](int m, int t) {   // PV of tile t (M-tile m) has completed
        while (o_seen[m] <= t) {
          if (!wait_or_abort(&o_done[m], o_seen[m] & 1, &s_abort, tmo)) return;
          ++o_seen[m];
        }
      };
      const uint32_t qa = smem_u32(q_s), ka = smem_u32(k_s), va = smem_u32(v_s);
      auto issue_s = [&](int j) {
        const int st = j % kKStages;
        wait_or_abort(&k_full[st], (j / kKStages) & 1, &s_abort, tmo);
        for (int m = 0; m < NM; ++m) {
          const int buf = j & 1;
          if (j >= 2) wait_pv(m, j - 2);   // S[m][buf] still holds P of tile j-2 until its PV is done
          fence_after_sync();
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks) {
            const uint64_t ad = sdesc(qa + m * C::kQTile + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024);
            const uint64_t bd = sdesc(ka + st * C::kKVTile + (ks >> 2) * 8192 + (ks & 3) * 32, 16, 1024);
            mma_ss(t_s0 + 64 * (2 * m + buf), ad, bd, kIdS, ks > 0);
          }
          commit(&s_full[m][buf]);
        }
        if (j + kKStages < n) commit(&k_empty[st]);
      };
      wait_or_abort(&q_full, 0, &s_abort, tmo);
      issue_s(0);
      for (int j = 0; j < n; ++j) {
        if (j + 1 < n) issue_s(j + 1);
        const int st = j % kVStages;
        wait_or_abort(&v_full[st], (j / kVStages) & 1, &s_abort, tmo);
        for (int m = 0; m < NM; ++m) {
          const int buf = j & 1;
          wait_or_abort(&p_full[m][buf], (j >> 1) & 1, &s_abort, tmo);
          fence_after_sync();
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t bd = sdesc(va + st * C::kKVTile + kk * 2048, 8192, 1024);
            mma_ts(t_o0 + m * D, t_s0 + 64 * (2 * m + buf) + 8 * kk, bd, kIdPV, (j > 0 || kk > 0) ? 1u : 0u);
          }
          commit(&o_done[m]);
        }
        if (j + kVStages < n) commit(&v_empty[st]);
      }
    }
  } else {
    // ============================================================== softmax
    const int m = (warp - 2) >> 2;          // M-tile of this warpgroup
    const int quarter = warp & 3;           // TMEM lane quarter this warp may access
    const int row = quarter * 32 + lane;    // row within the M-tile
    const int rb = 2 * m + (row >> 6);
    const int h = rb_head(rb), qt = rb_qt(rb);
    const bool rb_valid = qt < A.nQT;
    const int i = qt * kTile + (row & 63);  // query position
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t t_o = t_o0 + m * D + lane_off;
    const uint8_t* mrow = (!streaming && T.block_mask && rb_valid)
                              ? T.block_mask + (static_cast<long>(bg) * A.nQT + qt) * A.nQT
                              : nullptr;
    float m_run = kNegInf, l_run = 0.f;
    const float sc = A.scale_log2;
    TileListParams tp{0, A.Hkv, A.nQT, A.sink, A.local, nullptr, nullptr};

    for (int j = 0; j < n; ++j) {
      const int buf = j & 1;
      const uint32_t t_s = t_s0 + 64 * (2 * m + buf) + lane_off;
      wait_or_abort(&s_full[m][buf], (j >> 1) & 1, &s_abort, tmo);
      fence_after_sync();
      uint32_t x[64];
      tmem_ld32(t_s, *reinterpret_cast<uint32_t(*)[32]>(&x[0]));
      tmem_ld32(t_s + 32, *reinterpret_cast<uint32_t(*)[32]>(&x[32]));
      const int kt = cols[j];
      // keep mask of this row over the tile's 64 keys (bit c <-> key 64 kt + c)
      uint64_t keep = ~0ull;
      const bool keep_tile = rb_valid && (T.QG == 1 || tile_keep(tp, streaming, mrow, qt, kt));
      if (!keep_tile) {
        keep = 0ull;
      } else if (!tile_is_full(streaming, qt, kt, A.sink, A.local)) {
        const int d0 = i - kt * kTile;   // offset of the query position inside the tile
        keep = bits_upto(d0);
        if (streaming) keep &= bits_below(A.sink - kt * kTile) | bits_from(d0 - A.local + 1);
      }
      tmem_wait_ld();
      float mx[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) mx[e] = kNegInf;
      if (__all_sync(0xffffffffu, keep == ~0ull)) {
#pragma unroll
        for (int c = 0; c < 64; ++c) mx[c & 7] = fmaxf(mx[c & 7], __uint_as_float(x[c]));
      } else {
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          const float v = ((keep >> c) & 1ull) ? __uint_as_float(x[c]) : kNegInf;
          x[c] = __float_as_uint(v);
          mx[c & 7] = fmaxf(mx[c & 7], v);
        }
      }
      const float mloc = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                               fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7]))) * sc;
      // lazy rescale: move the reference max only when it grows by more than 8 (x256)
      const bool need = mloc > m_run + 8.f;
      const bool rescale = need && m_run != kNegInf;
      const float f = rescale ? fast_exp2(m_run - mloc) : 1.f;
      if (need) m_run = mloc;
      const float m_use = m_run == kNegInf ? 0.f : m_run;
      uint32_t pk[32];
      float ps[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        const float p0 = fast_exp2(fmaf(__uint_as_float(x[2 * c]), sc, -m_use));
        const float p1 = fast_exp2(fmaf(__uint_as_float(x[2 * c + 1]), sc, -m_use));
        ps[c & 3] += p0 + p1;
        pk[c] = pack_bf16x2(p0, p1);
      }
      l_run = l_run * f + ((ps[0] + ps[1]) + (ps[2] + ps[3]));
      tmem_st32(t_s, pk);   // P overwrites the first 32 columns of this S buffer
      // Observe the completion of PV of tile j-1 (every thread, every tile, in
      // order, so that the parity waits on o_done never fall two phases behind);
      // then O holds exactly the tiles < j and may be rescaled.
      if (j > 0) {
        wait_or_abort(&o_done[m], (j - 1) & 1, &s_abort, tmo);
        fence_after_sync();
      }
      if (__any_sync(0xffffffffu, rescale)) {
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
      mbar_arrive(&p_full[m][buf]);
    }
    // ---- epilogue
    if (rb_valid) {
      bf16* orow = A.out + (static_cast<long>(tok0 + i) * Hq + h) * D;
      const bool has = n > 0 && m_run != kNegInf && l_run > 0.f;
      if (n > 0) {
        wait_or_abort(&o_done[m], (n - 1) & 1, &s_abort, tmo);   // PV of the last tile
        fence_after_sync();
      }
      const float inv = has ? 1.f / l_run : 0.f;
#pragma unroll 1
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t ov[32];
        if (n > 0) {
          tmem_ld32(t_o + c0, ov);
          tmem_wait_ld();
        }
        uint32_t pk[16];
#pragma unroll
        for (int c = 0; c < 16; ++c)
          pk[c] = n > 0 ? pack_bf16x2(__uint_as_float(ov[2 * c]) * inv, __uint_as_float(ov[2 * c + 1]) * inv) : 0u;
#pragma unroll
        for (int c = 0; c < 4; ++c)
          *reinterpret_cast<uint4*>(orow + c0 + 8 * c) = make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
      }
      if (A.lse)
        A.lse[(static_cast<long>(b) * Hq + h) * A.S + i] =
            has ? (m_run + __log2f(l_run)) * 0.6931471805599453f : kNegInf;
    } else if (n > 0) {
      wait_or_abort(&o_done[m], (n - 1) & 1, &s_abort, tmo);
    }
  }
  fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    fence_after_sync();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

}  // namespace tc
}  // namespace lserve
