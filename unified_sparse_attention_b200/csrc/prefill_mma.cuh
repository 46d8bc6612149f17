// prefill_mma.cuh -- block-sparse causal prefill attention on mma.sync.
//
// LServe + SampleAttention blog post, "LServe - Prefill Phase", Fig. 1: a
// flash-attention kernel whose KV loop walks only the kept 64x64 tiles of its
// query tile (dense heads: causal tiles, optionally block-masked; streaming
// heads: the Lambda support).  Elements inside kept boundary tiles (the causal
// diagonal, the edges of the sink and of the local window) are masked exactly.
//
// One CTA per (kept-tile row, query head), launched longest row first.  Q (64
// rows) is loaded once by TMA; K/V tiles of the row's CSR list stream through a
// 2-stage TMA ring (128-byte swizzle); 4 warps own 16 query rows each and run
// S = Q K^T, online softmax (base-2, scale folded in) and O += P V on
// mma.sync m16n8k16 (bf16 in, fp32 accumulate).  This is the legacy tensor-core
// path: it is exported for comparison and as the reference point for the
// tcgen05 kernel.
#pragma once

#include "common.cuh"

namespace lserve {

constexpr int kPrefillThreads = 128;
constexpr int kPrefillStages = 2;

template <int D>
struct PrefillCfg {
  static constexpr int kBoxes = D / 64;
  static constexpr int kBoxBytes = 64 * 128;
  static constexpr int kTileBytes = kBoxes * kBoxBytes;   // 64 rows x D bf16
  static constexpr int kSmemBytes = (1 + 2 * kPrefillStages) * kTileBytes + 1024;
};

struct PrefillArgs {
  const int32_t* row_offsets;
  const uint16_t* cols;
  const int32_t* order;
  const uint8_t* head_kind;
  bf16* out;
  float* lse;
  int G, Hkv, nQT, S, sink, local;
  float scale_log2;
  unsigned long long timeout_ns;
};

// Is every element of tile (qt, kt) kept?  (Then no element mask is needed.)
__device__ __forceinline__ bool tile_is_full(bool streaming, int qt, int kt, int sink, int local) {
  if (kt >= qt) return false;   // diagonal (or beyond): causal mask needed
  if (!streaming) return true;
  return kTile * kt + kTile <= sink || kTile * qt + (kTile - 1) - kTile * kt < local;
}

template <int D>
__global__ void __launch_bounds__(kPrefillThreads) prefill_mma_kernel(const __grid_constant__ CUtensorMap tmQ,
                                                                      const __grid_constant__ CUtensorMap tmK,
                                                                      const __grid_constant__ CUtensorMap tmV,
                                                                      PrefillArgs A) {
  using Cfg = PrefillCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[kPrefillStages];
  __shared__ __align__(8) uint64_t q_bar;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* q_s = smem;
  uint8_t* kv_s = smem + Cfg::kTileBytes;   // stage st: K at 2*st, V at 2*st+1

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int w = blockIdx.x;
  const int r = A.order[w / A.G];
  const int hh = w % A.G;
  const int qt = r % A.nQT;
  const int bg = r / A.nQT;
  const int g = bg % A.Hkv, b = bg / A.Hkv;
  const int h = g * A.G + hh;
  const int Hq = A.Hkv * A.G;
  const bool streaming = A.head_kind[g] != LSERVE_HEAD_DENSE;
  const int beg = A.row_offsets[r];
  const int n = A.row_offsets[r + 1] - beg;
  const uint16_t* cols = A.cols + beg;
  const int tok0 = b * A.S;   // first token row of this sequence in the [B*S] view

  if (tid == 0) {
    prefetch_tensormap(&tmQ);
    prefetch_tensormap(&tmK);
    prefetch_tensormap(&tmV);
    mbar_init(&q_bar, 1);
    for (int s = 0; s < kPrefillStages; ++s) mbar_init(&full_bar[s], 1);
    fence_barrier_init();
  }
  __syncthreads();
  auto issue = [&](int it) {
    const int st = it % kPrefillStages;
    const int kt = cols[it];
    uint8_t* kd = kv_s + (2 * st) * Cfg::kTileBytes;
    uint8_t* vd = kd + Cfg::kTileBytes;
    mbar_arrive_expect_tx(&full_bar[st], 2 * Cfg::kTileBytes);
#pragma unroll
    for (int x = 0; x < Cfg::kBoxes; ++x) {
      tma_load_3d(kd + x * Cfg::kBoxBytes, &tmK, &full_bar[st], x * 64, g, tok0 + kt * kTile);
      tma_load_3d(vd + x * Cfg::kBoxBytes, &tmV, &full_bar[st], x * 64, g, tok0 + kt * kTile);
    }
  };
  if (tid == 0) {
    mbar_arrive_expect_tx(&q_bar, Cfg::kTileBytes);
#pragma unroll
    for (int x = 0; x < Cfg::kBoxes; ++x)
      tma_load_3d(q_s + x * Cfg::kBoxBytes, &tmQ, &q_bar, x * 64, h, tok0 + qt * kTile);
    for (int it = 0; it < min(kPrefillStages, n); ++it) issue(it);
  }

  const int mi = lane >> 3, rr = lane & 7;
  constexpr int KS = D / 16;
  bool timed_out = !mbar_wait_bounded(&q_bar, 0, A.timeout_ns);
  uint32_t qa[KS][4];
#pragma unroll
  for (int ks = 0; ks < KS; ++ks) {
    const int row = warp * 16 + (mi & 1) * 8 + rr;
    const int chunk = 2 * (ks & 3) + (mi >> 1);
    ldmatrix_x4(smem_u32(q_s + (ks >> 2) * Cfg::kBoxBytes + swz128(row, chunk)), qa[ks][0], qa[ks][1], qa[ks][2],
                qa[ks][3]);
  }

  float acc[D / 8][4];
#pragma unroll
  for (int j = 0; j < D / 8; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;
  float m_run[2] = {kNegInf, kNegInf}, l_run[2] = {0.f, 0.f};
  const int i_row0 = qt * kTile + warp * 16 + (lane >> 2);   // query positions of this lane's two rows
  const int tc = 2 * (lane & 3);

  for (int it = 0; it < n; ++it) {
    const int st = it % kPrefillStages;
    if (!mbar_wait_bounded(&full_bar[st], (it / kPrefillStages) & 1, A.timeout_ns)) timed_out = true;
    const uint8_t* ks_base = kv_s + (2 * st) * Cfg::kTileBytes;
    const uint8_t* vs_base = ks_base + Cfg::kTileBytes;
    const int kt = cols[it];

    float s[8][4];
#pragma unroll
    for (int j = 0; j < 8; ++j) s[j][0] = s[j][1] = s[j][2] = s[j][3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        const int row = np * 16 + (mi >> 1) * 8 + rr;
        const int chunk = 2 * (ks & 3) + (mi & 1);
        uint32_t b0, b1, b2, b3;
        ldmatrix_x4(smem_u32(ks_base + (ks >> 2) * Cfg::kBoxBytes + swz128(row, chunk)), b0, b1, b2, b3);
        mma_bf16_16816(s[2 * np], qa[ks], b0, b1);
        mma_bf16_16816(s[2 * np + 1], qa[ks], b2, b3);
      }
    }
    // scale (base 2) + element mask on boundary tiles
    if (tile_is_full(streaming, qt, kt, A.sink, A.local)) {
#pragma unroll
      for (int j = 0; j < 8; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) s[j][e] *= A.scale_log2;
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int i = i_row0 + (e >> 1) * 8;
          const int jj = kt * kTile + j * 8 + tc + (e & 1);
          const bool keep = jj <= i && (!streaming || jj < A.sink || i - jj < A.local);
          s[j][e] = keep ? s[j][e] * A.scale_log2 : kNegInf;
        }
    }
    float mloc[2] = {kNegInf, kNegInf};
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      mloc[0] = fmaxf(mloc[0], fmaxf(s[j][0], s[j][1]));
      mloc[1] = fmaxf(mloc[1], fmaxf(s[j][2], s[j][3]));
    }
    float corr[2];
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
      mloc[hr] = fmaxf(mloc[hr], __shfl_xor_sync(0xffffffffu, mloc[hr], 1));
      mloc[hr] = fmaxf(mloc[hr], __shfl_xor_sync(0xffffffffu, mloc[hr], 2));
      const float m_new = fmaxf(m_run[hr], mloc[hr]);
      const float m_use = m_new == kNegInf ? 0.f : m_new;
      corr[hr] = fast_exp2(m_run[hr] - m_use);
      m_run[hr] = m_new;
      mloc[hr] = m_use;
    }
    float psum[2] = {0.f, 0.f};
#pragma unroll
    for (int j = 0; j < 8; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        s[j][e] = fast_exp2(s[j][e] - mloc[e >> 1]);
        psum[e >> 1] += s[j][e];
      }
    l_run[0] = l_run[0] * corr[0] + psum[0];
    l_run[1] = l_run[1] * corr[1] + psum[1];
#pragma unroll
    for (int j = 0; j < D / 8; ++j) {
      acc[j][0] *= corr[0];
      acc[j][1] *= corr[0];
      acc[j][2] *= corr[1];
      acc[j][3] *= corr[1];
    }
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {   // 16 keys per k-step
      uint32_t pa[4];
      pa[0] = pack_bf16x2(s[2 * kk][0], s[2 * kk][1]);
      pa[1] = pack_bf16x2(s[2 * kk][2], s[2 * kk][3]);
      pa[2] = pack_bf16x2(s[2 * kk + 1][0], s[2 * kk + 1][1]);
      pa[3] = pack_bf16x2(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
      for (int np = 0; np < D / 16; ++np) {
        const int ch = np * 16 + (mi >> 1) * 8;
        const int row = kk * 16 + (mi & 1) * 8 + rr;
        uint32_t b0, b1, b2, b3;
        ldmatrix_x4_trans(smem_u32(vs_base + (ch >> 6) * Cfg::kBoxBytes + swz128(row, (ch & 63) >> 3)), b0, b1,
                          b2, b3);
        mma_bf16_16816(acc[2 * np], pa, b0, b1);
        mma_bf16_16816(acc[2 * np + 1], pa, b2, b3);
      }
    }
    if (__syncthreads_or(timed_out)) {
      timed_out = true;
      break;
    }
    if (tid == 0 && it + kPrefillStages < n) issue(it + kPrefillStages);
  }
  if (timed_out) {
    if (tid == 0) {
      mbar_wait_bounded(&q_bar, 0, A.timeout_ns);
      for (int it = 0; it < n; ++it)
        mbar_wait_bounded(&full_bar[it % kPrefillStages], (it / kPrefillStages) & 1, A.timeout_ns);
    }
    __syncthreads();
    return;
  }

  // epilogue: normalise, store bf16 rows and the optional LSE
#pragma unroll
  for (int hr = 0; hr < 2; ++hr) {
    l_run[hr] += __shfl_xor_sync(0xffffffffu, l_run[hr], 1);
    l_run[hr] += __shfl_xor_sync(0xffffffffu, l_run[hr], 2);
  }
#pragma unroll
  for (int hr = 0; hr < 2; ++hr) {
    const int i = i_row0 + hr * 8;
    const bool has = m_run[hr] != kNegInf && l_run[hr] > 0.f;
    const float inv = has ? 1.f / l_run[hr] : 0.f;
    if (A.out) {   // no output: only the LSE (CRA passes)
      bf16* orow = A.out + (static_cast<long>(tok0 + i) * Hq + h) * D;
#pragma unroll
      for (int j = 0; j < D / 8; ++j)
        *reinterpret_cast<uint32_t*>(orow + j * 8 + tc) = pack_bf16x2(acc[j][2 * hr] * inv, acc[j][2 * hr + 1] * inv);
    }
    if (A.lse && (lane & 3) == 0)
      A.lse[(static_cast<long>(b) * Hq + h) * A.S + i] =
          has ? (m_run[hr] + __log2f(l_run[hr])) * 0.6931471805599453f : kNegInf;
  }
}

}  // namespace lserve
