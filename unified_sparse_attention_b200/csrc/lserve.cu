// lserve.cu -- the C ABI of liblserve.so (declared in include/lserve.h).
//
// Host side only: argument validation (before any launch), workspace carving,
// TMA descriptor encoding and kernel launches on the caller's stream.  All
// arithmetic of the method runs in the kernels included below.
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <set>
#include <utility>

#include "common.cuh"
#include "cra.cuh"
#include "decode.cuh"
#include "page_stats.cuh"
#include "prefill_tc.cuh"
#include "quant.cuh"
#include "select.cuh"
#include "tile_lists.cuh"
#include "vslash.cuh"

using namespace lserve;

namespace {

thread_local char g_err[512] = "";

lserve_status fail(lserve_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return st;
}

lserve_status ok() {
  g_err[0] = '\0';
  return LSERVE_OK;
}

lserve_status check_launch(const char* what) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(LSERVE_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  return LSERVE_OK;
}

// Failure-detection test hook: with LSERVE_DEBUG_STALL_DECODE set, the decode
// attention kernel's page resolver publishes nothing, so its other waits run
// out and the call records LSERVE_ERR_DEVICE_TIMEOUT (no copy is in flight).
int debug_stall_decode() { return getenv("LSERVE_DEBUG_STALL_DECODE") ? 1 : 0; }
// The same for the tcgen05 prefill (LSERVE_DEBUG_STALL_PREFILL): its producer
// hands out no work item, so the MMA and softmax warps' waits run out.
int debug_stall_prefill() { return getenv("LSERVE_DEBUG_STALL_PREFILL") ? 1 : 0; }

// Limit of every bounded wait inside the kernels: LSERVE_WAIT_TIMEOUT_NS when it
// holds a positive integer (read at each launch), else 2 s.
unsigned long long wait_timeout_ns() {
  const char* s = getenv("LSERVE_WAIT_TIMEOUT_NS");
  const unsigned long long t = s ? strtoull(s, nullptr, 10) : 0ull;
  return t ? t : 2000000000ull;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Raise a kernel's dynamic shared-memory limit once per (kernel, device).
template <typename K>
void ensure_smem(K* kernel, int bytes) {
  static std::mutex mu;
  static std::set<std::pair<const void*, int>> done;
  int dev = 0;
  cudaGetDevice(&dev);
  const auto key = std::make_pair(reinterpret_cast<const void*>(kernel), dev);
  std::lock_guard<std::mutex> lk(mu);
  if (done.insert(key).second)
    cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

// ---------------------------------------------------------------- TMA maps
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      p = nullptr;
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }();
  return fn;
}

// 2-D bf16 view [rows, inner] (row stride = inner elements), box 64 x 64, 128B swizzle.
bool make_map_2d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {inner * 2};
  cuuint32_t box[2] = {64, 64};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D byte view [rows, inner] (row stride = inner bytes), box inner x 64, no swizzle:
// one page of INT4 codes per load.
bool make_map_2d_u8(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {inner};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(inner), 64};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D bf16 view [tokens, heads, D], box (64 channels, 1 head, 64 tokens), 128B swizzle.
bool make_map_3d(CUtensorMap* m, const void* base, uint64_t D, uint64_t H, uint64_t T) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {D, H, T};
  cuuint64_t strides[2] = {D * 2, H * D * 2};
  cuuint32_t box[3] = {64, 1, 64};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ------------------------------------------------------------- workspace
struct Carver {
  uintptr_t base, cur;
  explicit Carver(void* p) : base(reinterpret_cast<uintptr_t>(p)), cur(reinterpret_cast<uintptr_t>(p)) {}
  template <typename T>
  T* take(size_t count) {
    cur = (cur + 255) & ~uintptr_t(255);
    T* p = reinterpret_cast<T*>(cur);
    cur += count * sizeof(T);
    return p;
  }
  size_t used() const { return cur - base + 256; }
};

// SMs of the current device (148 if it cannot be asked).
int sm_count() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();
    return 148;
  }
  if (!cached[dev]) {
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0) {
      cudaGetLastError();
      sms = 148;
    }
    cached[dev] = sms;
  }
  return cached[dev];
}

// ---------------------------------------------------------------- prefill
struct PrefillWs {
  int* counts;
  int* offsets;
  int* order;
  int* hist;     // [B*Hkv][nQT + 1]
  int* fill;     // [B*Hkv][nQT + 1]  (contiguous with hist: one memset clears both)
  int* work_counter;   // next unclaimed work item of the persistent prefill (cleared with hist)
  int* bucket;   // [B*Hkv][nQT + 1]
  int* overflow;
  uint16_t* cols;
  long long max_nnz;
};

bool shape_valid(const lserve_shape* s) {
  return s && s->B > 0 && s->S > 0 && s->Hq > 0 && s->Hkv > 0 && s->d > 0 && s->Hq % s->Hkv == 0;
}

PrefillWs carve_prefill(const lserve_shape* s, void* ws, size_t* bytes) {
  const long long nQT = s->S / kTile;
  const long long R = static_cast<long long>(s->B) * s->Hkv * nQT;
  Carver c(ws);
  PrefillWs w;
  w.counts = c.take<int>(R);
  w.offsets = c.take<int>(R + 1);
  w.order = c.take<int>(R);
  const long long groups = static_cast<long long>(s->B) * s->Hkv;
  w.hist = c.take<int>(2 * groups * (nQT + 1) + 1);
  w.fill = w.hist + groups * (nQT + 1);
  w.work_counter = w.hist + 2 * groups * (nQT + 1);
  w.bucket = c.take<int>(groups * (nQT + 1));
  w.overflow = c.take<int>(1);
  w.max_nnz = R * (nQT + 1) / 2;
  w.cols = c.take<uint16_t>(w.max_nnz);
  if (bytes) *bytes = c.used();
  return w;
}

lserve_status validate_prefill(const lserve_shape* s, int sink, int local) {
  if (!shape_valid(s)) return fail(LSERVE_ERR_INVALID_ARG, "prefill: invalid shape");
  if (s->d != 64 && s->d != 128) return fail(LSERVE_ERR_UNSUPPORTED, "prefill: head dim %d not in {64,128}", s->d);
  if (s->S % kTile) return fail(LSERVE_ERR_UNSUPPORTED, "prefill: S=%d is not a multiple of 64", s->S);
  if (s->S / kTile > 65535) return fail(LSERVE_ERR_UNSUPPORTED, "prefill: S=%d too long", s->S);
  if (static_cast<long long>(s->B) * s->S > (1ll << 31) - 1)
    return fail(LSERVE_ERR_UNSUPPORTED, "prefill: B*S too large");
  if (sink < 0 || local < 0) return fail(LSERVE_ERR_INVALID_ARG, "prefill: sink/local must be >= 0");
  if (s->lambda_tiles != 0 && s->lambda_tiles != 1)
    return fail(LSERVE_ERR_INVALID_ARG, "prefill: lambda_tiles must be 0 or 1");
  const long long R = static_cast<long long>(s->B) * s->Hkv * (s->S / kTile);
  if (R * (s->S / kTile + 1) / 2 > (1ll << 31) - 1) return fail(LSERVE_ERR_UNSUPPORTED, "prefill: too many tiles");
  return LSERVE_OK;
}

lserve_status launch_tile_lists(const lserve_shape* s, const uint8_t* head_kind, int sink, int local,
                                const uint8_t* block_mask, const PrefillWs& w, int* offsets, uint16_t* cols,
                                long long max_nnz, int* order, cudaStream_t st, int qg = 1,
                                bool closed_form = false) {
  const int nQT = s->S / kTile;
  const int nRow = (nQT + qg - 1) / qg;
  const int R = s->B * s->Hkv * nRow;
  TileListParams P{s->B, s->Hkv, nQT, sink, local, head_kind, block_mask, qg, nRow, closed_form ? 1 : 0};
  const size_t hist_ints = 2ull * s->B * s->Hkv * (nQT + 1) + 1;   // + the work counter
  if (cudaMemsetAsync(w.hist, 0, sizeof(int) * hist_ints, st) != cudaSuccess)
    return fail(LSERVE_ERR_CUDA, "prefill: memset failed");
  const int blocks = (R + 7) / 8;
  tile_count_kernel<<<blocks, 256, 0, st>>>(P, w.counts, w.hist);
  tile_scan_kernel<<<1, 1024, 0, st>>>(w.counts, R, offsets, w.hist, nQT + 1, w.bucket, nRow, max_nnz,
                                       w.overflow);
  tile_fill_kernel<<<blocks, 256, 0, st>>>(P, offsets, w.counts, cols, w.bucket, w.fill, order, w.overflow);
  return check_launch("tile lists");
}

// Work-item shape from the GQA ratio (see prefill_tc.cuh): an item is 128 query
// rows that share one KV tile list.  Even G: two query heads of one query tile.
// Odd G (1, 3, ...): one query head, two adjacent query tiles walking the union
// of their lists.
struct TcPlan {
  int QG, HG;
};

TcPlan tc_plan(int G) { return G % 2 == 0 ? TcPlan{1, 2} : TcPlan{2, 1}; }

template <int D>
lserve_status launch_prefill_tc(const lserve_shape* s, const void* q, const void* k, const void* v,
                                const tc::TcArgs& T, int n_rows, cudaStream_t st) {
  using C = tc::Cfg<D>;
  CUtensorMap tq, tk, tv;
  const uint64_t Tn = static_cast<uint64_t>(s->B) * s->S;
  if (!make_map_3d(&tq, q, D, s->Hq, Tn) || !make_map_3d(&tk, k, D, s->Hkv, Tn) ||
      !make_map_3d(&tv, v, D, s->Hkv, Tn))
    return fail(LSERVE_ERR_CUDA, "prefill: cuTensorMapEncodeTiled failed");
  ensure_smem(tc::prefill_tc_kernel<D>, C::kSmem);
  // the kernel's register split (setmaxnreg) needs the launch to hand out at
  // least kRegsNeeded registers per thread, or its warpgroups would wait forever
  static const int regs = [] {
    cudaFuncAttributes fa{};
    return cudaFuncGetAttributes(&fa, tc::prefill_tc_kernel<D>) == cudaSuccess ? fa.numRegs : 0;
  }();
  if (regs < C::kRegsNeeded)
    return fail(LSERVE_ERR_UNSUPPORTED, "prefill: kernel built with %d registers per thread, its split needs %d",
                regs, C::kRegsNeeded);
  // persistent: one CTA per SM (its shared memory and TMEM admit no second), each
  // claiming work items from the counter until they run out
  const long long grid = std::min<long long>(T.n_items, sm_count());
  if (grid <= 0) return LSERVE_OK;
  tc::prefill_tc_kernel<D><<<static_cast<unsigned>(grid), C::kThreads, C::kSmem, st>>>(tq, tk, tv, T);
  return check_launch("prefill attention (tcgen05)");
}

// One prefill pass: tile lists, then the attention kernel.  out may be null
// (only the LSE is written: the CRA passes).
lserve_status run_prefill(const lserve_shape* shape, const void* q, const void* k, const void* v,
                          const uint8_t* head_kind, int sink, int local, const uint8_t* block_mask, void* out,
                          float* lse, void* workspace, cudaStream_t st);

size_t round_up256(size_t b) { return (b + 255) / 256 * 256; }

lserve_status run_prefill(const lserve_shape* shape, const void* q, const void* k, const void* v,
                          const uint8_t* head_kind, int sink, int local, const uint8_t* block_mask, void* out,
                          float* lse, void* workspace, cudaStream_t st) {
  PrefillWs w = carve_prefill(shape, workspace, nullptr);
  const int G = shape->Hq / shape->Hkv;
  const int nQT = shape->S / kTile;
  const float scale = shape->scale > 0.f ? shape->scale : 1.f / std::sqrt(static_cast<float>(shape->d));
  tc::PrefillArgs A{w.offsets, w.cols, w.order, head_kind, static_cast<bf16*>(out), lse, G,
                shape->Hkv, nQT, shape->S, sink, local, scale * 1.4426950408889634f, wait_timeout_ns(),
                shape->lambda_tiles ? 1 : 0};
  const TcPlan tp = tc_plan(G);
  // rows with a closed-form list (streaming heads; dense heads without a mask)
  // get no CSR entries: the kernel computes their tiles
  lserve_status s = launch_tile_lists(shape, head_kind, sink, local, block_mask, w, w.offsets, w.cols, w.max_nnz,
                                      w.order, st, tp.QG, /*closed_form=*/true);
  if (s != LSERVE_OK) return s;
  const int nRow = (nQT + tp.QG - 1) / tp.QG;
  const int n_rows = shape->B * shape->Hkv * nRow;
  tc::TcArgs T{A, block_mask, tp.QG, tp.HG, nRow, G / tp.HG, n_rows * (G / tp.HG), w.work_counter,
               debug_stall_prefill()};
  return shape->d == 128 ? launch_prefill_tc<128>(shape, q, k, v, T, n_rows, st)
                         : launch_prefill_tc<64>(shape, q, k, v, T, n_rows, st);
}

// ----------------------------------------------------------------- decode
struct DecodePlan {
  int kcap, budget_pages, G;
  int P;                 // CTAs of the attention grid (one wave)
  int R;                 // ranges of the flat page list (kRangesPerCta per CTA)
  float* scores;
  int32_t* sel;
  int32_t* sel_n;
  int32_t* off;          // [units + 1] flat offsets of the units' selections
  int4* flat;            // [units * kcap] pre-resolved flat page list (first off[units] entries used)
  int32_t* range_counter;   // next range to claim (zeroed by the partition step)
  float* part_o;         // [R + units][4 warps][G][d]
  float* part_lse;       // [R + units][4 warps][G]
  size_t bytes;
};


// Attention CTAs for the current device: SMs x resident CTAs per SM, or the
// value of LSERVE_DECODE_GRID (a positive integer) when that is set.
// CTAs of the attention grid: one wave (SMs x resident CTAs of the variant)
int decode_grid(bool q4) {
  if (const char* e = getenv("LSERVE_DECODE_GRID")) {
    const long v = strtol(e, nullptr, 10);
    if (v > 0 && v <= (1 << 20)) return static_cast<int>(v);
  }
  return sm_count() * (q4 ? kDecodeCtasPerSmQ4 : kDecodeCtasPerSm);
}

// Launch with programmatic stream serialisation: the kernel may start while its
// predecessor finishes and waits on griddepcontrol.wait before reading its output.
// With pdl = false (the first kernel of a step) it is an ordinary launch.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(bool pdl, void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

int streaming_page_bound(int sink, int local) {
  return (sink + kPage - 1) / kPage + (local + kPage - 1) / kPage + 1;
}

lserve_status validate_decode(const lserve_decode_args* a, bool need_stats = true) {
  if (!a) return fail(LSERVE_ERR_INVALID_ARG, "decode: null args");
  if (a->B <= 0 || a->Hq <= 0 || a->Hkv <= 0 || a->d <= 0 || a->Hq % a->Hkv || a->num_pages <= 0 || a->maxP <= 0)
    return fail(LSERVE_ERR_INVALID_ARG, "decode: invalid shape");
  if (a->d != 64 && a->d != 128) return fail(LSERVE_ERR_UNSUPPORTED, "decode: head dim %d not in {64,128}", a->d);
  if (a->Hkv > 256) return fail(LSERVE_ERR_UNSUPPORTED, "decode: more than 256 KV heads");
  const int G = a->Hq / a->Hkv;
  if (G != 1 && G != 2 && G != 4 && G != 8)
    return fail(LSERVE_ERR_UNSUPPORTED, "decode: Hq/Hkv=%d not in {1,2,4,8}", G);
  if (a->token_budget < kPage) return fail(LSERVE_ERR_INVALID_ARG, "decode: token_budget must be >= 64");
  if (a->sink < 0 || a->local < 0) return fail(LSERVE_ERR_INVALID_ARG, "decode: sink/local must be >= 0");
  if (static_cast<long long>(a->num_pages) * a->Hkv * kPage > (1ll << 31) - 1)
    return fail(LSERVE_ERR_UNSUPPORTED, "decode: page pool too large for 32-bit TMA coordinates");
  if (static_cast<long long>(a->B) * a->Hkv * std::max(1, std::min(a->maxP, std::max(a->token_budget / kPage,
                                                                    streaming_page_bound(a->sink, a->local)))) >
      (1ll << 31) - 1)
    return fail(LSERVE_ERR_UNSUPPORTED, "decode: B * Hkv * selected pages exceeds 32-bit offsets");
  if (static_cast<long long>(a->maxP) * kPage >= (1ll << 28))
    return fail(LSERVE_ERR_UNSUPPORTED, "decode: maxP * 64 tokens must stay below 2^28");
  if (!a->q || !a->k_pages || !a->v_pages || !a->page_table || !a->seq_lens || (need_stats && !a->stats) ||
      !a->head_kind)
    return fail(LSERVE_ERR_INVALID_ARG, "decode: null tensor pointer");
  if (!aligned16(a->q) || !aligned16(a->k_pages) || !aligned16(a->v_pages) || (a->stats && !aligned16(a->stats)))
    return fail(LSERVE_ERR_INVALID_ARG, "decode: tensors must be 16-byte aligned");
  return LSERVE_OK;
}

// grid > 0 sets the attention grid (CTAs) instead of one full wave.
DecodePlan plan_decode(const lserve_decode_args* a, void* ws, bool q4 = false, int grid = 0) {
  DecodePlan p{};
  p.G = a->Hq / a->Hkv;
  p.budget_pages = a->token_budget / kPage;
  const int dense_cap = std::min(p.budget_pages, a->maxP);
  p.kcap = std::max(1, std::max(dense_cap, std::min(streaming_page_bound(a->sink, a->local), a->maxP)));
  p.P = grid > 0 ? grid : decode_grid(q4);
  p.R = kRangesPerCta * p.P;

  Carver c(ws);
  const long long units = static_cast<long long>(a->B) * a->Hkv;
  p.scores = c.take<float>(units * a->maxP);
  p.sel = c.take<int32_t>(units * p.kcap);
  p.sel_n = c.take<int32_t>(units);
  p.off = c.take<int32_t>(units + 1);
  p.flat = c.take<int4>(units * p.kcap);
  p.range_counter = c.take<int32_t>(1);
  p.part_o = c.take<float>((p.R + units) * kDecodeWarps * p.G * a->d);
  p.part_lse = c.take<float>((p.R + units) * kDecodeWarps * p.G);
  p.bytes = c.used();
  return p;
}

template <int D>
lserve_status launch_decode_d(const lserve_decode_args* a, const DecodePlan& p, int32_t* sel, int32_t* sel_n,
                              void* out, float* lse, cudaStream_t st, const int32_t* sel_in = nullptr,
                              const int32_t* sel_n_in = nullptr, const float* kpar = nullptr,
                              const float* vpar = nullptr) {
  if (sel_in) {
    // a kept selection: no scoring (the top-k step copies the dense rows)
  } else if (p.G == 1) {
    // one query head per KV head: per-lane fp32 products over 16-byte summary
    // loads, one warp per (page, dense head); exactly one wave of CTAs, each
    // with an equal share of the (sequence, dense head, page) list
    static const int occ = [] {
      int o = 0;
      if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&o, score_pages_kernel<D, 1>, 256, 0) != cudaSuccess) o = 0;
      return std::max(1, o);
    }();
    const long long work = static_cast<long long>(a->B) * a->Hkv * a->maxP;
    const int grid = static_cast<int>(std::max(1ll, std::min<long long>(static_cast<long long>(sm_count()) * occ,
                                                                        (work + 63) / 64)));
    score_pages_kernel<D, 1><<<grid, 256, 0, st>>>(
        static_cast<const bf16*>(a->q), static_cast<const bf16*>(a->stats), a->page_table, a->B, a->maxP,
        a->seq_lens, a->head_kind, a->Hkv, a->num_pages, p.scores);
  } else {
    // G query heads per KV head: the bound as a contraction on the tensor cores,
    // one wave of SMs x resident CTAs (fewer when there is less work)
    const long long items = static_cast<long long>(a->B) * a->Hkv * ((a->maxP + 3) / 4);
    const long long want = (items + kScoreThreads / 32 - 1) / (kScoreThreads / 32);
    const int grid = static_cast<int>(std::min<long long>(want, static_cast<long long>(sm_count()) * kScoreCtasPerSm));
    score_pages_mma_kernel<D><<<grid, kScoreThreads, 0, st>>>(
        static_cast<const bf16*>(a->q), static_cast<const bf16*>(a->stats), a->page_table, a->B, a->maxP,
        a->seq_lens, a->head_kind, a->Hkv, p.G, a->num_pages, p.scores);
  }

  ensure_smem(topk_pages_kernel, kTopkSmemKeys * static_cast<int>(sizeof(uint32_t)));
  const int topk_smem = std::min(a->maxP, kTopkSmemKeys) * static_cast<int>(sizeof(uint32_t));
  const int units = a->B * a->Hkv;
  // one block per unit selects its pages; one more lays out the attention grid's work
  if (launch_pdl(sel_in == nullptr, topk_pages_kernel, dim3(units + 1), dim3(kTopkThreads), topk_smem, st,
                 static_cast<const float*>(p.scores), a->maxP, a->seq_lens, a->head_kind, a->page_table,
                 a->num_pages, a->Hkv, p.budget_pages, a->sink, a->local, sel, sel_n, p.kcap, units, p.G, D, p.off,
                 p.flat, p.range_counter, static_cast<bf16*>(out), lse, sel_in, sel_n_in) != cudaSuccess)
    return check_launch("decode top-k");
  // kpar set: INT4 pages (codes of d/2 bytes a row, steps and offsets in kpar, vpar)
  const bool q4 = kpar != nullptr;
  CUtensorMap tk, tv;
  const uint64_t rows = static_cast<uint64_t>(a->num_pages) * a->Hkv * kPage;
  const bool mapped = q4 ? make_map_2d_u8(&tk, a->k_pages, D / 2, rows) && make_map_2d_u8(&tv, a->v_pages, D / 2, rows)
                         : make_map_2d(&tk, a->k_pages, D, rows) && make_map_2d(&tv, a->v_pages, D, rows);
  if (!mapped) return fail(LSERVE_ERR_CUDA, "decode: cuTensorMapEncodeTiled failed");
  auto* kern = q4 ? paged_decode_kernel<D, true> : paged_decode_kernel<D, false>;
  ensure_smem(kern, q4 ? DecodeCfg<D>::smem_bytes_q4(kDecodeMaxG) : DecodeCfg<D>::smem_bytes(kDecodeMaxG));
  const int smem = q4 ? DecodeCfg<D>::smem_bytes_q4(p.G) : DecodeCfg<D>::smem_bytes(p.G);
  const float scale = a->scale > 0.f ? a->scale : 1.f / std::sqrt(static_cast<float>(D));
  if (launch_pdl(true, kern, dim3(p.P), dim3(kDecodeThreads), smem, st, tk,
                 tv, static_cast<const bf16*>(a->q), static_cast<const int4*>(p.flat),
                 static_cast<const int32_t*>(p.off), p.range_counter, p.R, p.kcap, units, a->Hkv, p.G,
                 a->sink, a->local, scale * 1.4426950408889634f, wait_timeout_ns(),
                 debug_stall_decode(), p.part_o, p.part_lse, kpar, vpar) != cudaSuccess)
    return check_launch("decode attention");
  if (launch_pdl(true, decode_merge_kernel, dim3(units), dim3(kMergeThreads), 0, st, static_cast<const int32_t*>(p.off),
                 units, p.R, p.G, D, static_cast<const float*>(p.part_o), static_cast<const float*>(p.part_lse),
                 static_cast<bf16*>(out), lse) != cudaSuccess)
    return check_launch("decode merge");
  return check_launch("decode");
}

// ------------------------------------------------------- vertical-slash masks
lserve_status validate_vslash(const lserve_shape* s, int stride, float tau) {
  if (!shape_valid(s)) return fail(LSERVE_ERR_INVALID_ARG, "vslash: invalid shape");
  if (s->d != 64 && s->d != 128) return fail(LSERVE_ERR_UNSUPPORTED, "vslash: head dim %d not in {64,128}", s->d);
  if (s->S % kTile) return fail(LSERVE_ERR_UNSUPPORTED, "vslash: S=%d is not a multiple of 64", s->S);
  if (stride < 1) return fail(LSERVE_ERR_INVALID_ARG, "vslash: sample stride must be >= 1");
  if (!(tau >= 0.f && tau <= 1.f)) return fail(LSERVE_ERR_INVALID_ARG, "vslash: tau must lie in [0, 1]");
  const int nQT = s->S / kTile, G = s->Hq / s->Hkv;
  if (G > kVsMaxG) return fail(LSERVE_ERR_UNSUPPORTED, "vslash: Hq/Hkv=%d above %d", G, kVsMaxG);
  if (nQT > kVsMaxTiles) return fail(LSERVE_ERR_UNSUPPORTED, "vslash: S=%d above %d tiles", s->S, kVsMaxTiles);
  if (static_cast<long long>(vs_rows(nQT, stride)) * G > kVsMaxEntries)
    return fail(LSERVE_ERR_UNSUPPORTED, "vslash: %d sampled rows x %d heads above %d; raise the stride",
                vs_rows(nQT, stride), G, kVsMaxEntries);
  if (static_cast<long long>(s->B) * s->Hkv > 65535) return fail(LSERVE_ERR_UNSUPPORTED, "vslash: B*Hkv too large");
  return LSERVE_OK;
}

size_t vslash_ws_bytes(const lserve_shape* s, int stride) {
  const long long nQT = s->S / kTile, G = s->Hq / s->Hkv;
  return static_cast<size_t>(s->B) * s->Hkv * vs_rows(static_cast<int>(nQT), stride) * G * nQT * sizeof(float) + 256;
}

}  // namespace

// ------------------------------------------------- decode without a workspace
// Scratch for lserve_decode_noalloc: one fixed array per device, part of the
// module image, so that callers who may not allocate device memory still get
// the decode step.  Its size is LSERVE_NOALLOC_SCRATCH_BYTES; the array lives
// (and holds its memory) for as long as the library stays loaded on a device.
static __device__ __align__(256) unsigned char g_noalloc_scratch[LSERVE_NOALLOC_SCRATCH_BYTES];

namespace {

// The driver's cuCtxGetCurrent, found through the runtime (no link to libcuda).
using CtxGetCurrentFn = CUresult (*)(CUcontext*);
CtxGetCurrentFn ctx_get_current_fn() {
  static CtxGetCurrentFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      p = nullptr;
    return reinterpret_cast<CtxGetCurrentFn>(p);
  }();
  return fn;
}

// Device address of g_noalloc_scratch in the current context.  Host code only
// sees a host-side stand-in under that name, so the address is asked for once
// per (device, context), with that device current, and cached.  The context is
// part of the key: after cudaDeviceReset the module is loaded again in a new
// primary context and the array may sit elsewhere.
lserve_status noalloc_scratch(void** out) {
  static std::mutex mu;
  static CUcontext ctx_of[64] = {};
  static void* addr[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
    return fail(LSERVE_ERR_CUDA, "decode_noalloc: no usable current device");
  auto get_ctx = ctx_get_current_fn();
  CUcontext ctx = nullptr;   // null: no context bound to this thread yet
  if (!get_ctx || get_ctx(&ctx) != CUDA_SUCCESS)
    return fail(LSERVE_ERR_CUDA, "decode_noalloc: cannot read the current CUDA context");
  std::lock_guard<std::mutex> lk(mu);
  if (ctx && addr[dev] && ctx_of[dev] == ctx) {
    *out = addr[dev];
    return LSERVE_OK;
  }
  // the lookup binds the device's primary context to this thread when none was
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
  if (e != cudaSuccess || !p)
    return fail(LSERVE_ERR_CUDA, "decode_noalloc: cudaGetSymbolAddress failed: %s", cudaGetErrorString(e));
  if (!ctx && (get_ctx(&ctx) != CUDA_SUCCESS || !ctx))
    return fail(LSERVE_ERR_CUDA, "decode_noalloc: no CUDA context after the symbol lookup");
  addr[dev] = p;
  ctx_of[dev] = ctx;
  *out = p;
  return LSERVE_OK;
}

}  // namespace

// =================================================================== C ABI
extern "C" {

const char* lserve_version(void) { return "0.1.0"; }

const char* lserve_last_error_string(void) { return g_err; }

size_t lserve_prefill_workspace_size(const lserve_shape* shape) {
  if (!shape_valid(shape) || shape->S % kTile) return 0;
  size_t bytes = 0;
  carve_prefill(shape, nullptr, &bytes);
  return bytes;
}

lserve_status lserve_prefill_tile_lists(const lserve_shape* shape, const uint8_t* head_kind, int32_t sink,
                                        int32_t local, const uint8_t* block_mask, int32_t* row_offsets,
                                        uint16_t* tile_cols, int64_t max_nnz, void* workspace, size_t ws_bytes,
                                        void* stream) {
  lserve_status s = validate_prefill(shape, sink, local);
  if (s != LSERVE_OK) return s;
  if (!head_kind || !row_offsets || !tile_cols || max_nnz < 0)
    return fail(LSERVE_ERR_INVALID_ARG, "tile lists: null pointer or negative capacity");
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) ||
      ws_bytes < lserve_prefill_workspace_size(shape))
    return fail(LSERVE_ERR_WORKSPACE, "tile lists: workspace missing, misaligned or smaller than %zu bytes",
                lserve_prefill_workspace_size(shape));
  PrefillWs w = carve_prefill(shape, workspace, nullptr);
  s = launch_tile_lists(shape, head_kind, sink, local, block_mask, w, row_offsets, tile_cols, max_nnz, nullptr,
                        static_cast<cudaStream_t>(stream));
  return s == LSERVE_OK ? ok() : s;
}

lserve_status lserve_prefill(const lserve_shape* shape, const void* q, const void* k, const void* v,
                             const uint8_t* head_kind, int32_t sink, int32_t local, const uint8_t* block_mask,
                             void* out, float* lse, void* workspace, size_t ws_bytes, void* stream) {
  lserve_status s = validate_prefill(shape, sink, local);
  if (s != LSERVE_OK) return s;
  if (!q || !k || !v || !head_kind || !out) return fail(LSERVE_ERR_INVALID_ARG, "prefill: null tensor pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))
    return fail(LSERVE_ERR_INVALID_ARG, "prefill: q/k/v/out must be 16-byte aligned");
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) ||
      ws_bytes < lserve_prefill_workspace_size(shape))
    return fail(LSERVE_ERR_WORKSPACE, "prefill: workspace missing, misaligned or smaller than %zu bytes",
                lserve_prefill_workspace_size(shape));
  s = run_prefill(shape, q, k, v, head_kind, sink, local, block_mask, out, lse, workspace,
                  static_cast<cudaStream_t>(stream));
  return s == LSERVE_OK ? ok() : s;
}

size_t lserve_vslash_workspace_size(const lserve_shape* shape, int32_t sample_stride) {
  if (validate_vslash(shape, sample_stride, 0.f) != LSERVE_OK) return 0;
  return vslash_ws_bytes(shape, sample_stride);
}

lserve_status lserve_build_vslash_mask(const lserve_shape* shape, const void* q, const void* k,
                                       const uint8_t* head_kind, int32_t sample_stride, float tau,
                                       uint8_t* block_mask, float* cra, int32_t* n_columns, int32_t* n_slashes,
                                       void* workspace, size_t ws_bytes, void* stream) {
  lserve_status s = validate_vslash(shape, sample_stride, tau);
  if (s != LSERVE_OK) return s;
  if (!q || !k || !head_kind || !block_mask) return fail(LSERVE_ERR_INVALID_ARG, "vslash: null tensor pointer");
  if (!aligned16(q) || !aligned16(k)) return fail(LSERVE_ERR_INVALID_ARG, "vslash: q/k must be 16-byte aligned");
  const size_t need = vslash_ws_bytes(shape, sample_stride);
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) || ws_bytes < need)
    return fail(LSERVE_ERR_WORKSPACE, "vslash: workspace missing, misaligned or smaller than %zu bytes", need);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int nQT = shape->S / kTile, G = shape->Hq / shape->Hkv, n_rows = vs_rows(nQT, sample_stride);
  const float scale = shape->scale > 0.f ? shape->scale : 1.f / std::sqrt(static_cast<float>(shape->d));
  float* r = static_cast<float*>(workspace);
  const dim3 grid_m(n_rows, shape->B * shape->Hkv);
  if (shape->d == 128)
    vslash_mass_kernel<128><<<grid_m, kVsThreads, 0, st>>>(static_cast<const bf16*>(q), static_cast<const bf16*>(k),
                                                          head_kind, shape->S, shape->Hkv, G, nQT, sample_stride,
                                                          n_rows, scale * 1.4426950408889634f, r);
  else
    vslash_mass_kernel<64><<<grid_m, kVsThreads, 0, st>>>(static_cast<const bf16*>(q), static_cast<const bf16*>(k),
                                                         head_kind, shape->S, shape->Hkv, G, nQT, sample_stride,
                                                         n_rows, scale * 1.4426950408889634f, r);
  s = check_launch("vslash tile masses");
  if (s != LSERVE_OK) return s;
  const size_t smem = vs_greedy_smem(n_rows * G, nQT);
  ensure_smem(vslash_greedy_kernel, static_cast<int>(vs_greedy_smem(kVsMaxEntries, kVsMaxTiles)));
  vslash_greedy_kernel<<<shape->B * shape->Hkv, kVsGreedyThreads, smem, st>>>(
      r, head_kind, shape->Hkv, G, nQT, sample_stride, n_rows, tau, block_mask, cra, n_columns, n_slashes);
  s = check_launch("vslash greedy");
  return s == LSERVE_OK ? ok() : s;
}

size_t lserve_cra_workspace_size(const lserve_shape* shape) {
  const size_t pw = lserve_prefill_workspace_size(shape);
  if (!pw) return 0;
  const size_t lse_bytes = static_cast<size_t>(shape->B) * shape->Hq * shape->S * sizeof(float);
  return round_up256(pw) + 2 * round_up256(lse_bytes) + round_up256(static_cast<size_t>(shape->Hkv));
}

lserve_status lserve_cra(const lserve_shape* shape, const void* q, const void* k, const void* v,
                         const uint8_t* head_kind, int32_t sink, int32_t local, const uint8_t* block_mask,
                         float* retained, float* cra, void* workspace, size_t ws_bytes, void* stream) {
  lserve_status s = validate_prefill(shape, sink, local);
  if (s != LSERVE_OK) return s;
  if (!q || !k || !v || !head_kind || !cra) return fail(LSERVE_ERR_INVALID_ARG, "cra: null tensor pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v))
    return fail(LSERVE_ERR_INVALID_ARG, "cra: q/k/v must be 16-byte aligned");
  const size_t need = lserve_cra_workspace_size(shape);
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) || ws_bytes < need)
    return fail(LSERVE_ERR_WORKSPACE, "cra: workspace missing, misaligned or smaller than %zu bytes", need);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* base = static_cast<uint8_t*>(workspace);
  const size_t pw = round_up256(lserve_prefill_workspace_size(shape));
  const size_t lse_bytes = round_up256(static_cast<size_t>(shape->B) * shape->Hq * shape->S * sizeof(float));
  float* lse_full = reinterpret_cast<float*>(base + pw);
  float* lse_sparse = reinterpret_cast<float*>(base + pw + lse_bytes);
  uint8_t* all_dense = base + pw + 2 * lse_bytes;
  if (cudaMemsetAsync(all_dense, LSERVE_HEAD_DENSE, static_cast<size_t>(shape->Hkv), st) != cudaSuccess)
    return fail(LSERVE_ERR_CUDA, "cra: memset failed");
  // the causal reference and the sparse mask, LSE only (no output written)
  s = run_prefill(shape, q, k, v, all_dense, 0, 0, nullptr, nullptr, lse_full, workspace, st);
  if (s != LSERVE_OK) return s;
  s = run_prefill(shape, q, k, v, head_kind, sink, local, block_mask, nullptr, lse_sparse, workspace, st);
  if (s != LSERVE_OK) return s;
  if (cudaMemsetAsync(cra, 0x7f, sizeof(float) * shape->B * shape->Hq, st) != cudaSuccess)
    return fail(LSERVE_ERR_CUDA, "cra: memset failed");
  const dim3 grid_r(shape->B * shape->Hq, (shape->S + kCraChunk - 1) / kCraChunk);
  cra_reduce_kernel<<<grid_r, kCraThreads, 0, st>>>(lse_sparse, lse_full, shape->S, retained, cra);
  s = check_launch("cra reduction");
  return s == LSERVE_OK ? ok() : s;
}

lserve_status lserve_update_page_stats(int32_t B, int32_t Hkv, int32_t d, int32_t num_pages, const void* k_pages,
                                       const int32_t* page_table, int32_t maxP, const int32_t* seq_lens,
                                       int32_t first_logical_page, const uint8_t* head_kind, void* stats,
                                       void* stream) {
  if (B <= 0 || Hkv <= 0 || num_pages <= 0 || maxP <= 0 || first_logical_page < 0)
    return fail(LSERVE_ERR_INVALID_ARG, "page stats: invalid sizes");
  if (d != 64 && d != 128) return fail(LSERVE_ERR_UNSUPPORTED, "page stats: head dim %d not in {64,128}", d);
  if (!k_pages || !page_table || !seq_lens || !head_kind || !stats)
    return fail(LSERVE_ERR_INVALID_ARG, "page stats: null pointer");
  if (!aligned16(k_pages) || !aligned16(stats))
    return fail(LSERVE_ERR_INVALID_ARG, "page stats: k_pages/stats must be 16-byte aligned");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const long long units = static_cast<long long>(maxP) * Hkv;
  dim3 grid(static_cast<unsigned>((units + 7) / 8), B);
  if (d == 128)
    page_stats_kernel<128><<<grid, 256, 0, st>>>(static_cast<const bf16*>(k_pages), page_table, maxP, seq_lens,
                                                 first_logical_page, head_kind, Hkv, num_pages,
                                                 static_cast<bf16*>(stats));
  else
    page_stats_kernel<64><<<grid, 256, 0, st>>>(static_cast<const bf16*>(k_pages), page_table, maxP, seq_lens,
                                                first_logical_page, head_kind, Hkv, num_pages,
                                                static_cast<bf16*>(stats));
  lserve_status s = check_launch("page stats");
  return s == LSERVE_OK ? ok() : s;
}

int32_t lserve_decode_max_selected(const lserve_decode_args* args) {
  if (!args || args->maxP <= 0 || args->token_budget < kPage) return 0;
  return std::max(1, std::max(std::min(args->token_budget / kPage, args->maxP),
                              std::min(streaming_page_bound(args->sink, args->local), args->maxP)));
}

size_t lserve_decode_workspace_size(const lserve_decode_args* args) {
  // the size depends on the shapes only: a call with stats = NULL (lserve_decode_reuse) asks too;
  // it covers the INT4 step's plan as well (a wider attention grid, more ranges)
  if (validate_decode(args, /*need_stats=*/false) != LSERVE_OK) return 0;
  return std::max(plan_decode(args, nullptr).bytes, plan_decode(args, nullptr, /*q4=*/true).bytes);
}

lserve_status lserve_decode(const lserve_decode_args* args, void* out, float* lse, int32_t* sel_out,
                            int32_t* sel_n, void* workspace, size_t ws_bytes, void* stream) {
  lserve_status s = validate_decode(args);
  if (s != LSERVE_OK) return s;
  if (!out || !aligned16(out)) return fail(LSERVE_ERR_INVALID_ARG, "decode: out must be non-null and 16-byte aligned");
  const size_t need = plan_decode(args, nullptr).bytes;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) || ws_bytes < need)
    return fail(LSERVE_ERR_WORKSPACE, "decode: workspace missing, misaligned or smaller than %zu bytes", need);
  DecodePlan p = plan_decode(args, workspace);
  int32_t* sel = sel_out ? sel_out : p.sel;
  int32_t* seln = sel_n ? sel_n : p.sel_n;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  s = args->d == 128 ? launch_decode_d<128>(args, p, sel, seln, out, lse, st)
                     : launch_decode_d<64>(args, p, sel, seln, out, lse, st);
  return s == LSERVE_OK ? ok() : s;
}

lserve_status lserve_decode_noalloc(const lserve_decode_args* args, void* out, float* lse, int32_t* sel_out,
                                    int32_t* sel_n, void* stream) {
  lserve_status s = validate_decode(args);
  if (s != LSERVE_OK) return s;
  if (!out || !aligned16(out)) return fail(LSERVE_ERR_INVALID_ARG, "decode: out must be non-null and 16-byte aligned");
  // The split partials of the attention grid grow with its width (one full wave
  // by default).  Where they would not fit, take the widest grid whose scratch
  // does: the result is the same attention, split over fewer ranges.
  const size_t cap = LSERVE_NOALLOC_SCRATCH_BYTES;
  int grid = decode_grid(false);
  if (plan_decode(args, nullptr, false, grid).bytes > cap) {
    const size_t need1 = plan_decode(args, nullptr, false, 1).bytes;
    if (need1 > cap)
      return fail(LSERVE_ERR_WORKSPACE,
                  "decode_noalloc: this batch needs %zu bytes of scratch even on a one-CTA grid but the built-in "
                  "array holds %zu; split the batch or call lserve_decode with a workspace",
                  need1, cap);
    int lo = 1, hi = grid - 1;   // plan(lo) fits, plan(grid) does not; the need grows with the grid
    while (lo < hi) {
      const int mid = lo + (hi - lo + 1) / 2;
      if (plan_decode(args, nullptr, false, mid).bytes <= cap) lo = mid;
      else hi = mid - 1;
    }
    grid = lo;
  }
  void* scratch = nullptr;
  s = noalloc_scratch(&scratch);
  if (s != LSERVE_OK) return s;
  // Every buffer carved here is fully written by the kernels before it is read,
  // so the previous call's leftovers need no clearing.
  DecodePlan p = plan_decode(args, scratch, false, grid);
  int32_t* sel = sel_out ? sel_out : p.sel;
  int32_t* seln = sel_n ? sel_n : p.sel_n;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  s = args->d == 128 ? launch_decode_d<128>(args, p, sel, seln, out, lse, st)
                     : launch_decode_d<64>(args, p, sel, seln, out, lse, st);
  return s == LSERVE_OK ? ok() : s;
}

lserve_status lserve_quantize_pages_int4(int32_t B, int32_t Hkv, int32_t d, int32_t num_pages, const void* k_pages,
                                        const void* v_pages, const int32_t* page_table, int32_t maxP,
                                        const int32_t* seq_lens, int32_t first_page, const uint8_t* head_kind,
                                        void* kq, float* kpar, void* vq, float* vpar, void* stats, void* stream) {
  if (B <= 0 || Hkv <= 0 || num_pages <= 0 || maxP <= 0 || first_page < 0 || B > 65535 || Hkv > 65535)
    return fail(LSERVE_ERR_INVALID_ARG, "quantize: invalid sizes");
  if (d != 64 && d != 128) return fail(LSERVE_ERR_UNSUPPORTED, "quantize: head dim %d not in {64,128}", d);
  if (!k_pages || !v_pages || !page_table || !seq_lens || !head_kind || !kq || !kpar || !vq || !vpar || !stats)
    return fail(LSERVE_ERR_INVALID_ARG, "quantize: null pointer");
  if (!aligned16(k_pages) || !aligned16(v_pages) || !aligned16(kq) || !aligned16(vq) || !aligned16(stats))
    return fail(LSERVE_ERR_INVALID_ARG, "quantize: pools and stats must be 16-byte aligned");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const dim3 grid(maxP, B, Hkv);
  if (d == 128)
    quant_int4_kernel<128><<<grid, 128, 0, st>>>(static_cast<const bf16*>(k_pages), static_cast<const bf16*>(v_pages),
                                                 page_table, maxP, seq_lens, first_page, head_kind, Hkv, num_pages,
                                                 static_cast<uint8_t*>(kq), kpar, static_cast<uint8_t*>(vq), vpar,
                                                 static_cast<bf16*>(stats));
  else
    quant_int4_kernel<64><<<grid, 128, 0, st>>>(static_cast<const bf16*>(k_pages), static_cast<const bf16*>(v_pages),
                                                page_table, maxP, seq_lens, first_page, head_kind, Hkv, num_pages,
                                                static_cast<uint8_t*>(kq), kpar, static_cast<uint8_t*>(vq), vpar,
                                                static_cast<bf16*>(stats));
  const lserve_status s = check_launch("quantize");
  return s == LSERVE_OK ? ok() : s;
}

lserve_status lserve_decode_int4(const lserve_decode_args* args, const float* kpar, const float* vpar, void* out,
                                 float* lse, int32_t* sel_out, int32_t* sel_n, void* workspace, size_t ws_bytes,
                                 void* stream) {
  lserve_status s = validate_decode(args);
  if (s != LSERVE_OK) return s;
  if (!kpar || !vpar || !aligned16(kpar) || !aligned16(vpar))
    return fail(LSERVE_ERR_INVALID_ARG, "decode int4: kpar and vpar must be non-null and 16-byte aligned");
  if (!out || !aligned16(out)) return fail(LSERVE_ERR_INVALID_ARG, "decode: out must be non-null and 16-byte aligned");
  const size_t need = plan_decode(args, nullptr, /*q4=*/true).bytes;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) || ws_bytes < need)
    return fail(LSERVE_ERR_WORKSPACE, "decode: workspace missing, misaligned or smaller than %zu bytes", need);
  DecodePlan p = plan_decode(args, workspace, /*q4=*/true);
  int32_t* sel = sel_out ? sel_out : p.sel;
  int32_t* seln = sel_n ? sel_n : p.sel_n;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  s = args->d == 128 ? launch_decode_d<128>(args, p, sel, seln, out, lse, st, nullptr, nullptr, kpar, vpar)
                     : launch_decode_d<64>(args, p, sel, seln, out, lse, st, nullptr, nullptr, kpar, vpar);
  return s == LSERVE_OK ? ok() : s;
}

lserve_status lserve_decode_reuse(const lserve_decode_args* args, const int32_t* sel_in, const int32_t* sel_n_in,
                                  void* out, float* lse, int32_t* sel_out, int32_t* sel_n, void* workspace,
                                  size_t ws_bytes, void* stream) {
  lserve_status s = validate_decode(args, /*need_stats=*/false);
  if (s != LSERVE_OK) return s;
  if (!sel_in || !sel_n_in) return fail(LSERVE_ERR_INVALID_ARG, "decode reuse: sel_in and sel_n_in are required");
  if (!out || !aligned16(out)) return fail(LSERVE_ERR_INVALID_ARG, "decode: out must be non-null and 16-byte aligned");
  const size_t need = plan_decode(args, nullptr).bytes;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) || ws_bytes < need)
    return fail(LSERVE_ERR_WORKSPACE, "decode: workspace missing, misaligned or smaller than %zu bytes", need);
  DecodePlan p = plan_decode(args, workspace);
  int32_t* sel = sel_out ? sel_out : p.sel;
  int32_t* seln = sel_n ? sel_n : p.sel_n;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  s = args->d == 128 ? launch_decode_d<128>(args, p, sel, seln, out, lse, st, sel_in, sel_n_in)
                     : launch_decode_d<64>(args, p, sel, seln, out, lse, st, sel_in, sel_n_in);
  return s == LSERVE_OK ? ok() : s;
}

lserve_status lserve_get_device_status(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return fail(LSERVE_ERR_CUDA, "device status: stream synchronisation failed: %s",
                cudaGetErrorString(cudaGetLastError()));
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_status, sizeof(int)) != cudaSuccess)
    return fail(LSERVE_ERR_CUDA, "device status: read failed");
  const int zero = 0;
  if (cudaMemcpyToSymbol(g_device_status, &zero, sizeof(int)) != cudaSuccess)
    return fail(LSERVE_ERR_CUDA, "device status: clear failed");
  if (v == 0) return ok();
  return fail(static_cast<lserve_status>(v), "kernel reported %s",
              v == LSERVE_ERR_DEVICE_TIMEOUT ? "a bounded wait that ran out" : "an out-of-range index");
}

}  // extern "C"
