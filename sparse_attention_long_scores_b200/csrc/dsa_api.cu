// dsa_api.cu - the C ABI declared in include/dsa.h: argument validation, TMA
// descriptor set-up, workspace carving and the launch schedule of the DSA
// forward path (indexer -> top-k -> sparse MLA; "DeepSeek-V3.2: Pushing the
// Frontier of Open Large Language Models", bud-325 paper digest, "Key claims",
// section 2.1 Eq. 1-2, and "Method").
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <string>

#include "../../include/dsa.h"
#include "dsa_kernels.h"

namespace {

thread_local std::string g_err;

// NVTX range around the enqueue of one kernel launch (or one entry point): a
// profiler attached to the process shows each stage of the path by name; with
// no tool attached a push/pop costs a few nanoseconds.
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

// Bound on device-side waits; DSA_WAIT_LIMIT_NS overrides the 2 s default.
unsigned long long initial_wait_ns() {
  const char* e = getenv("DSA_WAIT_LIMIT_NS");
  if (e != nullptr) {
    unsigned long long v = strtoull(e, nullptr, 10);
    if (v > 0) return v;
  }
  return 2000000000ull;
}
unsigned long long g_wait_ns = initial_wait_ns();

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_err = buf;
  return code;
}

int cuda_fail(cudaError_t e, const char* what) {
  return fail(DSA_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

#define DSA_TRY_CUDA(expr, what)            \
  do {                                      \
    cudaError_t e_ = (expr);                \
    if (e_ != cudaSuccess) return cuda_fail(e_, what); \
  } while (0)

// Device status word: [0] code, [1] site, [2] block, [3] wait id.
__device__ int g_status[4];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
int* g_status_ptr[kMaxDevices] = {nullptr};
int g_num_sms[kMaxDevices] = {0};

int device_ctl(dsa::DevCtl& ctl, int& num_sms) {
  int dev = 0;
  DSA_TRY_CUDA(cudaGetDevice(&dev), "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(DSA_ERR_CUDA, "device ordinal %d out of range", dev);
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_status_ptr[dev] == nullptr) {
    void* p = nullptr;
    DSA_TRY_CUDA(cudaGetSymbolAddress(&p, g_status), "cudaGetSymbolAddress(status)");
    g_status_ptr[dev] = static_cast<int*>(p);
    int sms = 0;
    DSA_TRY_CUDA(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev), "SM count");
    int major = 0, minor = 0;
    DSA_TRY_CUDA(cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev), "cc");
    DSA_TRY_CUDA(cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev), "cc");
    if (major != 10 || minor != 0)
      return fail(DSA_ERR_CUDA, "device %d is sm_%d%d; this library is built for sm_100a only",
                  dev, major, minor);
    g_num_sms[dev] = sms;
  }
  ctl.status = g_status_ptr[dev];
  ctl.wait_ns = g_wait_ns;
  num_sms = g_num_sms[dev];
  return DSA_OK;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D tiled tensor map over a row-major [rows, inner] array.
int make_map_2d(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int elem_bytes,
                uint64_t inner, uint64_t rows, uint32_t box_inner, uint32_t box_rows,
                CUtensorMapSwizzle swz) {
  auto fn = encode_fn();
  if (!fn) return fail(DSA_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable (driver too old?)");
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {inner * (uint64_t)elem_bytes};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(DSA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return DSA_OK;
}

// 3-D tiled tensor map over [depth][rows][inner] elements with row stride
// `row_stride` and depth stride `depth_stride` (in elements).
int make_map_3d(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int elem_bytes,
                uint64_t inner, uint64_t rows, uint64_t depth, uint64_t row_stride,
                uint64_t depth_stride, uint32_t box_inner, uint32_t box_rows,
                CUtensorMapSwizzle swz) {
  auto fn = encode_fn();
  if (!fn) return fail(DSA_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable (driver too old?)");
  cuuint64_t dims[3] = {inner, rows, depth};
  cuuint64_t strides[2] = {row_stride * (uint64_t)elem_bytes, depth_stride * (uint64_t)elem_bytes};
  cuuint32_t box[3] = {box_inner, box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, dt, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(DSA_ERR_CUDA, "cuTensorMapEncodeTiled (3-D) failed (%d)", (int)r);
  return DSA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_ptr(const void* p, const char* name, bool optional = false) {
  if (p == nullptr) {
    if (optional) return DSA_OK;
    return fail(DSA_ERR_INVALID_ARG, "%s is NULL", name);
  }
  if (!aligned16(p)) return fail(DSA_ERR_INVALID_ARG, "%s is not 16-byte aligned", name);
  return DSA_OK;
}

#define DSA_TRY(expr)          \
  do {                         \
    int r_ = (expr);           \
    if (r_ != DSA_OK) return r_; \
  } while (0)

int check_seq(int B, int Lq, int Lk, int q_pos0) {
  if (B < 1 || Lq < 1 || Lk < 1) return fail(DSA_ERR_INVALID_ARG, "B, Lq, Lk must be >= 1 (got %d, %d, %d)", B, Lq, Lk);
  if (q_pos0 < 0 || (long long)q_pos0 + Lq > Lk)
    return fail(DSA_ERR_INVALID_ARG, "need 0 <= q_pos0 and q_pos0 + Lq <= Lk (q_pos0=%d Lq=%d Lk=%d)", q_pos0, Lq, Lk);
  if ((long long)B * Lk > (1LL << 30) || (long long)B * Lq > (1LL << 30))
    return fail(DSA_ERR_UNSUPPORTED_SHAPE, "B*Lk and B*Lq must be <= 2^30");
  return DSA_OK;
}

int check_indexer_shape(int H_I, int d_I, int B, int Lq) {
  if (!((H_I == 64 && d_I == 128) || (H_I == 4 && d_I == 32)))
    return fail(DSA_ERR_UNSUPPORTED_SHAPE, "indexer (H_I, d_I) = (%d, %d) unsupported; use (64, 128) or (4, 32)", H_I, d_I);
  if ((long long)B * Lq * H_I > (1LL << 31) - 1)
    return fail(DSA_ERR_UNSUPPORTED_SHAPE, "B*Lq*H_I too large");
  return DSA_OK;
}

int check_mla_shape(int H, int Dqk, int Dv, int B, int Lq) {
  if (!((H == 128 && Dqk == 576 && Dv == 512) || (H == 8 && Dqk == 80 && Dv == 64)))
    return fail(DSA_ERR_UNSUPPORTED_SHAPE, "attention (H, Dqk, Dv) = (%d, %d, %d) unsupported; use (128, 576, 512) or (8, 80, 64)", H, Dqk, Dv);
  if ((long long)B * Lq * H > (1LL << 31) - 1)
    return fail(DSA_ERR_UNSUPPORTED_SHAPE, "B*Lq*H too large");
  return DSA_OK;
}

int check_k(int k, int kmax) {
  if (k < 32 || k > kmax || (k % 32) != 0)
    return fail(DSA_ERR_UNSUPPORTED_SHAPE, "k = %d unsupported: need a multiple of 32 in [32, %d]", k, kmax);
  return DSA_OK;
}

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Optional per-launch event recording (profiling entry point only).
struct Recorder {
  void* const* events = nullptr;  // events[0] before the first launch, events[i+1] after launch i
  int* kinds = nullptr;
  int cap = 0;
  int n = 0;
  int launched = 0;               // kernel launches so far (counted with or without events)
  int mark(int kind, cudaStream_t s) {
    ++launched;
    if (events == nullptr) return DSA_OK;
    if (n >= cap) return fail(DSA_ERR_INVALID_ARG, "profiling: more than %d launches", cap);
    kinds[n] = kind;
    ++n;
    DSA_TRY_CUDA(cudaEventRecord(static_cast<cudaEvent_t>(events[n]), s), "cudaEventRecord");
    return DSA_OK;
  }
};
Recorder g_no_rec;
thread_local int g_last_launches = 0;   // kernel launches of this thread's last forward call

// ---------------- schedule helpers ----------------
int indexer_piece_keys(int B, int rows, int t_blk, int keys_max, int num_sms) {
  int nblk = (rows + t_blk - 1) / t_blk;
  int R = 4096;
  while (R > 128 && (long long)B * nblk * ((keys_max + R - 1) / R) < 2LL * num_sms) R /= 2;
  return R;
}

int mla_n_dv(int Dv) { return Dv == 512 ? 2 : 1; }

// Key splits of the attention: as many as keep all CTAs in one wave. Every CTA
// pays a fixed cost (Q staging, pipeline fill, epilogue) of about three key
// tiles, so a second wave of short CTAs costs more than it saves; each split
// keeps at least 4 tiles, and at most 16 splits (the combine kernel's limit).
int mla_splits(int B, int Lq, int Dv, int k, int num_sms) {
  long long ctas = (long long)B * Lq * mla_n_dv(Dv);
  if (ctas >= num_sms) return 1;
  int tiles = k / 64 > 0 ? k / 64 : 1;   // 64-key tiles
  int s = (int)(num_sms / ctas);
  int max_s = tiles / 4 > 1 ? tiles / 4 : 1;
  if (s > max_s) s = max_s;
  if (s > 16) s = 16;
  return s < 1 ? 1 : s;
}

size_t mla_ws_bytes(int B, int Lq, int H, int Dv, int splits) {
  if (splits <= 1) return 0;
  size_t tok = (size_t)B * Lq;
  return align_up(tok * splits * H * Dv * sizeof(float), 256) +
         align_up(tok * splits * H * 2 * sizeof(float), 256);
}

int assumed_sms() {
  // Workspace sizing must not depend on a device being present; size for the
  // largest schedule (fewest SMs never needs more splits than this bound).
  return 148;
}

int run_mla(const uint16_t* q, const uint16_t* kv, const int32_t* idx, uint16_t* out, float* lse,
            int B, int Lq, int Lk, int H, int Dqk, int Dv, int k, float sm_scale, void* ws,
            size_t ws_bytes, const dsa::DevCtl& ctl, int num_sms, cudaStream_t stream,
            Recorder& rec = g_no_rec, bool fit_splits = false,
            const dsa_paged_cache* pc = nullptr) {
  // Key splits for this device's SM count. Workspaces are sized for assumed_sms()
  // (no device needed), and fewer SMs never need more splits, so a device with
  // more SMs than that is scheduled as if it had assumed_sms().
  const int sched_sms = (num_sms > 0 && num_sms < assumed_sms()) ? num_sms : assumed_sms();
  int splits = mla_splits(B, Lq, Dv, k, sched_sms);
  // fit_splits: use fewer key splits rather than fail when the partials of the
  // recommended count do not fit (one split needs none)
  while (fit_splits && splits > 1 && mla_ws_bytes(B, Lq, H, Dv, splits) > ws_bytes) --splits;
  size_t need = mla_ws_bytes(B, Lq, H, Dv, splits);
  if (ws_bytes < need)
    return fail(DSA_ERR_WORKSPACE_TOO_SMALL, "sparse MLA workspace: need %zu bytes, got %zu", need, ws_bytes);
  CUtensorMap tq;
  DSA_TRY(make_map_2d(&tq, q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)Dqk,
                      (uint64_t)B * Lq * H, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B));
  dsa::MlaArgs a{};
  a.q = q;
  a.idx = idx;
  a.out = out;
  a.lse = lse;
  a.B = B; a.Lq = Lq; a.Lk = Lk; a.H = H; a.Dqk = Dqk; a.Dv = Dv; a.k = k;
  a.scale_log2 = sm_scale * 1.4426950408889634f;
  a.n_dv = mla_n_dv(Dv);
  a.splits = splits;
  a.wave = num_sms > 0 ? num_sms : assumed_sms();
  if (pc != nullptr) {   // kv is a pool of pages
    a.block_table = pc->block_table;
    a.max_blocks = pc->max_blocks;
    a.page_size = pc->page_size;
    a.num_pages = pc->num_pages;
  }
  a.ctl = ctl;
  if (splits > 1) {
    size_t tok = (size_t)B * Lq;
    a.part_o = static_cast<float*>(ws);
    a.part_ml = reinterpret_cast<float*>(static_cast<char*>(ws) +
                                         align_up(tok * splits * H * Dv * sizeof(float), 256));
  }
  {
    NvtxRange r("dsa:sparse_mla");
    DSA_TRY_CUDA(dsa::launch_sparse_mla(tq, kv, a, stream), "sparse MLA launch");
  }
  DSA_TRY(rec.mark(DSA_KIND_SPARSE_MLA, stream));
  if (splits > 1) {
    NvtxRange r("dsa:mla_combine");
    DSA_TRY_CUDA(dsa::launch_mla_combine(a, stream), "split combine launch");
    DSA_TRY(rec.mark(DSA_KIND_COMBINE, stream));
  }
  return DSA_OK;
}

struct ForwardPlan {
  int chunk;         // query rows per chunk
  long long ld;      // score row stride (floats)
  size_t scores_bytes, idx_bytes, cnt_bytes, mla_bytes, total;
};

// Rows of problem p that are scored: those with p + 1 > k, or every row when the
// selected scores are returned.
int first_scored_row(const dsa_problem* p, bool score_all) {
  if (score_all) return 0;
  const int f = p->k - p->q_pos0;
  return f < 0 ? 0 : f;
}

// Workspace, in order: a score chunk of B x chunk x round4(Lk) fp32, the selected
// keys (when the caller does not want them back), one counter per row of a chunk
// (pieces scored, for the fused selection), and the attention's split partials.
ForwardPlan plan_forward(const dsa_problem* p, bool need_idx, size_t ws_bytes_or_zero,
                         bool score_all = false) {
  ForwardPlan f{};
  f.ld = (long long)align_up((size_t)p->Lk, 4);
  const size_t row_bytes = (size_t)p->B * f.ld * sizeof(float);
  f.idx_bytes = need_idx ? align_up((size_t)p->B * p->Lq * p->k * sizeof(int32_t), 256) : 0;
  f.mla_bytes = align_up(mla_ws_bytes(p->B, p->Lq, p->H, p->Dv,
                                      mla_splits(p->B, p->Lq, p->Dv, p->k, assumed_sms())), 256);
  const int scored_rows = p->Lq - first_scored_row(p, score_all);
  if (scored_rows <= 0) {
    f.chunk = p->Lq;
    f.scores_bytes = 0;
  } else {
    // default: about 64 MB of scores per chunk so one chunk stays in L2
    long long c = (64ll << 20) / (long long)row_bytes;
    if (c > scored_rows) c = scored_rows;
    if (c >= 4) c &= ~3ll;
    if (c < 4) c = scored_rows < 4 ? scored_rows : 4;
    if (ws_bytes_or_zero) {
      // as many rows as the given workspace holds (scores and counters), down to 1
      auto total_for = [&](long long rows) {
        return f.idx_bytes + f.mla_bytes + align_up((size_t)rows * row_bytes, 256) +
               align_up((size_t)p->B * rows * sizeof(int), 256) + 256;
      };
      const size_t fixed = f.idx_bytes + f.mla_bytes;
      c = ws_bytes_or_zero > fixed ? (long long)((ws_bytes_or_zero - fixed) / row_bytes) : 0;
      if (c > scored_rows) c = scored_rows;
      while (c > 0 && total_for(c) > ws_bytes_or_zero) --c;
      if (c >= 4) c &= ~3ll;
    }
    f.chunk = (int)c;
    f.scores_bytes = align_up((size_t)c * row_bytes, 256);
  }
  f.cnt_bytes = align_up((size_t)p->B * (f.chunk > 0 ? f.chunk : 1) * sizeof(int), 256);
  f.total = f.scores_bytes + f.idx_bytes + f.cnt_bytes + f.mla_bytes + (f.scores_bytes ? 256 : 0);
  return f;
}

// Smallest workspace dsa_forward accepts: the fixed parts plus score rows and
// counters for one chunk of min(4, scored rows) query rows.
size_t min_forward_bytes(const dsa_problem* p, const ForwardPlan& f, bool score_all = false) {
  const int scored_rows = p->Lq - first_scored_row(p, score_all);
  const size_t rows = scored_rows <= 0 ? 0 : (size_t)(scored_rows < 4 ? scored_rows : 4);
  if (rows == 0) return f.idx_bytes + f.mla_bytes + f.cnt_bytes;
  return f.idx_bytes + f.mla_bytes + align_up(rows * (size_t)p->B * f.ld * sizeof(float), 256) +
         align_up(rows * (size_t)p->B * sizeof(int), 256) + 256;
}

int validate_problem(const dsa_problem* p) {
  if (!p) return fail(DSA_ERR_INVALID_ARG, "problem is NULL");
  DSA_TRY(check_seq(p->B, p->Lq, p->Lk, p->q_pos0));
  DSA_TRY(check_indexer_shape(p->H_I, p->d_I, p->B, p->Lq));
  DSA_TRY(check_mla_shape(p->H, p->Dqk, p->Dv, p->B, p->Lq));
  DSA_TRY(check_k(p->k, 2048));
  if (p->w_dtype != DSA_DTYPE_F32 && p->w_dtype != DSA_DTYPE_BF16)
    return fail(DSA_ERR_INVALID_ARG, "w_dtype must be DSA_DTYPE_F32 or DSA_DTYPE_BF16");
  if (!(p->sm_scale > 0.f) || !std::isfinite(p->sm_scale))
    return fail(DSA_ERR_INVALID_ARG, "sm_scale must be finite and > 0");
  if (p->mode != DSA_MODE_PREFILL && p->mode != DSA_MODE_DECODE)
    return fail(DSA_ERR_INVALID_ARG, "mode must be DSA_MODE_PREFILL or DSA_MODE_DECODE");
  return DSA_OK;
}

int validate_tensors(const dsa_tensors* t) {
  if (!t) return fail(DSA_ERR_INVALID_ARG, "tensors is NULL");
  DSA_TRY(check_ptr(t->qI, "qI"));
  DSA_TRY(check_ptr(t->qI_scale, "qI_scale"));
  DSA_TRY(check_ptr(t->kI, "kI"));
  DSA_TRY(check_ptr(t->kI_scale, "kI_scale"));
  DSA_TRY(check_ptr(t->w, "w"));
  DSA_TRY(check_ptr(t->out, "out", true));
  DSA_TRY(check_ptr(t->idx_out, "idx_out", true));
  if (t->out == nullptr) {   // selection only: q, kv and lse are not read
    if (t->idx_out == nullptr)
      return fail(DSA_ERR_INVALID_ARG, "out is NULL: a selection-only call needs idx_out");
    return DSA_OK;
  }
  DSA_TRY(check_ptr(t->q, "q"));
  DSA_TRY(check_ptr(t->kv, "kv"));
  DSA_TRY(check_ptr(t->lse, "lse", true));
  return DSA_OK;
}

// Fused top-k selection of rows [t0, t1) of every sequence by the indexer launch.
struct FusedSelect {
  int k = 0;
  int t0 = 0, t1 = 0;
  int32_t* idx = nullptr;
  float* sel_scores = nullptr;
  int* row_cnt = nullptr;
};

int launch_indexer_rows(const uint8_t* qI, const float* qI_scale, const uint8_t* kI,
                        const float* kI_scale, const void* w, int w_dtype, float* scores,
                        long long sc_ld, long long sc_bstride, int sc_t0, int B, int Lq, int Lk,
                        int q_pos0, int H_I, int d_I, int t_lo, int t_hi, const dsa::DevCtl& ctl,
                        int num_sms, cudaStream_t stream, Recorder& rec = g_no_rec,
                        const dsa_paged_cache* pc = nullptr, const FusedSelect* fs = nullptr) {
  if (fs == nullptr && t_hi <= t_lo) return DSA_OK;
  if (t_hi < t_lo) t_hi = t_lo;
  const int n_tok = (H_I == 64) ? ((t_hi - t_lo == 1) ? 1 : 4) : 64;
  CUtensorMap tq, tk;
  DSA_TRY(make_map_2d(&tq, qI, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)d_I,
                      (uint64_t)B * Lq * H_I, (uint32_t)d_I, (uint32_t)(n_tok * H_I),
                      d_I == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_32B));
  // key rows: the sequences one after another, or the page pool
  const uint64_t k_rows = pc != nullptr ? (uint64_t)pc->num_pages * pc->page_size : (uint64_t)B * Lk;
  DSA_TRY(make_map_2d(&tk, kI, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)d_I, k_rows,
                      (uint32_t)d_I, 128,
                      d_I == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_32B));
  dsa::IndexerArgs a{};
  a.qI_scale = qI_scale;
  a.w = w;
  a.w_bf16 = w_dtype == DSA_DTYPE_BF16;
  a.kI_scale = kI_scale;
  a.scores = scores;
  a.sc_ld = sc_ld;
  a.sc_bstride = sc_bstride;
  a.sc_t0 = sc_t0;
  a.B = B; a.Lq = Lq; a.Lk = Lk; a.q_pos0 = q_pos0;
  a.t_lo = t_lo; a.t_hi = t_hi;
  if (pc != nullptr) {
    a.seq_lens = pc->seq_lens;
    a.block_table = pc->block_table;
    a.max_blocks = pc->max_blocks;
    a.page_size = pc->page_size;
    a.num_pages = pc->num_pages;
  }
  int keys_max = q_pos0 + t_hi < Lk ? q_pos0 + t_hi : Lk;
  a.piece_keys = t_hi > t_lo ? indexer_piece_keys(B, t_hi - t_lo, n_tok, keys_max, num_sms) : 128;
  a.ctl = ctl;
  if (fs != nullptr) {
    a.select = 1;
    a.k = fs->k;
    a.sel_t0 = fs->t0;
    a.sel_t1 = fs->t1;
    a.idx = fs->idx;
    a.sel_scores = fs->sel_scores;
    a.row_cnt = fs->row_cnt;
  }
  {
    NvtxRange r(fs != nullptr ? "dsa:indexer_topk" : "dsa:indexer");
    DSA_TRY_CUDA(dsa::launch_indexer(tq, tk, a, H_I, d_I, num_sms, stream),
                 fs != nullptr ? "indexer + top-k launch" : "indexer launch");
  }
  DSA_TRY(rec.mark(fs != nullptr ? DSA_KIND_INDEXER_TOPK : DSA_KIND_INDEXER, stream));
  return DSA_OK;
}

}  // namespace

extern "C" {

const char* dsa_last_error(void) { return g_err.c_str(); }

const char* dsa_version(void) { return "dsa-b200 0.1 (sm_100a)"; }

int dsa_indexer_scores(const uint8_t* qI, const float* qI_scale, const uint8_t* kI,
                       const float* kI_scale, const void* w, int w_dtype, float* scores, int B,
                       int Lq, int Lk, int q_pos0, int H_I, int d_I, void* stream) {
  DSA_TRY(check_ptr(qI, "qI"));
  DSA_TRY(check_ptr(qI_scale, "qI_scale"));
  DSA_TRY(check_ptr(kI, "kI"));
  DSA_TRY(check_ptr(kI_scale, "kI_scale"));
  DSA_TRY(check_ptr(w, "w"));
  DSA_TRY(check_ptr(scores, "scores"));
  DSA_TRY(check_seq(B, Lq, Lk, q_pos0));
  DSA_TRY(check_indexer_shape(H_I, d_I, B, Lq));
  if (w_dtype != DSA_DTYPE_F32 && w_dtype != DSA_DTYPE_BF16)
    return fail(DSA_ERR_INVALID_ARG, "w_dtype must be DSA_DTYPE_F32 or DSA_DTYPE_BF16");
  dsa::DevCtl ctl;
  int sms = 0;
  DSA_TRY(device_ctl(ctl, sms));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  DSA_TRY_CUDA(dsa::launch_fill_noncausal(scores, B, Lq, Lk, q_pos0, s), "fill launch");
  return launch_indexer_rows(qI, qI_scale, kI, kI_scale, w, w_dtype, scores, Lk, Lq, 0, B, Lq, Lk,
                             q_pos0, H_I, d_I, 0, Lq, ctl, sms, s);
}

int dsa_topk_select(const float* scores, int32_t* idx, int B, int Lq, int Lk, int q_pos0, int k,
                    void* stream) {
  DSA_TRY(check_ptr(scores, "scores"));
  DSA_TRY(check_ptr(idx, "idx"));
  DSA_TRY(check_seq(B, Lq, Lk, q_pos0));
  DSA_TRY(check_k(k, 4096));
  dsa::DevCtl ctl;
  int sms = 0;
  DSA_TRY(device_ctl(ctl, sms));
  dsa::TopkArgs a{};
  a.scores = scores;
  a.sc_ld = Lk;
  a.sc_bstride = Lq;
  a.sc_t0 = 0;
  a.idx = idx;
  a.B = B; a.Lq = Lq; a.Lk = Lk; a.q_pos0 = q_pos0; a.k = k;
  a.t_lo = 0; a.t_hi = Lq;
  a.vec4 = (Lk % 4) == 0;
  a.ctl = ctl;
  DSA_TRY_CUDA(dsa::launch_topk(a, sms, static_cast<cudaStream_t>(stream)), "top-k launch");
  return DSA_OK;
}

size_t dsa_sparse_mla_workspace_size(int B, int Lq, int Lk, int H, int Dqk, int Dv, int k) {
  (void)Lk; (void)Dqk;
  if (B < 1 || Lq < 1 || k < 32) return 0;
  return mla_ws_bytes(B, Lq, H, Dv, mla_splits(B, Lq, Dv, k, assumed_sms()));
}

int dsa_sparse_mla_fwd(const uint16_t* q, const uint16_t* kv, const int32_t* idx, uint16_t* out,
                       float* lse, int B, int Lq, int Lk, int H, int Dqk, int Dv, int k,
                       float sm_scale, void* ws, size_t ws_bytes, void* stream) {
  DSA_TRY(check_ptr(q, "q"));
  DSA_TRY(check_ptr(kv, "kv"));
  DSA_TRY(check_ptr(idx, "idx"));
  DSA_TRY(check_ptr(out, "out"));
  DSA_TRY(check_ptr(lse, "lse", true));
  DSA_TRY(check_ptr(ws, "ws", true));
  if (B < 1 || Lq < 1 || Lk < 1) return fail(DSA_ERR_INVALID_ARG, "B, Lq, Lk must be >= 1");
  if ((long long)B * Lk > (1LL << 30)) return fail(DSA_ERR_UNSUPPORTED_SHAPE, "B*Lk must be <= 2^30");
  DSA_TRY(check_mla_shape(H, Dqk, Dv, B, Lq));
  DSA_TRY(check_k(k, 4096));
  if (!(sm_scale > 0.f) || !std::isfinite(sm_scale))
    return fail(DSA_ERR_INVALID_ARG, "sm_scale must be finite and > 0");
  if (ws == nullptr && ws_bytes != 0) return fail(DSA_ERR_INVALID_ARG, "ws is NULL but ws_bytes > 0");
  dsa::DevCtl ctl;
  int sms = 0;
  DSA_TRY(device_ctl(ctl, sms));
  return run_mla(q, kv, idx, out, lse, B, Lq, Lk, H, Dqk, Dv, k, sm_scale, ws, ws_bytes, ctl, sms,
                 static_cast<cudaStream_t>(stream));
}

int dsa_indexer_kl(const uint16_t* q, const uint16_t* kv, const int32_t* idx, const float* lse,
                   const float* sel_scores, float* p_out, float* kl_out, int B, int Lq, int Lk,
                   int H, int Dqk, int k, float sm_scale, void* stream) {
  DSA_TRY(check_ptr(q, "q"));
  DSA_TRY(check_ptr(kv, "kv"));
  DSA_TRY(check_ptr(idx, "idx"));
  DSA_TRY(check_ptr(lse, "lse"));
  DSA_TRY(check_ptr(sel_scores, "sel_scores"));
  DSA_TRY(check_ptr(p_out, "p_out", true));
  DSA_TRY(check_ptr(kl_out, "kl_out"));
  if (B < 1 || Lq < 1 || Lk < 1) return fail(DSA_ERR_INVALID_ARG, "B, Lq, Lk must be >= 1");
  if ((long long)B * Lk > (1LL << 30)) return fail(DSA_ERR_UNSUPPORTED_SHAPE, "B*Lk must be <= 2^30");
  if (!((H == 128 && Dqk == 576) || (H == 8 && Dqk == 80)))
    return fail(DSA_ERR_UNSUPPORTED_SHAPE, "(H, Dqk) = (%d, %d) unsupported; use (128, 576) or (8, 80)", H, Dqk);
  if ((long long)B * Lq * H > (1LL << 31) - 1 || (long long)B * Lq > (1LL << 31) - 1)
    return fail(DSA_ERR_UNSUPPORTED_SHAPE, "B*Lq*H too large");
  DSA_TRY(check_k(k, 4096));
  if (!(sm_scale > 0.f) || !std::isfinite(sm_scale))
    return fail(DSA_ERR_INVALID_ARG, "sm_scale must be finite and > 0");
  dsa::DevCtl ctl;
  int sms = 0;
  DSA_TRY(device_ctl(ctl, sms));
  dsa::KlArgs a{};
  a.q = q;
  a.idx = idx;
  a.lse = lse;
  a.sel = sel_scores;
  a.p_out = p_out;
  a.kl_out = kl_out;
  a.B = B; a.Lq = Lq; a.Lk = Lk; a.H = H; a.Dqk = Dqk; a.k = k;
  a.scale_log2 = sm_scale * 1.4426950408889634f;
  a.ctl = ctl;
  DSA_TRY_CUDA(dsa::launch_indexer_kl(kv, a, static_cast<cudaStream_t>(stream)), "indexer KL launch");
  return DSA_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free variant of dsa_sparse_mla_fwd.
//
// Its key-split partials live in a fixed device array compiled into the
// library instead of a caller-provided workspace. Every GPU that loads the
// library holds this array until the process exits. Host code only sees a
// host-side stand-in for the symbol, so the device address is looked up once
// per device with cudaGetSymbolAddress (device current) and cached.
// ---------------------------------------------------------------------------
namespace {
constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;   // 16 MiB
__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];
void* g_noalloc_ptr[kMaxDevices] = {nullptr};

int noalloc_scratch(void** out) {
  int dev = 0;
  DSA_TRY_CUDA(cudaGetDevice(&dev), "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(DSA_ERR_CUDA, "device ordinal %d out of range", dev);
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* p = nullptr;
    DSA_TRY_CUDA(cudaGetSymbolAddress(&p, g_noalloc_scratch), "cudaGetSymbolAddress(scratch)");
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return DSA_OK;
}
}  // namespace

extern "C" {

int dsa_sparse_mla_fwd_noalloc(const uint16_t* q, const uint16_t* kv, const int32_t* idx,
                               uint16_t* out, float* lse, int B, int Lq, int Lk, int H, int Dqk,
                               int Dv, int k, float sm_scale, void* stream) {
  DSA_TRY(check_ptr(q, "q"));
  DSA_TRY(check_ptr(kv, "kv"));
  DSA_TRY(check_ptr(idx, "idx"));
  DSA_TRY(check_ptr(out, "out"));
  DSA_TRY(check_ptr(lse, "lse", true));
  if (B < 1 || Lq < 1 || Lk < 1) return fail(DSA_ERR_INVALID_ARG, "B, Lq, Lk must be >= 1");
  if ((long long)B * Lk > (1LL << 30)) return fail(DSA_ERR_UNSUPPORTED_SHAPE, "B*Lk must be <= 2^30");
  DSA_TRY(check_mla_shape(H, Dqk, Dv, B, Lq));
  DSA_TRY(check_k(k, 4096));
  if (!(sm_scale > 0.f) || !std::isfinite(sm_scale))
    return fail(DSA_ERR_INVALID_ARG, "sm_scale must be finite and > 0");
  dsa::DevCtl ctl;
  int sms = 0;
  DSA_TRY(device_ctl(ctl, sms));
  void* scratch = nullptr;
  DSA_TRY(noalloc_scratch(&scratch));
  return run_mla(q, kv, idx, out, lse, B, Lq, Lk, H, Dqk, Dv, k, sm_scale, scratch,
                 kNoAllocScratchBytes, ctl, sms, static_cast<cudaStream_t>(stream), g_no_rec,
                 /*fit_splits=*/true);
}

size_t dsa_forward_workspace_size(const dsa_problem* p) {
  if (validate_problem(p) != DSA_OK) return 0;
  // enough for either schedule: with sel_scores_out every row is scored
  const size_t a = plan_forward(p, true, 0, false).total, b = plan_forward(p, true, 0, true).total;
  return a > b ? a : b;
}

}  // extern "C"

namespace {
// Per-device side stream and events on which dsa_forward overlaps the top-k of
// one score chunk with the indexer of the next. Created on first use and kept for
// the life of the process; the mutex keeps one call's sequence of records and
// waits on them from interleaving with another call's.
struct SideStream {
  std::mutex mu;
  bool ready = false;
  cudaStream_t side = nullptr;
  cudaEvent_t scored[2] = {nullptr, nullptr};    // indexer of the chunk in buffer b done
  cudaEvent_t selected[2] = {nullptr, nullptr};  // top-k of the chunk in buffer b done
};
SideStream g_side[kMaxDevices];

int side_stream(SideStream** out) {
  int dev = 0;
  DSA_TRY_CUDA(cudaGetDevice(&dev), "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(DSA_ERR_UNSUPPORTED_SHAPE, "device index %d", dev);
  SideStream& r = g_side[dev];
  std::lock_guard<std::mutex> lk(r.mu);
  if (!r.ready) {
    DSA_TRY_CUDA(cudaStreamCreateWithFlags(&r.side, cudaStreamNonBlocking), "cudaStreamCreate");
    for (int b = 0; b < 2; ++b) {
      DSA_TRY_CUDA(cudaEventCreateWithFlags(&r.scored[b], cudaEventDisableTiming), "cudaEventCreate");
      DSA_TRY_CUDA(cudaEventCreateWithFlags(&r.selected[b], cudaEventDisableTiming), "cudaEventCreate");
    }
    r.ready = true;
  }
  *out = &r;
  return DSA_OK;
}

// Copy streams of dsa_forward_host's pipeline, per device, created on first use.
constexpr int kHostPipeRows = 4096;      // query rows per pipelined block
constexpr int kHostPipeMinRows = 1024;   // shorter problems are not split
constexpr int kHostPipeEvents = 64;      // ring of events (reused in order)
struct HostPipe {
  std::mutex mu;
  bool ready = false;
  cudaStream_t in = nullptr, out = nullptr;
  cudaEvent_t start = nullptr;
  cudaEvent_t in_done[kHostPipeEvents] = {};
  cudaEvent_t computed[kHostPipeEvents] = {};
};
HostPipe g_host_pipe[kMaxDevices];

int host_pipe(HostPipe** out) {
  int dev = 0;
  DSA_TRY_CUDA(cudaGetDevice(&dev), "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(DSA_ERR_UNSUPPORTED_SHAPE, "device index %d", dev);
  HostPipe& r = g_host_pipe[dev];
  std::lock_guard<std::mutex> lk(r.mu);
  if (!r.ready) {
    DSA_TRY_CUDA(cudaStreamCreateWithFlags(&r.in, cudaStreamNonBlocking), "cudaStreamCreate");
    DSA_TRY_CUDA(cudaStreamCreateWithFlags(&r.out, cudaStreamNonBlocking), "cudaStreamCreate");
    DSA_TRY_CUDA(cudaEventCreateWithFlags(&r.start, cudaEventDisableTiming), "cudaEventCreate");
    for (int i = 0; i < kHostPipeEvents; ++i) {
      DSA_TRY_CUDA(cudaEventCreateWithFlags(&r.in_done[i], cudaEventDisableTiming), "cudaEventCreate");
      DSA_TRY_CUDA(cudaEventCreateWithFlags(&r.computed[i], cudaEventDisableTiming), "cudaEventCreate");
    }
    r.ready = true;
  }
  *out = &r;
  return DSA_OK;
}

dsa::TopkArgs topk_args(const dsa_problem* p, const float* scores, long long ld, int bstride,
                        int t0, int t1, int32_t* idx, const dsa::DevCtl& ctl,
                        const dsa_paged_cache* pc, float* sel_scores = nullptr) {
  dsa::TopkArgs ta{};
  ta.scores = scores;
  ta.sc_ld = ld;
  ta.sc_bstride = bstride;
  ta.sc_t0 = t0;
  ta.idx = idx;
  ta.sel = sel_scores;
  ta.B = p->B; ta.Lq = p->Lq; ta.Lk = p->Lk; ta.q_pos0 = p->q_pos0; ta.k = p->k;
  ta.t_lo = t0; ta.t_hi = t1;
  ta.vec4 = 1;
  ta.seq_lens = pc != nullptr ? pc->seq_lens : nullptr;
  ta.ctl = ctl;
  return ta;
}

// fused: one cooperative indexer + top-k launch per score chunk (dsa_forward_fused);
// otherwise the indexer scores a chunk and a separate top-k kernel selects it
// (overlapped on a side stream: the indexer scores the next half-chunk meanwhile).
int forward_impl(const dsa_problem* p, const dsa_tensors* t, void* ws, size_t ws_bytes,
                 void* stream, Recorder& rec, const dsa_paged_cache* pc = nullptr,
                 bool fused = false) {
  NvtxRange whole("dsa_forward");
  DSA_TRY(validate_problem(p));
  DSA_TRY(validate_tensors(t));
  DSA_TRY(check_ptr(ws, "ws", true));
  const bool need_idx = t->idx_out == nullptr;
  const bool score_all = t->sel_scores_out != nullptr;
  if (score_all && need_idx)
    return fail(DSA_ERR_INVALID_ARG, "sel_scores_out needs idx_out (the scores are aligned with it)");
  ForwardPlan rec_plan = plan_forward(p, need_idx, 0, score_all);
  const size_t min_bytes = min_forward_bytes(p, rec_plan, score_all);
  if (ws_bytes < min_bytes)
    return fail(DSA_ERR_WORKSPACE_TOO_SMALL,
                "dsa_forward workspace: need at least %zu bytes (recommended %zu), got %zu",
                min_bytes, rec_plan.total, ws_bytes);
  if (ws == nullptr) return fail(DSA_ERR_INVALID_ARG, "ws is NULL");
  ForwardPlan f = plan_forward(p, need_idx, ws_bytes, score_all);
  dsa::DevCtl ctl;
  int sms = 0;
  DSA_TRY(device_ctl(ctl, sms));
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  char* wsb = static_cast<char*>(ws);
  float* scores = f.scores_bytes ? reinterpret_cast<float*>(wsb) : nullptr;
  int32_t* idx = need_idx ? reinterpret_cast<int32_t*>(wsb + f.scores_bytes) : t->idx_out;
  int* row_cnt = reinterpret_cast<int*>(wsb + f.scores_bytes + f.idx_bytes);
  void* mla_ws = wsb + f.scores_bytes + f.idx_bytes + f.cnt_bytes;

  // the attention step; a selection-only call (out == NULL) ends after the top-k
  auto attend = [&]() -> int {
    if (t->out == nullptr) return DSA_OK;
    return run_mla(t->q, t->kv, idx, t->out, t->lse, p->B, p->Lq, p->Lk, p->H, p->Dqk, p->Dv, p->k,
                   p->sm_scale, mla_ws, f.mla_bytes, ctl, sms, s, rec, false, pc);
  };
  const int first_scored = first_scored_row(p, score_all);
  if (first_scored < p->Lq && (f.chunk < 1 || f.scores_bytes == 0 || f.total > ws_bytes))
    return fail(DSA_ERR_WORKSPACE_TOO_SMALL, "dsa_forward workspace: no room for one score row");
  const int C = f.chunk > 0 ? f.chunk : p->Lq;
  // One fused indexer + top-k launch per chunk of C query rows: the chunk's scored
  // rows are scored into the workspace and every row of the chunk is selected by
  // the same kernel as soon as it is complete. The per-row piece counters start at
  // zero and each launch leaves them at zero.
  if (first_scored >= p->Lq) {
    // Short context: every row has at most k candidates and selects all of them, so
    // nothing is scored; one selection launch fills the index rows.
    dsa::TopkArgs ta{};
    ta.idx = idx;
    ta.B = p->B; ta.Lq = p->Lq; ta.Lk = p->Lk; ta.q_pos0 = p->q_pos0; ta.k = p->k;
    ta.t_lo = 0; ta.t_hi = p->Lq;
    ta.seq_lens = pc != nullptr ? pc->seq_lens : nullptr;
    ta.ctl = ctl;
    {
      NvtxRange nr("dsa:topk");
      DSA_TRY_CUDA(dsa::launch_topk(ta, sms, s), "top-k launch");
    }
    DSA_TRY(rec.mark(DSA_KIND_TOPK, s));
    return attend();
  }
  if (!fused) {
    // Overlapped schedule: the score area holds two half-size chunk buffers; the
    // top-k of a chunk runs on the side stream while the indexer scores the next
    // chunk into the other buffer (their CTAs fit on one SM together). The
    // profiling entry point keeps the serial schedule so that each launch's events
    // time that launch alone.
    const int C2 = (C / 2) & ~3;
    if (rec.events == nullptr && f.scores_bytes > 0 && C2 >= 4) {
      SideStream* r = nullptr;
      DSA_TRY(side_stream(&r));
      std::lock_guard<std::mutex> lk(r->mu);
      const size_t half = (size_t)p->B * C2 * (size_t)f.ld;   // floats per buffer
      int c = 0;
      for (int t0 = 0; t0 < p->Lq; t0 += C2, ++c) {
        const int t1 = t0 + C2 < p->Lq ? t0 + C2 : p->Lq;
        const int ts = t0 > first_scored ? t0 : first_scored;
        const int b = c & 1;
        float* sb = scores + b * half;
        // the buffer's previous chunk must have been selected before it is rewritten
        if (c >= 2) DSA_TRY_CUDA(cudaStreamWaitEvent(s, r->selected[b], 0), "cudaStreamWaitEvent");
        if (ts < t1) {
          DSA_TRY(launch_indexer_rows(t->qI, t->qI_scale, t->kI, t->kI_scale, t->w, p->w_dtype, sb,
                                      f.ld, C2, t0, p->B, p->Lq, p->Lk, p->q_pos0, p->H_I, p->d_I, ts,
                                      t1, ctl, sms, s, rec, pc));
        }
        DSA_TRY_CUDA(cudaEventRecord(r->scored[b], s), "cudaEventRecord");
        DSA_TRY_CUDA(cudaStreamWaitEvent(r->side, r->scored[b], 0), "cudaStreamWaitEvent");
        {
          NvtxRange nr("dsa:topk");
          DSA_TRY_CUDA(dsa::launch_topk(topk_args(p, sb, f.ld, C2, t0, t1, idx, ctl, pc, t->sel_scores_out),
                                        sms, r->side),
                       "top-k launch");
        }
        DSA_TRY(rec.mark(DSA_KIND_TOPK, r->side));   // counts it (no events on this path)
        DSA_TRY_CUDA(cudaEventRecord(r->selected[b], r->side), "cudaEventRecord");
      }
      // top-k launches run in order on the side stream: the last one covers all
      if (c >= 1) DSA_TRY_CUDA(cudaStreamWaitEvent(s, r->selected[(c - 1) & 1], 0), "cudaStreamWaitEvent");
    } else {
      for (int t0 = 0; t0 < p->Lq; t0 += C) {
        const int t1 = t0 + C < p->Lq ? t0 + C : p->Lq;
        const int ts = t0 > first_scored ? t0 : first_scored;
        if (ts < t1) {
          DSA_TRY(launch_indexer_rows(t->qI, t->qI_scale, t->kI, t->kI_scale, t->w, p->w_dtype, scores,
                                      f.ld, C, t0, p->B, p->Lq, p->Lk, p->q_pos0, p->H_I, p->d_I, ts,
                                      t1, ctl, sms, s, rec, pc));
        }
        {
          NvtxRange nr("dsa:topk");
          DSA_TRY_CUDA(dsa::launch_topk(topk_args(p, scores, f.ld, C, t0, t1, idx, ctl, pc, t->sel_scores_out),
                                        sms, s),
                       "top-k launch");
        }
        DSA_TRY(rec.mark(DSA_KIND_TOPK, s));
      }
    }
    return attend();
  }
  DSA_TRY_CUDA(cudaMemsetAsync(row_cnt, 0, f.cnt_bytes, s), "row counter clear");
  FusedSelect fs;
  fs.k = p->k;
  fs.idx = idx;
  fs.sel_scores = t->sel_scores_out;
  fs.row_cnt = row_cnt;
  for (int t0 = 0; t0 < p->Lq; t0 += C) {
    const int t1 = t0 + C < p->Lq ? t0 + C : p->Lq;
    const int ts = t0 > first_scored ? t0 : first_scored;
    fs.t0 = t0;
    fs.t1 = t1;
    DSA_TRY(launch_indexer_rows(t->qI, t->qI_scale, t->kI, t->kI_scale, t->w, p->w_dtype, scores,
                                f.ld, C, t0, p->B, p->Lq, p->Lk, p->q_pos0, p->H_I, p->d_I, ts,
                                ts < t1 ? t1 : ts, ctl, sms, s, rec, pc, &fs));
  }
  return attend();
}

// A paged problem is scheduled as the uniform problem whose rows sit as late as
// the capacity allows (q_pos0 = Lk - Lq): a row that needs no scores there needs
// none in any sequence, since every sequence is at most Lk tokens long.
dsa_problem paged_schedule_problem(const dsa_problem* p) {
  dsa_problem pp = *p;
  pp.q_pos0 = p->Lk - p->Lq;
  return pp;
}

int validate_paged(const dsa_problem* p, const dsa_paged_cache* pc) {
  if (pc == nullptr) return fail(DSA_ERR_INVALID_ARG, "paged cache is NULL");
  DSA_TRY(check_ptr(pc->block_table, "block_table"));
  DSA_TRY(check_ptr(pc->seq_lens, "seq_lens"));
  if (pc->page_size < 128 || pc->page_size % 128 != 0)
    return fail(DSA_ERR_UNSUPPORTED_SHAPE, "page_size = %d: need a multiple of 128", pc->page_size);
  if (pc->max_blocks < 1 || pc->num_pages < 1)
    return fail(DSA_ERR_INVALID_ARG, "max_blocks and num_pages must be >= 1");
  if ((long long)pc->max_blocks * pc->page_size != p->Lk)
    return fail(DSA_ERR_INVALID_ARG, "Lk = %d must equal max_blocks * page_size = %lld", p->Lk,
                (long long)pc->max_blocks * pc->page_size);
  if ((long long)pc->num_pages * pc->page_size > (1LL << 30))
    return fail(DSA_ERR_UNSUPPORTED_SHAPE, "num_pages * page_size must be <= 2^30");
  return DSA_OK;
}
}  // namespace

extern "C" {

int dsa_forward(const dsa_problem* p, const dsa_tensors* t, void* ws, size_t ws_bytes,
                void* stream) {
  Recorder none;
  const int rc = forward_impl(p, t, ws, ws_bytes, stream, none);
  g_last_launches = none.launched;
  return rc;
}

int dsa_forward_fused(const dsa_problem* p, const dsa_tensors* t, void* ws, size_t ws_bytes,
                      void* stream) {
  Recorder none;
  const int rc = forward_impl(p, t, ws, ws_bytes, stream, none, nullptr, /*fused=*/true);
  g_last_launches = none.launched;
  return rc;
}

int dsa_last_launch_count(void) { return g_last_launches; }

size_t dsa_forward_paged_workspace_size(const dsa_problem* p) {
  if (p == nullptr) return 0;
  const dsa_problem pp = paged_schedule_problem(p);
  return dsa_forward_workspace_size(&pp);
}

int dsa_forward_paged(const dsa_problem* p, const dsa_tensors* t, const dsa_paged_cache* pc,
                      void* ws, size_t ws_bytes, void* stream) {
  if (p == nullptr) return fail(DSA_ERR_INVALID_ARG, "problem is NULL");
  const dsa_problem pp = paged_schedule_problem(p);
  DSA_TRY(validate_problem(&pp));
  DSA_TRY(validate_paged(&pp, pc));
  Recorder none;
  const int rc = forward_impl(&pp, t, ws, ws_bytes, stream, none, pc);
  g_last_launches = none.launched;
  return rc;
}

int dsa_forward_profiled(const dsa_problem* p, const dsa_tensors* t, void* ws, size_t ws_bytes,
                         void* stream, void* const* events, int* kinds, int max_launches,
                         int* n_launches) {
  if (events == nullptr || kinds == nullptr || n_launches == nullptr || max_launches < 1)
    return fail(DSA_ERR_INVALID_ARG, "profiling arrays are NULL or empty");
  for (int i = 0; i <= max_launches; ++i)
    if (events[i] == nullptr) return fail(DSA_ERR_INVALID_ARG, "events[%d] is NULL", i);
  *n_launches = 0;
  Recorder rec;
  rec.events = events;
  rec.kinds = kinds;
  rec.cap = max_launches;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  DSA_TRY(validate_problem(p));
  DSA_TRY_CUDA(cudaEventRecord(static_cast<cudaEvent_t>(events[0]), s), "cudaEventRecord");
  int r = forward_impl(p, t, ws, ws_bytes, stream, rec);
  *n_launches = rec.n;
  g_last_launches = rec.launched;
  return r;
}

int dsa_forward_host(const dsa_problem* p, const dsa_tensors* host, const dsa_tensors* dev,
                     void* ws, size_t ws_bytes, void* stream) {
  DSA_TRY(validate_problem(p));
  if (!host) return fail(DSA_ERR_INVALID_ARG, "host tensors is NULL");
  DSA_TRY(validate_tensors(dev));
  const char* names[7] = {"host qI", "host qI_scale", "host kI", "host kI_scale", "host w", "host q", "host kv"};
  const void* hp[7] = {host->qI, host->qI_scale, host->kI, host->kI_scale, host->w, host->q, host->kv};
  for (int i = 0; i < 7; ++i)
    if (hp[i] == nullptr) return fail(DSA_ERR_INVALID_ARG, "%s is NULL", names[i]);
  if (host->out == nullptr) return fail(DSA_ERR_INVALID_ARG, "host out is NULL");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t B = p->B, Lq = p->Lq, Lk = p->Lk;
  const size_t wbytes = p->w_dtype == DSA_DTYPE_BF16 ? 2 : 4;
  // bytes per query row and per key of each tensor
  const size_t r_qI = (size_t)p->H_I * p->d_I, r_qs = (size_t)p->H_I * 4, r_w = (size_t)p->H_I * wbytes;
  const size_t r_q = (size_t)p->H * p->Dqk * 2, r_out = (size_t)p->H * p->Dv * 2;
  const size_t r_lse = (size_t)p->H * 4, r_idx = (size_t)p->k * 4;
  const size_t k_kI = (size_t)p->d_I, k_ks = 4, k_kv = (size_t)p->Dqk * 2;
  auto h2d = [&](void* d, const void* h, size_t off, size_t n, cudaStream_t st) -> int {
    if (n == 0) return DSA_OK;
    DSA_TRY_CUDA(cudaMemcpyAsync(static_cast<char*>(d) + off, static_cast<const char*>(h) + off, n,
                                 cudaMemcpyHostToDevice, st), "H2D copy");
    return DSA_OK;
  };
  auto d2h = [&](void* h, const void* d, size_t off, size_t n, cudaStream_t st) -> int {
    if (n == 0) return DSA_OK;
    DSA_TRY_CUDA(cudaMemcpyAsync(static_cast<char*>(h) + off, static_cast<const char*>(d) + off, n,
                                 cudaMemcpyDeviceToHost, st), "D2H copy");
    return DSA_OK;
  };
  int launched = 0;
  if (Lq < (size_t)kHostPipeMinRows) {
    // short problems: everything in, one forward, everything out
    DSA_TRY(h2d((void*)dev->qI, host->qI, 0, B * Lq * r_qI, s));
    DSA_TRY(h2d((void*)dev->qI_scale, host->qI_scale, 0, B * Lq * r_qs, s));
    DSA_TRY(h2d((void*)dev->kI, host->kI, 0, B * Lk * k_kI, s));
    DSA_TRY(h2d((void*)dev->kI_scale, host->kI_scale, 0, B * Lk * k_ks, s));
    DSA_TRY(h2d((void*)dev->w, host->w, 0, B * Lq * r_w, s));
    DSA_TRY(h2d((void*)dev->q, host->q, 0, B * Lq * r_q, s));
    DSA_TRY(h2d((void*)dev->kv, host->kv, 0, B * Lk * k_kv, s));
    DSA_TRY(dsa_forward(p, dev, ws, ws_bytes, stream));
    launched = g_last_launches;
    DSA_TRY(d2h(host->out, dev->out, 0, B * Lq * r_out, s));
    if (host->lse && dev->lse) DSA_TRY(d2h(host->lse, dev->lse, 0, B * Lq * r_lse, s));
    if (host->idx_out && dev->idx_out) DSA_TRY(d2h(host->idx_out, dev->idx_out, 0, B * Lq * r_idx, s));
    if (host->sel_scores_out && dev->sel_scores_out)
      DSA_TRY(d2h(host->sel_scores_out, dev->sel_scores_out, 0, B * Lq * r_idx, s));
    DSA_TRY_CUDA(cudaStreamSynchronize(s), "stream synchronize");
    g_last_launches = launched;
    return DSA_OK;
  }
  // Pipelined: per sequence, blocks of kHostPipeRows query rows. Block c's rows (and
  // the keys it newly needs) are copied in on the library's copy-in stream while
  // block c - 1 computes on the caller's stream and block c - 2's results go out
  // on the copy-out stream. Each block is an ordinary forward over one sequence
  // (B = 1) whose rows start at q_pos0 + t0: rows are independent, so the results
  // equal one forward over everything.
  HostPipe* hpipe = nullptr;
  DSA_TRY(host_pipe(&hpipe));
  std::lock_guard<std::mutex> lk(hpipe->mu);
  // the copies start after whatever the caller queued on its stream before
  DSA_TRY_CUDA(cudaEventRecord(hpipe->start, s), "cudaEventRecord");
  DSA_TRY_CUDA(cudaStreamWaitEvent(hpipe->in, hpipe->start, 0), "cudaStreamWaitEvent");
  auto run = [&]() -> int {
    int c = 0;
    for (size_t b = 0; b < B; ++b) {
      size_t keys_in = 0;
      for (size_t t0 = 0, t1 = 0; t0 < Lq; t0 = t1, ++c) {
        // a short remainder joins this block, so that every block has at least
        // kHostPipeMinRows rows (enough CTAs that the attention needs no key splits)
        t1 = t0 + kHostPipeRows;
        if (t1 + kHostPipeMinRows > Lq) t1 = Lq;
        // keys the block's rows can see (<= Lk, checked by validate_problem); the
        // sequence's last block brings in the rest of its keys too
        const size_t keys = t1 == Lq ? Lk : (size_t)p->q_pos0 + t1;
        cudaEvent_t ev_in = hpipe->in_done[c % kHostPipeEvents];
        cudaEvent_t ev_out = hpipe->computed[c % kHostPipeEvents];
        // A block's copies write only its own query rows and the keys that earlier
        // blocks did not need, which no launch in flight reads: they wait for nothing.
        const size_t row0 = b * Lq + t0, nrow = t1 - t0;
        DSA_TRY(h2d((void*)dev->qI, host->qI, row0 * r_qI, nrow * r_qI, hpipe->in));
        DSA_TRY(h2d((void*)dev->qI_scale, host->qI_scale, row0 * r_qs, nrow * r_qs, hpipe->in));
        DSA_TRY(h2d((void*)dev->w, host->w, row0 * r_w, nrow * r_w, hpipe->in));
        DSA_TRY(h2d((void*)dev->q, host->q, row0 * r_q, nrow * r_q, hpipe->in));
        const size_t key0 = b * Lk + keys_in, nkey = keys - keys_in;
        DSA_TRY(h2d((void*)dev->kI, host->kI, key0 * k_kI, nkey * k_kI, hpipe->in));
        DSA_TRY(h2d((void*)dev->kI_scale, host->kI_scale, key0 * k_ks, nkey * k_ks, hpipe->in));
        DSA_TRY(h2d((void*)dev->kv, host->kv, key0 * k_kv, nkey * k_kv, hpipe->in));
        keys_in = keys;
        DSA_TRY_CUDA(cudaEventRecord(ev_in, hpipe->in), "cudaEventRecord");
        DSA_TRY_CUDA(cudaStreamWaitEvent(s, ev_in, 0), "cudaStreamWaitEvent");
        dsa_problem sp = *p;
        sp.B = 1;
        sp.Lq = (int)nrow;
        sp.Lk = (int)keys;
        sp.q_pos0 = p->q_pos0 + (int)t0;
        dsa_tensors st = *dev;
        st.qI = dev->qI + row0 * r_qI;
        st.qI_scale = dev->qI_scale + row0 * p->H_I;
        st.kI = dev->kI + b * Lk * k_kI;
        st.kI_scale = dev->kI_scale + b * Lk;
        st.w = static_cast<const char*>(dev->w) + row0 * r_w;
        st.q = dev->q + row0 * (size_t)p->H * p->Dqk;
        st.kv = dev->kv + b * Lk * (size_t)p->Dqk;
        st.out = dev->out + row0 * (size_t)p->H * p->Dv;
        st.lse = dev->lse ? dev->lse + row0 * p->H : nullptr;
        st.idx_out = dev->idx_out ? dev->idx_out + row0 * p->k : nullptr;
        st.sel_scores_out = dev->sel_scores_out ? dev->sel_scores_out + row0 * p->k : nullptr;
        // at most the block's recommended workspace, so that its score chunks keep
        // the default size (a larger area would only make them spill out of L2)
        const size_t sub_rec = dsa_forward_workspace_size(&sp);
        DSA_TRY(dsa_forward(&sp, &st, ws, ws_bytes < sub_rec ? ws_bytes : sub_rec, stream));
        launched += g_last_launches;
        DSA_TRY_CUDA(cudaEventRecord(ev_out, s), "cudaEventRecord");
        DSA_TRY_CUDA(cudaStreamWaitEvent(hpipe->out, ev_out, 0), "cudaStreamWaitEvent");
        DSA_TRY(d2h(host->out, dev->out, row0 * r_out, nrow * r_out, hpipe->out));
        if (host->lse && dev->lse) DSA_TRY(d2h(host->lse, dev->lse, row0 * r_lse, nrow * r_lse, hpipe->out));
        if (host->idx_out && dev->idx_out)
          DSA_TRY(d2h(host->idx_out, dev->idx_out, row0 * r_idx, nrow * r_idx, hpipe->out));
        if (host->sel_scores_out && dev->sel_scores_out)
          DSA_TRY(d2h(host->sel_scores_out, dev->sel_scores_out, row0 * r_idx, nrow * r_idx, hpipe->out));
      }
    }
    return DSA_OK;
  };
  const int rc = run();
  // Wait for all three streams even after a failure, so that no copy still reads
  // or writes the caller's host buffers once the call has returned.
  const cudaError_t e_in = cudaStreamSynchronize(hpipe->in);
  const cudaError_t e_s = cudaStreamSynchronize(s);
  const cudaError_t e_out = cudaStreamSynchronize(hpipe->out);
  if (rc != DSA_OK) return rc;
  DSA_TRY_CUDA(e_in, "stream synchronize");
  DSA_TRY_CUDA(e_s, "stream synchronize");
  DSA_TRY_CUDA(e_out, "stream synchronize");
  g_last_launches = launched;
  return DSA_OK;
}

int dsa_check_status(void* stream) {
  dsa::DevCtl ctl{nullptr, 0};
  int sms = 0;
  DSA_TRY(device_ctl(ctl, sms));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  DSA_TRY_CUDA(cudaStreamSynchronize(s), "stream synchronize");
  DSA_TRY_CUDA(cudaGetLastError(), "pending CUDA error");
  int st[4] = {0, 0, 0, 0};
  DSA_TRY_CUDA(cudaMemcpy(st, ctl.status, sizeof(st), cudaMemcpyDeviceToHost), "status read");
  if (st[0] != 0) {
    int zero[4] = {0, 0, 0, 0};
    DSA_TRY_CUDA(cudaMemcpy(ctl.status, zero, sizeof(zero), cudaMemcpyHostToDevice), "status clear");
    const char* site = st[1] == dsa::kSiteIndexer ? "indexer" : st[1] == dsa::kSiteTopk ? "top-k"
                       : st[1] == dsa::kSiteMla ? "sparse MLA" : st[1] == dsa::kSiteDebug ? "debug wait" : "?";
    return fail(DSA_ERR_TIMEOUT, "device wait timed out in %s kernel (block %d, wait %d)", site, st[2], st[3]);
  }
  return DSA_OK;
}

int dsa_set_wait_limit_ns(unsigned long long ns) {
  if (ns == 0) return fail(DSA_ERR_INVALID_ARG, "wait limit must be > 0");
  g_wait_ns = ns;
  return DSA_OK;
}

int dsa_debug_wait_timeout(void* stream) {
  dsa::DevCtl ctl;
  int sms = 0;
  DSA_TRY(device_ctl(ctl, sms));
  DSA_TRY_CUDA(dsa::launch_debug_wait(ctl, static_cast<cudaStream_t>(stream)), "debug launch");
  return DSA_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Sparse-stage gradients (bud-325 digest, "Method": the main model learns
// through attention over the selected entries; the indexer through its own
// detached inputs with the KL on the selected tokens).
//
// Per chunk of T tokens the selected rows are gathered into a dense [T, k, D]
// block, the per-token contractions run as batched bf16 tensor-core GEMMs with
// fp32 accumulation (bgemm.cu), and the key-gradient products add their rows
// straight into the shared key rows with fp32 atomics. The indexer's code dots are exact up to
// fp32 rounding and the ReLU mask is re-decided exactly in fp64 wherever that
// rounding could change its sign; its real-valued gradient operands enter the
// products as three bf16 terms (24 significant bits).
// ---------------------------------------------------------------------------
namespace {

constexpr int kBwdChunkTokens = 64;                   // tokens per gathered block

// One operand of a batched product: `depth` blocks of `rows` rows of `inner`
// contiguous bf16 elements; mn says whether the contiguous dimension is M / N
// (else K). period: K tiles of 64 after which the operand repeats (0: none).
struct GemmOperand {
  const void* base;
  bool mn;
  uint64_t inner, rows, depth, row_stride, depth_stride;
  int period;
};

// Key-row scatter of a product's rows (see BgemmArgs): row m of batch z adds into
// row idx[(tok0 + z) * k + m] of sequence (tok0 + z) / Lq.
struct RowScatter {
  const int32_t* idx;
  long long tok0;
  int k, Lq, Lk;
};

// C[z] (fp32, element (z, m, n) at C + z sC + m c_sm + n c_sn) = A[z] B[z]^T, or,
// with a RowScatter, C's key rows += the rows of A[z] B[z]^T.
int tc_gemm(const GemmOperand& A, const GemmOperand& B, int M, int N, int K, float* C,
            long long c_sm, long long c_sn, long long sC, int batch, const dsa::DevCtl& ctl,
            cudaStream_t s, const char* what, const RowScatter* scatter = nullptr) {
  const int bn = dsa::bgemm_tile_n(N);
  CUtensorMap ta, tb;
  DSA_TRY(make_map_3d(&ta, A.base, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, A.inner, A.rows, A.depth,
                      A.row_stride, A.depth_stride, 64, A.mn ? 64 : 128,
                      CU_TENSOR_MAP_SWIZZLE_128B));
  DSA_TRY(make_map_3d(&tb, B.base, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, B.inner, B.rows, B.depth,
                      B.row_stride, B.depth_stride, 64, B.mn ? 64 : (uint32_t)bn,
                      CU_TENSOR_MAP_SWIZZLE_128B));
  const int kt = (K + 63) / 64;
  dsa::BgemmArgs a{};
  a.M = M;
  a.N = N;
  a.K = K;
  a.a_kt = A.period > 0 ? A.period : kt;
  a.b_kt = B.period > 0 ? B.period : kt;
  a.C = C;
  a.c_sm = c_sm;
  a.c_sn = c_sn;
  a.sC = sC;
  if (scatter != nullptr) {
    a.sidx = scatter->idx;
    a.s_tok0 = scatter->tok0;
    a.s_k = scatter->k;
    a.s_Lq = scatter->Lq;
    a.s_Lk = scatter->Lk;
  }
  a.ctl = ctl;
  DSA_TRY_CUDA(dsa::launch_bgemm(ta, tb, a, batch, A.mn, B.mn, bn, s), what);
  return DSA_OK;
}

char* align256(void* p) {
  return reinterpret_cast<char*>((reinterpret_cast<uintptr_t>(p) + 255) & ~uintptr_t(255));
}

// Workspace of the attention backward for T tokens (offsets from a 256-byte
// aligned base; total includes the alignment slack).
struct MlaBwdLayout {
  size_t cg, qo, sp, pz, total;
};
MlaBwdLayout mla_bwd_layout(int T, int H, int Dqk, int k) {
  MlaBwdLayout L{};
  size_t off = 0;
  auto take = [&off](size_t bytes) {
    const size_t o = off;
    off += align_up(bytes, 256);
    return o;
  };
  const size_t tk = (size_t)T * k, t2hk = (size_t)T * 2 * H * k;
  L.cg = take(tk * Dqk * sizeof(uint16_t));              // gathered latent rows, bf16
  L.qo = take((size_t)T * 2 * H * Dqk * sizeof(uint16_t));  // [q; dout padded], bf16
  L.sp = take(t2hk * sizeof(float));                     // [q . c; dout . c[:Dv]]
  L.pz = take(t2hk * sizeof(uint16_t));                  // [dz; P], bf16
  L.total = off + 256;
  return L;
}

// Workspace of the indexer backward for T tokens; kp = k rounded up to 64,
// hp = H_I rounded up to 64 (the K tiles of the split products).
struct IdxBwdLayout {
  size_t kb, qb, xt, g1, g2, total;
  int kp, hp;
};
IdxBwdLayout idx_bwd_layout(int T, int H_I, int d_I, int k) {
  IdxBwdLayout L{};
  size_t off = 0;
  auto take = [&off](size_t bytes) {
    const size_t o = off;
    off += align_up(bytes, 256);
    return o;
  };
  L.kp = (k + 63) / 64 * 64;
  L.hp = (H_I + 63) / 64 * 64;
  const size_t tk = (size_t)T * k;
  L.kb = take(tk * d_I * sizeof(uint16_t));                        // gathered key codes
  L.qb = take((size_t)T * H_I * d_I * sizeof(uint16_t));           // query codes
  L.xt = take(tk * H_I * sizeof(float));                           // code dots [T][k][H_I]
  L.g1 = take((size_t)T * H_I * 3 * L.kp * sizeof(uint16_t));      // G1 in three parts
  L.g2 = take((size_t)T * 3 * L.hp * k * sizeof(uint16_t));        // G2 in three parts
  L.total = off + 256;
  return L;
}

int bwd_chunk(long long tokens) {
  return tokens < kBwdChunkTokens ? static_cast<int>(tokens) : kBwdChunkTokens;
}

}  // namespace

extern "C" {

size_t dsa_sparse_mla_bwd_workspace_size(int B, int Lq, int H, int Dqk, int Dv, int k) {
  if (B < 1 || Lq < 1 || H < 1 || Dqk < 1 || Dv < 1 || k < 1) return 0;
  return mla_bwd_layout(bwd_chunk((long long)B * Lq), H, Dqk, k).total;
}

int dsa_sparse_mla_bwd(const uint16_t* q, const uint16_t* kv, const int32_t* idx,
                       const float* lse, const uint16_t* dout, float* dq, float* dkv,
                       int accumulate_dkv, int B, int Lq, int Lk, int H, int Dqk, int Dv, int k,
                       float sm_scale, void* ws, size_t ws_bytes, void* stream) {
  DSA_TRY(check_ptr(q, "q"));
  DSA_TRY(check_ptr(kv, "kv"));
  DSA_TRY(check_ptr(idx, "idx"));
  DSA_TRY(check_ptr(lse, "lse"));
  DSA_TRY(check_ptr(dout, "dout"));
  DSA_TRY(check_ptr(dq, "dq"));
  DSA_TRY(check_ptr(dkv, "dkv"));
  if (B < 1 || Lq < 1 || Lk < 1) return fail(DSA_ERR_INVALID_ARG, "B, Lq, Lk must be >= 1");
  if ((long long)B * Lk > (1LL << 30)) return fail(DSA_ERR_UNSUPPORTED_SHAPE, "B*Lk must be <= 2^30");
  DSA_TRY(check_mla_shape(H, Dqk, Dv, B, Lq));
  DSA_TRY(check_k(k, 4096));
  if (!(sm_scale > 0.f) || !std::isfinite(sm_scale))
    return fail(DSA_ERR_INVALID_ARG, "sm_scale must be finite and > 0");
  const long long n = (long long)B * Lq;
  int T = bwd_chunk(n);
  while (T > 1 && mla_bwd_layout(T, H, Dqk, k).total > ws_bytes) --T;
  const MlaBwdLayout L = mla_bwd_layout(T, H, Dqk, k);
  if (L.total > ws_bytes)
    return fail(DSA_ERR_WORKSPACE_TOO_SMALL, "sparse MLA backward workspace: need at least %zu bytes (recommended %zu), got %zu",
                L.total, dsa_sparse_mla_bwd_workspace_size(B, Lq, H, Dqk, Dv, k), ws_bytes);
  DSA_TRY(check_ptr(ws, "ws"));
  dsa::DevCtl ctl;
  int sms = 0;
  DSA_TRY(device_ctl(ctl, sms));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  char* base = align256(ws);
  uint16_t* cg = reinterpret_cast<uint16_t*>(base + L.cg);
  uint16_t* QO = reinterpret_cast<uint16_t*>(base + L.qo);
  float* SP = reinterpret_cast<float*>(base + L.sp);
  uint16_t* PZ = reinterpret_cast<uint16_t*>(base + L.pz);
  int launched = 0;
  if (!accumulate_dkv)
    DSA_TRY_CUDA(cudaMemsetAsync(dkv, 0, (size_t)B * Lk * Dqk * sizeof(float), s), "dkv clear");
  // Per token, with QO = [q; dout padded to Dqk] (2H x Dqk) and the gathered rows C
  // (k x Dqk): [S; dP] = QO C^T, dq = dz C, dC = [dz; P]^T QO (the padded columns of
  // dout make the second half of each product act on the value columns only).
  const uint64_t h2 = 2ull * H, uk = (uint64_t)k, ud = (uint64_t)Dqk, uT = (uint64_t)T;
  // operands, as blocks of the chunk's buffers (the maps span T tokens; a shorter
  // last chunk launches fewer blocks)
  const GemmOperand qo_k{QO, false, ud, h2, uT, ud, h2 * ud, 0};      // [2H][Dqk], K = Dqk
  const GemmOperand qo_mn{QO, true, ud, h2, uT, ud, h2 * ud, 0};      // K = 2H rows, N = Dqk
  const GemmOperand c_k{cg, false, ud, uk, uT, ud, uk * ud, 0};       // [k][Dqk], K = Dqk
  const GemmOperand c_mn{cg, true, ud, uk, uT, ud, uk * ud, 0};       // K = k rows, N = Dqk
  const GemmOperand dz_k{PZ, false, uk, (uint64_t)H, uT, uk, h2 * uk, 0};   // rows 0..H-1, K = k
  const GemmOperand pz_mn{PZ, true, uk, h2, uT, uk, h2 * uk, 0};      // K = 2H rows, M = k
  for (long long tok0 = 0; tok0 < n; tok0 += T) {
    const int Tc = (int)(n - tok0 < T ? n - tok0 : T);
    DSA_TRY_CUDA(dsa::launch_gather_rows_bf16(kv, idx, cg, tok0, Tc, Lq, Lk, k, Dqk, sms, s),
                 "latent row gather launch");
    DSA_TRY_CUDA(dsa::launch_pack_qo(q, dout, QO, tok0, Tc, H, Dqk, Dv, sms, s),
                 "query / output-gradient pack launch");
    DSA_TRY(tc_gemm(qo_k, c_k, 2 * H, k, Dqk, SP, k, 1, 2LL * H * k, Tc, ctl, s,
                    "[S; dP] = QO C^T"));
    DSA_TRY_CUDA(dsa::launch_mla_bwd_softmax(SP, lse, idx, PZ, tok0, Tc, H, k, Lk, sm_scale, sms,
                                             s),
                 "softmax gradient launch");
    DSA_TRY(tc_gemm(dz_k, c_mn, H, Dqk, k, dq + tok0 * H * Dqk, Dqk, 1, (long long)H * Dqk, Tc,
                    ctl, s, "dq = dz C"));
    // dC = [dz; P]^T QO, added row by row into the selected latent rows of dkv
    const RowScatter to_dkv{idx, tok0, k, Lq, Lk};
    DSA_TRY(tc_gemm(pz_mn, qo_mn, k, Dqk, 2 * H, dkv, Dqk, 1, 0, Tc, ctl, s,
                    "dkv += [dz; P]^T QO", &to_dkv));
    launched += 6;
  }
  g_last_launches = launched;
  return DSA_OK;
}

size_t dsa_indexer_bwd_workspace_size(int B, int Lq, int H_I, int d_I, int k) {
  if (B < 1 || Lq < 1 || H_I < 1 || d_I < 1 || k < 1) return 0;
  return idx_bwd_layout(bwd_chunk((long long)B * Lq), H_I, d_I, k).total;
}

int dsa_indexer_bwd(const uint8_t* qI, const float* qI_scale, const uint8_t* kI,
                    const float* kI_scale, const void* w, int w_dtype, const int32_t* idx,
                    const float* dI, float* dqI, float* dkI, float* dw, int accumulate_dkI, int B,
                    int Lq, int Lk, int H_I, int d_I, int k, void* ws, size_t ws_bytes,
                    void* stream) {
  DSA_TRY(check_ptr(qI, "qI"));
  DSA_TRY(check_ptr(qI_scale, "qI_scale"));
  DSA_TRY(check_ptr(kI, "kI"));
  DSA_TRY(check_ptr(kI_scale, "kI_scale"));
  DSA_TRY(check_ptr(w, "w"));
  DSA_TRY(check_ptr(idx, "idx"));
  DSA_TRY(check_ptr(dI, "dI"));
  DSA_TRY(check_ptr(dqI, "dqI"));
  DSA_TRY(check_ptr(dkI, "dkI"));
  DSA_TRY(check_ptr(dw, "dw"));
  if (B < 1 || Lq < 1 || Lk < 1) return fail(DSA_ERR_INVALID_ARG, "B, Lq, Lk must be >= 1");
  if ((long long)B * Lk > (1LL << 30)) return fail(DSA_ERR_UNSUPPORTED_SHAPE, "B*Lk must be <= 2^30");
  DSA_TRY(check_indexer_shape(H_I, d_I, B, Lq));
  DSA_TRY(check_k(k, 4096));
  if (w_dtype != DSA_DTYPE_F32 && w_dtype != DSA_DTYPE_BF16)
    return fail(DSA_ERR_INVALID_ARG, "w_dtype must be DSA_DTYPE_F32 or DSA_DTYPE_BF16");
  const long long n = (long long)B * Lq;
  int T = bwd_chunk(n);
  while (T > 1 && idx_bwd_layout(T, H_I, d_I, k).total > ws_bytes) --T;
  const IdxBwdLayout L = idx_bwd_layout(T, H_I, d_I, k);
  if (L.total > ws_bytes)
    return fail(DSA_ERR_WORKSPACE_TOO_SMALL, "indexer backward workspace: need at least %zu bytes (recommended %zu), got %zu",
                L.total, dsa_indexer_bwd_workspace_size(B, Lq, H_I, d_I, k), ws_bytes);
  DSA_TRY(check_ptr(ws, "ws"));
  dsa::DevCtl ctl;
  int sms = 0;
  DSA_TRY(device_ctl(ctl, sms));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  char* base = align256(ws);
  uint16_t* Kb = reinterpret_cast<uint16_t*>(base + L.kb);
  uint16_t* Qb = reinterpret_cast<uint16_t*>(base + L.qb);
  float* XT = reinterpret_cast<float*>(base + L.xt);
  uint16_t* G1s = reinterpret_cast<uint16_t*>(base + L.g1);
  uint16_t* G2s = reinterpret_cast<uint16_t*>(base + L.g2);
  int launched = 0;
  if (!accumulate_dkI)
    DSA_TRY_CUDA(cudaMemsetAsync(dkI, 0, (size_t)B * Lk * d_I * sizeof(float), s), "dkI clear");
  DSA_TRY_CUDA(cudaMemsetAsync(dw, 0, (size_t)n * H_I * sizeof(float), s), "dw clear");
  const long long qs = (long long)H_I * d_I;
  const uint64_t uk = (uint64_t)k, ud = (uint64_t)d_I, uh = (uint64_t)H_I, uT = (uint64_t)T;
  const uint64_t kp3 = 3ull * L.kp, hp3 = 3ull * L.hp;
  const GemmOperand kb_k{Kb, false, ud, uk, uT, ud, uk * ud, 0};            // [k][d_I], K = d_I
  const GemmOperand qb_k{Qb, false, ud, uh, uT, ud, uh * ud, 0};            // [H_I][d_I], K = d_I
  const GemmOperand kb_mn{Kb, true, ud, uk, uT, ud, uk * ud, L.kp / 64};    // K = slots, M = d_I
  const GemmOperand g1_k{G1s, false, kp3, uh, uT, kp3, uh * kp3, 0};        // [H_I][3 kp], K = 3 kp
  const GemmOperand g2_mn{G2s, true, uk, hp3, uT, uk, hp3 * uk, 0};         // K = 3 hp rows, M = k
  const GemmOperand qb_mn{Qb, true, ud, uh, uT, ud, uh * ud, L.hp / 64};    // K = heads, N = d_I
  for (long long tok0 = 0; tok0 < n; tok0 += T) {
    const int Tc = (int)(n - tok0 < T ? n - tok0 : T);
    DSA_TRY_CUDA(dsa::launch_decode_e4m3_bf16(qI + tok0 * qs, Qb, (long long)Tc * qs, sms, s),
                 "query code launch");
    DSA_TRY_CUDA(dsa::launch_gather_e4m3_rows_bf16(kI, idx, Kb, tok0, Tc, Lq, Lk, k, d_I, sms, s),
                 "indexer key gather launch");
    // X^T [k x H_I] = khat qhat^T (code dots, fp32 accumulation)
    DSA_TRY(tc_gemm(kb_k, qb_k, k, H_I, d_I, XT, H_I, 1, (long long)k * H_I, Tc, ctl, s,
                    "X^T = khat qhat^T"));
    DSA_TRY_CUDA(dsa::launch_indexer_bwd_relu_tc(XT, Kb, Qb, idx, dI, qI_scale, kI_scale, w,
                                                 w_dtype == DSA_DTYPE_BF16 ? 1 : 0, G1s, G2s, dw,
                                                 tok0, Tc, Lq, Lk, H_I, d_I, k, L.kp, L.hp, s),
                 "ReLU gradient launch");
    // dq^I [H_I x d_I], written transposed from (dq^I)^T = khat^T G1^T over K = 3 kp
    DSA_TRY(tc_gemm(kb_mn, g1_k, d_I, H_I, 3 * L.kp, dqI + tok0 * qs, 1, d_I, qs, Tc, ctl, s,
                    "dqI = G1 khat"));
    // G2^T qhat over K = 3 hp [k x d_I], added row by row into the selected keys of dkI
    const RowScatter to_dkI{idx, tok0, k, Lq, Lk};
    DSA_TRY(tc_gemm(g2_mn, qb_mn, k, d_I, 3 * L.hp, dkI, d_I, 1, 0, Tc, ctl, s,
                    "dkI += G2^T qhat", &to_dkI));
    launched += 6;
  }
  g_last_launches = launched;
  return DSA_OK;
}

int dsa_indexer_kl_grad(const float* sel_scores, const float* p, const int32_t* idx, float* dI,
                        int B, int Lq, int Lk, int k, float loss_scale, void* stream) {
  DSA_TRY(check_ptr(sel_scores, "sel_scores"));
  DSA_TRY(check_ptr(p, "p"));
  DSA_TRY(check_ptr(idx, "idx"));
  DSA_TRY(check_ptr(dI, "dI"));
  if (B < 1 || Lq < 1 || Lk < 1) return fail(DSA_ERR_INVALID_ARG, "B, Lq, Lk must be >= 1");
  if ((long long)B * Lq > (1LL << 30)) return fail(DSA_ERR_UNSUPPORTED_SHAPE, "B*Lq must be <= 2^30");
  DSA_TRY(check_k(k, 4096));
  if (!std::isfinite(loss_scale)) return fail(DSA_ERR_INVALID_ARG, "loss_scale must be finite");
  dsa::DevCtl ctl;
  int sms = 0;
  DSA_TRY(device_ctl(ctl, sms));
  DSA_TRY_CUDA(dsa::launch_kl_score_grad(sel_scores, p, idx, dI, (long long)B * Lq, k, Lk,
                                         loss_scale, sms, static_cast<cudaStream_t>(stream)),
               "KL score gradient launch");
  g_last_launches = 1;
  return DSA_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Decode with one sequence's key cache split over G devices (context_parallel.cu):
// the merge of the shards' candidates, the shard-local view of the merged
// selection, and the combine of the partial attentions.
// ---------------------------------------------------------------------------
namespace {

struct MergeLayout {
  size_t scores, idx, pos, total;
};
MergeLayout merge_layout(int G, int R, int k) {
  MergeLayout L{};
  size_t off = 0;
  auto take = [&off](size_t bytes) {
    const size_t o = off;
    off += align_up(bytes, 256);
    return o;
  };
  const size_t n = (size_t)R * G * k;
  L.scores = take(n * sizeof(float));
  L.idx = take(n * sizeof(int32_t));
  L.pos = take((size_t)R * k * sizeof(int32_t));
  L.total = off + 256;
  return L;
}

constexpr int kMaxShards = 16;

}  // namespace

extern "C" {

size_t dsa_topk_merge_workspace_size(int G, int R, int k) {
  if (G < 1 || G > kMaxShards || R < 1 || k < 1) return 0;
  return merge_layout(G, R, k).total;
}

int dsa_topk_merge(const float* cand_scores, const int32_t* cand_idx, const long long* shard_lo,
                   int G, int R, int k, int32_t* idx_out, float* sel_out, void* ws,
                   size_t ws_bytes, void* stream) {
  NvtxRange nr("dsa_topk_merge");
  DSA_TRY(check_ptr(cand_scores, "cand_scores"));
  DSA_TRY(check_ptr(cand_idx, "cand_idx"));
  DSA_TRY(check_ptr(idx_out, "idx_out"));
  DSA_TRY(check_ptr(sel_out, "sel_out", true));
  if (shard_lo == nullptr) return fail(DSA_ERR_INVALID_ARG, "shard_lo is NULL");
  if (G < 1 || G > kMaxShards) return fail(DSA_ERR_INVALID_ARG, "G must be in [1, %d]", kMaxShards);
  if (R < 1) return fail(DSA_ERR_INVALID_ARG, "R must be >= 1");
  DSA_TRY(check_k(k, 4096));
  if ((long long)R * G * k > (1LL << 31)) return fail(DSA_ERR_UNSUPPORTED_SHAPE, "R * G * k must be <= 2^31");
  dsa::ShardOffsets lo{};
  for (int g = 0; g < G; ++g) {
    if (shard_lo[g] < 0 || (g > 0 && shard_lo[g] <= shard_lo[g - 1]) || shard_lo[g] >= (1LL << 31))
      return fail(DSA_ERR_INVALID_ARG, "shard_lo must be increasing, >= 0 and < 2^31");
    lo.v[g] = shard_lo[g];
  }
  const MergeLayout L = merge_layout(G, R, k);
  if (ws_bytes < L.total)
    return fail(DSA_ERR_WORKSPACE_TOO_SMALL, "dsa_topk_merge workspace: need %zu bytes, got %zu",
                L.total, ws_bytes);
  DSA_TRY(check_ptr(ws, "ws"));
  dsa::DevCtl ctl;
  int sms = 0;
  DSA_TRY(device_ctl(ctl, sms));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  char* base = align256(ws);
  float* ext_scores = reinterpret_cast<float*>(base + L.scores);
  int32_t* ext_idx = reinterpret_cast<int32_t*>(base + L.idx);
  int32_t* pos = reinterpret_cast<int32_t*>(base + L.pos);
  const int n = G * k;
  DSA_TRY_CUDA(dsa::launch_cp_pack(cand_scores, cand_idx, lo, G, R, k, ext_scores, ext_idx, sms, s),
               "candidate pack launch");
  // every row has n = G k candidate positions: row r is "sequence" r, one query
  // row at position n - 1
  dsa::TopkArgs ta{};
  ta.scores = ext_scores;
  ta.sc_ld = n;
  ta.sc_bstride = 1;
  ta.sc_t0 = 0;
  ta.idx = pos;
  ta.B = R;
  ta.Lq = 1;
  ta.Lk = n;
  ta.q_pos0 = n - 1;
  ta.k = k;
  ta.t_lo = 0;
  ta.t_hi = 1;
  ta.vec4 = (n % 4 == 0) ? 1 : 0;
  ta.seq_lens = nullptr;
  ta.sel = sel_out;
  ta.ctl = ctl;
  DSA_TRY_CUDA(dsa::launch_topk(ta, sms, s), "candidate top-k launch");
  DSA_TRY_CUDA(dsa::launch_cp_map_compact(pos, ext_idx, R, n, k, idx_out, sel_out, sms, s),
               "candidate map launch");
  g_last_launches = 3;
  return DSA_OK;
}

int dsa_index_localize(const int32_t* idx, int32_t* idx_local, long long n, int lo, int len,
                       void* stream) {
  DSA_TRY(check_ptr(idx, "idx"));
  DSA_TRY(check_ptr(idx_local, "idx_local"));
  if (n < 1 || lo < 0 || len < 1) return fail(DSA_ERR_INVALID_ARG, "need n >= 1, lo >= 0, len >= 1");
  dsa::DevCtl ctl;
  int sms = 0;
  DSA_TRY(device_ctl(ctl, sms));
  DSA_TRY_CUDA(dsa::launch_cp_localize(idx, idx_local, n, lo, len, sms, static_cast<cudaStream_t>(stream)),
               "index localize launch");
  g_last_launches = 1;
  return DSA_OK;
}

int dsa_attn_combine(const uint16_t* part_out, const float* part_lse, int G, int R, int H, int Dv,
                     uint16_t* out, float* lse_out, void* stream) {
  DSA_TRY(check_ptr(part_out, "part_out"));
  DSA_TRY(check_ptr(part_lse, "part_lse"));
  DSA_TRY(check_ptr(out, "out"));
  DSA_TRY(check_ptr(lse_out, "lse_out", true));
  if (G < 1 || G > kMaxShards) return fail(DSA_ERR_INVALID_ARG, "G must be in [1, %d]", kMaxShards);
  if (R < 1 || H < 1 || Dv < 1) return fail(DSA_ERR_INVALID_ARG, "R, H, Dv must be >= 1");
  dsa::DevCtl ctl;
  int sms = 0;
  DSA_TRY(device_ctl(ctl, sms));
  DSA_TRY_CUDA(dsa::launch_cp_combine(part_out, part_lse, G, (long long)R * H, Dv, out, lse_out, sms,
                                      static_cast<cudaStream_t>(stream)),
               "partial attention combine launch");
  g_last_launches = 1;
  return DSA_OK;
}

}  // extern "C"
