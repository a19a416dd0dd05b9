// C ABI of libqmoe.so (declared in include/qmoe.h): argument validation, the
// handle (repacked weights + workspace), and the launch sequence
//   router logits -> router top-k -> schedule -> gate/up GEMM -> down GEMM -> combine
// on the caller's stream.  No call synchronises the stream on the hot path;
// the counts never travel to the host (the GEMMs read the device tile tables).
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "qmoe_internal.cuh"

using namespace qmoe;

namespace {

// Programmatic dependent launch of the kernels after the router.  Off: with
// it on, the mixed-format workload hit an unspecified launch failure whose
// cause was not found; every kernel still calls pdl_wait(), a no-op here.
constexpr bool kUsePdl = true;

thread_local std::string g_last_error;

qmoe_status fail(qmoe_status st, const std::string& msg) {
  g_last_error = msg;
  return st;
}

qmoe_status cuda_fail(cudaError_t e, const char* what) {
  return fail(QMOE_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
}

#define QMOE_CUDA(call, what)                       \
  do {                                              \
    cudaError_t e_ = (call);                        \
    if (e_ != cudaSuccess) return cuda_fail(e_, what); \
  } while (0)

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

struct Event {
  cudaEvent_t a = nullptr, b = nullptr;
  int stage = 0;
};

// cuTensorMapEncodeTiled, fetched from the driver through the runtime so the
// library does not link libcuda directly.
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// Row-major bf16 matrix [rows][cols] seen as 3-D (64 columns, rows, cols / 64
// column chunks) and read in boxes of 64 columns x box_rows rows x 2 chunks
// (one 128-column K stage) into 128-byte-swizzled shared memory laid out
// [chunk][row][64]; rows past the end read as zero.
bool encode_rows_map(CUtensorMap* m, const void* base, int rows, int cols, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {64, (cuuint64_t)rows, (cuuint64_t)cols / 64};
  const cuuint64_t strides[2] = {(cuuint64_t)cols * 2, 128};
  const cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 2};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

constexpr int kNumBn = 4;                 // token-block widths 16, 32, 64, 128
int bn_index(int bn) { return bn == 16 ? 0 : bn == 32 ? 1 : bn == 64 ? 2 : 3; }

}  // namespace

struct qmoe_handle {
  qmoe_config cfg{};
  int device = 0;
  int num_sms = 0;
  std::vector<void*> allocs;
  float* router_w = nullptr;
  float* router_b = nullptr;
  ExpertDev* d_experts = nullptr;
  // workspace
  int32_t *idx = nullptr, *inv_pos = nullptr, *counts = nullptr, *offsets = nullptr, *sorted_token = nullptr;
  int32_t *seg_off = nullptr, *seg_cnt = nullptr, *tiles = nullptr, *seg_fmt = nullptr, *sched_scratch = nullptr;
  bool fmt_present[4] = {false, false, false, false};
  bool mma_f16 = false;                  // all experts FP8: x rows, H and the MMAs in fp16
  CUtensorMap xp_map[kNumBn];            // permuted x rows (gate/up B operand), one per block width
  CUtensorMap h_map[kNumBn];             // H rows (down B operand), one per block width
  float *gates = nullptr, *zpart = nullptr;
  uint16_t *Xp = nullptr, *H = nullptr, *Y = nullptr, *x_stage = nullptr, *out_stage = nullptr;
  int* err = nullptr;
  int* tile_done = nullptr;              // router: per-32-token-tile completion counters (zero between calls)
  size_t zpart_floats = 0;               // capacity of the router's partial-logit buffer
  long long wait_limit = kWaitLimit;     // bound of the grouped GEMMs' mbarrier waits (SM cycles)
  // profiling
  bool profiling = false;
  int profiled_calls = 0;
  std::vector<Event> events;
  std::vector<Event> event_pool;

  template <class T>
  qmoe_status alloc(T** p, size_t count, const char* what) {
    void* ptr = nullptr;
    cudaError_t e = cudaMalloc(&ptr, count * sizeof(T) > 0 ? count * sizeof(T) : 16);
    if (e != cudaSuccess) {
      cudaGetLastError();
      return fail(QMOE_ERR_OOM, std::string("cudaMalloc failed for ") + what + ": " + cudaGetErrorString(e));
    }
    allocs.push_back(ptr);
    *p = static_cast<T*>(ptr);
    return QMOE_OK;
  }
  void release() {
    for (void* p : allocs) cudaFree(p);
    allocs.clear();
    for (auto& ev : event_pool) {
      cudaEventDestroy(ev.a);
      cudaEventDestroy(ev.b);
    }
    for (auto& ev : events) {
      cudaEventDestroy(ev.a);
      cudaEventDestroy(ev.b);
    }
    event_pool.clear();
    events.clear();
  }
};

namespace {

// Token-block width of the grouped GEMMs for T tokens: about 1.5x the mean
// rows per routed expert, rounded up to a supported width.
int choose_bn(const qmoe_config& c, int T) {
  const double mean = (double)T * c.k / c.E;
  const double want = 1.5 * mean;
  if (want <= 16) return 16;
  if (want <= 32) return 32;
  if (want <= 64) return 64;
  return 128;
}

// Bracket one launch with an event pair when profiling.
struct StageTimer {
  qmoe_handle* h;
  cudaStream_t s;
  Event ev;
  bool on;
  StageTimer(qmoe_handle* h_, cudaStream_t s_, int stage) : h(h_), s(s_), on(h_->profiling) {
    if (!on) return;
    if (!h->event_pool.empty()) {
      ev = h->event_pool.back();
      h->event_pool.pop_back();
    } else {
      cudaEventCreate(&ev.a);
      cudaEventCreate(&ev.b);
    }
    ev.stage = stage;
    cudaEventRecord(ev.a, s);
  }
  ~StageTimer() {
    if (!on) return;
    cudaEventRecord(ev.b, s);
    h->events.push_back(ev);
  }
};

qmoe_status check_device(int* device, int* sms) {
  QMOE_CUDA(cudaGetDevice(device), "cudaGetDevice");
  cudaDeviceProp prop;
  QMOE_CUDA(cudaGetDeviceProperties(&prop, *device), "cudaGetDeviceProperties");
  if (prop.major != 10 || prop.minor != 0)
    return fail(QMOE_ERR_UNSUPPORTED, "libqmoe is built for sm_100a (B200); device " + std::string(prop.name) +
                                          " is sm_" + std::to_string(prop.major) + std::to_string(prop.minor));
  *sms = prop.multiProcessorCount;
  return QMOE_OK;
}

qmoe_status route_impl(qmoe_handle* h, const uint16_t* x, const float* logits, int T, int32_t* idx, float* gates,
                       int32_t* counts, int32_t* offsets, int32_t* sorted_token, int32_t* inv_pos, bool tables, int bn,
                       cudaStream_t s) {
  const qmoe_config& c = h->cfg;
  {
    StageTimer tm(h, s, QMOE_STAGE_ROUTER);
    if (x) {
      int split = router_split(T, c.d, c.E, h->num_sms);
      while (split > 1 && (size_t)split * T * c.E > h->zpart_floats) split >>= 1;
      QMOE_CUDA(launch_router_fused(x, h->router_w, h->router_b, T, c.d, c.E, c.k, split, h->zpart, h->tile_done,
                                    idx, gates, s),
                "router launch");
    } else {
      QMOE_CUDA(launch_router_topk(logits, T, c.E, c.k, idx, gates, s), "router top-k launch");
    }
  }
  {
    StageTimer tm(h, s, QMOE_STAGE_SCHEDULE);
    QMOE_CUDA(launch_schedule(kUsePdl, idx, T, c.k, c.E, tables ? c.n_shared : 0, bn, 2 * c.I / kTileM, c.d / kTileM,
                              h->seg_fmt, counts, offsets, sorted_token, inv_pos, tables ? h->seg_off : nullptr,
                              tables ? h->seg_cnt : nullptr, h->tiles, h->sched_scratch, h->err, s),
              "schedule launch");
  }
  return QMOE_OK;
}

qmoe_status validate_tokens(const qmoe_handle* h, int T) {
  if (!h) return fail(QMOE_ERR_INVALID, "handle is NULL");
  if (T < 1 || T > h->cfg.max_tokens)
    return fail(QMOE_ERR_INVALID, "T=" + std::to_string(T) + " outside [1, max_tokens=" +
                                      std::to_string(h->cfg.max_tokens) + "]");
  return QMOE_OK;
}

}  // namespace

extern "C" {

const char* qmoe_last_error(void) { return g_last_error.c_str(); }

qmoe_status qmoe_create(const qmoe_config* cfg, const float* router_w, const float* router_bias,
                        const qmoe_expert* experts, qmoe_handle** out) {
  if (!out) return fail(QMOE_ERR_INVALID, "out is NULL");
  *out = nullptr;
  if (!cfg || !router_w || !experts) return fail(QMOE_ERR_INVALID, "cfg, router_w and experts must be non-NULL");
  const qmoe_config c = *cfg;
  if (c.d < 128 || c.d % 128) return fail(QMOE_ERR_INVALID, "d must be a positive multiple of 128");
  if (c.I < 128 || c.I % 128) return fail(QMOE_ERR_INVALID, "I must be a positive multiple of 128");
  if (c.E < 1 || c.E > kMaxE) return fail(QMOE_ERR_INVALID, "E must be in [1, 256]");
  if (c.k < 1 || c.k > c.E || c.k > kMaxK) return fail(QMOE_ERR_INVALID, "k must be in [1, min(E, 16)]");
  if (c.n_shared < 0 || c.n_shared > kMaxShared) return fail(QMOE_ERR_INVALID, "n_shared must be in [0, 8]");
  if (c.max_tokens < 1 || c.max_tokens > (1 << 20)) return fail(QMOE_ERR_INVALID, "max_tokens must be in [1, 2^20]");
  const long long rows_max = (long long)c.max_tokens * (c.k + c.n_shared);
  if (rows_max * (long long)(c.d > c.I ? c.d : c.I) >= (1ll << 40))
    return fail(QMOE_ERR_INVALID, "max_tokens too large for this layer");
  const int nexp = c.E + c.n_shared;
  for (int e = 0; e < nexp; ++e) {
    const qmoe_expert& x = experts[e];
    if (x.fmt != QMOE_W_INT8_PC && x.fmt != QMOE_W_INT4_G128 && x.fmt != QMOE_W_FP8_E4M3_PC)
      return fail(QMOE_ERR_INVALID, "expert " + std::to_string(e) + ": unknown weight format " + std::to_string(x.fmt));
    if (!x.w13 || !x.s13 || !x.w2 || !x.s2)
      return fail(QMOE_ERR_INVALID, "expert " + std::to_string(e) + ": NULL weight or scale pointer");
  }

  int device = 0, sms = 0;
  qmoe_status st = check_device(&device, &sms);
  if (st != QMOE_OK) return st;

  qmoe_handle* h = new qmoe_handle();
  h->cfg = c;
  h->device = device;
  h->num_sms = sms;
  auto bail = [&](qmoe_status s) {
    cudaDeviceSynchronize();
    h->release();
    delete h;
    return s;
  };
  const size_t Tm = (size_t)c.max_tokens;
  const size_t P = Tm * c.k + Tm * c.n_shared;  // permuted rows incl. shared segments

  // router
  if ((st = h->alloc(&h->router_w, (size_t)c.E * c.d, "router_w")) != QMOE_OK) return bail(st);
  if (cudaMemcpy(h->router_w, router_w, sizeof(float) * c.E * c.d, cudaMemcpyDefault) != cudaSuccess)
    return bail(cuda_fail(cudaGetLastError(), "copy router_w"));
  if (router_bias) {
    if ((st = h->alloc(&h->router_b, (size_t)c.E, "router_b")) != QMOE_OK) return bail(st);
    if (cudaMemcpy(h->router_b, router_bias, sizeof(float) * c.E, cudaMemcpyDefault) != cudaSuccess)
      return bail(cuda_fail(cudaGetLastError(), "copy router_b"));
  }

  // A layer whose experts are all FP8 computes in fp16: e4m3 codes convert to
  // fp16 exactly with one instruction per pair, so x rows and H are fp16 too.
  // Any other mix computes in bf16.
  h->mma_f16 = true;
  for (int e = 0; e < nexp; ++e) h->mma_f16 = h->mma_f16 && experts[e].fmt == QMOE_W_FP8_E4M3_PC;

  // experts: repack both matrices of each expert into handle-owned tiles
  std::vector<ExpertDev> host_desc(nexp);
  for (int e = 0; e < nexp; ++e) {
    const qmoe_expert& x = experts[e];
    ExpertDev& dv = host_desc[e];
    dv.fmt = x.fmt;
    dv.pad = 0;
    const int rows[2] = {2 * c.I, c.d};
    const int Ks[2] = {c.d, c.I};
    const void* ws[2] = {x.w13, x.w2};
    const void* ss[2] = {x.s13, x.s2};
    for (int m = 0; m < 2; ++m) {
      const size_t tiles = (size_t)(rows[m] / kTileM) * (Ks[m] / kBK);
      uint8_t* wdst = nullptr;
      float* sdst = nullptr;
      if ((st = h->alloc(&wdst, tiles * stage_bytes(x.fmt), "expert weights")) != QMOE_OK) return bail(st);
      if (x.fmt != QMOE_W_INT4_G128)
        if ((st = h->alloc(&sdst, (size_t)rows[m], "expert scales")) != QMOE_OK) return bail(st);
      cudaError_t e2 = launch_repack(h->mma_f16 ? kFmtFp8F16 : x.fmt, m, ws[m], ss[m], rows[m], Ks[m], c.I, wdst,
                                     sdst, 0);
      if (e2 != cudaSuccess) return bail(cuda_fail(e2, "repack launch"));
      dv.w[m] = wdst;
      dv.spc[m] = sdst;
    }
  }
  if ((st = h->alloc(&h->d_experts, (size_t)nexp, "expert table")) != QMOE_OK) return bail(st);
  if (cudaMemcpy(h->d_experts, host_desc.data(), sizeof(ExpertDev) * nexp, cudaMemcpyHostToDevice) != cudaSuccess)
    return bail(cuda_fail(cudaGetLastError(), "copy expert table"));

  // workspace
  const int n_seg = nexp;
  if ((st = h->alloc(&h->idx, Tm * c.k, "idx")) != QMOE_OK) return bail(st);
  if ((st = h->alloc(&h->gates, Tm * c.k, "gates")) != QMOE_OK) return bail(st);
  if ((st = h->alloc(&h->inv_pos, Tm * c.k, "inv_pos")) != QMOE_OK) return bail(st);
  if ((st = h->alloc(&h->counts, (size_t)c.E, "counts")) != QMOE_OK) return bail(st);
  if ((st = h->alloc(&h->offsets, (size_t)c.E + 1, "offsets")) != QMOE_OK) return bail(st);
  if ((st = h->alloc(&h->sorted_token, P, "sorted_token")) != QMOE_OK) return bail(st);
  if ((st = h->alloc(&h->seg_off, (size_t)n_seg, "seg_off")) != QMOE_OK) return bail(st);
  if ((st = h->alloc(&h->seg_cnt, (size_t)n_seg, "seg_cnt")) != QMOE_OK) return bail(st);
  if ((st = h->alloc(&h->tiles, (size_t)6 * (n_seg + 1), "tile tables")) != QMOE_OK) return bail(st);
  {
    std::vector<int32_t> fm(n_seg);
    for (int e = 0; e < n_seg; ++e) {
      fm[e] = experts[e].fmt;
      h->fmt_present[experts[e].fmt] = true;
    }
    if ((st = h->alloc(&h->seg_fmt, (size_t)n_seg, "segment formats")) != QMOE_OK) return bail(st);
    if (cudaMemcpy(h->seg_fmt, fm.data(), sizeof(int32_t) * n_seg, cudaMemcpyHostToDevice) != cudaSuccess)
      return bail(cuda_fail(cudaGetLastError(), "copy segment formats"));
  }
  if ((st = h->alloc(&h->sched_scratch, schedule_scratch_ints(c.max_tokens, c.E), "schedule scratch")) != QMOE_OK)
    return bail(st);
  // The router splits d into slices only while its grid of 32 x 32 tiles is
  // short of the SMs, so split * T * E stays below SMs * 1024 when split > 1;
  // with one slice the buffer holds the T x E logits themselves.
  h->zpart_floats = std::max(Tm * (size_t)c.E, (size_t)sms * 1024);
  if ((st = h->alloc(&h->zpart, h->zpart_floats, "router partials")) != QMOE_OK) return bail(st);
  if ((st = h->alloc(&h->tile_done, (Tm + 31) / 32, "router tile counters")) != QMOE_OK) return bail(st);
  if (cudaMemset(h->tile_done, 0, sizeof(int) * ((Tm + 31) / 32)) != cudaSuccess)
    return bail(cuda_fail(cudaGetLastError(), "memset"));
  if ((st = h->alloc(&h->Xp, P * c.d, "permuted x")) != QMOE_OK) return bail(st);
  if ((st = h->alloc(&h->H, P * c.I, "H")) != QMOE_OK) return bail(st);
  for (int b = 0; b < kNumBn; ++b) {
    if (!encode_rows_map(&h->xp_map[b], h->Xp, (int)P, c.d, 16 << b) ||
        !encode_rows_map(&h->h_map[b], h->H, (int)P, c.I, 16 << b))
      return bail(fail(QMOE_ERR_CUDA, "cuTensorMapEncodeTiled failed for the activation buffers"));
  }
  if ((st = h->alloc(&h->Y, P * c.d, "Y")) != QMOE_OK) return bail(st);
  if ((st = h->alloc(&h->x_stage, Tm * c.d, "x staging")) != QMOE_OK) return bail(st);
  if ((st = h->alloc(&h->out_stage, Tm * c.d, "out staging")) != QMOE_OK) return bail(st);
  if ((st = h->alloc(&h->err, 1, "error word")) != QMOE_OK) return bail(st);
  if (cudaMemset(h->err, 0, sizeof(int)) != cudaSuccess) return bail(cuda_fail(cudaGetLastError(), "memset"));
  cudaError_t se = cudaDeviceSynchronize();
  if (se != cudaSuccess) return bail(cuda_fail(se, "qmoe_create"));
  *out = h;
  return QMOE_OK;
}

qmoe_status qmoe_route(qmoe_handle* h, const uint16_t* x, const float* logits, int32_t T, int32_t* topk_idx,
                       float* topk_gate, int32_t* counts, int32_t* offsets, int32_t* sorted_token, int32_t* inv_pos,
                       void* stream) {
  qmoe_status st = validate_tokens(h, T);
  if (st != QMOE_OK) return st;
  if ((x == nullptr) == (logits == nullptr)) return fail(QMOE_ERR_INVALID, "exactly one of x and logits must be given");
  if (!topk_idx || !topk_gate || !counts || !offsets || !sorted_token || !inv_pos)
    return fail(QMOE_ERR_INVALID, "route outputs must be non-NULL");
  if ((x && !aligned16(x)) || (logits && !aligned16(logits)))
    return fail(QMOE_ERR_INVALID, "x / logits must be 16-byte aligned");
  const int bn = choose_bn(h->cfg, T);
  return route_impl(h, x, logits, T, topk_idx, topk_gate, counts, offsets, sorted_token, inv_pos, false, bn,
                    static_cast<cudaStream_t>(stream));
}

qmoe_status qmoe_forward(qmoe_handle* h, const uint16_t* x, int32_t T, uint16_t* out, void* stream) {
  qmoe_status st = validate_tokens(h, T);
  if (st != QMOE_OK) return st;
  if (!x || !out) return fail(QMOE_ERR_INVALID, "x and out must be non-NULL");
  if (!aligned16(x) || !aligned16(out)) return fail(QMOE_ERR_INVALID, "x and out must be 16-byte aligned");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const qmoe_config& c = h->cfg;
  const int bn = choose_bn(c, T);
  st = route_impl(h, x, nullptr, T, h->idx, h->gates, h->counts, h->offsets, h->sorted_token, h->inv_pos, true, bn, s);
  if (st != QMOE_OK) return st;

  {
    // x rows in schedule order (the permutation half of stage 2)
    StageTimer tm(h, s, QMOE_STAGE_SCHEDULE);
    QMOE_CUDA(launch_permute_rows(kUsePdl, x, h->sorted_token, T * (c.k + c.n_shared), c.d, h->Xp, h->mma_f16, T,
                                  h->err, s),
              "permute launch");
  }
  GemmArgs g{};
  g.experts = h->d_experts;
  g.seg_off = h->seg_off;
  g.seg_cnt = h->seg_cnt;
  g.n_seg = c.E + c.n_shared;
  g.err = h->err;
  g.rows = T * (c.k + c.n_shared);
  g.wait_limit = h->wait_limit;
  for (int mat = 0; mat < 2; ++mat) {
    StageTimer tm(h, s, mat == 0 ? QMOE_STAGE_GATE_UP : QMOE_STAGE_DOWN);
    g.mat = mat;
    g.act = mat == 0 ? h->Xp : h->H;
    g.act_ld = mat == 0 ? c.d : c.I;
    g.K = mat == 0 ? c.d : c.I;
    g.MB = mat == 0 ? 2 * c.I / kTileM : c.d / kTileM;
    g.out = mat == 0 ? h->H : h->Y;
    g.out_ld = mat == 0 ? c.I : c.d;
    for (int fmt = 1; fmt <= 3; ++fmt) {   // one launch per weight format present
      if (!h->fmt_present[fmt]) continue;
      g.tile_off = h->tiles + tile_table_offset(mat, fmt, g.n_seg);
      const int kfmt = h->mma_f16 ? kFmtFp8F16 : fmt;
      QMOE_CUDA(launch_grouped_gemm(kUsePdl, g, mat == 0 ? h->xp_map[bn_index(bn)] : h->h_map[bn_index(bn)], kfmt, bn,
                                    h->num_sms, s),
                mat == 0 ? "gate/up GEMM launch" : "down GEMM launch");
    }
  }
  {
    StageTimer tm(h, s, QMOE_STAGE_COMBINE);
    QMOE_CUDA(launch_combine(kUsePdl, h->Y, h->gates, h->inv_pos, T, c.k, c.n_shared, c.d, out, h->err, s),
              "combine launch");
  }
  if (h->profiling) h->profiled_calls++;
  return QMOE_OK;
}

qmoe_status qmoe_forward_host(qmoe_handle* h, const uint16_t* x_host, int32_t T, uint16_t* out_host, void* stream) {
  qmoe_status st = validate_tokens(h, T);
  if (st != QMOE_OK) return st;
  if (!x_host || !out_host) return fail(QMOE_ERR_INVALID, "x_host and out_host must be non-NULL");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t bytes = (size_t)T * h->cfg.d * sizeof(uint16_t);
  QMOE_CUDA(cudaMemcpyAsync(h->x_stage, x_host, bytes, cudaMemcpyHostToDevice, s), "copy x to device");
  st = qmoe_forward(h, h->x_stage, T, h->out_stage, stream);
  if (st != QMOE_OK) return st;
  QMOE_CUDA(cudaMemcpyAsync(out_host, h->out_stage, bytes, cudaMemcpyDeviceToHost, s), "copy out to host");
  QMOE_CUDA(cudaStreamSynchronize(s), "stream synchronize");
  return QMOE_OK;
}

qmoe_status qmoe_check_error(qmoe_handle* h, void* stream) {
  if (!h) return fail(QMOE_ERR_INVALID, "handle is NULL");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int flag = 0;
  QMOE_CUDA(cudaMemcpyAsync(&flag, h->err, sizeof(int), cudaMemcpyDeviceToHost, s), "read error word");
  QMOE_CUDA(cudaStreamSynchronize(s), "stream synchronize");
  if (flag) {
    QMOE_CUDA(cudaMemsetAsync(h->err, 0, sizeof(int), s), "clear error word");
    QMOE_CUDA(cudaStreamSynchronize(s), "stream synchronize");
    if (flag & kErrBounds) return fail(QMOE_ERR_BOUNDS, "a device-side bounds check failed (QMOE_DEBUG build)");
    return fail(QMOE_ERR_TIMEOUT, "a grouped GEMM kernel hit its bounded-wait limit and aborted");
  }
  return QMOE_OK;
}

int32_t qmoe_debug_build(void) {
#ifdef QMOE_DEBUG
  return 1;
#else
  return 0;
#endif
}

qmoe_status qmoe_set_wait_limit(qmoe_handle* h, int64_t cycles) {
  if (!h) return fail(QMOE_ERR_INVALID, "handle is NULL");
  if (cycles < 0) return fail(QMOE_ERR_INVALID, "cycles must be >= 0");
  h->wait_limit = cycles == 0 ? kWaitLimit : (long long)cycles;
  return QMOE_OK;
}

qmoe_status qmoe_profile(qmoe_handle* h, int32_t enable) {
  if (!h) return fail(QMOE_ERR_INVALID, "handle is NULL");
  h->profiling = enable != 0;
  return QMOE_OK;
}

qmoe_status qmoe_profile_read(qmoe_handle* h, float* ms, int32_t n, int32_t* calls) {
  if (!h || !ms || n < 0) return fail(QMOE_ERR_INVALID, "bad arguments");
  for (auto& ev : h->events) {
    QMOE_CUDA(cudaEventSynchronize(ev.b), "event synchronize");
    float t = 0.f;
    QMOE_CUDA(cudaEventElapsedTime(&t, ev.a, ev.b), "event elapsed");
    if (ev.stage < n) ms[ev.stage] += t;
    h->event_pool.push_back(ev);
  }
  h->events.clear();
  if (calls) *calls = h->profiled_calls;
  h->profiled_calls = 0;
  return QMOE_OK;
}

int32_t qmoe_launches_per_forward(const qmoe_handle* h, int32_t T) {
  (void)T;
  if (!h) return 0;
  int fmts = 0;
  for (int f = 1; f <= 3; ++f) fmts += h->fmt_present[f] ? 1 : 0;
  return 4 + 2 * fmts;  // router, schedule, row permutation, gate/up and down per format, combine
}

qmoe_status qmoe_destroy(qmoe_handle* h) {
  if (!h) return QMOE_OK;
  cudaDeviceSynchronize();
  h->release();
  delete h;
  return QMOE_OK;
}

}  // extern "C"

// ---- routing without a handle and without allocation ------------------------
// One fixed device array per device holds the router's partial logits (every
// element that is read is written first by the same call, so nothing needs
// clearing).  Nothing here allocates device memory.
namespace {

constexpr size_t kNoallocLogits = QMOE_ROUTE_STATIC_MAX_LOGITS;  // floats
static_assert(QMOE_ROUTE_STATIC_SCRATCH_BYTES == 4 * kNoallocLogits, "scratch size");
static __device__ __align__(256) unsigned char g_route_scratch[QMOE_ROUTE_STATIC_SCRATCH_BYTES];

constexpr int kNoallocMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_addr[kNoallocMaxDevices] = {};
int g_noalloc_sms[kNoallocMaxDevices] = {};

// Address of this device's copy of the array (looked up once per device).
qmoe_status noalloc_scratch(void** addr, int* sms) {
  int dev = 0;
  QMOE_CUDA(cudaGetDevice(&dev), "cudaGetDevice");
  if (dev < 0 || dev >= kNoallocMaxDevices) return fail(QMOE_ERR_UNSUPPORTED, "device ordinal out of range");
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_addr[dev]) {
    int d2 = 0, n = 0;
    qmoe_status st = check_device(&d2, &n);
    if (st != QMOE_OK) return st;
    void* p = nullptr;
    QMOE_CUDA(cudaGetSymbolAddress(&p, g_route_scratch), "cudaGetSymbolAddress for the routing scratch");
    g_noalloc_sms[dev] = n;
    g_noalloc_addr[dev] = p;
  }
  *addr = g_noalloc_addr[dev];
  *sms = g_noalloc_sms[dev];
  return QMOE_OK;
}

}  // namespace

qmoe_status qmoe_route_topk_noalloc(const uint16_t* x, const float* router_w, const float* router_bias, int32_t T,
                                    int32_t d, int32_t E, int32_t k, int32_t* topk_idx, float* topk_gate,
                                    void* stream) {
  if (!x || !router_w || !topk_idx || !topk_gate)
    return fail(QMOE_ERR_INVALID, "x, router_w, topk_idx and topk_gate must be non-NULL");
  if (!aligned16(x) || !aligned16(router_w)) return fail(QMOE_ERR_INVALID, "x and router_w must be 16-byte aligned");
  if (d < kBK || d % kBK != 0) return fail(QMOE_ERR_INVALID, "d must be a positive multiple of 128");
  if (E < 1 || E > kMaxE) return fail(QMOE_ERR_INVALID, "E must be in [1, 256]");
  if (k < 1 || k > E || k > kMaxK) return fail(QMOE_ERR_INVALID, "k must be in [1, min(E, 16)]");
  if (T < 1) return fail(QMOE_ERR_INVALID, "T must be >= 1");
  if ((long long)T * E > (long long)kNoallocLogits)
    return fail(QMOE_ERR_INVALID, "T*E=" + std::to_string((long long)T * E) + " exceeds the fixed routing scratch (" +
                                      std::to_string(kNoallocLogits) + " logits)");
  void* base = nullptr;
  int sms = 0;
  qmoe_status st = noalloc_scratch(&base, &sms);
  if (st != QMOE_OK) return st;
  float* zpart = static_cast<float*>(base);
  int split = router_split(T, d, E, sms);
  while (split > 1 && (long long)split * T * E > (long long)kNoallocLogits) split >>= 1;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  QMOE_CUDA(launch_router(x, router_w, router_bias, T, d, E, k, split, zpart, topk_idx, topk_gate, s),
            "router launch");
  return QMOE_OK;
}
