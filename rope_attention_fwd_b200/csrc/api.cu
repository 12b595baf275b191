// api.cu -- host implementation of the C ABI declared in include/rope_attn.h:
// argument validation, workspace carving, TMA tensor-map encoding, the launch
// sequence of each call and the optional per-kernel event timing.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <vector>

#include "common.h"
#include "launch.h"

using namespace ra;

namespace {

// ------------------------------------------------------------------ timing
struct TimedLaunch {
  int kid;
  cudaEvent_t start, stop;
};
std::mutex g_timing_mu;
bool g_timing = false;
std::vector<TimedLaunch> g_timed;
std::vector<cudaEvent_t> g_event_pool;

cudaEvent_t take_event() {
  if (!g_event_pool.empty()) {
    cudaEvent_t e = g_event_pool.back();
    g_event_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}

}  // namespace

namespace ra {

cudaEvent_t timing_begin(cudaStream_t s) {
  std::lock_guard<std::mutex> g(g_timing_mu);
  if (!g_timing) return nullptr;
  cudaEvent_t start = take_event();
  cudaEventRecord(start, s);
  return start;
}

void timing_end(cudaEvent_t start, int kid, cudaStream_t s) {
  if (!start) return;
  std::lock_guard<std::mutex> g(g_timing_mu);
  cudaEvent_t stop = take_event();
  cudaEventRecord(stop, s);
  g_timed.push_back({kid, start, stop});
}

}  // namespace ra

namespace {

struct LaunchScope {
  int kid;
  cudaStream_t s;
  cudaEvent_t start;
  LaunchScope(int k, cudaStream_t st) : kid(k), s(st), start(timing_begin(st)) {}
  void done() {
    timing_end(start, kid, s);
    start = nullptr;
  }
};

#define RA_LAUNCH(kid, stream, expr)              \
  do {                                            \
    LaunchScope _ls((kid), (stream));             \
    cudaError_t _e = (expr);                      \
    _ls.done();                                   \
    if (_e != cudaSuccess) return RA_ERR_CUDA;    \
  } while (0)

// ------------------------------------------------------------------ validation
bool aligned16(const void* ptr) { return ptr && (reinterpret_cast<uintptr_t>(ptr) % 16) == 0; }

ra_status check_problem(const ra_problem* p) {
  if (!p) return RA_ERR_INVALID_ARG;
  if (p->B < 1 || p->H < 1 || p->n < 1 || p->d < 2 || (p->d % 2) != 0) return RA_ERR_INVALID_ARG;
  if (p->dtype != RA_F32 && p->dtype != RA_BF16) return RA_ERR_INVALID_ARG;
  if (p->causal != 0 && p->causal != 1) return RA_ERR_INVALID_ARG;
  if (!(p->base > 0.0) || !std::isfinite(p->base)) return RA_ERR_INVALID_ARG;
  // Size limits, each tested before a product that could overflow: every byte count and
  // grid size the launchers form from B, H, n and d then fits its type (B H n d <= 2^38
  // elements is 512 GiB per bf16 tensor, beyond any one device).
  if (p->B > (int64_t(1) << 30) || p->H > (int64_t(1) << 30) || p->n > (int64_t(1) << 30))
    return RA_ERR_UNSUPPORTED;
  if (p->B * p->H > (int64_t(1) << 30)) return RA_ERR_UNSUPPORTED;
  if (p->d > 128) return RA_ERR_UNSUPPORTED;
  if (p->B * p->H * p->n > (int64_t(1) << 38) / p->d) return RA_ERR_UNSUPPORTED;
  // the fp32 kernels put (batch, head) on the grid's y dimension
  if (p->dtype == RA_F32 && p->B * p->H > 65535) return RA_ERR_UNSUPPORTED;
  if (p->fixed_bands < 0 || p->fixed_bands > p->d / 2 || p->reserved != 0)
    return RA_ERR_INVALID_ARG;
  if (p->d > 128) return RA_ERR_UNSUPPORTED;
  if (p->dtype == RA_BF16 && p->d != 64 && p->d != 128) return RA_ERR_UNSUPPORTED;
  return RA_OK;
}

// fwd_only: the forward needs only the leading regions of the layout (error word, loss
// partials, table, Q~, K~), so a smaller workspace is enough for it.
ra_status check_ws(const ra_problem* p, void* ws, size_t ws_bytes, bool fwd_only = false) {
  if (!ws || (reinterpret_cast<uintptr_t>(ws) % 256) != 0) return RA_ERR_WORKSPACE;
  const WsLayout L = ws_layout(*p);
  if (ws_bytes < (fwd_only ? L.fwd_total : L.total)) return RA_ERR_WORKSPACE;
  return RA_OK;
}


// Test hook for the bounded-wait path: RA_DEBUG_STARVE_BLOCK=<cta> makes that CTA of
// the bf16 forward skip its Q~ load, so its waits expire and it reports RA_ERR_TIMEOUT.
int starve_block() {
  const char* s = std::getenv("RA_DEBUG_STARVE_BLOCK");
  return s ? std::atoi(s) : -1;
}

template <typename T>
T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<uint8_t*>(ws) + off);
}

// ------------------------------------------------------------------ tensor maps
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return (EncodeTiledFn) nullptr;
    return reinterpret_cast<EncodeTiledFn>(f);
  }();
  return fn;
}

// 16-bit [BH][n][d] tensor (bf16 inputs, or the fp16 rotated Q~ / K~ when fp16 is set)
// viewed as (x = d, y = n, z = BH); box = 64 columns x `rows` rows.
bool make_map(CUtensorMap* map, const void* ptr, const ra_problem& p, int rows,
              bool fp16 = false) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)p.d, (cuuint64_t)p.n, (cuuint64_t)(p.B * p.H)};
  const cuuint64_t strides[2] = {(cuuint64_t)p.d * 2, (cuuint64_t)p.n * p.d * 2};
  const cuuint32_t box[3] = {64, (cuuint32_t)rows, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, fp16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
            const_cast<void*>(ptr), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Shared prefix of fwd and bwd: clear the error word, build the table, rotate Q and K.
ra_status prepare(const ra_problem* p, const void* q, const void* k, const float* alpha,
                  void* ws, const WsLayout& L, cudaStream_t s) {
  if (cudaMemsetAsync(at<uint8_t>(ws, L.err), 0, 64, s) != cudaSuccess) return RA_ERR_CUDA;
  RA_LAUNCH(K_TABLE, s, launch_table(*p, alpha, at<float2>(ws, L.table), s));
  RA_LAUNCH(K_ROTATE, s,
            launch_rotate(*p, q, k, at<void>(ws, L.qt), at<void>(ws, L.kt),
                          at<float2>(ws, L.table), at<uint32_t>(ws, L.err), s));
  return RA_OK;
}

}  // namespace

namespace ra {

uint64_t wait_limit_ns() {
  const char* s = std::getenv("RA_WAIT_LIMIT_MS");
  double ms = s ? std::atof(s) : 2000.0;
  if (!(ms > 0)) ms = 2000.0;
  return (uint64_t)(ms * 1e6);
}

bool tensor_map_rows(CUtensorMap* map, const void* ptr, uint64_t rows, uint64_t chunks,
                     uint64_t row_bytes, uint32_t box_rows, uint32_t box_chunks) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {64, (cuuint64_t)rows, (cuuint64_t)chunks};
  const cuuint64_t strides[2] = {(cuuint64_t)row_bytes, 128};
  const cuuint32_t box[3] = {64, box_rows, box_chunks};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool tensor_map_2d(CUtensorMap* map, const void* ptr, bool f32, uint64_t inner, uint64_t outer,
                   uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)outer};
  const cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
            const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace ra

extern "C" {

size_t rope_attn_workspace_bytes(const ra_problem* p) {
  if (check_problem(p) != RA_OK) return 0;
  return ws_layout(*p).total;
}

size_t rope_attn_fwd_workspace_bytes(const ra_problem* p) {
  if (check_problem(p) != RA_OK) return 0;
  return ws_layout(*p).fwd_total;
}

const char* rope_attn_status_string(ra_status s) {
  switch (s) {
    case RA_OK: return "ok";
    case RA_ERR_INVALID_ARG: return "invalid argument";
    case RA_ERR_UNSUPPORTED: return "unsupported problem";
    case RA_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case RA_ERR_CUDA: return "CUDA error";
    case RA_ERR_TIMEOUT: return "device-side wait timed out";
    case RA_ERR_RANGE: return "input entry beyond the fp16 range of the score operands";
  }
  return "unknown status";
}

ra_status rope_attn_fwd(const ra_problem* p, const void* q, const void* k, const void* v,
                        const float* alpha, void* o, float* lse, void* ws, size_t ws_bytes,
                        void* stream) {
  ra_status st = check_problem(p);
  if (st != RA_OK) return st;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(alpha) || !aligned16(o) ||
      !aligned16(lse))
    return RA_ERR_INVALID_ARG;
  if ((st = check_ws(p, ws, ws_bytes, true)) != RA_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const WsLayout L = ws_layout(*p);
  if ((st = prepare(p, q, k, alpha, ws, L, s)) != RA_OK) return st;
  if (p->dtype == RA_F32) {
    RA_LAUNCH(K_FWD_F32, s,
              launch_fwd_f32(*p, at<float>(ws, L.qt), at<float>(ws, L.kt), (const float*)v,
                             (float*)o, lse, s));
    return RA_OK;
  }
  Sm100Maps maps;
  std::memset(&maps, 0, sizeof(maps));
  if (!make_map(&maps.qt, at<void>(ws, L.qt), *p, 128, true) ||
      !make_map(&maps.kt, at<void>(ws, L.kt), *p, 128, true) || !make_map(&maps.v, v, *p, 128))
    return RA_ERR_CUDA;
  DevCtl ctl{at<uint32_t>(ws, L.err), wait_limit_ns(), starve_block()};
  RA_LAUNCH(K_FWD_SM100, s, launch_fwd_sm100(*p, maps, o, lse, ctl, s));
  return RA_OK;
}

ra_status rope_attn_loss(const ra_problem* p, const void* o, const void* e, float* Lout,
                         void* dO, void* ws, size_t ws_bytes, void* stream) {
  ra_status st = check_problem(p);
  if (st != RA_OK) return st;
  if (!aligned16(o) || !aligned16(e) || !aligned16(dO) || !Lout ||
      (reinterpret_cast<uintptr_t>(Lout) % 4) != 0)
    return RA_ERR_INVALID_ARG;
  if ((st = check_ws(p, ws, ws_bytes)) != RA_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const WsLayout L = ws_layout(*p);
  if (cudaMemsetAsync(at<uint8_t>(ws, L.err), 0, 64, s) != cudaSuccess) return RA_ERR_CUDA;
  RA_LAUNCH(K_LOSS_PARTIAL, s, launch_loss_partial(*p, o, e, dO, at<double>(ws, L.loss_part), s));
  RA_LAUNCH(K_LOSS_FINAL, s, launch_loss_final(at<double>(ws, L.loss_part), Lout, s));
  return RA_OK;
}

}  // extern "C"

namespace {

// Backward body shared by rope_attn_bwd (saved = false: clears the error word, builds the
// table and rotates q, k into ws) and rope_attn_bwd_saved (saved = true: uses the table,
// Q~ and K~ a previous forward left in ws and clears only the two max statistics).
ra_status bwd_impl(const ra_problem* p, const void* q, const void* k, const void* v,
                   const void* o, const float* lse, const void* dO, const float* alpha,
                   void* dq, void* dk, void* dv, float* dalpha, void* ws, size_t ws_bytes,
                   void* stream, bool saved) {
  ra_status st = check_problem(p);
  if (st != RA_OK) return st;
  // dalpha may be null: frozen frequencies, no frequency gradient (its partials and the
  // final reduction are skipped)
  if ((!saved && (!aligned16(q) || !aligned16(k))) || !aligned16(v) || !aligned16(o) ||
      !aligned16(lse) || !aligned16(dO) || !aligned16(alpha) || !aligned16(dq) ||
      !aligned16(dk) || !aligned16(dv) || (dalpha && !aligned16(dalpha)))
    return RA_ERR_INVALID_ARG;
  if ((st = check_ws(p, ws, ws_bytes)) != RA_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const WsLayout L = ws_layout(*p);
  if (saved) {
    // the two max statistics (words 8, 9 of the error region) start from zero
    if (cudaMemsetAsync(at<uint8_t>(ws, L.err) + 32, 0, 8, s) != cudaSuccess) return RA_ERR_CUDA;
  } else if ((st = prepare(p, q, k, alpha, ws, L, s)) != RA_OK) {
    return st;
  }
  float* delta = at<float>(ws, L.delta);
  float* dpart = dalpha ? at<float>(ws, L.dpart) : nullptr;
  const float2* table = at<float2>(ws, L.table);
  if (p->dtype == RA_F32) {
    RA_LAUNCH(K_BWD_DELTA, s, launch_delta(*p, o, dO, delta, s));
    const float* qt = at<float>(ws, L.qt);
    const float* kt = at<float>(ws, L.kt);
    RA_LAUNCH(K_BWD_DKDV_F32, s,
              launch_bwd_dkdv_f32(*p, qt, kt, (const float*)v, (const float*)dO, lse, delta,
                                  table, (float*)dk, (float*)dv, dpart, s));
    RA_LAUNCH(K_BWD_DQ_F32, s,
              launch_bwd_dq_f32(*p, qt, kt, (const float*)v, (const float*)dO, lse, delta, table,
                                (float*)dq, dpart, s));
  } else {
    float* lse2 = at<float>(ws, L.lse2);
    uint32_t* stats = at<uint32_t>(ws, L.err) + 8;  // zeroed with the error word in prepare()
    RA_LAUNCH(K_BWD_DELTA, s, launch_bwd_pre(*p, o, dO, v, lse, delta, lse2, stats, s));
    Sm100Maps maps;
    std::memset(&maps, 0, sizeof(maps));
    void* qt = at<void>(ws, L.qt);
    void* kt = at<void>(ws, L.kt);
    if (!make_map(&maps.qt, qt, *p, 128, true) || !make_map(&maps.kt, kt, *p, 128, true) ||
        !make_map(&maps.v, v, *p, 128) || !make_map(&maps.dO, dO, *p, 128) ||
        !make_map(&maps.qt64, qt, *p, 64, true) || !make_map(&maps.kt64, kt, *p, 64, true) ||
        !make_map(&maps.v64, v, *p, 64) || !make_map(&maps.dO64, dO, *p, 64))
      return RA_ERR_CUDA;
    DevCtl ctl{at<uint32_t>(ws, L.err), wait_limit_ns(), -1};
    // two passes: dK, dV (keys stationary), then dQ (queries stationary, S and dP
    // recomputed); every output bitwise reproducible
    RA_LAUNCH(K_BWD_DKDV_SM100, s,
              launch_bwd_dkdv_sm100(*p, maps, lse2, delta, table, stats, dk, dv, dpart, ctl, s));
    RA_LAUNCH(K_BWD_DQ_SM100, s,
              launch_bwd_dq_sm100(*p, maps, lse2, delta, table, stats, dq, dpart, ctl, s));
  }
  if (dalpha) RA_LAUNCH(K_DALPHA, s, launch_dalpha_final(*p, dpart, alpha, dalpha, s));
  return RA_OK;
}

}  // namespace

extern "C" {

ra_status rope_attn_bwd(const ra_problem* p, const void* q, const void* k, const void* v,
                        const void* o, const float* lse, const void* dO, const float* alpha,
                        void* dq, void* dk, void* dv, float* dalpha, void* ws, size_t ws_bytes,
                        void* stream) {
  return bwd_impl(p, q, k, v, o, lse, dO, alpha, dq, dk, dv, dalpha, ws, ws_bytes, stream,
                  false);
}

ra_status rope_attn_bwd_saved(const ra_problem* p, const void* v, const void* o,
                              const float* lse, const void* dO, const float* alpha, void* dq,
                              void* dk, void* dv, float* dalpha, void* ws, size_t ws_bytes,
                              void* stream) {
  return bwd_impl(p, nullptr, nullptr, v, o, lse, dO, alpha, dq, dk, dv, dalpha, ws, ws_bytes,
                  stream, true);
}

ra_status rope_attn_alpha_adam(const ra_adam* opt, int64_t count, float* alpha,
                               const float* dalpha, float* m1, float* m2, void* stream) {
  if (!opt || count < 1 || count > (int64_t(1) << 20)) return RA_ERR_INVALID_ARG;
  if (!aligned16(alpha) || !aligned16(dalpha) || !aligned16(m1) || !aligned16(m2))
    return RA_ERR_INVALID_ARG;
  if (!(opt->lr >= 0.f) || !(opt->beta1 >= 0.f && opt->beta1 < 1.f) ||
      !(opt->beta2 >= 0.f && opt->beta2 < 1.f) || !(opt->eps > 0.f) || opt->step < 1 ||
      !std::isfinite(opt->clip_norm))
    return RA_ERR_INVALID_ARG;
  const float bc1 = (float)(1.0 - std::pow((double)opt->beta1, (double)opt->step));
  const float bc2 = (float)(1.0 - std::pow((double)opt->beta2, (double)opt->step));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  RA_LAUNCH(K_ALPHA_ADAM, s,
            launch_alpha_adam(alpha, dalpha, m1, m2, count, opt->lr, opt->beta1, opt->beta2,
                              opt->eps, opt->clip_norm, bc1, bc2, s));
  return RA_OK;
}

ra_status rope_attn_device_status(void* ws, size_t ws_bytes, void* stream, int32_t info[3]) {
  if (!ws || ws_bytes < 64 || (reinterpret_cast<uintptr_t>(ws) % 256) != 0)
    return RA_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t word[4] = {0, 0, 0, 0};
  // The error word is the first region of every workspace layout.
  if (cudaMemcpyAsync(word, ws, sizeof(word), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return RA_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return RA_ERR_CUDA;
  if (cudaMemsetAsync(ws, 0, 16, s) != cudaSuccess) return RA_ERR_CUDA;
  if (info) {
    info[0] = (int32_t)word[1];
    info[1] = (int32_t)word[2];
    info[2] = (int32_t)word[3];
  }
  if (word[0] == 0) return RA_OK;
  return word[0] == (uint32_t)RA_ERR_RANGE ? RA_ERR_RANGE : RA_ERR_TIMEOUT;
}

void rope_attn_timing_enable(int on) {
  std::lock_guard<std::mutex> g(g_timing_mu);
  g_timing = on != 0;
}

int rope_attn_timing_read(int32_t* launches, double* total_ms, int max_ids) {
  std::vector<TimedLaunch> rec;
  {
    std::lock_guard<std::mutex> g(g_timing_mu);
    rec.swap(g_timed);
  }
  const int nid = max_ids < K_COUNT ? max_ids : (int)K_COUNT;
  for (int i = 0; i < nid; ++i) {
    launches[i] = 0;
    total_ms[i] = 0.0;
  }
  for (auto& r : rec) {
    cudaEventSynchronize(r.stop);
    float ms = 0.f;
    cudaEventElapsedTime(&ms, r.start, r.stop);
    if (r.kid < nid) {
      launches[r.kid] += 1;
      total_ms[r.kid] += ms;
    }
  }
  std::lock_guard<std::mutex> g(g_timing_mu);
  for (auto& r : rec) {
    g_event_pool.push_back(r.start);
    g_event_pool.push_back(r.stop);
  }
  return nid;
}

const char* rope_attn_kernel_name(int id) {
  static const char* names[K_COUNT] = {
      "rope_table",       "rotate",       "fwd_f32",      "fwd_sm100",
      "loss_partial",     "loss_final",   "bwd_delta",    "bwd_dq_f32",
      "bwd_dkdv_f32",     "bwd_dq_sm100", "bwd_dkdv_sm100", "dalpha_final",
      "proj_gemm",        "proj_dw_gemm", "proj_dx_gemm", "merge_heads",
      "spectrum",         "alpha_adam"};
  return (id >= 0 && id < K_COUNT) ? names[id] : "unknown";
}

}  // extern "C"
