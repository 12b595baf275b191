// proj.cu -- the projections on either side of the path, on the library's own GEMMs
// (gemm_sm100.cu: tcgen05 tensor cores for bf16, CUDA cores for the exact fp32 path):
//   forward:  [q | k | v] = X [W_Q | W_K | W_V], one GEMM (the three weights side by side
//             along N), written in the [B, H, n, d] layout the attention kernels read;
//   backward: each gradient is first merged to [B n, H d] rows (a copy kernel into the
//             caller's workspace, the three side by side), then
//             [dW_Q | dW_K | dW_V] = X^T [dQ | dK | dV]     (one GEMM, segmented along N)
//             dX = [dQ | dK | dV] [W_Q | W_K | W_V]^T       (one GEMM, segmented along K)
// ("RoPE attention can be trained in almost-linear time", Lemma 4.1: the loss gradient with
// respect to the weights, reached from the gradient of the attention inputs through X).
//
// Layouts (row-major): X [B, n, d_model]; W [d_model, H d] with head h in columns
// h d .. h d + d - 1; Q, K, V, dQ, dK, dV [B, H, n, d]; dW [d_model, H d] fp32;
// dX [B, n, d_model] fp32.  Accumulation is fp32 in a fixed order (no atomics), so the
// results are deterministic.
#include <cuda.h>
#include <cuda_runtime.h>

#include "common.h"
#include "gemm.h"
#include "launch.h"
#include "rope_attn.h"

namespace {

constexpr size_t kProjErrBytes = 1024;  // the error word region at the start of ws

bool aligned16(const void* p) { return p && (reinterpret_cast<uintptr_t>(p) % 16) == 0; }

ra_status check(const ra_problem* p, int64_t d_model) {
  if (!p || p->B < 1 || p->H < 1 || p->n < 1 || p->d < 2 || (p->d % 2) != 0)
    return RA_ERR_INVALID_ARG;
  if (p->dtype != RA_F32 && p->dtype != RA_BF16) return RA_ERR_INVALID_ARG;
  if (d_model < 1 || d_model > (int64_t(1) << 20)) return RA_ERR_INVALID_ARG;
  // 32-bit GEMM sizes; each factor is bounded before a product is formed, so no product
  // overflows and every byte count fits a size_t
  if (p->B > (int64_t(1) << 30) || p->n > (int64_t(1) << 30) || p->H > (int64_t(1) << 30) ||
      p->d > (int64_t(1) << 30))
    return RA_ERR_UNSUPPORTED;
  if (p->B * p->n > (int64_t(1) << 30) || 3 * p->H * p->d > (int64_t(1) << 30))
    return RA_ERR_UNSUPPORTED;
  if (p->B * p->n * p->H * p->d > (int64_t(1) << 38)) return RA_ERR_UNSUPPORTED;
  // the tensor-core GEMM: every 64-wide box inside one head and one weight (d in {64, 128}),
  // 16-byte rows for the tensor maps (d_model a multiple of 8)
  if (p->dtype == RA_BF16 && ((p->d != 64 && p->d != 128) || d_model % 8 != 0))
    return RA_ERR_UNSUPPORTED;
  return RA_OK;
}

size_t elem(const ra_problem* p) { return p->dtype == RA_BF16 ? 2 : 4; }

size_t merged_bytes(const ra_problem* p) {
  return (size_t)(p->B * p->n * p->H * p->d) * elem(p);
}

ra_status check_ws(const ra_problem* p, void* ws, size_t ws_bytes, bool merged) {
  if (!ws || (reinterpret_cast<uintptr_t>(ws) % 256) != 0) return RA_ERR_WORKSPACE;
  if (ws_bytes < kProjErrBytes + (merged ? 3 * ra::align_up(merged_bytes(p), 1024) : 0))
    return RA_ERR_WORKSPACE;
  return RA_OK;
}

uint8_t* merged_at(void* ws, const ra_problem* p, int which) {
  return static_cast<uint8_t*>(ws) + kProjErrBytes +
         (size_t)which * ra::align_up(merged_bytes(p), 1024);
}

}  // namespace

extern "C" {

size_t rope_attn_proj_workspace_bytes(const ra_problem* p) {
  if (check(p, 8) != RA_OK) return 0;
  return kProjErrBytes + 3 * ra::align_up(merged_bytes(p), 1024);
}

ra_status rope_attn_proj_fwd(const ra_problem* p, int64_t d_model, const void* x, const void* wq,
                             const void* wk, const void* wv, void* q, void* k, void* v, void* ws,
                             size_t ws_bytes, void* stream) {
  ra_status st = check(p, d_model);
  if (st != RA_OK) return st;
  if (!aligned16(x) || !aligned16(wq) || !aligned16(wk) || !aligned16(wv) || !aligned16(q) ||
      !aligned16(k) || !aligned16(v))
    return RA_ERR_INVALID_ARG;
  if ((st = check_ws(p, ws, ws_bytes, false)) != RA_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(ws, 0, 64, s) != cudaSuccess) return RA_ERR_CUDA;
  const int rows = (int)(p->B * p->n), hd = (int)(p->H * p->d), dm = (int)d_model;
  // C[B n][3 H d] = X [W_Q | W_K | W_V]: A = X K-major, B = W MN-major (segmented along N)
  ra::GemmSpec spec{rows, 3 * hd, dm, 0, 0, 0, 1, 1, 0, hd, 3};
  spec.bk = 64;  // four stages in flight: both operands already stream as whole rows
  spec.b_rowbox = hd % 256 == 0;
  const ra::GemmOut out{{q, k, v}, ra::GEMM_OUT_HEADS, hd, 3, 0, (int)p->n, (int)p->H,
                        (int)p->d};
  const void* W[3] = {wq, wk, wv};
  cudaError_t e;
  if (p->dtype == RA_BF16) {
    CUtensorMap am[1], bm[3];
    if (!ra::gemm_operand_map(&am[0], spec, false, x, rows, dm)) return RA_ERR_CUDA;
    for (int w = 0; w < 3; ++w)
      if (!ra::gemm_operand_map(&bm[w], spec, true, W[w], dm, hd)) return RA_ERR_CUDA;
    const ra::TimingScope timed(ra::K_PROJ_GEMM, s);
    e = ra::launch_gemm_bf16(spec, am, bm, out, static_cast<uint32_t*>(ws), ra::wait_limit_ns(),
                             s);
  } else {
    const void* a[1] = {x};
    const ra::TimingScope timed(ra::K_PROJ_GEMM, s);
    e = ra::launch_gemm_f32(spec, a, dm, 0, W, hd, 0, out, s);
  }
  return e == cudaSuccess ? RA_OK : RA_ERR_CUDA;
}

ra_status rope_attn_proj_bwd(const ra_problem* p, int64_t d_model, const void* x, const void* wq,
                             const void* wk, const void* wv, const void* dq, const void* dk,
                             const void* dv, float* dwq, float* dwk, float* dwv, float* dx,
                             void* ws, size_t ws_bytes, void* stream) {
  ra_status st = check(p, d_model);
  if (st != RA_OK) return st;
  if (!aligned16(x) || !aligned16(wq) || !aligned16(wk) || !aligned16(wv) || !aligned16(dq) ||
      !aligned16(dk) || !aligned16(dv) || !aligned16(dwq) || !aligned16(dwk) ||
      !aligned16(dwv) || !aligned16(dx))
    return RA_ERR_INVALID_ARG;
  if ((st = check_ws(p, ws, ws_bytes, true)) != RA_OK) return st;
  // the head merge moves 16-byte vectors: a d-row must be a whole number of them
  if (((size_t)p->d * elem(p)) % 16 != 0) return RA_ERR_UNSUPPORTED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(ws, 0, 64, s) != cudaSuccess) return RA_ERR_CUDA;
  const int rows = (int)(p->B * p->n), hd = (int)(p->H * p->d), dm = (int)d_model;
  const void* G[3] = {dq, dk, dv};
  const void* W[3] = {wq, wk, wv};
  void* Y[3];
  for (int w = 0; w < 3; ++w) {
    Y[w] = merged_at(ws, p, w);
    // Y_w = the gradient merged to [B n, H d] rows (row (b, i) holds every head of position i)
    cudaError_t em;
    {
      const ra::TimingScope timed(ra::K_MERGE_HEADS, s);
      em = ra::launch_merge_heads(*p, G[w], Y[w], s);
    }
    if (em != cudaSuccess) return RA_ERR_CUDA;
  }
  // [dW_Q | dW_K | dW_V] (d_model x 3 H d) = X^T [Y_Q | Y_K | Y_V]: A = X MN-major,
  // B = Y MN-major segmented along N; K = B n
  ra::GemmSpec sw{dm, 3 * hd, rows, 1, 0, 0, 1, 1, 0, hd, 3};
  sw.bk = 64;
  sw.a_rowbox = dm % 64 == 0;
  sw.b_rowbox = hd % 256 == 0;
  const ra::GemmOut ow{{dwq, dwk, dwv}, ra::GEMM_OUT_F32, hd, 3, hd, 0, 0, 0};
  // dX (B n x d_model) = [Y_Q | Y_K | Y_V] [W_Q | W_K | W_V]^T: A = Y K-major segmented along
  // K, B = W K-major ([d_model][H d] rows) segmented along K; K = 3 H d
  ra::GemmSpec sx{rows, dm, 3 * hd, 0, 1, hd, 3, 0, 1, hd, 3};
  // K-major operands: 128-wide K chunks make every row piece 256 contiguous bytes
  sx.bk = 128;
  sx.a_rowbox = sx.b_rowbox = hd % 128 == 0;
  const ra::GemmOut ox{{dx, dx, dx}, ra::GEMM_OUT_F32, dm, 1, dm, 0, 0, 0};
  cudaError_t e;
  if (p->dtype == RA_BF16) {
    uint32_t* err = static_cast<uint32_t*>(ws);
    const uint64_t wait = ra::wait_limit_ns();
    CUtensorMap xa[1], yb[3], ya[3], wb[3];
    if (!ra::gemm_operand_map(&xa[0], sw, false, x, rows, dm)) return RA_ERR_CUDA;
    for (int w = 0; w < 3; ++w)
      if (!ra::gemm_operand_map(&yb[w], sw, true, Y[w], rows, hd) ||
          !ra::gemm_operand_map(&ya[w], sx, false, Y[w], rows, hd) ||
          !ra::gemm_operand_map(&wb[w], sx, true, W[w], dm, hd))
        return RA_ERR_CUDA;
    {
      const ra::TimingScope timed(ra::K_PROJ_DW, s);
      e = ra::launch_gemm_bf16(sw, xa, yb, ow, err, wait, s);
    }
    if (e == cudaSuccess) {
      const ra::TimingScope timed(ra::K_PROJ_DX, s);
      e = ra::launch_gemm_bf16(sx, ya, wb, ox, err, wait, s);
    }
  } else {
    const void* xs[1] = {x};
    const void* ys[3] = {Y[0], Y[1], Y[2]};
    {
      const ra::TimingScope timed(ra::K_PROJ_DW, s);
      e = ra::launch_gemm_f32(sw, xs, dm, 0, ys, hd, 0, ow, s);
    }
    if (e == cudaSuccess) {
      const ra::TimingScope timed(ra::K_PROJ_DX, s);
      e = ra::launch_gemm_f32(sx, ys, hd, 0, W, hd, 0, ox, s);
    }
  }
  return e == cudaSuccess ? RA_OK : RA_ERR_CUDA;
}

}  // extern "C"
