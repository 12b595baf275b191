// launch.h -- host-side launchers of every kernel (defined next to the kernels).
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include "common.h"

namespace ra {

// Bound on every device-side wait: RA_WAIT_LIMIT_MS (default 2000 ms), read per call.
uint64_t wait_limit_ns();

// A 2-D row-major tensor map (inner x outer elements, rows row_bytes apart), 128-byte
// swizzle, box box_inner x box_outer; false if the driver rejects it.
// bf16 row-major [rows][row_elems] tensor viewed as (x = 64 columns of a chunk, y = row,
// z = 64-column chunk), the chunk stride (128 B) below the row stride; box {64, box_rows,
// box_chunks} is box_rows whole row segments of 64 * box_chunks columns in one request,
// stored chunk-major in shared memory (128-byte swizzle).
bool tensor_map_rows(CUtensorMap* map, const void* ptr, uint64_t rows, uint64_t chunks,
                     uint64_t row_bytes, uint32_t box_rows, uint32_t box_chunks);
bool tensor_map_2d(CUtensorMap* map, const void* ptr, bool f32, uint64_t inner, uint64_t outer,
                   uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer);

// Per-kernel event timing (rope_attn_timing_enable).  While it is on, timing_begin records a
// start event on s and timing_end a stop event, the pair filed under kernel id kid; while it
// is off timing_begin returns nullptr and timing_end does nothing.
cudaEvent_t timing_begin(cudaStream_t s);
void timing_end(cudaEvent_t start, int kid, cudaStream_t s);

// timing_begin at construction, timing_end when the scope is left (early returns included).
struct TimingScope {
  cudaEvent_t start;
  int kid;
  cudaStream_t s;
  TimingScope(int k, cudaStream_t st) : start(timing_begin(st)), kid(k), s(st) {}
  ~TimingScope() { timing_end(start, kid, s); }
  TimingScope(const TimingScope&) = delete;
  TimingScope& operator=(const TimingScope&) = delete;
};

struct DevCtl {
  uint32_t* err;        // workspace error word
  uint64_t wait_ns;     // bound on every device-side wait
  int starve_block;     // test hook: this CTA of the forward skips its Q~ load (-1 = off)
};

cudaError_t launch_table(const ra_problem& p, const float* alpha, float2* table, cudaStream_t s);
// bf16 problems: Q~, K~ written as fp16; an entry beyond fp16 range sets err[0] = 6.
cudaError_t launch_rotate(const ra_problem& p, const void* q, const void* k, void* qt, void* kt,
                          const float2* table, uint32_t* err, cudaStream_t s);
cudaError_t launch_loss_partial(const ra_problem& p, const void* o, const void* e, void* dO,
                                double* part, cudaStream_t s);
cudaError_t launch_loss_final(const double* part, float* L, cudaStream_t s);
cudaError_t launch_delta(const ra_problem& p, const void* o, const void* dO, float* delta,
                         cudaStream_t s);
// One Adam step for alpha with dalpha clipped to L2 norm clip first (one block).
cudaError_t launch_alpha_adam(float* alpha, const float* dalpha, float* m1, float* m2,
                              long long count, float lr, float b1, float b2, float eps,
                              float clip, float bc1, float bc2, cudaStream_t s);
// A [B, H, n, d] tensor as [B n, H d] rows (row (b, i) holds every head of position i).
cudaError_t launch_merge_heads(const ra_problem& p, const void* g, void* y, cudaStream_t s);
cudaError_t launch_dalpha_final(const ra_problem& p, const float* part, const float* alpha,
                                float* dalpha, cudaStream_t s);

// fp32 CUDA-core attention (any even d <= 128)
cudaError_t launch_fwd_f32(const ra_problem& p, const float* qt, const float* kt, const float* v,
                           float* o, float* lse, cudaStream_t s);
cudaError_t launch_bwd_dq_f32(const ra_problem& p, const float* qt, const float* kt,
                              const float* v, const float* dO, const float* lse,
                              const float* delta, const float2* table, float* dq, float* dpart,
                              cudaStream_t s);
cudaError_t launch_bwd_dkdv_f32(const ra_problem& p, const float* qt, const float* kt,
                                const float* v, const float* dO, const float* lse,
                                const float* delta, const float2* table, float* dk, float* dv,
                                float* dpart, cudaStream_t s);

// bf16 tcgen05 attention (d in {64, 128}); tensor maps are built by the caller.
struct Sm100Maps {
  CUtensorMap qt, kt, v, dO;         // boxes of 64 columns x 128 rows
  CUtensorMap qt64, kt64, v64, dO64; // boxes of 64 columns x 64 rows
};
cudaError_t launch_fwd_sm100(const ra_problem& p, const Sm100Maps& maps, void* o, float* lse,
                             const DevCtl& ctl, cudaStream_t s);
// Padded per-row vectors for the tensor-core backward, delta and lse * log2(e), plus
// max_i |dO_i| into stats[0] and max_j |v_j| into stats[1] (fp32 bits, atomic max; stats
// zeroed by the caller), in one pass over O, dO and V.
cudaError_t launch_bwd_pre(const ra_problem& p, const void* o, const void* dO, const void* v,
                           const float* lse, float* deltap, float* lse2p, uint32_t* stats,
                           cudaStream_t s);
// stats: [0] max_i |dO_i|, [1] max_j |v_j| (fp32 bits) for the fp16 scale of dS.
cudaError_t launch_bwd_dkdv_sm100(const ra_problem& p, const Sm100Maps& maps,
                                  const float* lse2p, const float* deltap, const float2* table,
                                  const uint32_t* stats, void* dk, void* dv, float* dpart,
                                  const DevCtl& ctl, cudaStream_t s);
cudaError_t launch_bwd_dq_sm100(const ra_problem& p, const Sm100Maps& maps, const float* lse2p,
                                const float* deltap, const float2* table, const uint32_t* stats,
                                void* dq, float* dpart, const DevCtl& ctl, cudaStream_t s);

}  // namespace ra
