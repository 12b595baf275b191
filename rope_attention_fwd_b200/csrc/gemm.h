// gemm.h -- the projection GEMMs (gemm_sm100.cu): C[M][N] = sum_k A(m, k) B(n, k) over
// segmented operands, for the projections on either side of the attention path.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

namespace ra {

// Shape and operand layout.  An operand is K-major (row-major [MN][K]) or MN-major
// (row-major [K][MN]); it may be up to three tensors side by side along its MN dimension
// (seg_k = 0) or its K dimension (seg_k = 1), each seg_len long (a multiple of 64 for the
// tensor-core kernel).
struct GemmSpec {
  int M, N, K;
  int a_mn, a_seg_k, a_seg_len, a_nseg;
  int b_mn, b_seg_k, b_seg_len, b_nseg;
};

enum GemmOutKind { GEMM_OUT_F32 = 0, GEMM_OUT_HEADS = 1 };

// Output: up to three tensors side by side along N (seg_len columns each).
//   GEMM_OUT_F32:   fp32 row-major [M][ld] per segment;
//   GEMM_OUT_HEADS: row m = (b, i) with i < n, segment column (h, c) with c < d, written to
//                   [B, H, n, d] in the problem dtype (bf16 from the tensor-core kernel,
//                   fp32 from the CUDA-core one).
struct GemmOut {
  void* ptr[3];
  int kind, seg_len, nseg, ld;
  int n, H, d;
};

// bf16 operands on the tensor cores; amaps / bmaps hold one 2-D tensor map per segment
// (bf16, 128-byte swizzle; boxes: K-major A 64 x 128, every other 64 x 64).
cudaError_t launch_gemm_bf16(const GemmSpec& spec, const CUtensorMap* amaps,
                             const CUtensorMap* bmaps, const GemmOut& out, uint32_t* err,
                             uint64_t wait_ns, cudaStream_t s);

// fp32 arithmetic on CUDA cores (exact fp32 products and sums of the operands' values); a / b:
// one pointer per segment, each row-major with leading dimension a_ld / b_ld, fp32 or (flag
// set) bf16.
cudaError_t launch_gemm_f32(const GemmSpec& spec, const void* const* a, int a_ld, int a_bf16,
                            const void* const* b, int b_ld, int b_bf16, const GemmOut& out,
                            cudaStream_t s);

}  // namespace ra
