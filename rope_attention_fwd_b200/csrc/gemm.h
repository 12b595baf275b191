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
  // K chunk of one pipeline stage of the tensor-core kernel: 64 (four stages) or 128 (two).
  int bk = 64;
  // Operand given as a 3-D whole-row view (tensor_map_rows: x = 64 columns of a chunk, y = row,
  // z = 64-column chunk), so that one request brings the operand's whole stage: MN-major
  // y = K row, z = MN chunk (B only for segments along N whose length is a multiple of 256);
  // K-major y = MN row, z = K chunk (bk = 128 only; segments along K a multiple of 128
  // long).  0: 2-D maps.
  int a_rowbox = 0;
  int b_rowbox = 0;
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

// Tensor map of one bf16 operand segment with the box the tensor-core kernel loads under
// spec (bk, majorness, rowbox flag): ptr is row-major [rows][cols] (cols = K for a K-major
// operand, MN for an MN-major one), rows 16-byte aligned, cols a multiple of 64 for a rowbox
// view.  False if the map cannot be encoded.
bool gemm_operand_map(CUtensorMap* map, const GemmSpec& spec, bool is_b, const void* ptr,
                      uint64_t rows, uint64_t cols);

// bf16 operands on the tensor cores; amaps / bmaps hold one gemm_operand_map per segment.
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
