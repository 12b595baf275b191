// blas.h -- the library's cuBLAS handle (one per device, created on first use).
#pragma once
#include <cublas_v2.h>

namespace ra {

// The current device's handle, or nullptr if it cannot be created.
cublasHandle_t cublas_handle();

}  // namespace ra
