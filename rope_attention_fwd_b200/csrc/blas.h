// blas.h -- the library's cuBLAS handles (one per host thread and device, created on
// first use, destroyed when the thread exits).
#pragma once
#include <cublas_v2.h>

namespace ra {

// This thread's handle for the current device, or nullptr if it cannot be created.
cublasHandle_t cublas_handle();

}  // namespace ra
