// Internal interface between the module code and the library's GEMM kernel
// (gemm_sm100.cuh, compiled into libbsa.cu's translation unit so that it
// shares the device status word and the TMA descriptor encoder).
#pragma once

#include <cstdint>

#include <cuda_runtime.h>

namespace bsa {

// D[m, n] (row-major, row stride ldd) = A[m, k] B[k, n] (+ bias[n]), bf16 in,
// fp32 accumulation, bf16 out. A is stored [m][k] (a_mn_major = false, row
// stride lda) or [k][m] (true); B is stored [n][k] (b_mn_major = false, an
// nn.Linear weight) or [k][n] (true). Returns a bsa_status code; asynchronous.
int gemm_bf16(const void *a, int64_t lda, bool a_mn_major, const void *b, int64_t ldb,
              bool b_mn_major, const void *bias, void *d, int64_t ldd, int64_t m, int64_t n,
              int64_t k, cudaStream_t stream);

}  // namespace bsa
