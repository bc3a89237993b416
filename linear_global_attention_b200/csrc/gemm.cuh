#pragma once
#include <cuda_runtime.h>
#include <stddef.h>

namespace zebra {

constexpr size_t GEMM_WS_BYTES = 32u << 20;

// Row-major Cout[M_rows, N_cols] = A[M_rows, K] * B[N_cols, K]^T + beta * Cin (bf16, fp32 accumulate).
int gemm_bf16_nt(const void* A, const void* B, const void* Cin, void* Cout, long long M_rows, long long N_cols,
                 long long K, float beta, void* ws, size_t ws_bytes, cudaStream_t st);

}  // namespace zebra
