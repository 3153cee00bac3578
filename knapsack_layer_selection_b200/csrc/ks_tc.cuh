// Tensor-core (tcgen05 / TMEM / TMA) kernels of the bf16 sublayer forward.
#pragma once

#include "ks_common.cuh"

namespace ks {

// Fused epilogues of the tensor-core GEMM C[M][N] = A[M][K] . B[N][K]^T.
enum Epilogue {
  EPI_RESID_F32 = 0,    // out fp32 [M][N] = acc + resid[M][N]
  EPI_ROPE_BF16 = 1,    // out bf16 [M][N] = rotate-half RoPE(acc) per head (row r = token r % T)
  EPI_SWIGLU_BF16 = 2,  // out bf16 [M][N] = silu(A.Bg^T) * (A.Bu^T)  (B = gate, B2 = up)
  EPI_STORE_BF16 = 3,   // out bf16 [M][N] = acc
  EPI_STORE_F32 = 4,    // out fp32 [M][N] = acc
};

// True when the model's contractions run on the tensor cores (bf16 weights).
bool use_tensor_cores(const ks_model_desc* m);

// A [M][K], B/B2 [N][K] bf16 row-major; K a multiple of 64; N a multiple of 256
// (128 for SwiGLU, whose output has N columns).  status: device word for a
// bounded-wait timeout, or NULL.
ks_status tc_gemm(const void* A, const void* B, const void* B2, void* out, const float* resid,
                  int M, int N, int K, int epi, const float2* rope_cs, int T, int head_dim,
                  int32_t* status, cudaStream_t st);

}  // namespace ks
