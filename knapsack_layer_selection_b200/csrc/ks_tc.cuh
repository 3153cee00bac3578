// Tensor-core (tcgen05 / TMEM / TMA) kernels of the bf16 sublayer forward.
#pragma once

#include <cuda.h>

#include "ks_common.cuh"

namespace ks {

// Fused epilogues of the tensor-core GEMM C[M][N] = A[M][K] . B[N][K]^T.
enum Epilogue {
  EPI_RESID_F32 = 0,    // out fp32 [M][N] = acc + resid[M][N]
  EPI_ROPE_BF16 = 1,    // out bf16 [M][N] = rotate-half RoPE(acc) per head (row r = token r % T)
  EPI_SWIGLU_BF16 = 2,  // out bf16 [M][N] = silu(A.Bg^T) * (A.Bu^T)  (B = gate, B2 = up)
  EPI_STORE_BF16 = 3,   // out bf16 [M][N] = acc
  EPI_STORE_F32 = 4,    // out fp32 [M][N] = acc
  EPI_ROWMAX = 5,       // out float4 [M][N/256]: per row and 256-column tile, of
                        // v = scale * acc + col_bias[n]: {top-1, index (int bits), top-2, 0}
};

// Parameters of the row-maximum epilogue (EPI_ROWMAX).
struct RowMaxArgs {
  float scale;
  const float* col_bias;   // [N] or NULL
};

// True when the model's contractions run on the tensor cores (bf16 weights).
bool use_tensor_cores(const ks_model_desc* m);

// A [M][K], B/B2 [N][K] bf16 row-major; K a multiple of 64; N a multiple of 256
// (128 for SwiGLU, whose output has N columns).  status: device word for a
// bounded-wait timeout, or NULL.
// dyn_cells (device int, optional): only the first *dyn_cells x T rows are live
// (a batch compacted on the device); M is then an upper bound.
ks_status tc_gemm(const void* A, const void* B, const void* B2, void* out, const float* resid,
                  int M, int N, int K, int epi, const float2* rope_cs, int T, int head_dim,
                  int32_t* status, cudaStream_t st, const int* dyn_cells = nullptr,
                  RowMaxArgs rowmax = RowMaxArgs{1.0f, nullptr});

// Up to kGemmMaxGroups independent row groups multiplied by the same B (and
// B2) in one launch: group g computes out_g = epi(A_g . B^T) for its M_g rows
// (its own residual and RoPE table).  One tile walk covers every group's row
// tiles, so a weight tile read once serves all groups; each output element is
// the same fixed-order sum over K as in a one-group launch.
constexpr int kGemmMaxGroups = 4;
struct GemmGroupArg {
  const void* A;
  void* out;
  const float* resid;
  const float2* rope_cs;
  int M;
};
ks_status tc_gemm_groups(const GemmGroupArg* groups, int n_groups, const void* B, const void* B2,
                         int N, int K, int epi, int T, int head_dim, int32_t* status,
                         cudaStream_t st, const int* dyn_cells = nullptr,
                         RowMaxArgs rowmax = RowMaxArgs{1.0f, nullptr});

// Tensor map of a row-major bf16 matrix [rows][cols] (row_stride elements apart)
// read in boxes of box_rows x box_cols with the 128-byte swizzle; reads outside
// [rows) x [cols) return zeros.
ks_status make_tmap_2d(CUtensorMap* m, const void* base, long long rows, long long cols,
                       long long row_stride, int box_cols, int box_rows);

// Causal GQA attention on the tensor cores: q, out [R][Hq][hd] bf16 (row r is
// evaluation token r % T), kc/vc one layer of the cache [cache_rows][Hkv][hd]
// bf16; token t attends to positions 0 .. ctx + t.  hd = 64 or 128.  With kw,
// vw ([R][Hkv][hd] bf16, T dividing 128) the window positions ctx .. ctx + t
// take row r's own state's keys / values (rows r - t .. r) instead of the cache.
ks_status tc_attention(const void* q, const void* kc, const void* vc, long long cache_rows, int R,
                       int T, int Hq, int Hkv, int hd, int ctx, void* out, int32_t* status,
                       cudaStream_t st, const int* dyn_cells = nullptr,
                       const void* kw = nullptr, const void* vw = nullptr);

int sm_count();

}  // namespace ks
