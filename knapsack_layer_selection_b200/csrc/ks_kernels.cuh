// Internal kernel launchers of the KnapSpec library (not part of the C ABI).
#pragma once

#include "ks_common.cuh"

namespace ks {

// Activation (GEMM operand) storage type: fp32 for fp32 models, bf16 otherwise.
enum ActType { ACT_F32 = 0, ACT_BF16 = 1 };

inline size_t act_bytes(int act) { return act == ACT_F32 ? 4 : 2; }

// y[r] = x[r] / sqrt(mean(x[r]^2) + eps) * g  for R rows of length d.
// x fp32; g in the weight dtype; y in the activation dtype.
ks_status launch_rmsnorm(const float* x, const void* g, int wdt, void* y, int act, int R, int d,
                         float eps, cudaStream_t st);

// C[M][N] = A[M][K] . B[N][K]^T (+ resid[M][N]) on CUDA cores, fp32 accumulation in
// increasing k.  A in the activation dtype, B in the weight dtype; the output is fp32
// when out_f32, else the activation dtype.
ks_status launch_gemm_simt(const void* A, int act, const void* B, int wdt, void* C, bool out_f32,
                           const float* resid, int M, int N, int K, cudaStream_t st);

// cos/sin table [T][hd/2] for rotate-half RoPE at positions ctx + t (fp64 angles).
ks_status launch_rope_table(float2* cs, int T, int hd, int ctx, double base, cudaStream_t st);

// In-place rotate-half RoPE of q [R][H][hd] (activation dtype), row r is token r % T.
ks_status launch_rope_inplace(void* q, int act, const float2* cs, int R, int H, int hd, int T,
                              cudaStream_t st);

// g[i] = silu(g[i]) * u[i] for n elements (activation dtype, in place).
ks_status launch_swiglu_inplace(void* g, const void* u, int act, long long n, cudaStream_t st);

// o[r][h] = softmax(q[r][h] . K[0..ctx+t]^T / sqrt(hd)) . V  with t = r % T and kv head
// h / (Hq / Hkv).  q, o: [R][Hq][hd] activation dtype; kc, vc: one layer's cache
// [rows][Hkv][hd] in the weight dtype.  With kw, vw ([R][Hkv][hd], activation
// dtype) the positions ctx + j, j = 0 .. t, take key / value row (r - t + j) of
// kw / vw -- the window of row r's own state -- instead of the cache.
// CUDA-core version.
ks_status launch_attention_simt(const void* q, int act, const void* kc, const void* vc, int wdt,
                                int R, int T, int Hq, int Hkv, int hd, int ctx, void* o,
                                cudaStream_t st, const void* kw = nullptr,
                                const void* vw = nullptr);

// dst[c] = src for c in [0, n_copies), each copy n_elems floats.
ks_status launch_broadcast(float* dst, const float* src, int n_copies, long long n_elems,
                           cudaStream_t st);

// ---- DP step kernels (ks_select.cu)
ks_status launch_select(const float* prev, const float* exec, const float* target, int C, int T,
                        int d, int w, float* cur, float* val, uint8_t* bp, float* cos_s,
                        float* cos_e, cudaStream_t st);

// The DP loop's select on a buffer whose slot 0 is the reference state (see
// ks_select.cu); also writes the next item's normalised operand when g_next.
// valid_prev / valid_cur (both NULL: every cell valid) carry the exact-budget
// validity of the cells from row to row.  cur may equal prev (the states are
// then updated in place: a cell whose skip candidate wins is not rewritten).
ks_status launch_select_fused(const float* prev, const float* exec, const float* target, int C,
                              int T, int d, int w, float eps, const void* g_next, int wdt,
                              float* cur, void* xh_next, float* val, uint8_t* bp, float* cos_s,
                              float* cos_e, float* ref_out, const uint8_t* valid_prev,
                              uint8_t* valid_cur, double prune_tau, int min_valid_b,
                              const int* exec_map, uint64_t* hash_cur, cudaStream_t st);

// Slots 0..n_slots-1 of a state buffer <- x0, and their normalised operands.
ks_status launch_init_states(const float* x0, int n_slots, int T, int d, float eps, const void* g,
                             int wdt, float* states, void* xh, float* ref_out, uint64_t* hash_out,
                             cudaStream_t st);

// Distinct-state compaction of the next execute batch (slots 0..n-1): see ks_select.cu.
ks_status launch_dedup(const uint64_t* hash, const uint8_t* valid, int n, int* map, int* uniq,
                       int* count, int32_t* count_out, bool weak, cudaStream_t st);
// Byte comparison of every fold launch_dedup made; a slot whose state differs
// from its representative's gets its own compacted entry.
ks_status launch_dedup_verify(const float* states, long long cell, int n, int* map, int* uniq,
                              int* count, int32_t* count_out, int32_t* rejected_out,
                              cudaStream_t st);
ks_status launch_gather(const int* uniq, const int* count, int max_count, long long cell,
                        const float* states, const void* xh, int act, float* states_c, void* xh_c,
                        cudaStream_t st);

struct ItemTable {
  static constexpr int kMaxItems = 256;
  int32_t w[kMaxItems];
  double t[kMaxItems];
};

// valid (NULL: all valid): invalid cells get an empty set, used weight -1, NaN t_draft.
ks_status launch_reconstruct(const uint8_t* bp, const int32_t* w, const double* t,
                             const ItemTable* tab, int n_items, int C, uint64_t* sets,
                             int32_t* used_w, double* t_draft, int32_t* status,
                             const uint8_t* valid, cudaStream_t st);

// *p = v (device word).
ks_status launch_fill_i32(int32_t* p, int32_t v, cudaStream_t st);

// Initial validity: only b == 0 in the exact-budget mode, every cell otherwise.
ks_status launch_init_valid(uint8_t* valid, int C, bool exact, cudaStream_t st);

ks_status launch_tpt(const float* values, const double* t_draft, int C, double t_target,
                     int gamma_max, double lo, double scale, double amax, double* tpt,
                     int32_t* best, double* best_tpt, cudaStream_t st);

}  // namespace ks
