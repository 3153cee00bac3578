// Lemma 4.1 checker on the GPU (KnapSpec review page, §4 Lemma 4.1, referee
// major 2; "What would settle it" asks for exactly this measurement).
//
// For the final normalised states h' of the DP cells (rescaled to the
// reference's norm, the lemma's equal-norm premise) and the full model's
// h: logits z = W h through an LM head W [V][d]; i* = argmax z, margin
// xi = z_i* - max_{j != i*} z_j, D = max_j ||w_i* - w_j||.  The lemma's
// sufficient condition ||h - h'|| < xi / D (with ||h - h'||^2 = 2||h||^2 (1 -
// cos)) guarantees argmax W h' = i*; the checker reports, per cell and token,
// whether the condition holds and whether the greedy tokens agree.
//
// Both vocabulary-sized products run on the tensor-core GEMM with a row-maximum
// epilogue (top-2 per 256-column tile), so no V-wide logits row is stored:
//   z rows of every state and of the reference:   scale 1, no bias;
//   D^2_t = ||w_i*||^2 + max_j (||w_j||^2 - 2 w_i* . w_j):  A = the rows w_i*, scale -2, bias ||w_j||^2.
#include <math.h>

#include "ks_kernels.cuh"
#include "ks_tc.cuh"

namespace ks {
namespace {

constexpr int kPrepThreads = 256;

template <typename T>
__device__ __forceinline__ double block_sum(double v, T* sh) {
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  __syncthreads();
  if ((threadIdx.x & 31) == 0) sh[threadIdx.x >> 5] = v;
  __syncthreads();
  double s = 0.0;
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) s += sh[w];
  return s;
}

// One block per row r of [states (N*T rows); reference (T rows)]: final RMSNorm
// (gain g or 1), states rescaled to the same token's reference norm; bf16 rows
// for the logits GEMM, fp64-summed cosines and reference norms.
template <typename TG>
__global__ void __launch_bounds__(kPrepThreads) lemma_prep_kernel(
    const float* __restrict__ states, const float* __restrict__ ref, int N, int T, int d,
    const TG* __restrict__ g, float eps, __nv_bfloat16* __restrict__ A, float* __restrict__ cos_out,
    float* __restrict__ refnorm2) {
  __shared__ double sh[32];
  const long long r = blockIdx.x;
  const bool is_state = r < (long long)N * T;
  const int t = is_state ? (int)(r % T) : (int)(r - (long long)N * T);
  const float* x = is_state ? states + r * d : ref + (long long)t * d;
  const float* rr = ref + (long long)t * d;
  double sx2 = 0, sxs2 = 0, srs2 = 0, sxr = 0, sr2 = 0;
  for (int i = threadIdx.x; i < d; i += blockDim.x) {
    const double gi = g ? (double)Elem<TG>::to_f(g[i]) : 1.0;
    const double xv = x[i], rv = rr[i];
    sx2 += xv * xv;
    sr2 += rv * rv;
    sxs2 += (xv * gi) * (xv * gi);
    srs2 += (rv * gi) * (rv * gi);
    sxr += (xv * gi) * (rv * gi);
  }
  sx2 = block_sum(sx2, sh);
  sr2 = block_sum(sr2, sh);
  sxs2 = block_sum(sxs2, sh);
  srs2 = block_sum(srs2, sh);
  sxr = block_sum(sxr, sh);
  // reference: h = r g / sqrt(mean(r^2) + eps);  ||h||^2 = sum((r g)^2) / (mean(r^2) + eps)
  const double href2 = srs2 / (sr2 / d + eps);
  double scale;
  if (is_state) {
    scale = sqrt(href2 / sxs2);                  // x g rescaled to ||h||
    if (threadIdx.x == 0) cos_out[r] = (float)(sxr / sqrt(sxs2 * srs2));
  } else {
    scale = 1.0 / sqrt(sr2 / d + eps);
    if (threadIdx.x == 0) refnorm2[t] = (float)href2;
  }
  __nv_bfloat16* out = A + r * d;
  for (int i = threadIdx.x; i < d; i += blockDim.x) {
    const double gi = g ? (double)Elem<TG>::to_f(g[i]) : 1.0;
    out[i] = __float2bfloat16_rn((float)((double)x[i] * gi * scale));
  }
}

// Combines the per-tile top-2 of each row: top-1 value and index (first on
// ties, as the tiles and columns are scanned in increasing order) and top-2.
__global__ void rowmax_reduce_kernel(const float4* __restrict__ part, int rows, int tiles,
                                     int* __restrict__ idx, float* __restrict__ top1,
                                     float* __restrict__ top2) {
  const int r = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (r >= rows) return;
  float v1 = -INFINITY, v2 = -INFINITY;
  int i1 = 0x7fffffff;
  for (int k = lane; k < tiles; k += 32) {
    const float4 q = part[(long long)r * tiles + k];
    const int qi = __float_as_int(q.y);
    if (q.x > v1 || (q.x == v1 && qi < i1)) {
      v2 = fmaxf(v1, q.z);
      v1 = q.x;
      i1 = qi;
    } else {
      v2 = fmaxf(v2, q.x);
    }
  }
  for (int o = 16; o > 0; o >>= 1) {
    const float ov1 = __shfl_xor_sync(0xffffffffu, v1, o);
    const float ov2 = __shfl_xor_sync(0xffffffffu, v2, o);
    const int oi1 = __shfl_xor_sync(0xffffffffu, i1, o);
    if (ov1 > v1 || (ov1 == v1 && oi1 < i1)) {
      v2 = fmaxf(v1, ov2);
      v1 = ov1;
      i1 = oi1;
    } else {
      v2 = fmaxf(v2, ov1);
    }
  }
  if (lane == 0) {
    if (idx) idx[r] = i1;
    if (top1) top1[r] = v1;
    if (top2) top2[r] = v2;
  }
}

// ||w_j||^2 for every LM-head row (fp64 sums of the bf16 values).
__global__ void rownorm2_kernel(const __nv_bfloat16* __restrict__ W, int V, int d,
                                float* __restrict__ n2) {
  const int j = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (j >= V) return;
  double s = 0;
  for (int i = lane; i < d; i += 32) {
    const double v = __bfloat162float(W[(long long)j * d + i]);
    s += v * v;
  }
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (lane == 0) n2[j] = (float)s;
}

// A2[t] = W[i*_t]
__global__ void gather_head_rows_kernel(const __nv_bfloat16* __restrict__ W,
                                        const int* __restrict__ istar, int d,
                                        __nv_bfloat16* __restrict__ A2) {
  const int t = blockIdx.x;
  const long long src = istar[t];
  for (int i = threadIdx.x; i < d; i += blockDim.x) A2[(long long)t * d + i] = W[src * d + i];
}

// Per cell n and token t: the lemma's condition and greedy agreement.
__global__ void lemma_eval_kernel(int N, int T, const float* __restrict__ cos,
                                  const float* __restrict__ refnorm2,
                                  const int* __restrict__ istar, const float* __restrict__ ref_top1,
                                  const float* __restrict__ ref_top2,
                                  const float* __restrict__ dmax, const float* __restrict__ n2,
                                  const int* __restrict__ state_idx, float* __restrict__ margin_out,
                                  float* __restrict__ dist_out, uint8_t* __restrict__ bound,
                                  uint8_t* __restrict__ agree, int32_t* __restrict__ counts) {
  const long long r = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (r < T) {
    const int t = (int)r;
    margin_out[t] = ref_top1[t] - ref_top2[t];
    dist_out[t] = sqrtf(fmaxf(0.f, n2[istar[t]] + dmax[t]));
  }
  if (r >= (long long)N * T) return;
  const int t = (int)(r % T);
  const float xi = ref_top1[t] - ref_top2[t];
  const float D = sqrtf(fmaxf(0.f, n2[istar[t]] + dmax[t]));
  const float gap = sqrtf(fmaxf(0.f, 2.f * refnorm2[t] * (1.f - cos[r])));
  const bool b = gap * D < xi;
  const bool a = state_idx[r] == istar[t];
  bound[r] = b;
  agree[r] = a;
  if (b) atomicAdd(&counts[0], 1);
  if (a) atomicAdd(&counts[1], 1);
  if (b && !a) atomicAdd(&counts[2], 1);
}

__global__ void zero3_kernel(int32_t* c) {
  if (threadIdx.x < 3) c[threadIdx.x] = 0;
}

struct LemmaWs {
  __nv_bfloat16 *A, *A2;
  float4 *part, *part2;
  float *refnorm2, *n2, *top1, *top2, *dmax;
  int* idx;
  size_t total;
};

size_t al(size_t x) { return (x + 255) & ~size_t(255); }

LemmaWs lemma_carve(long long N, long long T, long long d, long long V, char* base) {
  LemmaWs w{};
  size_t off = 0;
  auto take = [&](size_t bytes) -> char* {
    char* p = base ? base + off : nullptr;
    off += al(bytes);
    return p;
  };
  const long long rows = (N + 1) * T, tiles = V / 256;
  w.A = (__nv_bfloat16*)take(rows * d * 2);
  w.part = (float4*)take(rows * tiles * 16);
  w.A2 = (__nv_bfloat16*)take(T * d * 2);
  w.part2 = (float4*)take(T * tiles * 16);
  w.refnorm2 = (float*)take(T * 4);
  w.n2 = (float*)take(V * 4);
  w.top1 = (float*)take(rows * 4);
  w.top2 = (float*)take(rows * 4);
  w.dmax = (float*)take(T * 4);
  w.idx = (int*)take(rows * 4);
  w.total = off;
  return w;
}

}  // namespace
}  // namespace ks

using namespace ks;

extern "C" {

KS_API ks_status ks_lemma_workspace_size(int32_t N, int32_t T, int32_t d, int32_t V, size_t* bytes) {
  if (!bytes || N < 1 || T < 1 || d < 64 || V < 256) return fail(KS_ERR_INVALID_ARG, "lemma: bad size");
  *bytes = lemma_carve(N, T, d, V, nullptr).total;
  return KS_OK;
}

KS_API ks_status ks_lemma_check(const float* states, int32_t N, const float* ref, int32_t T,
                                int32_t d, const void* final_norm, float eps, const void* lm_head,
                                int32_t V, void* workspace, size_t workspace_bytes,
                                ks_lemma_result* out, int32_t* status, ks_stream_t stream) {
  if (!states || !ref || !lm_head || !workspace || !out)
    return fail(KS_ERR_INVALID_ARG, "lemma: NULL argument");
  if (!out->istar || !out->margin || !out->dist || !out->cos || !out->bound || !out->agree ||
      !out->counts)
    return fail(KS_ERR_INVALID_ARG, "lemma: result buffers missing");
  if (N < 1 || T < 1) return fail(KS_ERR_INVALID_ARG, "lemma: N, T >= 1");
  if (d % 64 || d < 64) return fail(KS_ERR_UNSUPPORTED, "lemma: d must be a multiple of 64");
  if (V % 256 || V < 256) return fail(KS_ERR_UNSUPPORTED, "lemma: V must be a multiple of 256");
  if ((uintptr_t)workspace % 256) return fail(KS_ERR_INVALID_ARG, "lemma: workspace alignment");
  KS_TRY(check_aligned16({states, ref, lm_head, final_norm}, "lemma"));
  const LemmaWs need = lemma_carve(N, T, d, V, nullptr);
  if (workspace_bytes < need.total) return fail(KS_ERR_WORKSPACE, "lemma: workspace too small");
  LemmaWs w = lemma_carve(N, T, d, V, (char*)workspace);
  cudaStream_t st = (cudaStream_t)stream;
  const long long rows = (long long)(N + 1) * T;
  const int tiles = V / 256;
  const __nv_bfloat16* W = (const __nv_bfloat16*)lm_head;

  zero3_kernel<<<1, 32, 0, st>>>(out->counts);
  lemma_prep_kernel<__nv_bfloat16><<<(unsigned)rows, kPrepThreads, 0, st>>>(
      states, ref, N, T, d, (const __nv_bfloat16*)final_norm, eps, w.A, out->cos, w.refnorm2);
  KS_LAUNCH_CHECK();
  // logits top-2 of every state row and of the reference rows
  KS_TRY(tc_gemm(w.A, W, nullptr, w.part, nullptr, (int)rows, V, d, EPI_ROWMAX, nullptr, 1, 64,
                 status, st, nullptr, RowMaxArgs{1.0f, nullptr}));
  rowmax_reduce_kernel<<<ceil_div(rows, 8), 256, 0, st>>>(w.part, (int)rows, tiles, w.idx, w.top1,
                                                          w.top2);
  KS_LAUNCH_CHECK();
  const int* istar = w.idx + (long long)N * T;
  KS_CUDA_TRY(cudaMemcpyAsync(out->istar, istar, T * sizeof(int32_t), cudaMemcpyDeviceToDevice, st));
  // D^2 = ||w_i*||^2 + max_j (||w_j||^2 - 2 w_i* . w_j)
  rownorm2_kernel<<<ceil_div(V, 8), 256, 0, st>>>(W, V, d, w.n2);
  KS_LAUNCH_CHECK();
  gather_head_rows_kernel<<<T, 256, 0, st>>>(W, istar, d, w.A2);
  KS_LAUNCH_CHECK();
  KS_TRY(tc_gemm(w.A2, W, nullptr, w.part2, nullptr, T, V, d, EPI_ROWMAX, nullptr, 1, 64, status,
                 st, nullptr, RowMaxArgs{-2.0f, w.n2}));
  rowmax_reduce_kernel<<<ceil_div(T, 8), 256, 0, st>>>(w.part2, T, tiles, nullptr, w.dmax, nullptr);
  KS_LAUNCH_CHECK();
  lemma_eval_kernel<<<ceil_div((long long)N * T + T, 256), 256, 0, st>>>(
      N, T, out->cos, w.refnorm2, istar, w.top1 + (long long)N * T, w.top2 + (long long)N * T,
      w.dmax, w.n2, w.idx, out->margin, out->dist, out->bound, out->agree, out->counts);
  KS_LAUNCH_CHECK();
  return KS_OK;
}

}  // extern "C"
