// CUDA-core kernels of the sublayer forward: RMSNorm, RoPE, SwiGLU, a tiled fp32
// GEMM and a one-row-per-block attention.  They carry the fp32 model exactly
// (tensor-core tf32 would not) and compute the same sublayers the paper's items
// are made of (KnapSpec review page, "What carries the argument": each Attention
// and each MLP sublayer is an item).
#include "ks_kernels.cuh"

#include <math.h>

namespace ks {

// ---------------------------------------------------------------- RMSNorm
template <typename TW, typename TY>
__global__ void rmsnorm_kernel(const float* __restrict__ x, const TW* __restrict__ g,
                               TY* __restrict__ y, int d, float eps) {
  const long long row = blockIdx.x;
  const float* xr = x + row * d;
  float ss = 0.f;
  for (int i = threadIdx.x; i < d; i += blockDim.x) {
    float v = xr[i];
    ss = fmaf(v, v, ss);
  }
  __shared__ float red[32];
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  if (threadIdx.x < 32) {
    float v = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.f;
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (threadIdx.x == 0) red[0] = v;
  }
  __syncthreads();
  const float inv = 1.0f / sqrtf(red[0] / (float)d + eps);
  TY* yr = y + row * d;
  for (int i = threadIdx.x; i < d; i += blockDim.x)
    yr[i] = Elem<TY>::from_f(xr[i] * inv * Elem<TW>::to_f(g[i]));
}

ks_status launch_rmsnorm(const float* x, const void* g, int wdt, void* y, int act, int R, int d,
                         float eps, cudaStream_t st) {
  if (R <= 0) return KS_OK;
  dim3 grid(R), block(256);
  if (wdt == KS_F32 && act == ACT_F32)
    rmsnorm_kernel<float, float><<<grid, block, 0, st>>>(x, (const float*)g, (float*)y, d, eps);
  else if (wdt == KS_BF16 && act == ACT_BF16)
    rmsnorm_kernel<__nv_bfloat16, __nv_bfloat16><<<grid, block, 0, st>>>(
        x, (const __nv_bfloat16*)g, (__nv_bfloat16*)y, d, eps);
  else
    return fail(KS_ERR_UNSUPPORTED, "rmsnorm: dtype combination");
  KS_LAUNCH_CHECK();
  return KS_OK;
}

// ---------------------------------------------------------------- SIMT GEMM
// C[M][N] = A[M][K] . B[N][K]^T.  64x64 tile, 16-deep k slices, 4x4 per thread.
// Each output accumulates over k in increasing order whatever M is, so a row's
// result does not depend on the other rows of the batch.
template <typename TA, typename TB, typename TC>
__global__ void __launch_bounds__(256) gemm_simt_kernel(const TA* __restrict__ A,
                                                        const TB* __restrict__ B,
                                                        TC* __restrict__ C,
                                                        const float* __restrict__ resid,
                                                        int M, int N, int K) {
  constexpr int BM = 64, BN = 64, BK = 16;
  __shared__ float As[BK][BM + 4];
  __shared__ float Bs[BK][BN + 4];
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  const long long m0 = (long long)blockIdx.y * BM, n0 = (long long)blockIdx.x * BN;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += BK) {
    for (int e = threadIdx.x; e < BM * BK; e += 256) {
      int r = e / BK, kk = e % BK;
      long long m = m0 + r;
      int k = k0 + kk;
      As[kk][r] = (m < M && k < K) ? Elem<TA>::to_f(A[m * K + k]) : 0.f;
      long long n = n0 + r;
      Bs[kk][r] = (n < N && k < K) ? Elem<TB>::to_f(B[n * K + k]) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < BK; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    long long m = m0 + ty * 4 + i;
    if (m >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      long long n = n0 + tx * 4 + j;
      if (n >= N) continue;
      float v = acc[i][j];
      if (resid) v += resid[m * N + n];
      C[m * N + n] = Elem<TC>::from_f(v);
    }
  }
}

template <typename TA, typename TB>
static ks_status gemm_simt_dispatch_out(const void* A, const void* B, void* C, bool out_f32,
                                        const float* resid, int M, int N, int K, cudaStream_t st) {
  dim3 grid(ceil_div(N, 64), ceil_div(M, 64)), block(256);
  if (out_f32 || sizeof(TA) == 4)
    gemm_simt_kernel<TA, TB, float><<<grid, block, 0, st>>>((const TA*)A, (const TB*)B,
                                                           (float*)C, resid, M, N, K);
  else
    gemm_simt_kernel<TA, TB, __nv_bfloat16><<<grid, block, 0, st>>>(
        (const TA*)A, (const TB*)B, (__nv_bfloat16*)C, resid, M, N, K);
  KS_LAUNCH_CHECK();
  return KS_OK;
}

ks_status launch_gemm_simt(const void* A, int act, const void* B, int wdt, void* C, bool out_f32,
                           const float* resid, int M, int N, int K, cudaStream_t st) {
  if (M <= 0) return KS_OK;
  if (act == ACT_F32 && wdt == KS_F32)
    return gemm_simt_dispatch_out<float, float>(A, B, C, true, resid, M, N, K, st);
  if (act == ACT_BF16 && wdt == KS_BF16)
    return gemm_simt_dispatch_out<__nv_bfloat16, __nv_bfloat16>(A, B, C, out_f32, resid, M, N,
                                                                K, st);
  return fail(KS_ERR_UNSUPPORTED, "gemm_simt: dtype combination");
}

// ---------------------------------------------------------------- RoPE
__global__ void rope_table_kernel(float2* cs, int T, int hd, int ctx, double base) {
  const int half = hd / 2;
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= T * half) return;
  const int t = i / half, j = i % half;
  const double theta = pow(base, -2.0 * (double)j / (double)hd);
  const double ang = (double)(ctx + t) * theta;
  cs[i] = make_float2((float)cos(ang), (float)sin(ang));
}

ks_status launch_rope_table(float2* cs, int T, int hd, int ctx, double base, cudaStream_t st) {
  const int n = T * (hd / 2);
  rope_table_kernel<<<ceil_div(n, 256), 256, 0, st>>>(cs, T, hd, ctx, base);
  KS_LAUNCH_CHECK();
  return KS_OK;
}

template <typename TQ>
__global__ void rope_kernel(TQ* q, const float2* __restrict__ cs, int R, int H, int hd, int T) {
  const int half = hd / 2;
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long total = (long long)R * H * half;
  if (i >= total) return;
  const int j = (int)(i % half);
  const long long rh = i / half;
  const int r = (int)(rh / H);
  const int t = r % T;
  TQ* p = q + rh * hd;
  const float2 c = cs[t * half + j];
  const float x1 = Elem<TQ>::to_f(p[j]), x2 = Elem<TQ>::to_f(p[j + half]);
  p[j] = Elem<TQ>::from_f(x1 * c.x - x2 * c.y);
  p[j + half] = Elem<TQ>::from_f(x2 * c.x + x1 * c.y);
}

ks_status launch_rope_inplace(void* q, int act, const float2* cs, int R, int H, int hd, int T,
                              cudaStream_t st) {
  const long long n = (long long)R * H * (hd / 2);
  if (n == 0) return KS_OK;
  if (act == ACT_F32)
    rope_kernel<float><<<ceil_div(n, 256), 256, 0, st>>>((float*)q, cs, R, H, hd, T);
  else
    rope_kernel<__nv_bfloat16><<<ceil_div(n, 256), 256, 0, st>>>((__nv_bfloat16*)q, cs, R, H,
                                                                 hd, T);
  KS_LAUNCH_CHECK();
  return KS_OK;
}

// ---------------------------------------------------------------- SwiGLU
template <typename TA>
__global__ void swiglu_kernel(TA* g, const TA* __restrict__ u, long long n) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const float a = Elem<TA>::to_f(g[i]);
  const float b = Elem<TA>::to_f(u[i]);
  g[i] = Elem<TA>::from_f(a / (1.0f + expf(-a)) * b);
}

ks_status launch_swiglu_inplace(void* g, const void* u, int act, long long n, cudaStream_t st) {
  if (n == 0) return KS_OK;
  if (act == ACT_F32)
    swiglu_kernel<float><<<ceil_div(n, 256), 256, 0, st>>>((float*)g, (const float*)u, n);
  else
    swiglu_kernel<__nv_bfloat16><<<ceil_div(n, 256), 256, 0, st>>>(
        (__nv_bfloat16*)g, (const __nv_bfloat16*)u, n);
  KS_LAUNCH_CHECK();
  return KS_OK;
}

// ---------------------------------------------------------------- attention (CUDA cores)
// One block per (row, q head).  Scores of all visible keys sit in shared memory.
template <typename TQ, typename TKV>
__global__ void __launch_bounds__(128) attention_simt_kernel(const TQ* __restrict__ q,
                                                             const TKV* __restrict__ kc,
                                                             const TKV* __restrict__ vc,
                                                             TQ* __restrict__ o, int T, int Hq,
                                                             int Hkv, int hd, int ctx,
                                                             float scale,
                                                             const TQ* __restrict__ kw,
                                                             const TQ* __restrict__ vw) {
  extern __shared__ float sm[];
  float* qs = sm;             // [hd]
  float* sc = sm + hd;        // [ctx + T]
  __shared__ float red[32];
  const long long r = blockIdx.x;
  const int h = blockIdx.y;
  const int t = (int)(r % T);
  const int n = ctx + t + 1;
  const int g = h / (Hq / Hkv);
  const long long kv_row = (long long)Hkv * hd;
  const TQ* qp = q + (r * Hq + h) * hd;
  for (int i = threadIdx.x; i < hd; i += blockDim.x) qs[i] = Elem<TQ>::to_f(qp[i]);
  __syncthreads();
  // window reading: positions ctx + j' (j' <= t) are row (r - t + j') of kw / vw
  const long long w0 = r - t - ctx;
  const bool window = kw != nullptr;
  float mx = -INFINITY;
  for (int j = threadIdx.x; j < n; j += blockDim.x) {
    float s = 0.f;
    if (window && j >= ctx) {
      const TQ* kp = kw + (w0 + j) * kv_row + (long long)g * hd;
      for (int i = 0; i < hd; ++i) s = fmaf(qs[i], Elem<TQ>::to_f(kp[i]), s);
    } else {
      const TKV* kp = kc + j * kv_row + (long long)g * hd;
      for (int i = 0; i < hd; ++i) s = fmaf(qs[i], Elem<TKV>::to_f(kp[i]), s);
    }
    s *= scale;
    sc[j] = s;
    mx = fmaxf(mx, s);
  }
  for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = mx;
  __syncthreads();
  mx = red[0];
  for (int w = 1; w < (int)(blockDim.x >> 5); ++w) mx = fmaxf(mx, red[w]);
  __syncthreads();
  float sum = 0.f;
  for (int j = threadIdx.x; j < n; j += blockDim.x) {
    float p = expf(sc[j] - mx);
    sc[j] = p;
    sum += p;
  }
  for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = sum;
  __syncthreads();
  sum = 0.f;
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) sum += red[w];
  const float inv = 1.0f / sum;
  TQ* op = o + (r * Hq + h) * hd;
  for (int i = threadIdx.x; i < hd; i += blockDim.x) {
    const TKV* vp = vc + (long long)g * hd + i;
    const int nc = window ? ctx : n;             // keys read from the cache
    float acc = 0.f;
    for (int j = 0; j < nc; ++j) acc = fmaf(sc[j], Elem<TKV>::to_f(vp[j * kv_row]), acc);
    if (window) {
      const TQ* wp = vw + (long long)g * hd + i;
      for (int j = ctx; j < n; ++j) acc = fmaf(sc[j], Elem<TQ>::to_f(wp[(w0 + j) * kv_row]), acc);
    }
    op[i] = Elem<TQ>::from_f(acc * inv);
  }
}

ks_status launch_attention_simt(const void* q, int act, const void* kc, const void* vc, int wdt,
                                int R, int T, int Hq, int Hkv, int hd, int ctx, void* o,
                                cudaStream_t st, const void* kw, const void* vw) {
  if ((kw == nullptr) != (vw == nullptr))
    return fail(KS_ERR_INVALID_ARG, "attention_simt: window keys and values go together");
  if (R <= 0) return KS_OK;
  const size_t smem = (size_t)(hd + ctx + T) * sizeof(float);
  if (smem > 200 * 1024) return fail(KS_ERR_UNSUPPORTED, "attention_simt: context too long");
  dim3 grid(R, Hq), block(128);
  const float scale = (float)(1.0 / sqrt((double)hd));
  if (act == ACT_F32 && wdt == KS_F32) {
    auto k = attention_simt_kernel<float, float>;
    KS_CUDA_TRY(cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
    k<<<grid, block, smem, st>>>((const float*)q, (const float*)kc, (const float*)vc, (float*)o,
                                 T, Hq, Hkv, hd, ctx, scale, (const float*)kw, (const float*)vw);
  } else if (act == ACT_BF16 && wdt == KS_BF16) {
    auto k = attention_simt_kernel<__nv_bfloat16, __nv_bfloat16>;
    KS_CUDA_TRY(cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
    k<<<grid, block, smem, st>>>((const __nv_bfloat16*)q, (const __nv_bfloat16*)kc,
                                 (const __nv_bfloat16*)vc, (__nv_bfloat16*)o, T, Hq, Hkv, hd, ctx,
                                 scale, (const __nv_bfloat16*)kw, (const __nv_bfloat16*)vw);
  } else {
    return fail(KS_ERR_UNSUPPORTED, "attention_simt: dtype combination");
  }
  KS_LAUNCH_CHECK();
  return KS_OK;
}

// ---------------------------------------------------------------- broadcast
__global__ void broadcast_kernel(float4* dst, const float4* __restrict__ src, int n_copies,
                                 long long n4) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n4 * n_copies) return;
  dst[i] = src[i % n4];
}

ks_status launch_broadcast(float* dst, const float* src, int n_copies, long long n_elems,
                           cudaStream_t st) {
  if (n_elems % 4 != 0) return fail(KS_ERR_UNSUPPORTED, "broadcast: size not a multiple of 4");
  const long long n4 = n_elems / 4;
  const long long total = n4 * n_copies;
  if (total == 0) return KS_OK;
  broadcast_kernel<<<ceil_div(total, 256), 256, 0, st>>>((float4*)dst, (const float4*)src,
                                                         n_copies, n4);
  KS_LAUNCH_CHECK();
  return KS_OK;
}

}  // namespace ks
