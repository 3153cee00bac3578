// Tensor-core attention of the candidate states' queries over the full model's
// KV cache (sm_100a, tcgen05 + TMEM + TMA).
//
// In the KnapSpec DP every budget cell that executes an Attention item runs
// that sublayer on its own hidden state, while keys and values come from the
// full model's cache (KnapSpec review page, "What carries the argument"; the
// cache reading is R7 of the oracle).  So all E cells x T tokens x group query
// rows of one KV head read the same K/V tiles, and this is a prefill-shaped,
// compute-bound contraction: O = softmax(Q K^T / sqrt(hd)) V with token t
// seeing cache positions 0 .. ctx + t.
//
// One CTA per (128 query rows, query head); 192 threads:
//   warp 0    -- TMA: the Q tile once, then K and V blocks of 128 keys into a
//                2-stage ring (64-column panels, 128-byte swizzle);
//   warp 1    -- TMEM owner; one lane issues S_j = Q K_j^T (M=128, N=128) into
//                one of two S buffers, and O_j = P_j V_j (M=128, N=hd, V read
//                MN-major straight from the cache layout) into one of two O
//                buffers, in the order S_0, S_1, O_0, S_2, O_1, ... so the
//                softmax of block j+1 overlaps the P.V product of block j;
//   warps 2-5 -- one thread per query row: online softmax (running max and sum
//                in the exp2 domain), P_j to shared memory as bf16 in the
//                swizzled K-major layout the MMA reads, and O accumulated in
//                registers as O <- O * alpha + O_j.
// Every row uses the same block order and the same arithmetic whatever the
// batch, so a row's output does not depend on the other rows.
#include <cuda.h>

#include "ks_sm100.cuh"
#include "ks_tc.cuh"

namespace ks {

using namespace sm100;

namespace {

template <int HD>
struct Cfg {
  static constexpr int BM = 128, BN = 128, STAGES = 2;
  static constexpr int PANELS = HD / 64;              // 64-wide panels along head_dim
  static constexpr int KV_PANEL = BN * 128;           // [128 keys][64] bf16
  static constexpr int Q_BYTES = BM * HD * 2;
  static constexpr int K_BYTES = PANELS * KV_PANEL;
  static constexpr int V_BYTES = PANELS * KV_PANEL;
  static constexpr int STAGE = K_BYTES + V_BYTES;
  static constexpr int P_PANEL = BM * 128;            // [128 rows][64 keys] bf16
  static constexpr int P_BYTES = (BN / 64) * P_PANEL;
  static constexpr int OFF_STAGE = Q_BYTES;
  static constexpr int OFF_P = Q_BYTES + STAGES * STAGE;
  static constexpr int OFF_TAIL = OFF_P + 2 * P_BYTES;
  static constexpr int SMEM = OFF_TAIL + 256 + 1024;
  static constexpr int TMEM_S = 0;                    // S buffers: columns [0, 2*BN)
  static constexpr int TMEM_O = 2 * BN;               // O buffers: [2*BN, 2*BN + 2*HD)
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t IDESC_S = idesc_bf16_f32(BM, BN);
  static constexpr uint32_t IDESC_O = idesc_bf16_f32(BM, HD) | (1u << 16);   // B (V) MN-major
};

struct Tail {
  uint64_t q_full;
  uint64_t k_full[2], v_full[2], kv_empty[2];
  uint64_t s_full[2], s_free[2], p_full[2], o_full[2], o_free[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

struct AttnParams {
  void* out;
  int32_t* status;
  int R, T, Hq, Hkv, ctx, n_keys, n_blocks;
  float scale_log2;
};

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack2(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

// MN-major, 128-byte-swizzled operand: 64 elements contiguous along N in each
// 128-byte row, rows along K 128 bytes apart (8-row atoms of 1024 bytes, SBO),
// 64-wide N panels `panel_bytes` apart (LBO).
__device__ __forceinline__ uint64_t desc_mnmajor_sw128(uint32_t smem_addr, uint32_t panel_bytes) {
  uint64_t d = 0;
  d |= (uint64_t)((smem_addr & 0x3FFFF) >> 4);
  d |= (uint64_t)((panel_bytes >> 4) & 0x3FFF) << 16;
  d |= (uint64_t)(1024 >> 4) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}

// Warp-uniform wait: every lane polls, and the warp leaves together if any lane gave up.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int* abort,
                                          int32_t* status) {
  const bool ok = mbar_wait(bar, parity, abort, status);
  return __all_sync(0xffffffffu, ok);
}

template <int HD>
__global__ void __launch_bounds__(192, 1)
    attn_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const AttnParams p) {
  using C = Cfg<HD>;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = (unsigned char*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  Tail* tail = reinterpret_cast<Tail*>(smem + C::OFF_TAIL);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * C::BM;
  const int h = blockIdx.y;
  const int g = h / (p.Hq / p.Hkv);
  const int J = p.n_blocks;
  volatile int* abort = &tail->abort;
  const uint32_t sbase = smem_u32(smem);

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&tail->q_full), 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(smem_u32(&tail->k_full[s]), 1);
      mbar_init(smem_u32(&tail->v_full[s]), 1);
      mbar_init(smem_u32(&tail->kv_empty[s]), 1);
      mbar_init(smem_u32(&tail->s_full[s]), 1);
      mbar_init(smem_u32(&tail->s_free[s]), 128);
      mbar_init(smem_u32(&tail->p_full[s]), 128);
      mbar_init(smem_u32(&tail->o_full[s]), 1);
      mbar_init(smem_u32(&tail->o_free[s]), 128);
    }
    mbar_init(smem_u32(&tail->drain), 1);
    tail->abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&tail->tmem_base), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tail->tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      const uint32_t qf = smem_u32(&tail->q_full);
      mbar_arrive_expect_tx(qf, C::Q_BYTES);
      for (int pn = 0; pn < C::PANELS; ++pn)
        tma_load_2d(sbase + pn * (C::BM * 128), &tmQ, h * HD + pn * 64, m0, qf);
      int j = 0;
      for (; j < J; ++j) {
        const int s = j & 1;
        const uint32_t r = (uint32_t)(j >> 1);
        if (!mbar_wait(smem_u32(&tail->kv_empty[s]), (r & 1u) ^ 1u, abort, p.status)) break;
        const uint32_t kst = sbase + C::OFF_STAGE + s * C::STAGE;
        const uint32_t vst = kst + C::K_BYTES;
        const uint32_t kf = smem_u32(&tail->k_full[s]), vf = smem_u32(&tail->v_full[s]);
        mbar_arrive_expect_tx(kf, C::K_BYTES);
        for (int pn = 0; pn < C::PANELS; ++pn)
          tma_load_2d(kst + pn * C::KV_PANEL, &tmK, g * HD + pn * 64, j * C::BN, kf);
        mbar_arrive_expect_tx(vf, C::V_BYTES);
        for (int pn = 0; pn < C::PANELS; ++pn)
          tma_load_2d(vst + pn * C::KV_PANEL, &tmV, g * HD + pn * 64, j * C::BN, vf);
      }
      // drain the copies still in flight before leaving
      mbar_wait_drain(qf, 0, p.status);
      for (int i = (j > 2 ? j - 2 : 0); i < j; ++i) {
        mbar_wait_drain(smem_u32(&tail->k_full[i & 1]), (uint32_t)(i >> 1) & 1u, p.status);
        mbar_wait_drain(smem_u32(&tail->v_full[i & 1]), (uint32_t)(i >> 1) & 1u, p.status);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = mbar_wait(smem_u32(&tail->q_full), 0, abort, p.status);
      tc_fence_after();
      for (int j = 0; ok && j <= J; ++j) {
        if (j < J) {
          const int s = j & 1;
          const uint32_t r = (uint32_t)(j >> 1);
          if (!mbar_wait(smem_u32(&tail->k_full[s]), r & 1u, abort, p.status) ||
              !mbar_wait(smem_u32(&tail->s_free[s]), (r & 1u) ^ 1u, abort, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t kst = sbase + C::OFF_STAGE + s * C::STAGE;
#pragma unroll
          for (int kk = 0; kk < HD / 16; ++kk) {
            const uint64_t a = desc_kmajor_sw128(sbase + (kk / 4) * (C::BM * 128)) + 2 * (kk % 4);
            const uint64_t b = desc_kmajor_sw128(kst + (kk / 4) * C::KV_PANEL) + 2 * (kk % 4);
            mma_bf16(tmem + C::TMEM_S + s * C::BN, a, b, C::IDESC_S, kk > 0);
          }
          mma_commit(smem_u32(&tail->s_full[s]));
        }
        if (j >= 1) {
          const int i = j - 1;
          const int s = i & 1;
          const uint32_t r = (uint32_t)(i >> 1);
          if (!mbar_wait(smem_u32(&tail->p_full[s]), r & 1u, abort, p.status) ||
              !mbar_wait(smem_u32(&tail->v_full[s]), r & 1u, abort, p.status) ||
              !mbar_wait(smem_u32(&tail->o_free[s]), (r & 1u) ^ 1u, abort, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t pb = sbase + C::OFF_P + s * C::P_BYTES;
          const uint32_t vst = sbase + C::OFF_STAGE + s * C::STAGE + C::K_BYTES;
#pragma unroll
          for (int kk = 0; kk < C::BN / 16; ++kk) {
            const uint64_t a = desc_kmajor_sw128(pb + (kk / 4) * C::P_PANEL) + 2 * (kk % 4);
            // 16 keys = 16 rows of 128 bytes further along K
            const uint64_t b = desc_mnmajor_sw128(vst + kk * 16 * 128, C::KV_PANEL);
            mma_bf16(tmem + C::TMEM_O + s * HD, a, b, C::IDESC_O, kk > 0);
          }
          mma_commit(smem_u32(&tail->o_full[s]));
          mma_commit(smem_u32(&tail->kv_empty[s]));
        }
      }
      mma_commit(smem_u32(&tail->drain));
      mbar_wait_drain(smem_u32(&tail->drain), 0, p.status);
    }
  } else {
    // ------------------------------------------------------------ softmax + output (warps 2-5)
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;                 // row of the tile = TMEM lane
    const int row = m0 + r;
    const bool live = row < p.R;
    const int limit = p.ctx + (live ? row % p.T : 0);   // last visible cache position
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    const float sl2 = p.scale_log2;
    float o[HD];
#pragma unroll
    for (int i = 0; i < HD; ++i) o[i] = 0.f;
    float m = -INFINITY, l = 0.f, alpha_prev = 0.f;
    bool ok = true;

    auto correct = [&](int i, float a) -> bool {
      const int s = i & 1;
      if (!warp_wait(smem_u32(&tail->o_full[s]), (uint32_t)(i >> 1) & 1u, abort, p.status))
        return false;
      tc_fence_after();
      float v[32];
#pragma unroll
      for (int c = 0; c < HD / 32; ++c) {
        tmem_ld32(tmem + lane_off + C::TMEM_O + s * HD + c * 32, v);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) o[c * 32 + e] = fmaf(o[c * 32 + e], a, v[e]);
      }
      tc_fence_before();
      mbar_arrive(smem_u32(&tail->o_free[s]));
      return true;
    };

    for (int j = 0; j < J; ++j) {
      const int s = j & 1;
      if (!warp_wait(smem_u32(&tail->s_full[s]), (uint32_t)(j >> 1) & 1u, abort, p.status)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t ts = tmem + lane_off + C::TMEM_S + s * C::BN;
      const int key0 = j * C::BN;
      float v[32];
      // pass 1: block maximum of the scaled scores over visible keys
      float bmax = -INFINITY;
#pragma unroll
      for (int c = 0; c < C::BN / 32; ++c) {
        tmem_ld32(ts + c * 32, v);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const float x = (key0 + c * 32 + e <= limit) ? v[e] * sl2 : -INFINITY;
          bmax = fmaxf(bmax, x);
        }
      }
      const float m_new = fmaxf(m, bmax);
      const float alpha = ex2(m - m_new);
      // pass 2: probabilities, their sum, and P (bf16) into the swizzled K-major tile
      float sum = 0.f;
      unsigned char* pb = smem + C::OFF_P + s * C::P_BYTES;
#pragma unroll
      for (int c = 0; c < C::BN / 32; ++c) {
        tmem_ld32(ts + c * 32, v);
        tmem_wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          const float p0 = (key0 + c * 32 + e <= limit) ? ex2(fmaf(v[e], sl2, -m_new)) : 0.f;
          const float p1 = (key0 + c * 32 + e + 1 <= limit) ? ex2(fmaf(v[e + 1], sl2, -m_new)) : 0.f;
          sum += p0 + p1;
          pk[e / 2] = pack2(p0, p1);
        }
        unsigned char* panel = pb + (c >> 1) * C::P_PANEL + (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll
        for (int k4 = 0; k4 < 4; ++k4) {
          const int chunk = ((c & 1) * 4 + k4) ^ (r & 7);
          *reinterpret_cast<uint4*>(panel + chunk * 16) =
              make_uint4(pk[4 * k4], pk[4 * k4 + 1], pk[4 * k4 + 2], pk[4 * k4 + 3]);
        }
      }
      l = l * alpha + sum;
      m = m_new;
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // P visible to the MMA
      tc_fence_before();
      mbar_arrive(smem_u32(&tail->p_full[s]));
      mbar_arrive(smem_u32(&tail->s_free[s]));
      if (j >= 1 && !correct(j - 1, alpha_prev)) {
        ok = false;
        break;
      }
      alpha_prev = alpha;
    }
    if (ok && J > 0) ok = correct(J - 1, alpha_prev);
    if (ok && live) {
      const float inv = 1.0f / l;
      uint4* dst = reinterpret_cast<uint4*>((__nv_bfloat16*)p.out +
                                            ((long long)row * p.Hq + h) * HD);
#pragma unroll
      for (int c = 0; c < HD / 8; ++c)
        dst[c] = make_uint4(pack2(o[8 * c] * inv, o[8 * c + 1] * inv),
                            pack2(o[8 * c + 2] * inv, o[8 * c + 3] * inv),
                            pack2(o[8 * c + 4] * inv, o[8 * c + 5] * inv),
                            pack2(o[8 * c + 6] * inv, o[8 * c + 7] * inv));
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

template <int HD>
ks_status launch_attn(const void* q, const void* kc, const void* vc, long long cache_rows, int R,
                      int T, int Hq, int Hkv, int ctx, void* out, int32_t* status,
                      cudaStream_t st) {
  using C = Cfg<HD>;
  static bool attr = false;
  auto k = attn_kernel<HD>;
  if (!attr) {
    KS_CUDA_TRY(cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM));
    attr = true;
  }
  const int n_keys = ctx + T;
  CUtensorMap tq, tk, tv;
  KS_TRY(make_tmap_2d(&tq, q, R, (long long)Hq * HD, (long long)Hq * HD, 64, C::BM));
  KS_TRY(make_tmap_2d(&tk, kc, n_keys, (long long)Hkv * HD, (long long)Hkv * HD, 64, C::BN));
  KS_TRY(make_tmap_2d(&tv, vc, n_keys, (long long)Hkv * HD, (long long)Hkv * HD, 64, C::BN));
  (void)cache_rows;
  AttnParams ap;
  ap.out = out;
  ap.status = status;
  ap.R = R;
  ap.T = T;
  ap.Hq = Hq;
  ap.Hkv = Hkv;
  ap.ctx = ctx;
  ap.n_keys = n_keys;
  ap.n_blocks = (n_keys + C::BN - 1) / C::BN;
  ap.scale_log2 = (float)(1.4426950408889634 / sqrt((double)HD));
  dim3 grid((R + C::BM - 1) / C::BM, Hq);
  k<<<grid, 192, C::SMEM, st>>>(tq, tk, tv, ap);
  KS_LAUNCH_CHECK();
  return KS_OK;
}

}  // namespace

ks_status tc_attention(const void* q, const void* kc, const void* vc, long long cache_rows, int R,
                       int T, int Hq, int Hkv, int hd, int ctx, void* out, int32_t* status,
                       cudaStream_t st) {
  if (R <= 0) return KS_OK;
  if (Hq % Hkv) return fail(KS_ERR_INVALID_ARG, "attention: Hq must be a multiple of Hkv");
  if (cache_rows < (long long)ctx + T) return fail(KS_ERR_INVALID_ARG, "attention: cache too short");
  if (hd == 128) return launch_attn<128>(q, kc, vc, cache_rows, R, T, Hq, Hkv, ctx, out, status, st);
  if (hd == 64) return launch_attn<64>(q, kc, vc, cache_rows, R, T, Hq, Hkv, ctx, out, status, st);
  return fail(KS_ERR_UNSUPPORTED, "attention: head_dim must be 64 or 128");
}

}  // namespace ks
