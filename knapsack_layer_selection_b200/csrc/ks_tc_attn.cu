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
// One CTA per (128 query rows, query head); 320 threads:
//   warp 0    -- TMA: the Q tile once, then K and V blocks of 128 keys into two
//                2-slot rings (64-column panels, 128-byte swizzle), K two blocks
//                ahead of V;
//   warp 1    -- TMEM owner; one lane issues S_j = Q K_j^T (M=128, N=128) into
//                one of three S buffers and O += P_j V_j (M=128, N=hd, V read
//                MN-major straight from the cache layout) into one TMEM
//                accumulator, in the order S_0, S_1, S_2, PV_0, S_3, PV_1, ...
//                so two score blocks are in flight while block j's softmax runs;
//   warps 2-9 -- two threads per query row, each with half of the block's 128
//                scores and half of the row's O columns (they swap partial row
//                maxima and, at the end, row sums through shared memory); the
//                scores of a block go from TMEM to registers once; the running maximum is kept "stale": P is taken
//                relative to a reference maximum that moves only when the row's
//                maximum grows by more than 2^8, and only then is the row's O in
//                TMEM rescaled (after the previous P.V has landed).  exp2 runs
//                on the MUFU unit for five of every eight scores and as a cubic
//                on the FMA/integer pipes for the other three.  Only blocks that reach past
//                position ctx are masked.  P goes to shared memory as bf16 in the
//                swizzled K-major layout the MMA reads; O is normalised by the
//                running sum once, at the end.
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
  static constexpr int OFF_X = OFF_TAIL + 256;        // [2 blocks][2 halves][128 rows] fp32
  static constexpr int SMEM = OFF_X + 2 * 2 * BM * 4; // the base is checked to be 1024-aligned
  static constexpr int THREADS = 320;                 // TMA, MMA, 8 softmax warps
  static constexpr int S_BUFS = 3;
  static constexpr int TMEM_S = 0;                    // S buffers: columns [0, 3*BN)
  static constexpr int TMEM_O = S_BUFS * BN;          // O accumulator: [3*BN, 3*BN + HD)
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t IDESC_S = idesc_bf16_f32(BM, BN);
  static constexpr uint32_t IDESC_O = idesc_bf16_f32(BM, HD) | (1u << 16);   // B (V) MN-major
};

struct Tail {
  uint64_t q_full;
  uint64_t k_full[2], v_full[2], k_empty[2], v_empty[2];
  uint64_t s_full[3], s_free[3], p_full[2], o_done[2];
  uint64_t pair[2][4];   // per block parity and lane quarter: both halves' values posted
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

struct AttnParams {
  void* out;
  int32_t* status;
  int R, T, Hq, Hkv, ctx, n_keys, n_blocks;
  float scale_log2;
  const int* dyn_cells;   // optional device count: R = min(R, *dyn_cells * T) at run time
};

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Packed pairs of fp32 (Blackwell f32x2 arithmetic: two lanes per instruction).
__device__ __forceinline__ uint64_t pk2(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void upk2(uint64_t v, float& a, float& b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// 2^x for a pair of arguments as 2^n * q(x - n) with n = round(x): adding
// 1.5 * 2^23 leaves n in the low mantissa bits (and, shifted by 23, exactly the
// exponent increment), so no conversion instruction is needed; q is a cubic
// fitted to 2^f on [-1/2, 1/2] for minimal relative error (7.5e-5, far below
// the bf16 rounding of P).  Every step runs on the FMA or integer pipes, two
// lanes per f32x2 instruction, which takes load off the MUFU unit.
__device__ __forceinline__ void exp2_cubic2(float x0, float x1, float& y0, float& y1) {
  const uint64_t x = pk2(fmaxf(x0, -125.0f), fmaxf(x1, -125.0f));   // results stay normal
  const uint64_t t = add2(x, pk2(12582912.0f, 12582912.0f));
  const uint64_t n = add2(t, pk2(-12582912.0f, -12582912.0f));     // round(x) as a float
  const uint64_t f = fma2(n, pk2(-1.0f, -1.0f), x);                // x - round(x)
  uint64_t q = fma2(pk2(0.055171434f, 0.055171434f), f, pk2(0.24261081f, 0.24261081f));
  q = fma2(q, f, pk2(0.69326097f, 0.69326097f));
  q = fma2(q, f, pk2(0.99992812f, 0.99992812f));
  float q0, q1, t0, t1;
  upk2(q, q0, q1);
  upk2(t, t0, t1);
  y0 = __int_as_float(__float_as_int(q0) + (__float_as_int(t0) << 23));
  y1 = __int_as_float(__float_as_int(q1) + (__float_as_int(t1) << 23));
}

// 32 consecutive fp32 columns into this thread's TMEM lane (32x32b shape, x32).
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]),
      "f"(v[8]), "f"(v[9]), "f"(v[10]), "f"(v[11]), "f"(v[12]), "f"(v[13]), "f"(v[14]),
      "f"(v[15]), "f"(v[16]), "f"(v[17]), "f"(v[18]), "f"(v[19]), "f"(v[20]), "f"(v[21]),
      "f"(v[22]), "f"(v[23]), "f"(v[24]), "f"(v[25]), "f"(v[26]), "f"(v[27]), "f"(v[28]),
      "f"(v[29]), "f"(v[30]), "f"(v[31])
      : "memory");
}

__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
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
__global__ void __launch_bounds__(320, 1)
    attn_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const AttnParams p_in) {
  using C = Cfg<HD>;
  AttnParams p = p_in;
  if (p.dyn_cells) {
    const long long live = (long long)(*p.dyn_cells) * p.T;
    p.R = (int)(live < p.R ? live : p.R);
  }
  if ((int)blockIdx.x * C::BM >= p.R) return;   // a row tile past the live rows: nothing to do
  extern __shared__ __align__(1024) unsigned char smem[];
  // the 128-byte-swizzled tiles need a 1024-aligned base; the layout uses all of
  // shared memory, so there is no room to realign -- refuse instead
  if (smem_u32(smem) & 1023u) {
    if (threadIdx.x == 0) raise_status(p.status, KS_ERR_INTERNAL);
    return;
  }
  Tail* tail = reinterpret_cast<Tail*>(smem + C::OFF_TAIL);
  float* xchg = reinterpret_cast<float*>(smem + C::OFF_X);
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
      mbar_init(smem_u32(&tail->k_empty[s]), 1);
      mbar_init(smem_u32(&tail->v_empty[s]), 1);
      mbar_init(smem_u32(&tail->p_full[s]), 256);
      mbar_init(smem_u32(&tail->o_done[s]), 1);
    }
    for (int s = 0; s < C::S_BUFS; ++s) {
      mbar_init(smem_u32(&tail->s_full[s]), 1);
      mbar_init(smem_u32(&tail->s_free[s]), 256);
    }
    for (int s = 0; s < 2; ++s)
      for (int q = 0; q < 4; ++q) mbar_init(smem_u32(&tail->pair[s][q]), 64);
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
      // K runs two blocks ahead of V, in the order the MMA consumes them:
      // K_0, K_1, then K_{j+2}, V_j for j = 0, 1, ...
      auto load_k = [&](int j) -> bool {
        const int s = j & 1;
        if (!mbar_wait(smem_u32(&tail->k_empty[s]), ((uint32_t)(j >> 1) & 1u) ^ 1u, abort,
                       p.status))
          return false;
        const uint32_t kst = sbase + C::OFF_STAGE + s * C::STAGE;
        const uint32_t kf = smem_u32(&tail->k_full[s]);
        mbar_arrive_expect_tx(kf, C::K_BYTES);
        for (int pn = 0; pn < C::PANELS; ++pn)
          tma_load_2d(kst + pn * C::KV_PANEL, &tmK, g * HD + pn * 64, j * C::BN, kf);
        return true;
      };
      auto load_v = [&](int j) -> bool {
        const int s = j & 1;
        if (!mbar_wait(smem_u32(&tail->v_empty[s]), ((uint32_t)(j >> 1) & 1u) ^ 1u, abort,
                       p.status))
          return false;
        const uint32_t vst = sbase + C::OFF_STAGE + s * C::STAGE + C::K_BYTES;
        const uint32_t vf = smem_u32(&tail->v_full[s]);
        mbar_arrive_expect_tx(vf, C::V_BYTES);
        for (int pn = 0; pn < C::PANELS; ++pn)
          tma_load_2d(vst + pn * C::KV_PANEL, &tmV, g * HD + pn * 64, j * C::BN, vf);
        return true;
      };
      int nk = 0, nv = 0;                       // blocks whose K / V loads were issued
      bool ok = true;
      while (ok && nk < J && nk < 2) ok = load_k(nk++);
      while (ok && nv < J) {
        if (nk < J) {
          if (!(ok = load_k(nk))) break;
          ++nk;
        }
        if (!(ok = load_v(nv))) break;
        ++nv;
      }
      // drain the copies still in flight before leaving
      mbar_wait_drain(qf, 0, p.status);
      for (int i = (nk > 2 ? nk - 2 : 0); i < nk; ++i)
        mbar_wait_drain(smem_u32(&tail->k_full[i & 1]), (uint32_t)(i >> 1) & 1u, p.status);
      for (int i = (nv > 2 ? nv - 2 : 0); i < nv; ++i)
        mbar_wait_drain(smem_u32(&tail->v_full[i & 1]), (uint32_t)(i >> 1) & 1u, p.status);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = mbar_wait(smem_u32(&tail->q_full), 0, abort, p.status);
      tc_fence_after();
      // S_j = Q K_j^T into S buffer j % 3; released by the softmax once read
      auto issue_s = [&](int j) -> bool {
        const int ks = j & 1, sb = j % C::S_BUFS;
        if (!mbar_wait(smem_u32(&tail->k_full[ks]), (uint32_t)(j >> 1) & 1u, abort, p.status) ||
            !mbar_wait(smem_u32(&tail->s_free[sb]), ((uint32_t)(j / C::S_BUFS) & 1u) ^ 1u, abort,
                       p.status))
          return false;
        tc_fence_after();
        const uint32_t kst = sbase + C::OFF_STAGE + ks * C::STAGE;
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint64_t a = desc_kmajor_sw128(sbase + (kk / 4) * (C::BM * 128)) + 2 * (kk % 4);
          const uint64_t b = desc_kmajor_sw128(kst + (kk / 4) * C::KV_PANEL) + 2 * (kk % 4);
          mma_bf16(tmem + C::TMEM_S + sb * C::BN, a, b, C::IDESC_S, kk > 0);
        }
        mma_commit(smem_u32(&tail->s_full[sb]));
        mma_commit(smem_u32(&tail->k_empty[ks]));
        return true;
      };
      // O += P_j V_j once the softmax has written P_j
      auto issue_pv = [&](int i) -> bool {
        const int s = i & 1;
        const uint32_t r = (uint32_t)(i >> 1);
        if (!mbar_wait(smem_u32(&tail->p_full[s]), r & 1u, abort, p.status) ||
            !mbar_wait(smem_u32(&tail->v_full[s]), r & 1u, abort, p.status))
          return false;
        tc_fence_after();
        const uint32_t pb = sbase + C::OFF_P + s * C::P_BYTES;
        const uint32_t vst = sbase + C::OFF_STAGE + s * C::STAGE + C::K_BYTES;
#pragma unroll
        for (int kk = 0; kk < C::BN / 16; ++kk) {
          const uint64_t a = desc_kmajor_sw128(pb + (kk / 4) * C::P_PANEL) + 2 * (kk % 4);
          // 16 keys = 16 rows of 128 bytes further along K
          const uint64_t b = desc_mnmajor_sw128(vst + kk * 16 * 128, C::KV_PANEL);
          mma_bf16(tmem + C::TMEM_O, a, b, C::IDESC_O, (i > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(smem_u32(&tail->o_done[s]));
        mma_commit(smem_u32(&tail->v_empty[s]));
        return true;
      };
      // order: S_0, S_1, then S_{j+2} ahead of PV_j, so two score blocks are in
      // flight while the softmax of block j runs
      for (int j = 0; ok && j < J && j < 2; ++j) ok = issue_s(j);
      for (int j = 0; ok && j < J; ++j) {
        if (j + 2 < J) ok = issue_s(j + 2);
        if (ok) ok = issue_pv(j);
      }
      mma_commit(smem_u32(&tail->drain));
      mbar_wait_drain(smem_u32(&tail->drain), 0, p.status);
    }
  } else {
    // ------------------------------------------------------------ softmax + output (warps 2-9)
    // Two warps share each 32-lane quarter of the tile: warp half 0 takes score
    // and O columns [0, 64) of those rows, half 1 columns [64, 128); they swap
    // their partial row maxima (and, at the end, row sums) through shared memory.
    const int q4 = warp & 3;
    const int half = (warp - 2) >> 2;
    const int r = q4 * 32 + lane;                 // row of the tile = TMEM lane
    const int row = m0 + r;
    const bool live = row < p.R;
    const int limit = p.ctx + (live ? row % p.T : 0);   // last visible cache position
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    constexpr int NC = C::BN / 2;                 // score columns per warp
    constexpr int OC = HD / 2;                    // O columns per warp
    const float sl2 = p.scale_log2;
    constexpr float kStale = 8.0f;                // rescale once the max grows by > 2^8
    float m_ref = -INFINITY;                      // reference maximum (raw score units)
    float l = 0.f;                                // this half's running sum relative to m_ref
    bool ok = true;
    for (int j = 0; j < J; ++j) {
      const int s = j & 1;                        // P buffer / O-done barrier of this block
      const int sb = j % C::S_BUFS;               // S buffer of this block
      if (!warp_wait(smem_u32(&tail->s_full[sb]), (uint32_t)(j / C::S_BUFS) & 1u, abort,
                     p.status)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t ts = tmem + lane_off + C::TMEM_S + sb * C::BN + half * NC;
      const int key0 = j * C::BN + half * NC;
      const bool masked = j * C::BN + C::BN - 1 > p.ctx;   // a key may be past a row's window
      float sc[NC];
#pragma unroll
      for (int c = 0; c < NC / 32; ++c)
        tmem_ld32(ts + c * 32, *reinterpret_cast<float(*)[32]>(&sc[c * 32]));
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(smem_u32(&tail->s_free[sb]));   // S buffer may be overwritten now
      if (masked) {
#pragma unroll
        for (int e = 0; e < NC; ++e)
          if (key0 + e > limit) sc[e] = -INFINITY;
      }
      static_assert(NC % 2 == 0 && NC >= 4, "pairs of scores");
      float mx[4] = {sc[0], sc[1], sc[2], sc[3]};
#pragma unroll
      for (int e = 4; e < NC; e += 2)             // columns 4 .. NC-1, two at a time
        mx[(e >> 1) & 3] = fmax3(mx[(e >> 1) & 3], sc[e], sc[e + 1]);
      const float hmax = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
      // swap half maxima with the partner warp (a bounded wait, like every other)
      float* xb = xchg + s * (2 * C::BM);
      xb[half * C::BM + r] = hmax;
      mbar_arrive(smem_u32(&tail->pair[s][q4]));
      if (!warp_wait(smem_u32(&tail->pair[s][q4]), (uint32_t)(j >> 1) & 1u, abort, p.status)) {
        ok = false;
        break;
      }
      const float bmax = fmaxf(hmax, xb[(1 - half) * C::BM + r]);
      const bool grow = (bmax - m_ref) * sl2 > kStale;   // true on the first block
      if (__any_sync(0xffffffffu, grow && j > 0)) {
        // rescale this warp's O columns once the previous P.V has landed in TMEM
        const int i = j - 1;
        if (!warp_wait(smem_u32(&tail->o_done[i & 1]), (uint32_t)(i >> 1) & 1u, abort,
                       p.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const float a = grow ? ex2((m_ref - bmax) * sl2) : 1.0f;
        float v[32];
#pragma unroll
        for (int c = 0; c < OC / 32; ++c) {
          const uint32_t to = tmem + lane_off + C::TMEM_O + half * OC + c * 32;
          tmem_ld32(to, v);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] *= a;
          tmem_st32(to, v);
        }
        tmem_wait_st();
        l *= a;
      }
      if (grow) m_ref = bmax;
      // P_j into shared buffer s: the P.V that last read it (block j-2) must be done
      if (j >= 2) {
        const int i = j - 2;
        if (!warp_wait(smem_u32(&tail->o_done[i & 1]), (uint32_t)(i >> 1) & 1u, abort,
                       p.status)) {
          ok = false;
          break;
        }
      }
      const uint64_t scale2 = pk2(sl2, sl2);
      const uint64_t moff2 = pk2(-m_ref * sl2, -m_ref * sl2);
      uint64_t sum2[4] = {0, 0, 0, 0};
      unsigned char* rowp = smem + C::OFF_P + s * C::P_BYTES + half * C::P_PANEL +
                            (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll
      for (int c8 = 0; c8 < NC / 8; ++c8) {       // 8 keys = one 16-byte chunk of the P row
        uint32_t pk[4];
#pragma unroll
        for (int e = 0; e < 8; e += 2) {
          const int k = c8 * 8 + e;
          float x0, x1, p0, p1;
          upk2(fma2(pk2(sc[k], sc[k + 1]), scale2, moff2), x0, x1);
          if ((c8 & 1) ? (e == 2 || e == 6) : (e == 6)) {
            exp2_cubic2(x0, x1, p0, p1);           // three pairs in eight on the FMA pipe
          } else {
            p0 = ex2(x0);
            p1 = ex2(x1);
          }
          sum2[e >> 1] = add2(sum2[e >> 1], pk2(p0, p1));
          pk[e >> 1] = pack2(p0, p1);
        }
        *reinterpret_cast<uint4*>(rowp + ((c8 ^ (r & 7)) * 16)) =
            make_uint4(pk[0], pk[1], pk[2], pk[3]);
      }
      float t0, t1, t2, t3, t4, t5, t6, t7;
      upk2(sum2[0], t0, t1);
      upk2(sum2[1], t2, t3);
      upk2(sum2[2], t4, t5);
      upk2(sum2[3], t6, t7);
      l += ((t0 + t1) + (t2 + t3)) + ((t4 + t5) + (t6 + t7));
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // P visible to the MMA
      tc_fence_before();                          // and any O rescale stores ordered first
      mbar_arrive(smem_u32(&tail->p_full[s]));
    }
    if (ok && J > 0) {
      const int i = J - 1;
      ok = warp_wait(smem_u32(&tail->o_done[i & 1]), (uint32_t)(i >> 1) & 1u, abort, p.status);
    }
    if (ok) {
      // row sum = both halves' sums (exchanged in the block buffer no block uses now)
      float* xb = xchg + (J & 1) * (2 * C::BM);
      xb[half * C::BM + r] = l;
      mbar_arrive(smem_u32(&tail->pair[J & 1][q4]));
      ok = warp_wait(smem_u32(&tail->pair[J & 1][q4]), (uint32_t)(J >> 1) & 1u, abort, p.status);
    }
    if (ok) {
      float* xb = xchg + (J & 1) * (2 * C::BM);
      const float inv = 1.0f / (l + xb[(1 - half) * C::BM + r]);
      tc_fence_after();
      uint4* dst = reinterpret_cast<uint4*>((__nv_bfloat16*)p.out +
                                            ((long long)row * p.Hq + h) * HD + half * OC);
      float v[32];
#pragma unroll
      for (int c = 0; c < OC / 32; ++c) {
        tmem_ld32(tmem + lane_off + C::TMEM_O + half * OC + c * 32, v);
        tmem_wait_ld();
        if (live) {
#pragma unroll
          for (int q8 = 0; q8 < 4; ++q8)
            dst[c * 4 + q8] = make_uint4(pack2(v[8 * q8] * inv, v[8 * q8 + 1] * inv),
                                         pack2(v[8 * q8 + 2] * inv, v[8 * q8 + 3] * inv),
                                         pack2(v[8 * q8 + 4] * inv, v[8 * q8 + 5] * inv),
                                         pack2(v[8 * q8 + 6] * inv, v[8 * q8 + 7] * inv));
        }
      }
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
                      cudaStream_t st, const int* dyn_cells) {
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
  ap.dyn_cells = dyn_cells;
  dim3 grid((R + C::BM - 1) / C::BM, Hq);
  k<<<grid, C::THREADS, C::SMEM, st>>>(tq, tk, tv, ap);
  KS_LAUNCH_CHECK();
  return KS_OK;
}

}  // namespace

ks_status tc_attention(const void* q, const void* kc, const void* vc, long long cache_rows, int R,
                       int T, int Hq, int Hkv, int hd, int ctx, void* out, int32_t* status,
                       cudaStream_t st, const int* dyn_cells) {
  if (R <= 0) return KS_OK;
  if (Hq % Hkv) return fail(KS_ERR_INVALID_ARG, "attention: Hq must be a multiple of Hkv");
  if (cache_rows < (long long)ctx + T) return fail(KS_ERR_INVALID_ARG, "attention: cache too short");
  if (hd == 128)
    return launch_attn<128>(q, kc, vc, cache_rows, R, T, Hq, Hkv, ctx, out, status, st, dyn_cells);
  if (hd == 64)
    return launch_attn<64>(q, kc, vc, cache_rows, R, T, Hq, Hkv, ctx, out, status, st, dyn_cells);
  return fail(KS_ERR_UNSUPPORTED, "attention: head_dim must be 64 or 128");
}

}  // namespace ks
