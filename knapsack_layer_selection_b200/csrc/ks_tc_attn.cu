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
// One CTA per (128 query rows, query head); 384 threads in three warpgroups:
//   warp 0    -- TMA: the Q tile once, then K blocks of 128 keys into a 3-slot
//                ring and V blocks into a 2-slot ring (64-column panels,
//                128-byte swizzle); each V slot ends with a panel of ones;
//   warp 1    -- TMEM owner; one lane issues S_i = Q K_i^T (M=128, N=128) into
//                S buffer i%2, as soon as the softmax has copied S_{i-2} out
//                (the softmax group that sees S_i complete also frees K_i's
//                slot, so each S group ends with a single commit);
//   warp 2    -- one lane issues [O | l] += P_i [V_i | 1] (M=128, N=hd+16) with
//                P_i read from TMEM and V read MN-major straight from the cache
//                layout, as soon as P_i is written: the 16 columns after O
//                collect P's row sums, so the softmax never adds its
//                probabilities up.  An MMA issue returns only as the tensor
//                core takes the work, so with one issuing thread every barrier
//                wait, fence and commit would leave the tensor core idle; with
//                two, one thread's waits overlap the other's MMAs (each commit
//                tracks its own thread's MMAs, and S and P.V never touch the
//                same TMEM columns);
//   warp 3    -- idle (it only gives its registers to the softmax);
//   warps 4-7 and 8-11 -- two softmax groups, one thread per query row (its
//                TMEM lane) in each: group 0 takes the even blocks, group 1 the
//                odd ones, so two blocks' softmax run at once.  A group copies
//                its block's 128 scores from TMEM to registers once and frees
//                the S buffer at once, so S_{i+2} is computed while block i's P
//                is produced; P goes to TMEM (one buffer) once PV_{i-1} has read
//                the previous one.  The running maximum is "stale": block i's
//                reference m_i is m_{i-1} unless the block's maximum exceeds it
//                by more than 2^8 (in exp2 units), in which case it is the
//                block's maximum and O with its row sums is rescaled in TMEM
//                (after PV_{i-1} has landed).  m_i passes from the group of block
//                i to the other through shared memory, so both groups' P are taken
//                relative to the same sequence of references.  exp2 runs on the
//                MUFU unit (with the row sums on the tensor core, the softmax is
//                bound by its instruction count, not by MUFU: moving part of the
//                exponentials to an FMA-pipe polynomial was measured slower); only
//                blocks that reach past position ctx are masked.  The group of
//                the last block divides O by its row sum and stores it.
// Registers: the softmax threads hold a block's 128 scores, so the kernel
// launches with 168 registers a thread and moves them with setmaxnreg from the
// first warpgroup (56) to the two softmax warpgroups (224): 128*56 + 256*224 =
// 384*168, the launch's whole allocation.  The host refuses to launch a build
// whose register count is not 168, since a larger share could never be met.
// Every row uses the same block order and the same arithmetic whatever the
// batch, so a row's output does not depend on the other rows.
#include <cuda.h>

#include "ks_sm100.cuh"
#include "ks_tc.cuh"

namespace ks {

using namespace sm100;

namespace {

struct Tail {
  uint64_t q_full;
  uint64_t k_full[3], k_empty[3], v_full[2], v_empty[2];
  uint64_t s_full[2], s_free[2];                           // [softmax group = S buffer]
  uint64_t p_full;                                         // one phase per block
  uint64_t pv_done[2];                                     // [block parity]: PV_i on pv_done[i % 2]
  uint64_t m_ready[2];                                     // [group of the publishing block]
  uint64_t drain[2];                                       // [S issuer, PV issuer]
  uint32_t tmem_base;
  int abort;
  float m_pub[2][128];                                     // block references, by block parity
};

template <int HD>
struct Cfg {
  static constexpr int BM = 128, BN = 128, KST = 3, VST = 2;   // rows, keys per block, K / V slots
  static constexpr int PANELS = HD / 64;              // 64-wide panels along head_dim
  static constexpr int Q_PANEL = BM * 128;            // [128 rows][64] bf16
  static constexpr int Q_TILE = PANELS * Q_PANEL;
  static constexpr int KV_PANEL = BN * 128;           // [128 keys][64] bf16
  static constexpr int KV_BLOCK = PANELS * KV_PANEL;
  // a V slot holds the block's PANELS panels of V and one panel of ones after
  // them: the P.V MMA reads N = HD + 16 columns, the last 16 giving P's row sums
  static constexpr int V_SLOT = (PANELS + 1) * KV_PANEL;
  static constexpr int N_O = HD + 16;
  static constexpr int OFF_K = Q_TILE;
  static constexpr int OFF_V = OFF_K + KST * KV_BLOCK;
  static constexpr int OFF_TAIL = OFF_V + VST * V_SLOT;
  static constexpr int USED = OFF_TAIL + (int)((sizeof(Tail) + 255) / 256 * 256);
  // at least 116 KB, so one CTA holds an SM and its 512 TMEM columns
  static constexpr int SMEM = USED > 118784 ? USED : 118784;   // base checked 1024-aligned
  static constexpr int THREADS = 384;                 // TMA, MMA, 2 idle, 2 x 4 softmax warps
  static constexpr int REGS = 168, REGS_LOW = 56, REGS_HIGH = 224;
  static_assert(128 * REGS_LOW + 256 * REGS_HIGH == THREADS * REGS, "register split");
  static constexpr int TMEM_S = 0;                    // S[b]: columns b * BN (fp32)
  static constexpr int TMEM_P = 2 * BN;               // P: TMEM_P .. + BN/2 (bf16 pairs)
  static constexpr int TMEM_O = 2 * BN + BN / 2;      // O: HD columns, then 16 of row sums
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t IDESC_S = idesc_bf16_f32(BM, BN);
  static constexpr uint32_t IDESC_O = idesc_bf16_f32(BM, N_O) | (1u << 16);   // B (V) MN-major
  static_assert(TMEM_O + N_O <= (int)TMEM_COLS, "TMEM budget");
  static_assert(USED <= 232448, "shared memory budget");
};

struct AttnParams {
  void* out;
  int32_t* status;
  int R, T, Hq, Hkv, ctx, n_keys, n_blocks;
  float scale_log2;
  const int* dyn_cells;   // optional device count: R = min(R, *dyn_cells * T) at run time
  int window;             // window reading: the last block holds the tile's own window keys
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
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
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

// Ties 32 registers filled by tcgen05.ld to the point after tcgen05.wait::ld:
// the compiler sees no dependency between the two instructions, so without
// this a use of the registers could be scheduled before the wait.
__device__ __forceinline__ void reg_fence32(float (&v)[32]) {
  asm volatile(""
               : "+f"(v[0]), "+f"(v[1]), "+f"(v[2]), "+f"(v[3]), "+f"(v[4]), "+f"(v[5]),
                 "+f"(v[6]), "+f"(v[7]), "+f"(v[8]), "+f"(v[9]), "+f"(v[10]), "+f"(v[11]),
                 "+f"(v[12]), "+f"(v[13]), "+f"(v[14]), "+f"(v[15]), "+f"(v[16]), "+f"(v[17]),
                 "+f"(v[18]), "+f"(v[19]), "+f"(v[20]), "+f"(v[21]), "+f"(v[22]), "+f"(v[23]),
                 "+f"(v[24]), "+f"(v[25]), "+f"(v[26]), "+f"(v[27]), "+f"(v[28]), "+f"(v[29]),
                 "+f"(v[30]), "+f"(v[31]));
}

// 16 consecutive 32-bit columns (packed bf16 pairs) into this thread's TMEM lane.
__device__ __forceinline__ void tmem_st16u(uint32_t taddr, const uint32_t* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
      "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
      "r"(v[15])
      : "memory");
}

template <uint32_t N>
__device__ __forceinline__ void regs_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}
template <uint32_t N>
__device__ __forceinline__ void regs_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}

template <int HD>
__global__ void __launch_bounds__(384, 1)
    attn_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmKw,
                const __grid_constant__ CUtensorMap tmVw, const AttnParams p_in) {
  using C = Cfg<HD>;
  AttnParams p = p_in;
  if (p.dyn_cells) {
    const long long live = (long long)(*p.dyn_cells) * p.T;
    p.R = (int)(live < p.R ? live : p.R);
  }
  const int m0 = blockIdx.x * C::BM;
  if (m0 >= p.R) return;                        // a row tile past the live rows: nothing to do
  extern __shared__ __align__(1024) unsigned char smem[];
  // the 128-byte-swizzled tiles need a 1024-aligned base; refuse rather than realign
  if (smem_u32(smem) & 1023u) {
    if (threadIdx.x == 0) raise_status(p.status, KS_ERR_INTERNAL);
    return;
  }
  Tail* tail = reinterpret_cast<Tail*>(smem + C::OFF_TAIL);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y;
  const int g = h / (p.Hq / p.Hkv);
  const int J = p.n_blocks;
  volatile int* abort = &tail->abort;
  const uint32_t sbase = smem_u32(smem);

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&tail->q_full), 1);
    for (int s = 0; s < C::KST; ++s) {
      mbar_init(smem_u32(&tail->k_full[s]), 1);
      mbar_init(smem_u32(&tail->k_empty[s]), 1);
    }
    for (int s = 0; s < C::VST; ++s) {
      mbar_init(smem_u32(&tail->v_full[s]), 1);
      mbar_init(smem_u32(&tail->v_empty[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&tail->s_full[b]), 1);
      mbar_init(smem_u32(&tail->s_free[b]), 4);         // one arrival per softmax warp
      mbar_init(smem_u32(&tail->m_ready[b]), 4);
    }
    mbar_init(smem_u32(&tail->p_full), 4);
    mbar_init(smem_u32(&tail->pv_done[0]), 1);
    mbar_init(smem_u32(&tail->pv_done[1]), 1);
    mbar_init(smem_u32(&tail->drain[0]), 1);
    mbar_init(smem_u32(&tail->drain[1]), 1);
    tail->abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&tail->tmem_base), C::TMEM_COLS);
    tmem_relinquish();
  }
  // the ones panel of each V slot (every element 1.0, so its swizzle is moot);
  // the TMA only ever writes the V panels before it
  for (int s = 0; s < C::VST; ++s) {
    uint4* ones = reinterpret_cast<uint4*>(smem + C::OFF_V + s * C::V_SLOT + C::PANELS * C::KV_PANEL);
    for (int e = threadIdx.x; e < C::KV_PANEL / 16; e += blockDim.x)
      ones[e] = make_uint4(0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u);
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // visible to the tensor core
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tail->tmem_base;

  if (warp < 4) {
    regs_dec<C::REGS_LOW>();
    if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      if (p.window) {
        prefetch_tmap(&tmKw);
        prefetch_tmap(&tmVw);
      }
      const uint32_t qf = smem_u32(&tail->q_full);
      mbar_arrive_expect_tx(qf, C::Q_TILE);
      for (int pn = 0; pn < C::PANELS; ++pn)
        tma_load_2d(sbase + pn * C::Q_PANEL, &tmQ, h * HD + pn * 64, m0, qf);
      // block m of K (V) goes to ring slot m % KST once the MMA of block m - KST is done.
      // Under the window reading the last block is the tile's own rows of the window
      // keys / values (whole states: T divides 128 and m0 is a multiple of 128).
      auto load_kv = [&](const CUtensorMap* tm, const CUtensorMap* tmw, int off, uint64_t* full,
                         uint64_t* empty, int m, int nst, int slot_bytes) -> bool {
        const int s = m % nst;
        if (!mbar_wait(smem_u32(&empty[s]), ((uint32_t)(m / nst) & 1u) ^ 1u, abort, p.status))
          return false;
        const uint32_t dst = sbase + off + s * slot_bytes;
        const uint32_t fb = smem_u32(&full[s]);
        const bool win = p.window && m == J - 1;
        const CUtensorMap* src = win ? tmw : tm;
        const int row0 = win ? m0 : m * C::BN;
        mbar_arrive_expect_tx(fb, C::KV_BLOCK);
        for (int pn = 0; pn < C::PANELS; ++pn)
          tma_load_2d(dst + pn * C::KV_PANEL, src, g * HD + pn * 64, row0, fb);
        return true;
      };
      // in the order the MMAs consume them: K_0, K_1, then K_{j+2}, V_j for j = 0, 1, ...
      int nk = 0, nv = 0;                       // blocks whose K / V loads were issued
      bool ok = true;
      while (ok && nk < J && nk < 2) {
        ok = load_kv(&tmK, &tmKw, C::OFF_K, tail->k_full, tail->k_empty, nk, C::KST, C::KV_BLOCK);
        if (ok) ++nk;
      }
      while (ok && nv < J) {
        if (nk < J) {
          if (!(ok = load_kv(&tmK, &tmKw, C::OFF_K, tail->k_full, tail->k_empty, nk, C::KST,
                             C::KV_BLOCK)))
            break;
          ++nk;
        }
        if (!(ok = load_kv(&tmV, &tmVw, C::OFF_V, tail->v_full, tail->v_empty, nv, C::VST,
                           C::V_SLOT)))
          break;
        ++nv;
      }
      // drain the copies still in flight before leaving
      mbar_wait_drain(qf, 0, p.status);
      for (int i = (nk > C::KST ? nk - C::KST : 0); i < nk; ++i)
        mbar_wait_drain(smem_u32(&tail->k_full[i % C::KST]), (uint32_t)(i / C::KST) & 1u,
                        p.status);
      for (int i = (nv > C::VST ? nv - C::VST : 0); i < nv; ++i)
        mbar_wait_drain(smem_u32(&tail->v_full[i % C::VST]), (uint32_t)(i / C::VST) & 1u,
                        p.status);
    }
    } else if (warp == 1) {
      // ---------------------------------------------------------- S issuer
      if (lane == 0) {
        bool ok = mbar_wait(smem_u32(&tail->q_full), 0, abort, p.status);
        const uint64_t dq0 = desc_kmajor_sw128(sbase);
        const uint64_t dk0 = desc_kmajor_sw128(sbase + C::OFF_K);
        for (int i = 0; ok && i < J; ++i) {
          // S_i = Q K_i^T into S buffer i % 2, free once the softmax has copied S_{i-2}
          const int ks = i % C::KST, b = i & 1;
          if (i >= 2 && !(ok = mbar_wait(smem_u32(&tail->s_free[b]), ((uint32_t)(i - 2) >> 1) & 1u,
                                         abort, p.status)))
            break;
          if (!(ok = mbar_wait(smem_u32(&tail->k_full[ks]), (uint32_t)(i / C::KST) & 1u, abort,
                               p.status)))
            break;
          tc_fence_after();
          // descriptors of a tile: the base's plus the byte offset / 16 (shared
          // addresses stay below 2^18, so the 14-bit start field never carries)
          const uint64_t dk = dk0 + (uint64_t)((ks * C::KV_BLOCK) >> 4);
          const uint32_t ds = tmem + C::TMEM_S + b * C::BN;
#pragma unroll
          for (int kk = 0; kk < HD / 16; ++kk)
            mma_bf16(ds, dq0 + (uint64_t)((kk / 4) * (C::Q_PANEL >> 4) + 2 * (kk % 4)),
                     dk + (uint64_t)((kk / 4) * (C::KV_PANEL >> 4) + 2 * (kk % 4)), C::IDESC_S,
                     kk > 0);
          // one commit: the softmax group that sees S_i complete frees K slot ks
          mma_commit(smem_u32(&tail->s_full[b]));
        }
        mma_commit(smem_u32(&tail->drain[0]));
        mbar_wait_drain(smem_u32(&tail->drain[0]), 0, p.status);
      }
    } else if (warp == 2) {
      // ---------------------------------------------------------- P.V issuer
      if (lane == 0) {
        bool ok = true;
        const uint64_t dv0 = desc_mnmajor_sw128(sbase + C::OFF_V, C::KV_PANEL);
        for (int i = 0; ok && i < J; ++i) {
          // [O | row sums] += P_i [V_i | ones] once the softmax has written P_i
          const int vs = i % C::VST;
          if (!(ok = mbar_wait(smem_u32(&tail->p_full), (uint32_t)i & 1u, abort, p.status)))
            break;
          if (!(ok = mbar_wait(smem_u32(&tail->v_full[vs]), (uint32_t)(i / C::VST) & 1u, abort,
                               p.status)))
            break;
          tc_fence_after();
          const uint64_t dv = dv0 + (uint64_t)((vs * C::V_SLOT) >> 4);
          const uint32_t pt = tmem + C::TMEM_P;
#pragma unroll
          for (int kk = 0; kk < C::BN / 16; ++kk)
            // 16 keys = 8 packed TMEM columns of P, 16 rows of 128 bytes further along V
            mma_bf16_tmem_a(tmem + C::TMEM_O, pt + kk * 8, dv + (uint64_t)(kk * ((16 * 128) >> 4)),
                            C::IDESC_O, (i > 0 || kk > 0) ? 1u : 0u);
          mma_commit(smem_u32(&tail->pv_done[i & 1]));
          mma_commit(smem_u32(&tail->v_empty[vs]));
        }
        mma_commit(smem_u32(&tail->drain[1]));
        mbar_wait_drain(smem_u32(&tail->drain[1]), 0, p.status);
      }
    }
  } else {
    regs_inc<C::REGS_HIGH>();
    // ------------------------------------------------------------ softmax groups (warps 4-11)
    const int G = (warp - 4) >> 2;               // group: blocks i with i % 2 == G
    const int q4 = warp & 3;                     // TMEM lane quarter this warp may access
    const int r = q4 * 32 + lane;                // row of the tile = TMEM lane
    const int row = m0 + r;
    const bool live = row < p.R;
    const int limit = p.ctx + (live ? row % p.T : 0);   // last visible cache position
    // window reading: context blocks show positions < ctx; the last block shows the
    // keys lo .. r of the tile (this row's own state, tokens 0 .. t)
    const int ctx_last = p.ctx - 1;
    const int win_lo = (r / p.T) * p.T;
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    const uint32_t ts = tmem + lane_off + C::TMEM_S + G * C::BN;
    const uint32_t tp = tmem + lane_off + C::TMEM_P;
    constexpr int NC = C::BN;                    // scores per row and block
    const float sl2 = p.scale_log2;
    constexpr float kStale = 8.0f;               // a new reference once the max grows by > 2^8
    bool ok = true;
    // waits until PV_q has completed.  PV_q commits to pv_done[q % 2], whose phases
    // are PV_{q-2}, PV_q, PV_{q+2}...; at every wait below PV_{q-2} has completed
    // (this group waited for it, or for a later P.V, whose commit covers it) and
    // PV_{q+2} cannot have (it needs a P this group has not yet written), so a
    // parity wait sees the right phase
    auto wait_pv = [&](int q) -> bool {
      if (!warp_wait(smem_u32(&tail->pv_done[q & 1]), ((uint32_t)q >> 1) & 1u, abort, p.status))
        return false;
      tc_fence_after();
      return true;
    };
    for (int i = G; i < J; i += 2) {
      const uint32_t k = (uint32_t)(i >> 1);     // this group's k-th block
      if (!warp_wait(smem_u32(&tail->s_full[G]), k & 1u, abort, p.status)) {
        ok = false;
        break;
      }
      if (q4 == 0 && lane == 0) mbar_arrive(smem_u32(&tail->k_empty[i % C::KST]));   // K_i read
      tc_fence_after();
      float sc[NC];
#pragma unroll
      for (int c = 0; c < NC / 32; ++c)
        tmem_ld32(ts + c * 32, *reinterpret_cast<float(*)[32]>(&sc[c * 32]));
      tmem_wait_ld();
#pragma unroll
      for (int c = 0; c < NC / 32; ++c) reg_fence32(*reinterpret_cast<float(*)[32]>(&sc[c * 32]));
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&tail->s_free[G]));   // S_{i+2} may be computed now
      if (p.window) {
        if (i == J - 1) {                        // the tile's own window keys
#pragma unroll
          for (int e = 0; e < NC; ++e)
            if (e < win_lo || e > r) sc[e] = -INFINITY;
        } else if (i * C::BN + C::BN - 1 > ctx_last) {   // a context block reaching past ctx
          const int key0 = i * C::BN;
#pragma unroll
          for (int e = 0; e < NC; ++e)
            if (key0 + e > ctx_last) sc[e] = -INFINITY;
        }
      } else if (i * C::BN + C::BN - 1 > p.ctx) {   // a key of this block may be past the window
        const int key0 = i * C::BN;
#pragma unroll
        for (int e = 0; e < NC; ++e)
          if (key0 + e > limit) sc[e] = -INFINITY;
      }
      float mx[4] = {sc[0], sc[1], sc[2], sc[3]};
#pragma unroll
      for (int e = 4; e < NC; e += 2)            // columns 4 .. NC-1, two at a time
        mx[(e >> 1) & 3] = fmax3(mx[(e >> 1) & 3], sc[e], sc[e + 1]);
      const float bmax = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
      // the reference of the previous block, from the other group
      float m_in = -INFINITY;
      if (i > 0) {
        const int q = i - 1;
        if (!warp_wait(smem_u32(&tail->m_ready[1 - G]), ((uint32_t)q >> 1) & 1u, abort,
                       p.status)) {
          ok = false;
          break;
        }
        m_in = tail->m_pub[1 - G][r];
      }
      const bool grow = (bmax - m_in) * sl2 > kStale;   // true on block 0
      const float m_new = grow ? bmax : m_in;
      tail->m_pub[G][r] = m_new;
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&tail->m_ready[G]));
      if (__any_sync(0xffffffffu, grow && i > 0)) {
        // O and its row sums hold the P.V of blocks < i relative to m_in: rescale them
        // once PV_{i-1} has landed
        if (!wait_pv(i - 1)) {
          ok = false;
          break;
        }
        const float a = grow ? ex2((m_in - m_new) * sl2) : 1.0f;
        float v[32];
#pragma unroll
        for (int c = 0; c < HD / 32; ++c) {
          const uint32_t to = tmem + lane_off + C::TMEM_O + c * 32;
          tmem_ld32(to, v);
          tmem_wait_ld();
          reg_fence32(v);
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] *= a;
          tmem_st32(to, v);
        }
        {
          const uint32_t to = tmem + lane_off + C::TMEM_O + HD;   // the 16 row-sum columns
          tmem_wait_st();                        // the stores above land before this reload
          tmem_ld32(to - 16, v);                 // 32 columns ending at the sums: HD-16 .. HD+15
          tmem_wait_ld();
          reg_fence32(v);
#pragma unroll
          for (int e = 16; e < 32; ++e) v[e] *= a;   // the first 16 were rescaled above
          tmem_st32(to - 16, v);
        }
      }
      const uint64_t scale2 = pk2(sl2, sl2);
      const uint64_t moff2 = pk2(-m_new * sl2, -m_new * sl2);
      uint32_t pk[NC / 2];                       // P of the block as bf16 pairs
#pragma unroll
      for (int e = 0; e < NC; e += 2) {
        float x0, x1, p0, p1;
        upk2(fma2(pk2(sc[e], sc[e + 1]), scale2, moff2), x0, x1);
        p0 = ex2(x0);
        p1 = ex2(x1);
        pk[e >> 1] = pack2(p0, p1);
      }
      // the P buffer was last read by PV_{i-1}: wait for it only now, with P in registers
      if (i >= 1 && !wait_pv(i - 1)) {
        ok = false;
        break;
      }
#pragma unroll
      for (int c = 0; c < NC / 32; ++c) tmem_st16u(tp + c * 16, &pk[c * 16]);
      tmem_wait_st();                            // P and any O rescale stores complete
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&tail->p_full));
    }
    // the group of the last block writes the output: O over its row sum
    const int last = J - 1;
    if (ok && G == (last & 1) && wait_pv(last)) {
      float v[32];
      tmem_ld32(tmem + lane_off + C::TMEM_O + HD - 16, v);   // HD-16 .. HD+15: the sum at 16
      tmem_wait_ld();
      reg_fence32(v);
      const float inv = 1.0f / v[16];
      uint4* dst = reinterpret_cast<uint4*>((__nv_bfloat16*)p.out +
                                            ((long long)row * p.Hq + h) * HD);
#pragma unroll
      for (int c = 0; c < HD / 32; ++c) {
        tmem_ld32(tmem + lane_off + C::TMEM_O + c * 32, v);
        tmem_wait_ld();
        reg_fence32(v);
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
ks_status launch_attn(const void* q, const void* kc, const void* vc, int R, int T, int Hq, int Hkv,
                      int ctx, void* out, int32_t* status, cudaStream_t st,
                      const int* dyn_cells, const void* kw, const void* vw) {
  using C = Cfg<HD>;
  static std::atomic<unsigned long long> attr{0};
  auto k = attn_kernel<HD>;
  KS_TRY(once_per_device(attr, [&]() -> ks_status {
    // the setmaxnreg split assumes exactly C::REGS registers a thread at launch
    cudaFuncAttributes fa;
    KS_CUDA_TRY(cudaFuncGetAttributes(&fa, k));
    if (fa.numRegs != C::REGS)
      return fail(KS_ERR_INTERNAL, "attention: kernel built with " + std::to_string(fa.numRegs) +
                                       " registers a thread, the register split needs " +
                                       std::to_string(C::REGS));
    KS_CUDA_TRY(cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM));
    return KS_OK;
  }));
  const bool window = kw != nullptr;
  // keys read from the cache: all ctx + T positions, or the ctx context positions
  // when the window comes from kw / vw (at least one row, so the map is valid)
  const int n_keys = window ? ctx : ctx + T;
  const long long kvd = (long long)Hkv * HD;
  CUtensorMap tq, tk, tv, tkw, tvw;
  KS_TRY(make_tmap_2d(&tq, q, R, (long long)Hq * HD, (long long)Hq * HD, 64, C::BM));
  KS_TRY(make_tmap_2d(&tk, kc, n_keys > 0 ? n_keys : 1, kvd, kvd, 64, C::BN));
  KS_TRY(make_tmap_2d(&tv, vc, n_keys > 0 ? n_keys : 1, kvd, kvd, 64, C::BN));
  if (window) {
    KS_TRY(make_tmap_2d(&tkw, kw, R, kvd, kvd, 64, C::BN));
    KS_TRY(make_tmap_2d(&tvw, vw, R, kvd, kvd, 64, C::BN));
  } else {
    tkw = tk;
    tvw = tv;
  }
  AttnParams ap;
  ap.out = out;
  ap.status = status;
  ap.R = R;
  ap.T = T;
  ap.Hq = Hq;
  ap.Hkv = Hkv;
  ap.ctx = ctx;
  ap.n_keys = n_keys;
  ap.n_blocks = (n_keys + C::BN - 1) / C::BN + (window ? 1 : 0);
  ap.scale_log2 = (float)(1.4426950408889634 / sqrt((double)HD));
  ap.dyn_cells = dyn_cells;
  ap.window = window ? 1 : 0;
  const dim3 grid((R + C::BM - 1) / C::BM, Hq);
  k<<<grid, C::THREADS, C::SMEM, st>>>(tq, tk, tv, tkw, tvw, ap);
  KS_LAUNCH_CHECK();
  return KS_OK;
}

}  // namespace

ks_status tc_attention(const void* q, const void* kc, const void* vc, long long cache_rows, int R,
                       int T, int Hq, int Hkv, int hd, int ctx, void* out, int32_t* status,
                       cudaStream_t st, const int* dyn_cells, const void* kw, const void* vw) {
  if (R <= 0) return KS_OK;
  if (Hq % Hkv) return fail(KS_ERR_INVALID_ARG, "attention: Hq must be a multiple of Hkv");
  if (cache_rows < (long long)ctx + T) return fail(KS_ERR_INVALID_ARG, "attention: cache too short");
  if ((kw == nullptr) != (vw == nullptr))
    return fail(KS_ERR_INVALID_ARG, "attention: window keys and values go together");
  if (kw && (T < 1 || 128 % T))
    return fail(KS_ERR_UNSUPPORTED, "attention: the window reading needs T to divide 128");
  if (hd == 128)
    return launch_attn<128>(q, kc, vc, R, T, Hq, Hkv, ctx, out, status, st, dyn_cells, kw, vw);
  if (hd == 64)
    return launch_attn<64>(q, kc, vc, R, T, Hq, Hkv, ctx, out, status, st, dyn_cells, kw, vw);
  return fail(KS_ERR_UNSUPPORTED, "attention: head_dim must be 64 or 128");
}

}  // namespace ks
