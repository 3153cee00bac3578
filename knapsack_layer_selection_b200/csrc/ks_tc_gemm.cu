// Tensor-core GEMM of the bf16 sublayer forward on sm_100a:
//   C[M][N] = A[M][K] . B[N][K]^T   (A = activations, B = a [out][in] weight)
// with the sublayer's elementwise work fused into the epilogue (RoPE on the
// query projection, SwiGLU on the gate/up projection, the fp32 residual add on
// the output/down projections).  These are the contractions the KnapSpec DP
// runs for every budget cell that executes an item (KnapSpec review page,
// "What carries the argument": Attention and MLP sublayers are the items).
//
// Design (one persistent CTA per SM, 192 threads, warp-specialised):
//   warp 0  -- TMA producer: 128x64 A tile and 256x64 B tile per stage, 128-byte
//              swizzle, 4-stage ring of 48 KB stages guarded by full/empty mbarriers;
//   warp 1  -- allocates 512 TMEM columns and one lane issues tcgen05.mma
//              (M=128, N=256, K=16) into one of two 256-column fp32 accumulators;
//   warps 2-5 -- epilogue: tcgen05.ld 32 columns at a time from their 32-lane
//              quarter, apply the fused epilogue, store to global memory.
// The accumulator double buffer lets the epilogue of tile i overlap the MMAs of
// tile i+1.  Tiles are walked in groups of m-tiles (m fastest inside a group):
// the CTAs running together share a few weight tiles through L2, and a group's
// activation rows stay resident while its weight columns stream.  No split-K: every output is the same fixed-order
// sum over K whatever M is, so a row's result does not depend on its batch.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "ks_sm100.cuh"
#include "ks_tc.cuh"

namespace ks {

using namespace sm100;

namespace {

constexpr int BM = 128, BN = 256, BK = 64;
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;         // 16 KB
constexpr int B_BYTES = BN * BK * 2;         // 32 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int TMEM_COLS = 512;               // two 256-column fp32 accumulators
constexpr int THREADS = 192;
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 /*align*/ + 256 /*barriers*/;
constexpr uint32_t IDESC = idesc_bf16_f32(BM, BN);

struct SharedTail {
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Stores 32 consecutive bf16 values (64 bytes) at p (16-byte aligned).
__device__ __forceinline__ void store_bf16x32(__nv_bfloat16* p, const float (&v)[32]) {
  uint4* q = reinterpret_cast<uint4*>(p);
#pragma unroll
  for (int j = 0; j < 4; ++j)
    q[j] = make_uint4(pack_bf16(v[8 * j + 0], v[8 * j + 1]), pack_bf16(v[8 * j + 2], v[8 * j + 3]),
                      pack_bf16(v[8 * j + 4], v[8 * j + 5]), pack_bf16(v[8 * j + 6], v[8 * j + 7]));
}

// One row group of a launch: its rows are m-tiles tile_m0 .. tile_m0 + ceil(M/BM) - 1
// of the walk.
struct GemmGroupDev {
  void* out;
  const float* resid;
  const float2* rope_cs;
  int M;
  int tile_m0;
};

struct GemmParams {
  int32_t* status;
  int N_out, K;
  int tiles_m, tiles_n;  // m-tiles of all row groups together
  int group_m;          // tile walk: groups of group_m m-tiles, m fastest inside a group
  int group_n;          // > 0: bands of group_n n-tiles instead, n fastest inside a band
  int T, head_dim;
  const int* dyn_cells; // optional device count (one row group only): M = min(M, *dyn_cells * T)
  RowMaxArgs rowmax;    // EPI_ROWMAX only
  int n_groups;
  GemmGroupDev grp[kGemmMaxGroups];
};

// Tile t of the walk -> (m-tile of all row groups, n-tile).  Tiles go in groups
// of group_m m-tiles; inside a group the m index runs fastest, so the CTAs in
// flight share a few weight tiles and the group's A rows stay in L2 while its
// weight columns stream.
__device__ __forceinline__ void tile_coords(const GemmParams& p, int t, int& tm, int& tn) {
  if (p.group_n > 0) {
    // a band of group_n weight tiles stays in L2 while every row tile passes it
    // once; the CTAs in flight read the same activation tile at about the same time
    const int per_band = p.group_n * p.tiles_m;
    const int g = t / per_band;
    const int local = t - g * per_band;
    const int n_base = g * p.group_n;
    const int cols = min(p.group_n, p.tiles_n - n_base);
    tn = n_base + local % cols;
    tm = local / cols;
    return;
  }
  const int per_group = p.group_m * p.tiles_n;
  const int g = t / per_group;
  const int local = t - g * per_group;
  const int m_base = g * p.group_m;
  const int rows = min(p.group_m, p.tiles_m - m_base);
  tm = m_base + local % rows;
  tn = local / rows;
}

// m-tile of the walk -> (row group, m-tile inside it).
__device__ __forceinline__ int tile_group(const GemmParams& p, int tm, int& local_tm) {
  int g = 0, m0 = 0;
#pragma unroll
  for (int i = 1; i < kGemmMaxGroups; ++i)
    if (i < p.n_groups && tm >= p.grp[i].tile_m0) {
      g = i;
      m0 = p.grp[i].tile_m0;
    }
  local_tm = tm - m0;
  return g;
}

// The fused epilogue of one accumulator row: this thread's TMEM lane holds row
// `row` of the tile, 256 columns from tbase, for output columns tn * 256 (tn * 128
// for SwiGLU).  Stores nothing for a row past M (but still reads TMEM, a
// warp-collective operation).
template <int EPI>
__device__ __forceinline__ void epilogue_row(const GemmParams& p, void* g_out, const float* g_resid,
                                             const float2* g_rope, int row, bool live, int tn,
                                             uint32_t tbase) {
  float v[32], u[32];
  if (EPI == EPI_RESID_F32 || EPI == EPI_STORE_F32 || EPI == EPI_STORE_BF16) {
    const int n0 = tn * BN;
#pragma unroll 1
    for (int c = 0; c < BN / 32; ++c) {
      tmem_ld32(tbase + c * 32, v);
      tmem_wait_ld();
      if (!live) continue;
      const long long off = (long long)row * p.N_out + n0 + c * 32;
      if (EPI == EPI_STORE_BF16) {
        store_bf16x32((__nv_bfloat16*)g_out + off, v);
      } else {
        float4* o = reinterpret_cast<float4*>((float*)g_out + off);
        if (EPI == EPI_RESID_F32) {
          const float4* rr = reinterpret_cast<const float4*>(g_resid + off);
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const float4 x = rr[j];
            o[j] = make_float4(v[4 * j] + x.x, v[4 * j + 1] + x.y, v[4 * j + 2] + x.z,
                               v[4 * j + 3] + x.w);
          }
        } else {
#pragma unroll
          for (int j = 0; j < 8; ++j)
            o[j] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
        }
      }
    }
  } else if (EPI == EPI_ROWMAX) {
    // top-2 of scale * acc + bias over this tile's 256 columns of the row
    const int n0 = tn * BN;
    float v1 = -INFINITY, v2 = -INFINITY;
    int i1 = -1;
#pragma unroll 1
    for (int c = 0; c < BN / 32; ++c) {
      tmem_ld32(tbase + c * 32, v);
      tmem_wait_ld();
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const int col = n0 + c * 32 + j;
        const float x = p.rowmax.scale * v[j] + (p.rowmax.col_bias ? p.rowmax.col_bias[col] : 0.f);
        if (x > v1) {
          v2 = v1;
          v1 = x;
          i1 = col;
        } else if (x > v2) {
          v2 = x;
        }
      }
    }
    if (live)
      reinterpret_cast<float4*>(g_out)[(long long)row * p.tiles_n + tn] =
          make_float4(v1, __int_as_float(i1), v2, 0.f);
  } else if (EPI == EPI_SWIGLU_BF16) {
    // columns 0..127: gate, 128..255: up, for output columns tn*128 ..
    const int n0 = tn * (BN / 2);
#pragma unroll 1
    for (int c = 0; c < BN / 64; ++c) {
      tmem_ld32(tbase + c * 32, v);
      tmem_ld32(tbase + BN / 2 + c * 32, u);
      tmem_wait_ld();
      if (!live) continue;
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] = v[j] / (1.0f + __expf(-v[j])) * u[j];
      store_bf16x32((__nv_bfloat16*)g_out + (long long)row * p.N_out + n0 + c * 32, v);
    }
  } else if (EPI == EPI_ROPE_BF16) {
    // rotate-half RoPE inside each head of this tile: column j pairs with j + hd/2
    const int half = p.head_dim / 2;
    const int tok = row % p.T;
    const float2* cs = g_rope + (long long)tok * half;
    const int n0 = tn * BN;
#pragma unroll 1
    for (int h0 = 0; h0 < BN; h0 += p.head_dim) {
#pragma unroll 1
      for (int c = 0; c < half; c += 32) {
        tmem_ld32(tbase + h0 + c, v);
        tmem_ld32(tbase + h0 + half + c, u);
        tmem_wait_ld();
        if (!live) continue;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const float2 r = cs[c + j];
          const float x1 = v[j], x2 = u[j];
          v[j] = x1 * r.x - x2 * r.y;
          u[j] = x2 * r.x + x1 * r.y;
        }
        __nv_bfloat16* o = (__nv_bfloat16*)g_out + (long long)row * p.N_out + n0 + h0 + c;
        store_bf16x32(o, v);
        store_bf16x32(o + half, u);
      }
    }
  }
}

template <int EPI>
__global__ void __launch_bounds__(THREADS, 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmA1,
                   const __grid_constant__ CUtensorMap tmA2, const __grid_constant__ CUtensorMap tmA3,
                   const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmB2, const GemmParams p_in) {
  // rows can be decided on the device (a compacted batch): the walk uses the live
  // count.  Group fields are read from the parameter space (dynamically indexed);
  // only group 0's row count can change, and it is kept in m_live0.
  GemmParams p = p_in;
  int m_live0 = p_in.grp[0].M;
  if (p.dyn_cells) {
    const long long live = (long long)(*p.dyn_cells) * p.T;
    m_live0 = (int)(live < m_live0 ? live : m_live0);
    p.tiles_m = (m_live0 + BM - 1) / BM;
    if (p.group_m > p.tiles_m) p.group_m = p.tiles_m > 0 ? p.tiles_m : 1;
  }
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = (unsigned char*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  SharedTail* tail = reinterpret_cast<SharedTail*>(smem + STAGES * STAGE_BYTES);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_tiles = p.tiles_m * p.tiles_n;
  const int KB = p.K / BK;
  volatile int* abort = &tail->abort;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(smem_u32(&tail->full[s]), 1);
      mbar_init(smem_u32(&tail->empty[s]), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(smem_u32(&tail->tfull[a]), 1);
      mbar_init(smem_u32(&tail->tempty[a]), 128);
    }
    mbar_init(smem_u32(&tail->drain), 1);
    tail->abort = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA);
    if (p.n_groups > 1) prefetch_tmap(&tmA1);
    if (p.n_groups > 2) prefetch_tmap(&tmA2);
    if (p.n_groups > 3) prefetch_tmap(&tmA3);
    prefetch_tmap(&tmB);
    if (EPI == EPI_SWIGLU_BF16) prefetch_tmap(&tmB2);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&tail->tmem_base), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = tail->tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int it = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x) {
        int tmg, tn, tm;
        tile_coords(p, t, tmg, tn);
        const int grp = tile_group(p, tmg, tm);
        const CUtensorMap* am = grp == 0 ? &tmA : grp == 1 ? &tmA1 : grp == 2 ? &tmA2 : &tmA3;
        const int m0 = tm * BM;
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t r = (uint32_t)(it / STAGES);
          if (!mbar_wait(smem_u32(&tail->empty[s]), (r & 1u) ^ 1u, abort, p.status)) {
            ok = false;
            break;
          }
          const uint32_t full = smem_u32(&tail->full[s]);
          const uint32_t a_dst = smem_u32(smem + s * STAGE_BYTES);
          const uint32_t b_dst = a_dst + A_BYTES;
          mbar_arrive_expect_tx(full, STAGE_BYTES);
          tma_load_2d(a_dst, am, kb * BK, m0, full);
          if (EPI == EPI_SWIGLU_BF16) {
            tma_load_2d(b_dst, &tmB, kb * BK, tn * (BN / 2), full);
            tma_load_2d(b_dst + B_BYTES / 2, &tmB2, kb * BK, tn * (BN / 2), full);
          } else {
            tma_load_2d(b_dst, &tmB, kb * BK, tn * BN, full);
          }
        }
      }
      // never leave while a copy this thread issued may still be landing
      for (int j = (it > STAGES ? it - STAGES : 0); j < it; ++j)
        mbar_wait_drain(smem_u32(&tail->full[j % STAGES]), (uint32_t)(j / STAGES) & 1u, p.status);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int it = 0, i = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x, ++i) {
        const int acc = i & 1;
        const uint32_t ar = (uint32_t)(i >> 1);
        if (!mbar_wait(smem_u32(&tail->tempty[acc]), (ar & 1u) ^ 1u, abort, p.status)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t r = (uint32_t)(it / STAGES);
          if (!mbar_wait(smem_u32(&tail->full[s]), r & 1u, abort, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + s * STAGE_BYTES);
          const uint64_t a_desc = desc_kmajor_sw128(a_addr);
          const uint64_t b_desc = desc_kmajor_sw128(a_addr + A_BYTES);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k)   // advance 16 elements = 32 bytes = 2 units
            mma_bf16(d_tmem, a_desc + 2 * k, b_desc + 2 * k, IDESC, (kb | k) != 0);
          mma_commit(smem_u32(&tail->empty[s]));
        }
        if (!ok) break;
        mma_commit(smem_u32(&tail->tfull[acc]));
      }
      // wait until every MMA issued above has retired before TMEM is released
      mma_commit(smem_u32(&tail->drain));
      mbar_wait_drain(smem_u32(&tail->drain), 0, p.status);
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 2-5)
    const int q = warp & 3;                       // TMEM lane quarter this warp may read
    int i = 0;
    for (int t = blockIdx.x; t < n_tiles; t += gridDim.x, ++i) {
      const int acc = i & 1;
      const uint32_t ar = (uint32_t)(i >> 1);
      // the whole warp leaves together: tcgen05.ld below is warp-collective
      const bool got = mbar_wait(smem_u32(&tail->tfull[acc]), ar & 1u, abort, p.status);
      if (!__all_sync(0xffffffffu, got)) break;
      tc_fence_after();
      int tmg, tn, tm;
      tile_coords(p, t, tmg, tn);
      const int gi = tile_group(p, tmg, tm);
      const GemmGroupDev& gr = p_in.grp[gi];
      void* const g_out = gr.out;
      const float* const g_resid = gr.resid;
      const float2* const g_rope = gr.rope_cs;
      const int m0 = tm * BM;
      const int row = m0 + q * 32 + lane;
      const bool live = row < (gi == 0 ? m_live0 : gr.M);
      const uint32_t tbase = tmem_base + (uint32_t)(acc * BN) + ((uint32_t)(q * 32) << 16);
      epilogue_row<EPI>(p, g_out, g_resid, g_rope, row, live, tn, tbase);
      tc_fence_before();
      mbar_arrive(smem_u32(&tail->tempty[acc]));
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// ---------------------------------------------------------------- the CTA-pair GEMM
// The same product and epilogues on 256 x 256 tiles computed by a pair of CTAs
// on two SMs (a 2-CTA cluster) with the pair MMA (tcgen05.mma.cta_group::2, M =
// 256): each CTA loads its own 128 rows of A and its half of the tile's 256
// weight rows, so per SM a k-step moves 32 KB instead of 48 KB for the same
// tensor work, and six stages fit where four did -- half again as much time to
// hide each stage's load behind the MMAs.  The leader CTA (rank 0) arms each
// stage's barrier for both CTAs' bytes and issues the MMAs; its commits arrive
// on both CTAs' barriers; both CTAs' epilogues read their own 128 TMEM rows and
// release the accumulator on the leader's barrier.  Every wait is bounded, and
// a cluster barrier at the end keeps either CTA from leaving while the other may
// still touch its shared memory.  A tile's arithmetic is the same fixed-order
// sum over K as in tc_gemm_kernel.
// ---------------------------------------------------------------- transposing epilogue
// One epilogue warp's 32 rows (rows row0 .. row0 + 31, one per lane, as TMEM holds
// them) x 32 consecutive output columns from col0: the lanes write their rows into
// a padded 32 x 33 staging block in shared memory, then read it back across rows, so
// each global load and store covers whole row segments (fp32: 8 lanes x 16 B = one
// row's 128 bytes, four rows an instruction; bf16: 4 lanes x 16 B, eight rows) instead
// of 16 bytes of 32 different rows.  Row stride 33 keeps both directions free of bank
// conflicts.  Rows at or past m_live are neither read nor written.
constexpr int kStageStride = 33;
constexpr int kStageFloats = 32 * kStageStride;

template <bool RESID, bool F32>
__device__ __forceinline__ void flush_chunk(float* stage, const float (&v)[32], int lane, int row0,
                                            int m_live, int n_out, int col0, void* g_out,
                                            const float* g_resid) {
#pragma unroll
  for (int j = 0; j < 32; ++j) stage[lane * kStageStride + j] = v[j];
  __syncwarp();
  if (F32) {
    const int c4 = (lane & 7) * 4;
    float4 r[8];
    if (RESID) {
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int row = row0 + 4 * k + (lane >> 3);
        if (row < m_live)
          r[k] = *reinterpret_cast<const float4*>(g_resid + (long long)row * n_out + col0 + c4);
      }
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int rr = 4 * k + (lane >> 3);
      const int row = row0 + rr;
      if (row >= m_live) continue;
      const float* sv = stage + rr * kStageStride + c4;
      float4 x = make_float4(sv[0], sv[1], sv[2], sv[3]);
      if (RESID) {
        x.x += r[k].x;
        x.y += r[k].y;
        x.z += r[k].z;
        x.w += r[k].w;
      }
      *reinterpret_cast<float4*>((float*)g_out + (long long)row * n_out + col0 + c4) = x;
    }
  } else {
    const int c8 = (lane & 3) * 8;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int rr = 8 * k + (lane >> 2);
      const int row = row0 + rr;
      if (row >= m_live) continue;
      const float* sv = stage + rr * kStageStride + c8;
      *reinterpret_cast<uint4*>((__nv_bfloat16*)g_out + (long long)row * n_out + col0 + c8) =
          make_uint4(pack_bf16(sv[0], sv[1]), pack_bf16(sv[2], sv[3]), pack_bf16(sv[4], sv[5]),
                     pack_bf16(sv[6], sv[7]));
    }
  }
  __syncwarp();                 // the block is read before the next chunk overwrites it
}

// The fused epilogue of one epilogue warp's 32 accumulator rows (this lane's TMEM lane
// holds row row0 + lane, 256 columns from tbase) for output columns tn * 256 (tn * 128
// for SwiGLU), through flush_chunk.  Same arithmetic as epilogue_row, which the
// SwiGLU (and row-max) epilogues still use.
template <int EPI>
__device__ __forceinline__ void epilogue_rows(const GemmParams& p, void* g_out, const float* g_resid,
                                              const float2* g_rope, int row0, int m_live, int tn,
                                              uint32_t tbase, float* stage) {
  const int lane = threadIdx.x & 31;
  float v[32], u[32];
  if (EPI == EPI_RESID_F32 || EPI == EPI_STORE_F32 || EPI == EPI_STORE_BF16) {
    const int n0 = tn * BN;
#pragma unroll 1
    for (int c = 0; c < BN / 32; ++c) {
      tmem_ld32(tbase + c * 32, v);
      tmem_wait_ld();
      flush_chunk<EPI == EPI_RESID_F32, EPI != EPI_STORE_BF16>(stage, v, lane, row0, m_live,
                                                               p.N_out, n0 + c * 32, g_out, g_resid);
    }
  } else if (EPI == EPI_SWIGLU_BF16 || EPI == EPI_ROWMAX) {
    // SwiGLU writes half as many bf16 columns as it reads and was measured faster
    // row by row (the staging costs more than its stores gain)
    epilogue_row<EPI>(p, g_out, g_resid, g_rope, row0 + lane, row0 + lane < m_live, tn, tbase);
  } else if (EPI == EPI_ROPE_BF16) {
    // rotate-half RoPE inside each head of this tile: column j pairs with j + hd/2
    const int half = p.head_dim / 2;
    const int tok = (row0 + lane) % p.T;
    const float4* cs = reinterpret_cast<const float4*>(g_rope + (long long)tok * half);
    const int n0 = tn * BN;
#pragma unroll 1
    for (int h0 = 0; h0 < BN; h0 += p.head_dim) {
#pragma unroll 1
      for (int c = 0; c < half; c += 32) {
        tmem_ld32(tbase + h0 + c, v);
        tmem_ld32(tbase + h0 + half + c, u);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 32; j += 2) {
          const float4 r = cs[(c + j) >> 1];   // (cos, sin) of columns c + j and c + j + 1
          const float x1 = v[j], x2 = u[j], y1 = v[j + 1], y2 = u[j + 1];
          v[j] = x1 * r.x - x2 * r.y;
          u[j] = x2 * r.x + x1 * r.y;
          v[j + 1] = y1 * r.z - y2 * r.w;
          u[j + 1] = y2 * r.z + y1 * r.w;
        }
        flush_chunk<false, false>(stage, v, lane, row0, m_live, p.N_out, n0 + h0 + c, g_out,
                                  nullptr);
        flush_chunk<false, false>(stage, u, lane, row0, m_live, p.N_out, n0 + h0 + half + c, g_out,
                                  nullptr);
      }
    }
  }
}

constexpr int BM2 = 256;
constexpr int STAGES2 = 6;
constexpr int A2_BYTES = 128 * BK * 2;       // this CTA's 128 rows of A: 16 KB
constexpr int B2_BYTES = 128 * BK * 2;       // this CTA's half of the 256 weight rows: 16 KB
constexpr int STAGE2_BYTES = A2_BYTES + B2_BYTES;
// the ring, the barriers, then one transposing-epilogue staging block per epilogue warp
constexpr int STAGE_OFF2 = STAGES2 * STAGE2_BYTES + 256;
constexpr int SMEM2_BYTES = STAGE_OFF2 + 4 * kStageFloats * 4 + 1024 /*align*/;
constexpr uint32_t IDESC2 = idesc_bf16_f32(BM2, BN);

struct SharedTail2 {
  uint64_t full[STAGES2];   // leader: both CTAs' bytes of a stage have landed
  uint64_t empty[STAGES2];  // each CTA: the pair MMAs reading a stage are done
  uint64_t tfull[2];        // each CTA: an accumulator is complete
  uint64_t tempty[2];       // leader: both CTAs' epilogues have read an accumulator
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(SharedTail2) <= 256, "barrier block");

template <int EPI>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(THREADS, 1)
    tc_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA,
                        const __grid_constant__ CUtensorMap tmA1,
                        const __grid_constant__ CUtensorMap tmA2,
                        const __grid_constant__ CUtensorMap tmA3,
                        const __grid_constant__ CUtensorMap tmB,
                        const __grid_constant__ CUtensorMap tmB2, const GemmParams p_in) {
  GemmParams p = p_in;
  int m_live0 = p_in.grp[0].M;
  if (p.dyn_cells) {
    const long long live = (long long)(*p.dyn_cells) * p.T;
    m_live0 = (int)(live < m_live0 ? live : m_live0);
    p.tiles_m = (m_live0 + BM2 - 1) / BM2;
    if (p.group_m > p.tiles_m) p.group_m = p.tiles_m > 0 ? p.tiles_m : 1;
  }
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = (unsigned char*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  SharedTail2* tail = reinterpret_cast<SharedTail2*>(smem + STAGES2 * STAGE2_BYTES);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = (int)(blockIdx.x >> 1), n_pairs = (int)(gridDim.x >> 1);
  const int n_tiles = p.tiles_m * p.tiles_n;
  const int KB = p.K / BK;
  volatile int* abort = &tail->abort;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES2; ++s) {
      mbar_init(smem_u32(&tail->full[s]), 1);
      mbar_init(smem_u32(&tail->empty[s]), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(smem_u32(&tail->tfull[a]), 1);
      mbar_init(smem_u32(&tail->tempty[a]), 2 * 128);   // every epilogue thread of both CTAs
    }
    mbar_init(smem_u32(&tail->drain), 1);
    tail->abort = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA);
    if (p.n_groups > 1) prefetch_tmap(&tmA1);
    if (p.n_groups > 2) prefetch_tmap(&tmA2);
    if (p.n_groups > 3) prefetch_tmap(&tmA3);
    prefetch_tmap(&tmB);
    if (EPI == EPI_SWIGLU_BF16) prefetch_tmap(&tmB2);
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(&tail->tmem_base), TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  cluster_sync_all();           // the peer's barriers exist before any remote arrival
  const uint32_t tmem_base = tail->tmem_base;
  const uint32_t full_leader = cluster_addr(smem_u32(&tail->full[0]), 0);
  const uint32_t tempty_leader = cluster_addr(smem_u32(&tail->tempty[0]), 0);

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (both CTAs)
    if (lane == 0) {
      int it = 0;
      bool ok = true;
      for (int t = pair; t < n_tiles && ok; t += n_pairs) {
        int tmg, tn, tm;
        tile_coords(p, t, tmg, tn);
        const int grp = tile_group(p, tmg, tm);
        const CUtensorMap* am = grp == 0 ? &tmA : grp == 1 ? &tmA1 : grp == 2 ? &tmA2 : &tmA3;
        const int m0 = tm * BM2 + (int)rank * 128;
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = it % STAGES2;
          const uint32_t r = (uint32_t)(it / STAGES2);
          if (!mbar_wait(smem_u32(&tail->empty[s]), (r & 1u) ^ 1u, abort, p.status)) {
            ok = false;
            break;
          }
          const uint32_t fb = full_leader + 8u * (uint32_t)s;
          if (leader) mbar_arrive_expect_tx(smem_u32(&tail->full[s]), 2 * STAGE2_BYTES);
          const uint32_t a_dst = smem_u32(smem + s * STAGE2_BYTES);
          const uint32_t b_dst = a_dst + A2_BYTES;
          tma_load_2d_pair(a_dst, am, kb * BK, m0, fb);
          if (EPI == EPI_SWIGLU_BF16)   // gate rows in the leader, up rows in the peer
            tma_load_2d_pair(b_dst, leader ? &tmB : &tmB2, kb * BK, tn * (BN / 2), fb);
          else
            tma_load_2d_pair(b_dst, &tmB, kb * BK, tn * BN + (int)rank * 128, fb);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ pair MMA issuer (leader)
    if (lane == 0 && leader) {
      int it = 0, i = 0;
      bool ok = true;
      for (int t = pair; t < n_tiles && ok; t += n_pairs, ++i) {
        const int acc = i & 1;
        const uint32_t ar = (uint32_t)(i >> 1);
        if (!mbar_wait(smem_u32(&tail->tempty[acc]), (ar & 1u) ^ 1u, abort, p.status)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = it % STAGES2;
          const uint32_t r = (uint32_t)(it / STAGES2);
          if (!mbar_wait(smem_u32(&tail->full[s]), r & 1u, abort, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + s * STAGE2_BYTES);
          const uint64_t a_desc = desc_kmajor_sw128(a_addr);
          const uint64_t b_desc = desc_kmajor_sw128(a_addr + A2_BYTES);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k)
            mma_bf16_pair(d_tmem, a_desc + 2 * k, b_desc + 2 * k, IDESC2, (kb | k) != 0);
          mma_commit_pair_both(smem_u32(&tail->empty[s]));
        }
        if (!ok) break;
        mma_commit_pair_both(smem_u32(&tail->tfull[acc]));
      }
      // every pair MMA issued above retires before TMEM is released
      mma_commit_pair_self(smem_u32(&tail->drain));
      mbar_wait_drain(smem_u32(&tail->drain), 0, p.status);
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 2-5, both CTAs)
    const int q = warp & 3;
    float* stage = reinterpret_cast<float*>(smem + STAGE_OFF2) + q * kStageFloats;
    int i = 0;
    for (int t = pair; t < n_tiles; t += n_pairs, ++i) {
      const int acc = i & 1;
      const uint32_t ar = (uint32_t)(i >> 1);
      const bool got = mbar_wait(smem_u32(&tail->tfull[acc]), ar & 1u, abort, p.status);
      if (!__all_sync(0xffffffffu, got)) break;
      tc_fence_after();
      int tmg, tn, tm;
      tile_coords(p, t, tmg, tn);
      const int gi = tile_group(p, tmg, tm);
      const GemmGroupDev& gr = p_in.grp[gi];
      const int row0 = tm * BM2 + (int)rank * 128 + q * 32;
      const uint32_t tbase = tmem_base + (uint32_t)(acc * BN) + ((uint32_t)(q * 32) << 16);
      epilogue_rows<EPI>(p, gr.out, gr.resid, gr.rope_cs, row0, gi == 0 ? m_live0 : gr.M, tn,
                         tbase, stage);
      tc_fence_before();
      mbar_arrive_cluster(tempty_leader + 8u * (uint32_t)acc);
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync_all();           // neither CTA leaves while its peer may still reach it
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, TMEM_COLS);
  }
}

// ---------------------------------------------------------------- host side
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (PFN_cuTensorMapEncodeTiled_v12000)f;
  });
  return fn;
}

template <int EPI>
ks_status launch(const CUtensorMap* a, const CUtensorMap& b, const CUtensorMap& b2,
                 const GemmParams& gp, cudaStream_t st) {
  static std::atomic<unsigned long long> attr_set{0};
  auto k = tc_gemm_kernel<EPI>;
  KS_TRY(once_per_device(attr_set, [&]() -> ks_status {
    KS_CUDA_TRY(cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES));
    return KS_OK;
  }));
  const int n_tiles = gp.tiles_m * gp.tiles_n;
  const int grid = n_tiles < sm_count() ? n_tiles : sm_count();
  k<<<grid, THREADS, SMEM_BYTES, st>>>(a[0], a[1], a[2], a[3], b, b2, gp);
  KS_LAUNCH_CHECK();
  return KS_OK;
}

// Pairs of CTAs that can be resident at once (a persistent grid of that many pairs).
template <int EPI>
ks_status launch_pair(const CUtensorMap* a, const CUtensorMap& b, const CUtensorMap& b2,
                      const GemmParams& gp, cudaStream_t st) {
  static std::atomic<unsigned long long> attr_set{0};
  static int max_pairs = 0;
  auto k = tc_gemm_pair_kernel<EPI>;
  KS_TRY(once_per_device(attr_set, [&]() -> ks_status {
    KS_CUDA_TRY(cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM2_BYTES));
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * sm_count());
    cfg.blockDim = dim3(THREADS);
    cfg.dynamicSmemBytes = SMEM2_BYTES;
    cudaLaunchAttribute at;
    at.id = cudaLaunchAttributeClusterDimension;
    at.val.clusterDim.x = 2;
    at.val.clusterDim.y = 1;
    at.val.clusterDim.z = 1;
    cfg.attrs = &at;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, k, &cfg) != cudaSuccess || n < 1) n = sm_count() / 2;
    max_pairs = n;
    return KS_OK;
  }));
  const int n_tiles = gp.tiles_m * gp.tiles_n;
  const int pairs = n_tiles < max_pairs ? n_tiles : max_pairs;
  k<<<2 * pairs, THREADS, SMEM2_BYTES, st>>>(a[0], a[1], a[2], a[3], b, b2, gp);
  KS_LAUNCH_CHECK();
  return KS_OK;
}

}  // namespace

// SMs of the current device (read once).
int sm_count() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

ks_status make_tmap_2d(CUtensorMap* m, const void* base, long long rows, long long cols,
                       long long row_stride, int box_cols, int box_rows) {
  auto fn = encode_fn();
  if (!fn) return fail(KS_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
  if ((uintptr_t)base % 16) return fail(KS_ERR_INVALID_ARG, "tensor base not 16-byte aligned");
  if ((row_stride * 2) % 16) return fail(KS_ERR_UNSUPPORTED, "tensor row stride not a multiple of 16 bytes");
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)row_stride * 2};
  cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return fail(KS_ERR_CUDA, "cuTensorMapEncodeTiled failed: " + std::to_string((int)r));
  return KS_OK;
}

bool use_tensor_cores(const ks_model_desc* m) { return m->wdtype == KS_BF16; }

ks_status tc_gemm(const void* A, const void* B, const void* B2, void* out, const float* resid,
                  int M, int N, int K, int epi, const float2* rope_cs, int T, int head_dim,
                  int32_t* status, cudaStream_t st, const int* dyn_cells, RowMaxArgs rowmax) {
  const GemmGroupArg g{A, out, resid, rope_cs, M};
  return tc_gemm_groups(&g, 1, B, B2, N, K, epi, T, head_dim, status, st, dyn_cells, rowmax);
}

ks_status tc_gemm_groups(const GemmGroupArg* groups, int n_groups, const void* B, const void* B2,
                         int N, int K, int epi, int T, int head_dim, int32_t* status,
                         cudaStream_t st, const int* dyn_cells, RowMaxArgs rowmax) {
  if (n_groups < 1 || n_groups > kGemmMaxGroups)
    return fail(KS_ERR_INVALID_ARG, "tensor-core GEMM: 1 to 4 row groups");
  if (dyn_cells && n_groups != 1)
    return fail(KS_ERR_INVALID_ARG, "tensor-core GEMM: a device row count needs one row group");
  if (K % BK) return fail(KS_ERR_UNSUPPORTED, "tensor-core GEMM: K must be a multiple of 64");
  const int bn_out = epi == EPI_SWIGLU_BF16 ? BN / 2 : BN;
  if (N % bn_out)
    return fail(KS_ERR_UNSUPPORTED, "tensor-core GEMM: N must be a multiple of " + std::to_string(bn_out));
  if (epi == EPI_SWIGLU_BF16 && !B2) return fail(KS_ERR_INVALID_ARG, "tensor-core GEMM: up weight is NULL");
  GemmParams gp{};
  CUtensorMap ta[kGemmMaxGroups], tb, tb2;
  int tiles_m = 0, n_live = 0;
  // CTA pairs for every product but the row-maximum scan; each CTA then loads
  // 128-row boxes of A and of the weights
  const bool pair = epi != EPI_ROWMAX;
  const int bm = pair ? BM2 : BM;
  for (int g = 0; g < n_groups; ++g) {
    const GemmGroupArg& a = groups[g];
    if (a.M <= 0) continue;                     // an empty group takes no tiles
    if (epi == EPI_ROPE_BF16 && (head_dim % 64 || BN % head_dim || !a.rope_cs || T < 1))
      return fail(KS_ERR_UNSUPPORTED, "tensor-core GEMM: RoPE epilogue needs head_dim 64 or 128");
    if (epi == EPI_RESID_F32 && !a.resid)
      return fail(KS_ERR_INVALID_ARG, "tensor-core GEMM: resid is NULL");
    KS_TRY(make_tmap_2d(&ta[n_live], a.A, a.M, K, K, BK, BM));
    gp.grp[n_live] = GemmGroupDev{a.out, a.resid, a.rope_cs, a.M, tiles_m};
    tiles_m += (a.M + bm - 1) / bm;
    ++n_live;
  }
  if (n_live == 0) return KS_OK;
  for (int g = n_live; g < kGemmMaxGroups; ++g) ta[g] = ta[0];
  if (epi == EPI_SWIGLU_BF16) {
    KS_TRY(make_tmap_2d(&tb, B, N, K, K, BK, BN / 2));
    KS_TRY(make_tmap_2d(&tb2, B2, N, K, K, BK, BN / 2));
  } else {
    KS_TRY(make_tmap_2d(&tb, B, N, K, K, BK, pair ? BN / 2 : BN));
    tb2 = tb;
  }
  gp.n_groups = n_live;
  gp.status = status;
  gp.N_out = N;
  gp.K = K;
  gp.tiles_m = tiles_m;
  gp.tiles_n = N / bn_out;
  // Tile walk: either groups of group_m row tiles whose A rows (group_m x 128 x K,
  // at most ~32 MB, well inside one die's half of L2) stay resident while the
  // weight columns stream past them -- B is then read once per group -- or bands
  // of group_n weight tiles (at most ~48 MB of B) that stay resident while every
  // row tile passes -- A is then read once per band.  The walk with the smaller
  // estimated DRAM traffic is taken (a long-K, narrow-N product like the MLP's
  // down projection reads its weights ~8 times under the first and A twice under
  // the second).  The walk changes only which CTA computes a tile and when, never
  // a tile's arithmetic.
  {
    const long long a_tile = (long long)bm * K * 2;
    const long long b_tile = (long long)BN * K * 2;
    long long g = (32ll << 20) / a_tile;
    if (g < 8) g = 8;
    if (g > 32) g = 32;
    gp.group_m = (int)(g < gp.tiles_m ? g : gp.tiles_m);
    long long h = (48ll << 20) / b_tile;
    if (h < 1) h = 1;
    if (h > gp.tiles_n) h = gp.tiles_n;
    const long long a_all = a_tile * gp.tiles_m, b_all = b_tile * gp.tiles_n;
    const long long by_m = a_all + b_all * ((gp.tiles_m + gp.group_m - 1) / gp.group_m);
    const long long by_n = b_all + a_all * ((gp.tiles_n + h - 1) / h);
    gp.group_n = (epi != EPI_ROWMAX && !dyn_cells && by_n < by_m) ? (int)h : 0;
  }
  gp.T = T;
  gp.head_dim = head_dim;
  gp.dyn_cells = dyn_cells;
  gp.rowmax = rowmax;
  switch (epi) {
    case EPI_RESID_F32: return launch_pair<EPI_RESID_F32>(ta, tb, tb2, gp, st);
    case EPI_ROPE_BF16: return launch_pair<EPI_ROPE_BF16>(ta, tb, tb2, gp, st);
    case EPI_SWIGLU_BF16: return launch_pair<EPI_SWIGLU_BF16>(ta, tb, tb2, gp, st);
    case EPI_STORE_BF16: return launch_pair<EPI_STORE_BF16>(ta, tb, tb2, gp, st);
    case EPI_STORE_F32: return launch_pair<EPI_STORE_F32>(ta, tb, tb2, gp, st);
    case EPI_ROWMAX: return launch<EPI_ROWMAX>(ta, tb, tb2, gp, st);
  }
  return fail(KS_ERR_INVALID_ARG, "tensor-core GEMM: unknown epilogue");
}

}  // namespace ks
