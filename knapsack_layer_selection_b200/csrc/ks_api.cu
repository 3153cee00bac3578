// C ABI of the KnapSpec DP library and its host orchestrator.
//
// ks_solve runs KnapSpec's DP (KnapSpec review page: Eq. 6-8 / Algorithm 1 in
// referee major 1, Algorithm 2 in referee minor 4, TPT Eq. 4/5 in "What carries
// the argument") as one stream of kernel launches: the reference states, then
// for every item a batched sublayer forward over all budget cells that can
// afford it followed by the select step, then reconstruction and the TPT search.
// The host never waits on the device inside a solve.
#include <math.h>
#include <stdio.h>

#include <algorithm>
#include <mutex>
#include <string>
#include <vector>

#include "ks_kernels.cuh"
#include "ks_prof.cuh"
#include "ks_tc.cuh"

namespace ks {

static thread_local std::string g_last_error;

void set_error(const std::string& msg) { g_last_error = msg; }

ks_status fail(ks_status s, const std::string& msg) {
  set_error(msg);
  return s;
}

// ---------------------------------------------------------------- validation
static ks_status check_model(const ks_model_desc* m) {
  if (!m) return fail(KS_ERR_INVALID_ARG, "model is NULL");
  if (m->n_layers < 1 || 2 * m->n_layers > ItemTable::kMaxItems)
    return fail(KS_ERR_INVALID_ARG, "n_layers must be in 1..128");
  if (m->d_model < 64 || m->d_model % 64)
    return fail(KS_ERR_INVALID_ARG, "d_model must be a positive multiple of 64");
  if (m->head_dim != 64 && m->head_dim != 128)
    return fail(KS_ERR_UNSUPPORTED, "head_dim must be 64 or 128");
  if (m->n_kv_heads < 1 || m->n_q_heads < 1 || m->n_q_heads % m->n_kv_heads)
    return fail(KS_ERR_INVALID_ARG, "n_q_heads must be a positive multiple of n_kv_heads");
  if (m->ffn < 16 || m->ffn % 16) return fail(KS_ERR_INVALID_ARG, "ffn must be a positive multiple of 16");
  if (m->wdtype != KS_F32 && m->wdtype != KS_BF16) return fail(KS_ERR_INVALID_ARG, "wdtype");
  if (!(m->rms_eps >= 0.f)) return fail(KS_ERR_INVALID_ARG, "rms_eps must be >= 0");
  if (!(m->rope_base > 0.0)) return fail(KS_ERR_INVALID_ARG, "rope_base must be > 0");
  if (m->wdtype == KS_BF16) {
    // the tensor-core GEMM's output tiles: 256 columns (Q, O, down), 128 (gate/up)
    if (m->d_model % 256 || (m->n_q_heads * m->head_dim) % 256)
      return fail(KS_ERR_UNSUPPORTED,
                  "bf16 weights: d_model and n_q_heads * head_dim must be multiples of 256");
    if (m->ffn % 128) return fail(KS_ERR_UNSUPPORTED, "bf16 weights: ffn must be a multiple of 128");
  }
  return KS_OK;
}

static ks_status check_T(int T) {
  if (T < 1 || T > 256) return fail(KS_ERR_INVALID_ARG, "T must be in 1..256");
  return KS_OK;
}

static ks_status check_cache(const ks_model_desc* m, const ks_cache_desc* c, int T) {
  if (!c || !c->k_cache || !c->v_cache) return fail(KS_ERR_INVALID_ARG, "cache is NULL");
  KS_TRY(check_aligned16({c->k_cache, c->v_cache}, "cache"));
  if (c->ctx < 0) return fail(KS_ERR_INVALID_ARG, "ctx must be >= 0");
  if (c->kv_mode != KS_KV_CACHE && c->kv_mode != KS_KV_WINDOW)
    return fail(KS_ERR_INVALID_ARG, "cache kv_mode must be KS_KV_CACHE or KS_KV_WINDOW");
  if (c->kv_mode == KS_KV_WINDOW && m->wdtype == KS_BF16 && 128 % T)
    return fail(KS_ERR_UNSUPPORTED,
                "KS_KV_WINDOW with bf16 weights needs T to divide 128 (whole states per row tile)");
  if (c->cache_rows < (int64_t)c->ctx + T)
    return fail(KS_ERR_INVALID_ARG, "cache_rows must be >= ctx + T");
  // fp32 weights run the SIMT attention, which keeps a row's scores in shared memory
  if (m->wdtype == KS_F32 && (int64_t)m->head_dim + c->ctx + T > 51200)
    return fail(KS_ERR_UNSUPPORTED, "fp32 weights: ctx + T + head_dim must be at most 51200");
  return KS_OK;
}

static ks_status check_layers(const ks_model_desc* m, const ks_layer_weights* layers,
                              const ks_cache_desc* c) {
  if (!layers) return fail(KS_ERR_INVALID_ARG, "layers is NULL");
  const bool window = c && c->kv_mode == KS_KV_WINDOW;
  for (int l = 0; l < m->n_layers; ++l) {
    const ks_layer_weights& L = layers[l];
    if (!L.attn_norm || !L.wq || !L.wo || !L.mlp_norm || !L.w_gate || !L.w_up || !L.w_down)
      return fail(KS_ERR_INVALID_ARG, "layer " + std::to_string(l) + " has a NULL weight");
    KS_TRY(check_aligned16({L.attn_norm, L.wq, L.wo, L.mlp_norm, L.w_gate, L.w_up, L.w_down},
                           "layer weights"));
    if (window) {
      if (!L.wk || !L.wv)
        return fail(KS_ERR_INVALID_ARG,
                    "layer " + std::to_string(l) + ": KS_KV_WINDOW needs wk and wv");
      KS_TRY(check_aligned16({L.wk, L.wv}, "layer weights"));
    }
  }
  return KS_OK;
}

// ---------------------------------------------------------------- workspace
struct Workspace {
  int32_t* status;            // [1] device status word of the last call (first in the buffer)
  float *prev, *cur, *exec;   // [C+1][T][d] fp32 states: slot 0 = reference, slot b+1 = cell b
  void *xh;                   // [C+1][T][d] act: the current item's normalised operand
  void *q, *att;              // [(C+1)T][qd] act
  void *gb, *ub;              // [(C+1)T][ffn] act
  void *kw, *vw;              // [(C+1)T][Hkv*hd] act: window keys / values (KS_KV_WINDOW)
  uint8_t* bp;                // [n_items][C]
  uint8_t *valid_a, *valid_b; // [C] exact-budget validity, ping-pong
  uint64_t *hash_a, *hash_b;  // [C+1] state fingerprints (distinct-state execution), ping-pong
  int *map, *uniq, *count;    // [C+1], [C+1], [1] compaction of the execute batch
  float* prev_c;              // [C+1][T][d] fp32 distinct source states
  void* xh_c;                 // [C+1][T][d] act: their normalised operands
  float* val;                 // [C]
  double* t_draft;            // [C]
  float2* rope;               // [T][hd/2]
  size_t total;
};

static size_t align_up(size_t x) { return (x + 255) & ~size_t(255); }

// Lays the workspace out for batches of up to n_slots states of T tokens.
static Workspace carve(const ks_model_desc* m, long long n_slots, long long T, char* base) {
  Workspace w{};
  const int act = m->wdtype == KS_F32 ? ACT_F32 : ACT_BF16;
  const size_t ab = act_bytes(act);
  const long long R = n_slots * T;
  const long long d = m->d_model, qd = (long long)m->n_q_heads * m->head_dim, F = m->ffn;
  const long long n_items = 2LL * m->n_layers;
  const long long C = n_slots;
  size_t off = 0;
  auto take = [&](size_t bytes) -> char* {
    char* p = base ? base + off : nullptr;
    off += align_up(bytes);
    return p;
  };
  w.status = (int32_t*)take(256);
  w.prev = (float*)take(R * d * 4);
  w.cur = (float*)take(R * d * 4);
  w.exec = (float*)take(R * d * 4);
  w.xh = take(R * d * ab);
  w.q = take(R * qd * ab);
  w.att = take(R * qd * ab);
  w.gb = take(R * F * ab);
  w.ub = take(R * F * ab);
  const long long kvd = (long long)m->n_kv_heads * m->head_dim;
  w.kw = take(R * kvd * ab);
  w.vw = take(R * kvd * ab);
  w.bp = (uint8_t*)take(n_items * C);
  w.valid_a = (uint8_t*)take(C);
  w.valid_b = (uint8_t*)take(C);
  w.hash_a = (uint64_t*)take((C + 1) * 8);
  w.hash_b = (uint64_t*)take((C + 1) * 8);
  w.map = (int*)take((C + 1) * 4);
  w.uniq = (int*)take((C + 1) * 4);
  w.count = (int*)take(4);
  w.prev_c = (float*)take(R * d * 4);
  w.xh_c = take(R * d * ab);
  w.val = (float*)take(C * 4);
  w.t_draft = (double*)take(C * 8);
  w.rope = (float2*)take(T * (m->head_dim / 2) * sizeof(float2));
  w.total = off;
  return w;
}

// ---------------------------------------------------------------- sublayer forward
struct Ctx {
  const ks_model_desc* m;
  const ks_layer_weights* layers;
  const ks_cache_desc* cache;
  int T;
  int act;
  Workspace ws;
  int32_t* status;   // device word a timed-out wait reports into (may be NULL)
  cudaStream_t st;
};

// Applies item k to E states in[0..E) -> out[0..E) (fp32 [E][T][d]).
// The RoPE table in ws.rope must hold positions ctx .. ctx+T-1.  With
// xh_ready, ws.xh already holds the item's normalised operand of `in`.
static ks_status sublayer(const Ctx& c, int k, const float* in, int E, float* out,
                          bool xh_ready = false, const void* xh_src = nullptr,
                          const int* dyn_cells = nullptr) {
  const ks_model_desc* m = c.m;
  const int l = k / 2;
  const ks_layer_weights& L = c.layers[l];
  const int R = E * c.T;
  const int d = m->d_model, qd = m->n_q_heads * m->head_dim, F = m->ffn;
  if (E <= 0) return KS_OK;
  const bool tc = use_tensor_cores(m);
  const double ab = (double)act_bytes(c.act);
  const double wb = m->wdtype == KS_F32 ? 4.0 : 2.0;
  const double Rd = (double)R;
  const void* xh = xh_src ? xh_src : c.ws.xh;   // the item's normalised operand
  if (!xh_ready) {
    ProfScope ps(KK_RMSNORM, c.st, 3.0 * Rd * d, Rd * d * (4.0 + ab));
    KS_TRY(launch_rmsnorm(in, k % 2 == 0 ? L.attn_norm : L.mlp_norm, m->wdtype, c.ws.xh, c.act, R,
                          d, m->rms_eps, c.st));
  }
  if (k % 2 == 0) {
    // Attention sublayer: x^ = RMSNorm(H); q = RoPE(x^ Wq^T); o = Attn(q); out = H + o Wo^T
    const size_t elem = m->wdtype == KS_F32 ? 4 : 2;
    const size_t layer_off = (size_t)l * c.cache->cache_rows * m->n_kv_heads * m->head_dim * elem;
    const char* kc = (const char*)c.cache->k_cache + layer_off;
    const char* vc = (const char*)c.cache->v_cache + layer_off;
    {
      ProfScope ps(KK_GEMM_Q, c.st, 2.0 * Rd * qd * d, (Rd * d + (double)qd * d) * ab + Rd * qd * ab,
                   tc ? 1 : 2);
      if (tc) {
        KS_TRY(tc_gemm(xh, L.wq, nullptr, c.ws.q, nullptr, R, qd, d, EPI_ROPE_BF16, c.ws.rope,
                       c.T, m->head_dim, c.status, c.st, dyn_cells));
      } else {
        KS_TRY(launch_gemm_simt(xh, c.act, L.wq, m->wdtype, c.ws.q, false, nullptr, R, qd, d,
                                c.st));
        KS_TRY(launch_rope_inplace(c.ws.q, c.act, c.ws.rope, R, m->n_q_heads, m->head_dim, c.T,
                                   c.st));
      }
    }
    const bool window = c.cache->kv_mode == KS_KV_WINDOW;
    const void* kw = nullptr;
    const void* vw = nullptr;
    if (window) {
      // the window positions' keys and values from the candidates' own normalised
      // state: k = RoPE(x^ Wk^T) at position ctx + t (the query's rotation), v = x^ Wv^T
      const int kvd = m->n_kv_heads * m->head_dim;
      ProfScope ps(KK_GEMM_KV, c.st, 2.0 * 2.0 * Rd * kvd * d,
                   (Rd * d + 2.0 * kvd * d) * ab + 2.0 * Rd * kvd * ab, tc ? 2 : 3);
      if (tc) {
        KS_TRY(tc_gemm(xh, L.wk, nullptr, c.ws.kw, nullptr, R, kvd, d, EPI_ROPE_BF16, c.ws.rope,
                       c.T, m->head_dim, c.status, c.st, dyn_cells));
        KS_TRY(tc_gemm(xh, L.wv, nullptr, c.ws.vw, nullptr, R, kvd, d, EPI_STORE_BF16, nullptr,
                       c.T, m->head_dim, c.status, c.st, dyn_cells));
      } else {
        KS_TRY(launch_gemm_simt(xh, c.act, L.wk, m->wdtype, c.ws.kw, false, nullptr, R, kvd, d,
                                c.st));
        KS_TRY(launch_rope_inplace(c.ws.kw, c.act, c.ws.rope, R, m->n_kv_heads, m->head_dim, c.T,
                                   c.st));
        KS_TRY(launch_gemm_simt(xh, c.act, L.wv, m->wdtype, c.ws.vw, false, nullptr, R, kvd, d,
                                c.st));
      }
      kw = c.ws.kw;
      vw = c.ws.vw;
    }
    {
      const double T = c.T, ctx = c.cache->ctx;
      const double keys = (double)E * (T * ctx + T * (T + 1) / 2);   // sum over rows of visible keys
      // cache keys/values read: ctx + T rows, or ctx rows plus the window tensors
      const double kv_bytes = window ? 2.0 * ctx * m->n_kv_heads * m->head_dim * wb +
                                           2.0 * Rd * m->n_kv_heads * m->head_dim * ab
                                     : 2.0 * (ctx + T) * m->n_kv_heads * m->head_dim * wb;
      ProfScope ps(KK_ATTN, c.st, 4.0 * m->n_q_heads * m->head_dim * keys,
                   2.0 * Rd * qd * ab + kv_bytes);
      if (tc) {
        KS_TRY(tc_attention(c.ws.q, kc, vc, c.cache->cache_rows, R, c.T, m->n_q_heads,
                            m->n_kv_heads, m->head_dim, c.cache->ctx, c.ws.att, c.status, c.st,
                            dyn_cells, kw, vw));
      } else {
        KS_TRY(launch_attention_simt(c.ws.q, c.act, kc, vc, m->wdtype, R, c.T, m->n_q_heads,
                                     m->n_kv_heads, m->head_dim, c.cache->ctx, c.ws.att, c.st,
                                     kw, vw));
      }
    }
    {
      ProfScope ps(KK_GEMM_O, c.st, 2.0 * Rd * d * qd,
                   (Rd * qd + (double)d * qd) * ab + Rd * d * 8.0);
      if (tc) {
        KS_TRY(tc_gemm(c.ws.att, L.wo, nullptr, out, in, R, d, qd, EPI_RESID_F32, nullptr, c.T,
                       m->head_dim, c.status, c.st, dyn_cells));
      } else {
        KS_TRY(launch_gemm_simt(c.ws.att, c.act, L.wo, m->wdtype, out, true, in, R, d, qd, c.st));
      }
    }
  } else {
    // MLP sublayer: x^ = RMSNorm(H); u = silu(x^ Wg^T) * (x^ Wu^T); out = H + u Wd^T
    {
      ProfScope ps(KK_GEMM_GATEUP, c.st, 2.0 * Rd * 2.0 * F * d,
                   (Rd * d + 2.0 * F * d) * ab + Rd * F * ab, tc ? 1 : 3);
      if (tc) {
        KS_TRY(tc_gemm(xh, L.w_gate, L.w_up, c.ws.gb, nullptr, R, F, d, EPI_SWIGLU_BF16,
                       nullptr, c.T, m->head_dim, c.status, c.st, dyn_cells));
      } else {
        KS_TRY(launch_gemm_simt(xh, c.act, L.w_gate, m->wdtype, c.ws.gb, false, nullptr, R, F,
                                d, c.st));
        KS_TRY(launch_gemm_simt(xh, c.act, L.w_up, m->wdtype, c.ws.ub, false, nullptr, R, F,
                                d, c.st));
        KS_TRY(launch_swiglu_inplace(c.ws.gb, c.ws.ub, c.act, (long long)R * F, c.st));
      }
    }
    {
      ProfScope ps(KK_GEMM_DOWN, c.st, 2.0 * Rd * d * F, (Rd * F + (double)d * F) * ab + Rd * d * 8.0);
      if (tc) {
        KS_TRY(tc_gemm(c.ws.gb, L.w_down, nullptr, out, in, R, d, F, EPI_RESID_F32, nullptr, c.T,
                       m->head_dim, c.status, c.st, dyn_cells));
      } else {
        KS_TRY(launch_gemm_simt(c.ws.gb, c.act, L.w_down, m->wdtype, out, true, in, R, d, F, c.st));
      }
    }
  }
  return KS_OK;
}

static ks_status reference_chain(const Ctx& c, const float* x0, float* ref) {
  const long long cell = (long long)c.T * c.m->d_model;
  if (ref != x0)
    KS_CUDA_TRY(cudaMemcpyAsync(ref, x0, cell * sizeof(float), cudaMemcpyDeviceToDevice, c.st));
  for (int k = 0; k < 2 * c.m->n_layers; ++k)
    KS_TRY(sublayer(c, k, ref + k * cell, 1, ref + (k + 1) * cell));
  return KS_OK;
}

// Item k on several contexts' batches at once (bf16 weights, tensor cores):
// group g applies the item to E[g] states in[g] -> out[g] of context cs[g], with
// the normalised operand already in that context's workspace (xh).  Every GEMM
// runs once over all groups' rows, so the item's weights are read once for all
// contexts; the attention runs once per context (each has its own context
// length and cache).  A group's rows get exactly the arithmetic of a one-group
// call: the same kernels, the same fixed-order sums.
static ks_status sublayer_multi(const Ctx* const* cs, int n, int k, const float* const* in,
                                const int* E, float* const* out) {
  const Ctx& c0 = *cs[0];
  const ks_model_desc* m = c0.m;
  const int l = k / 2;
  const ks_layer_weights& L = c0.layers[l];
  const int d = m->d_model, qd = m->n_q_heads * m->head_dim, F = m->ffn;
  const int kvd = m->n_kv_heads * m->head_dim;
  const double ab = (double)act_bytes(c0.act);
  double Rd = 0.0;
  for (int g = 0; g < n; ++g) Rd += (double)E[g] * c0.T;
  if (Rd <= 0.0) return KS_OK;
  GemmGroupArg grp[kGemmMaxGroups];
  auto groups = [&](auto&& fill) {
    for (int g = 0; g < n; ++g) grp[g] = fill(g, *cs[g], E[g] * cs[g]->T);
  };
  if (k % 2 == 0) {
    {
      ProfScope ps(KK_GEMM_Q, c0.st, 2.0 * Rd * qd * d, (Rd * d + (double)qd * d) * ab + Rd * qd * ab);
      groups([&](int g, const Ctx& c, int R) {
        return GemmGroupArg{c.ws.xh, c.ws.q, nullptr, c.ws.rope, R};
      });
      KS_TRY(tc_gemm_groups(grp, n, L.wq, nullptr, qd, d, EPI_ROPE_BF16, c0.T, m->head_dim,
                            c0.status, c0.st));
    }
    const bool window = c0.cache->kv_mode == KS_KV_WINDOW;
    if (window) {
      ProfScope ps(KK_GEMM_KV, c0.st, 2.0 * 2.0 * Rd * kvd * d,
                   (Rd * d + 2.0 * kvd * d) * ab + 2.0 * Rd * kvd * ab, 2);
      groups([&](int g, const Ctx& c, int R) {
        return GemmGroupArg{c.ws.xh, c.ws.kw, nullptr, c.ws.rope, R};
      });
      KS_TRY(tc_gemm_groups(grp, n, L.wk, nullptr, kvd, d, EPI_ROPE_BF16, c0.T, m->head_dim,
                            c0.status, c0.st));
      groups([&](int g, const Ctx& c, int R) {
        return GemmGroupArg{c.ws.xh, c.ws.vw, nullptr, nullptr, R};
      });
      KS_TRY(tc_gemm_groups(grp, n, L.wv, nullptr, kvd, d, EPI_STORE_BF16, c0.T, m->head_dim,
                            c0.status, c0.st));
    }
    for (int g = 0; g < n; ++g) {
      const Ctx& c = *cs[g];
      if (E[g] <= 0) continue;
      const double T = c.T, ctx = c.cache->ctx, R = (double)E[g] * c.T;
      const double keys = (double)E[g] * (T * ctx + T * (T + 1) / 2);
      const double kv_bytes = window ? 2.0 * ctx * kvd * 2.0 + 2.0 * R * kvd * ab
                                     : 2.0 * (ctx + T) * kvd * 2.0;
      ProfScope ps(KK_ATTN, c.st, 4.0 * m->n_q_heads * m->head_dim * keys, 2.0 * R * qd * ab + kv_bytes);
      const size_t layer_off = (size_t)l * c.cache->cache_rows * kvd * 2;
      KS_TRY(tc_attention(c.ws.q, (const char*)c.cache->k_cache + layer_off,
                          (const char*)c.cache->v_cache + layer_off, c.cache->cache_rows,
                          E[g] * c.T, c.T, m->n_q_heads, m->n_kv_heads, m->head_dim, c.cache->ctx,
                          c.ws.att, c.status, c.st, nullptr, window ? c.ws.kw : nullptr,
                          window ? c.ws.vw : nullptr));
    }
    {
      ProfScope ps(KK_GEMM_O, c0.st, 2.0 * Rd * d * qd, (Rd * qd + (double)d * qd) * ab + Rd * d * 8.0);
      groups([&](int g, const Ctx& c, int R) {
        return GemmGroupArg{c.ws.att, out[g], in[g], nullptr, R};
      });
      KS_TRY(tc_gemm_groups(grp, n, L.wo, nullptr, d, qd, EPI_RESID_F32, c0.T, m->head_dim,
                            c0.status, c0.st));
    }
  } else {
    {
      ProfScope ps(KK_GEMM_GATEUP, c0.st, 2.0 * Rd * 2.0 * F * d,
                   (Rd * d + 2.0 * F * d) * ab + Rd * F * ab);
      groups([&](int g, const Ctx& c, int R) {
        return GemmGroupArg{c.ws.xh, c.ws.gb, nullptr, nullptr, R};
      });
      KS_TRY(tc_gemm_groups(grp, n, L.w_gate, L.w_up, F, d, EPI_SWIGLU_BF16, c0.T, m->head_dim,
                            c0.status, c0.st));
    }
    {
      ProfScope ps(KK_GEMM_DOWN, c0.st, 2.0 * Rd * d * F, (Rd * F + (double)d * F) * ab + Rd * d * 8.0);
      groups([&](int g, const Ctx& c, int R) {
        return GemmGroupArg{c.ws.gb, out[g], in[g], nullptr, R};
      });
      KS_TRY(tc_gemm_groups(grp, n, L.w_down, nullptr, d, F, EPI_RESID_F32, c0.T, m->head_dim,
                            c0.status, c0.st));
    }
  }
  return KS_OK;
}

// ---------------------------------------------------------------- allocation-free variant
// Scratch for ks_reference_forward_noalloc: a fixed device array that every GPU
// loading this library holds until the process exits.  Host code must not use
// the symbol itself as a pointer (that is a host-side stand-in); it asks the
// runtime for the device address once per device.
constexpr size_t kStaticScratchBytes = size_t(8) << 20;
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];
constexpr int kMaxDevices = 64;

// Carves only the per-call operands of the sublayer forward (x^, q, o, gate,
// up, RoPE table) for R = T rows; returns the bytes needed.
static size_t carve_sublayer_only(const ks_model_desc* m, long long T, char* base, Workspace* w) {
  const int act = m->wdtype == KS_F32 ? ACT_F32 : ACT_BF16;
  const size_t ab = act_bytes(act);
  const long long d = m->d_model, qd = (long long)m->n_q_heads * m->head_dim, F = m->ffn;
  size_t off = 0;
  auto take = [&](size_t bytes) -> char* {
    char* p = base ? base + off : nullptr;
    off += align_up(bytes);
    return p;
  };
  *w = Workspace{};
  w->xh = take(T * d * ab);
  w->q = take(T * qd * ab);
  w->att = take(T * qd * ab);
  w->gb = take(T * F * ab);
  w->ub = take(T * F * ab);
  w->rope = (float2*)take(T * (m->head_dim / 2) * sizeof(float2));
  w->total = off;
  return off;
}

// Device address of g_static_scratch on the current device, looked up on the
// first call for that device (with the device current) and cached.
static ks_status static_scratch(char** out) {
  int dev = -1;
  KS_CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kMaxDevices) return fail(KS_ERR_UNSUPPORTED, "device index above 63");
  static std::mutex mu;
  static char* addr[kMaxDevices] = {};
  std::lock_guard<std::mutex> g(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess || !p)
      return fail(KS_ERR_CUDA, std::string("cudaGetSymbolAddress(static scratch): ") +
                                   cudaGetErrorString(e));
    addr[dev] = (char*)p;
  }
  *out = addr[dev];
  return KS_OK;
}

}  // namespace ks

using namespace ks;

// ==================================================================== C ABI
extern "C" {

const char* ks_version(void) { return "knapspec-b200 0.1 (sm_100a)"; }

const char* ks_last_error(void) { return g_last_error.c_str(); }

const char* ks_status_string(ks_status s) {
  switch (s) {
    case KS_OK: return "ok";
    case KS_ERR_INVALID_ARG: return "invalid argument";
    case KS_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case KS_ERR_WORKSPACE: return "workspace too small";
    case KS_ERR_CUDA: return "CUDA error";
    case KS_ERR_TIMEOUT: return "device wait timed out";
    case KS_ERR_INTERNAL: return "internal error";
  }
  return "unknown status";
}

ks_status ks_quantize_weights(const double* t, int32_t n_items, int32_t n_bins, int32_t* w_out) {
  if (!t || !w_out) return fail(KS_ERR_INVALID_ARG, "quantize: NULL pointer");
  if (n_items < 1 || n_bins < 1) return fail(KS_ERR_INVALID_ARG, "quantize: n_items, n_bins >= 1");
  double total = 0.0;
  for (int i = 0; i < n_items; ++i) {
    if (!(t[i] > 0.0)) return fail(KS_ERR_INVALID_ARG, "quantize: latencies must be positive");
    total += t[i];
  }
  const double delta = total / (double)n_bins;
  for (int i = 0; i < n_items; ++i) {
    const double q = floor(t[i] / delta + 0.5);
    w_out[i] = q < 1.0 ? 1 : (int32_t)q;
  }
  return KS_OK;
}

ks_status ks_workspace_size(const ks_model_desc* model, int32_t n_cells, int32_t T, size_t* bytes) {
  KS_TRY(check_model(model));
  KS_TRY(check_T(T));
  if (!bytes) return fail(KS_ERR_INVALID_ARG, "bytes is NULL");
  if (n_cells < 1) return fail(KS_ERR_INVALID_ARG, "n_cells must be >= 1");
  // a solve over n_cells cells keeps one more state slot (the reference)
  *bytes = carve(model, (long long)n_cells + 1, T, nullptr).total;
  return KS_OK;
}

static ks_status make_ctx(const ks_model_desc* model, const ks_layer_weights* layers,
                          const ks_cache_desc* cache, int T, long long n_cells, void* workspace,
                          size_t ws_bytes, cudaStream_t st, Ctx* c) {
  KS_TRY(check_model(model));
  KS_TRY(check_T(T));
  KS_TRY(check_cache(model, cache, T));
  KS_TRY(check_layers(model, layers, cache));
  if (!workspace) return fail(KS_ERR_INVALID_ARG, "workspace is NULL");
  if ((uintptr_t)workspace % 256) return fail(KS_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  const size_t need = carve(model, n_cells, T, nullptr).total;
  if (ws_bytes < need)
    return fail(KS_ERR_WORKSPACE, "workspace has " + std::to_string(ws_bytes) + " bytes, needs " +
                                      std::to_string(need));
  c->m = model;
  c->layers = layers;
  c->cache = cache;
  c->T = T;
  c->act = model->wdtype == KS_F32 ? ACT_F32 : ACT_BF16;
  c->ws = carve(model, n_cells, T, (char*)workspace);
  c->status = c->ws.status;
  c->st = st;
  return KS_OK;
}

ks_status ks_sublayer_forward(const ks_model_desc* model, const ks_layer_weights* layers,
                              const ks_cache_desc* cache, int32_t T, int32_t item,
                              const float* states_in, int32_t E, float* states_out,
                              void* workspace, size_t workspace_bytes, ks_stream_t stream) {
  Ctx c;
  KS_TRY(make_ctx(model, layers, cache, T, std::max(E, 1), workspace, workspace_bytes,
                  (cudaStream_t)stream, &c));
  if (item < 0 || item >= 2 * model->n_layers) return fail(KS_ERR_INVALID_ARG, "item out of range");
  if (E < 0) return fail(KS_ERR_INVALID_ARG, "E must be >= 0");
  if (E > 0 && (!states_in || !states_out)) return fail(KS_ERR_INVALID_ARG, "states are NULL");
  KS_TRY(check_aligned16({states_in, states_out}, "sublayer_forward"));
  KS_CUDA_TRY(cudaMemsetAsync(c.status, 0, sizeof(int32_t), c.st));
  KS_TRY(launch_rope_table(c.ws.rope, T, model->head_dim, cache->ctx, model->rope_base, c.st));
  return sublayer(c, item, states_in, E, states_out);
}

ks_status ks_reference_forward(const ks_model_desc* model, const ks_layer_weights* layers,
                               const ks_cache_desc* cache, int32_t T, const float* x0,
                               float* ref_out, void* workspace, size_t workspace_bytes,
                               ks_stream_t stream) {
  Ctx c;
  KS_TRY(make_ctx(model, layers, cache, T, 1, workspace, workspace_bytes, (cudaStream_t)stream, &c));
  if (!x0 || !ref_out) return fail(KS_ERR_INVALID_ARG, "x0 / ref_out is NULL");
  KS_TRY(check_aligned16({x0, ref_out}, "reference_forward"));
  KS_CUDA_TRY(cudaMemsetAsync(c.status, 0, sizeof(int32_t), c.st));
  KS_TRY(launch_rope_table(c.ws.rope, T, model->head_dim, cache->ctx, model->rope_base, c.st));
  return reference_chain(c, x0, ref_out);
}

ks_status ks_select_step(const float* prev, const float* exec, const float* target, int32_t C,
                         int32_t T, int32_t d, int32_t w, float* cur, float* val, uint8_t* bp,
                         float* cos_skip, float* cos_exec, ks_stream_t stream) {
  if (!prev || !target || !cur || !val || !bp) return fail(KS_ERR_INVALID_ARG, "select: NULL pointer");
  if (C < 1 || T < 1 || d < 4 || w < 1) return fail(KS_ERR_INVALID_ARG, "select: C, T >= 1, d >= 4, w >= 1");
  if (C > w && !exec) return fail(KS_ERR_INVALID_ARG, "select: exec is NULL");
  if (prev == cur) return fail(KS_ERR_INVALID_ARG, "select: prev and cur must differ");
  KS_TRY(check_aligned16({prev, exec, target, cur}, "select"));
  return launch_select(prev, exec, target, C, T, d, w, cur, val, bp, cos_skip, cos_exec,
                       (cudaStream_t)stream);
}

ks_status ks_reconstruct(const uint8_t* bp, const int32_t* w, const double* t, int32_t n_items,
                         int32_t C, uint64_t* sets, int32_t* used_w, double* t_draft,
                         int32_t* status, ks_stream_t stream) {
  if (!bp || !w || !t || !sets) return fail(KS_ERR_INVALID_ARG, "reconstruct: NULL pointer");
  if (n_items < 1 || n_items > ItemTable::kMaxItems || C < 1)
    return fail(KS_ERR_INVALID_ARG, "reconstruct: n_items in 1..256, C >= 1");
  return launch_reconstruct(bp, w, t, nullptr, n_items, C, sets, used_w, t_draft, status,
                            nullptr, (cudaStream_t)stream);
}

ks_status ks_tpt_argmax(const float* values, const double* t_draft, int32_t C, double t_target,
                        const ks_params* p, double* tpt, int32_t* best, double* best_tpt,
                        ks_stream_t stream) {
  if (!values || !t_draft || !p || !best) return fail(KS_ERR_INVALID_ARG, "tpt: NULL pointer");
  if (C < 1 || p->gamma_max < 1) return fail(KS_ERR_INVALID_ARG, "tpt: C >= 1, gamma_max >= 1");
  if (!(p->alpha_scale > 0.0)) return fail(KS_ERR_INVALID_ARG, "tpt: alpha_scale must be > 0");
  if (!(t_target > 0.0)) return fail(KS_ERR_INVALID_ARG, "tpt: t_target must be > 0");
  return launch_tpt(values, t_draft, C, t_target, p->gamma_max, p->alpha_lo, p->alpha_scale,
                    p->alpha_max, tpt, best, best_tpt, (cudaStream_t)stream);
}

static ks_status resolve_weights(int32_t n_items, const int32_t* w, const double* t,
                                 const ks_params* p, std::vector<int32_t>* out) {
  out->assign(n_items, 0);
  if (w) {
    for (int i = 0; i < n_items; ++i) {
      if (w[i] < 1) return fail(KS_ERR_INVALID_ARG, "item weights must be >= 1");
      (*out)[i] = w[i];
    }
    return KS_OK;
  }
  if (!p) return fail(KS_ERR_INVALID_ARG, "params is NULL");
  return ks_quantize_weights(t, n_items, p->n_bins, out->data());
}

ks_status ks_solve_cells(int32_t n_items, const int32_t* w, const double* t, const ks_params* p,
                         int32_t* n_cells) {
  if (!n_cells || n_items < 1) return fail(KS_ERR_INVALID_ARG, "solve_cells: bad argument");
  if (!w && !t) return fail(KS_ERR_INVALID_ARG, "solve_cells: need w or t");
  std::vector<int32_t> ww;
  KS_TRY(resolve_weights(n_items, w, t, p, &ww));
  long long K = 0;
  for (int x : ww) K += x;
  if (K + 1 > (1 << 20)) return fail(KS_ERR_UNSUPPORTED, "more than 2^20 budget cells");
  *n_cells = (int32_t)(K + 1);
  return KS_OK;
}

// ---------------------------------------------------------------- the DP over one or more contexts
// One context of a solve: its cache (context length), evaluation tokens, item
// weights and latencies, result buffers and its slice of the workspace.
struct SolveCtx {
  Ctx c;
  const float* x0 = nullptr;
  const float* ref = nullptr;
  ks_result* out = nullptr;
  std::vector<int32_t> w;
  ItemTable tab;
  int C = 0;
  double t_target = 0.0;
};

static ks_status check_params(const ks_params* params) {
  if (!params) return fail(KS_ERR_INVALID_ARG, "solve: params is NULL");
  if (params->gamma_max < 1 || !(params->alpha_scale > 0.0))
    return fail(KS_ERR_INVALID_ARG, "solve: gamma_max >= 1 and alpha_scale > 0");
  if (params->budget_mode != KS_BUDGET_AT_MOST && params->budget_mode != KS_BUDGET_EXACT)
    return fail(KS_ERR_INVALID_ARG, "solve: budget_mode must be KS_BUDGET_AT_MOST or KS_BUDGET_EXACT");
  if (params->prune_tau != params->prune_tau)
    return fail(KS_ERR_INVALID_ARG, "solve: prune_tau is NaN (use -INFINITY to turn it off)");
  if (params->dedup < 0 || params->dedup > 2)
    return fail(KS_ERR_INVALID_ARG, "solve: dedup must be 0 (off), 1 (on) or 2 (8-bit fingerprints)");
  return KS_OK;
}

// Host checks of one context's inputs and results; its item weights (given, or
// quantised from t) and grid size.
static ks_status prepare_context(const ks_model_desc* model, const int32_t* w, const double* t,
                                 const ks_params* params, const float* x0, const float* ref,
                                 ks_result* out, SolveCtx* s) {
  if (!t || !out || !x0) return fail(KS_ERR_INVALID_ARG, "solve: NULL argument");
  if (!out->status || !out->values || !out->sets || !out->best)
    return fail(KS_ERR_INVALID_ARG, "solve: result needs status, values, sets and best");
  KS_TRY(check_aligned16({x0, ref, out->ref_states, out->final_states}, "solve"));
  const int n_items = 2 * model->n_layers;
  KS_TRY(resolve_weights(n_items, w, t, params, &s->w));
  long long K = 0;
  double t_target = 0.0;
  for (int i = 0; i < n_items; ++i) {
    if (!(t[i] > 0.0)) return fail(KS_ERR_INVALID_ARG, "solve: latencies must be positive");
    s->tab.w[i] = s->w[i];
    s->tab.t[i] = t[i];
    K += s->w[i];
    t_target += t[i];
  }
  if (K + 1 > (1 << 20)) return fail(KS_ERR_UNSUPPORTED, "more than 2^20 budget cells");
  s->C = (int)(K + 1);
  s->t_target = t_target;
  s->x0 = x0;
  s->ref = ref;
  s->out = out;
  return KS_OK;
}

// The DP of n contexts that share the model's weights (one context: ks_solve).
// Slot 0 of every state buffer carries the context's full-model state X^(k)
// through the same batched kernels as its cells, so the select target X^(k+1)
// comes out of each item's batch (exec slot 0) and no separate reference chain
// runs.  Cells start from X^(0).  For every item, the contexts' batches go
// through one grouped sublayer (tensor cores) and then one select each.
static ks_status solve_run(const ks_model_desc* model, const ks_layer_weights* layers, int n,
                           SolveCtx* ss, const ks_params* params) {
  const int n_items = 2 * model->n_layers;
  const cudaStream_t st = ss[0].c.st;
  const int T = ss[0].c.T;
  const long long cell = (long long)T * model->d_model;
  const double xb = model->wdtype == KS_F32 ? 4.0 : 2.0;
  const bool dedup = params->dedup != 0;
  const bool exact = params->budget_mode == KS_BUDGET_EXACT;
  const bool pruning = params->prune_tau > -INFINITY || params->skip_cap >= 0;
  const bool track = exact || pruning;       // validity is carried only when it can change
  struct Run {
    float* prev;
    uint8_t *bp, *vprev, *vcur;
    uint64_t *hprev, *hcur;
    long long W_k;
  };
  std::vector<Run> run(n);
  for (int j = 0; j < n; ++j) {
    SolveCtx& s = ss[j];
    Ctx& c = s.c;
    ks_result* out = s.out;
    c.status = out->status;
    const int C = s.C;
    if (dedup && C + 1 > 3072)
      return fail(KS_ERR_UNSUPPORTED, "solve: distinct-state execution handles up to 3071 cells");
    KS_CUDA_TRY(cudaMemsetAsync(out->status, 0, sizeof(int32_t), st));
    if (c.cache->kv_mode == KS_KV_WINDOW && dedup) {
      // rows past a compacted batch's live count are read (and masked) by the
      // attention's window block: they must hold finite values from the start
      const size_t kvb = (size_t)(C + 1) * T * model->n_kv_heads * model->head_dim *
                         act_bytes(c.act);
      KS_CUDA_TRY(cudaMemsetAsync(c.ws.kw, 0, kvb, st));
      KS_CUDA_TRY(cudaMemsetAsync(c.ws.vw, 0, kvb, st));
    }
    {
      ProfScope ps(KK_ROPE_TABLE, st, 0.0, 0.0);
      KS_TRY(launch_rope_table(c.ws.rope, T, model->head_dim, c.cache->ctx, model->rope_base, st));
    }
    Run& r = run[j];
    r.hprev = dedup ? c.ws.hash_a : nullptr;
    r.hcur = dedup ? c.ws.hash_b : nullptr;
    {
      ProfScope ps(KK_BROADCAST, st, 0.0, (double)(C + 1) * cell * (4.0 + xb));
      KS_TRY(launch_init_states(s.x0, C + 1, T, model->d_model, model->rms_eps,
                                layers[0].attn_norm, model->wdtype, c.ws.prev, c.ws.xh,
                                out->ref_states, r.hprev, st));
    }
    // the cells' states are updated in place: a select writes slot b only when
    // its execute candidate wins (every select block reads only its own slot)
    r.prev = c.ws.prev;
    r.bp = out->bp ? out->bp : c.ws.bp;
    r.vprev = track ? c.ws.valid_a : nullptr;
    r.vcur = track ? c.ws.valid_b : nullptr;
    if (track) KS_TRY(launch_init_valid(r.vprev, C, exact, st));
    r.W_k = 0;
  }
  const bool tc = use_tensor_cores(model);
  std::vector<const Ctx*> cs(n);
  std::vector<const float*> ins(n);
  std::vector<float*> outs(n);
  std::vector<int> Es(n);
  for (int k = 0; k < n_items; ++k) {
    // the item's batched forward over every context's executing cells
    for (int j = 0; j < n; ++j) {
      SolveCtx& s = ss[j];
      Ctx& c = s.c;
      Run& r = run[j];
      const int E = s.C - s.w[k];
      cs[j] = &c;
      ins[j] = r.prev;
      outs[j] = c.ws.exec;
      Es[j] = E + 1;
      if (dedup) {
        // fold equal source states together, then run the item once per distinct state
        ks_result* out = s.out;
        {
          ProfScope ps(KK_DEDUP, st, 0.0, (E + 1.0) * 9.0);
          KS_TRY(launch_dedup(r.hprev, r.vprev, E + 1, c.ws.map, c.ws.uniq, c.ws.count,
                              out->exec_counts ? out->exec_counts + k : nullptr,
                              params->dedup == 2, st));
        }
        {
          ProfScope ps(KK_DEDUP_VERIFY, st, 0.0, 2.0 * (E + 1.0) * cell * 4.0);
          KS_TRY(launch_dedup_verify(r.prev, cell, E + 1, c.ws.map, c.ws.uniq, c.ws.count,
                                     out->exec_counts ? out->exec_counts + k : nullptr,
                                     out->dedup_rejected ? out->dedup_rejected + k : nullptr, st));
        }
        {
          ProfScope ps(KK_GATHER, st, 0.0, 2.0 * (E + 1.0) * cell * (4.0 + xb));
          KS_TRY(launch_gather(c.ws.uniq, c.ws.count, E + 1, cell, r.prev, c.ws.xh, c.act,
                               c.ws.prev_c, c.ws.xh_c, st));
        }
        KS_TRY(sublayer(c, k, c.ws.prev_c, E + 1, c.ws.exec, /*xh_ready=*/true, c.ws.xh_c,
                        c.ws.count));
      } else if (s.out->exec_counts) {
        KS_TRY(launch_fill_i32(s.out->exec_counts + k, E + 1, st));
      }
    }
    if (!dedup) {
      if (tc) {
        KS_TRY(sublayer_multi(cs.data(), n, k, ins.data(), Es.data(), outs.data()));
      } else {
        for (int j = 0; j < n; ++j)
          KS_TRY(sublayer(*cs[j], k, ins[j], Es[j], outs[j], /*xh_ready=*/true));
      }
    }
    // each context's select
    const void* g_next = nullptr;
    if (k + 1 < n_items) g_next = (k + 1) % 2 == 0 ? layers[(k + 1) / 2].attn_norm
                                                    : layers[(k + 1) / 2].mlp_norm;
    for (int j = 0; j < n; ++j) {
      SolveCtx& s = ss[j];
      Ctx& c = s.c;
      Run& r = run[j];
      ks_result* out = s.out;
      const int C = s.C, wk = s.w[k];
      r.W_k += wk;
      const int min_valid_b =
          params->skip_cap >= 0 ? (int)std::max(0LL, r.W_k - (long long)params->skip_cap) : 0;
      float* val = (k == n_items - 1) ? out->values : c.ws.val;
      const float* target = s.ref ? s.ref + (long long)(k + 1) * cell : nullptr;
      ProfScope ps(KK_SELECT, st, 10.0 * (2.0 * C - wk) * cell,
                   (3.0 * C - wk + 2.0) * cell * 4.0 + (g_next ? (C + 1.0) * cell * xb : 0.0));
      KS_TRY(launch_select_fused(
          r.prev, c.ws.exec, target, C, T, model->d_model, wk, model->rms_eps, g_next,
          model->wdtype, r.prev, c.ws.xh, val, r.bp + (long long)k * C,
          out->cos_skip ? out->cos_skip + (long long)k * C : nullptr,
          out->cos_exec ? out->cos_exec + (long long)k * C : nullptr,
          out->ref_states ? out->ref_states + (long long)(k + 1) * cell : nullptr, r.vprev,
          r.vcur, params->prune_tau, min_valid_b, dedup ? c.ws.map : nullptr, r.hcur, st));
      std::swap(r.vprev, r.vcur);
      std::swap(r.hprev, r.hcur);
    }
  }
  for (int j = 0; j < n; ++j) {
    SolveCtx& s = ss[j];
    Ctx& c = s.c;
    Run& r = run[j];
    ks_result* out = s.out;
    const int C = s.C;
    if (out->final_states)
      KS_CUDA_TRY(cudaMemcpyAsync(out->final_states, r.prev + cell,
                                  (size_t)C * cell * sizeof(float), cudaMemcpyDeviceToDevice, st));
    double* tdp = out->t_draft ? out->t_draft : c.ws.t_draft;
    {
      ProfScope ps(KK_RECONSTRUCT, st, 0.0, (double)n_items * C);
      KS_TRY(launch_reconstruct(r.bp, nullptr, nullptr, &s.tab, n_items, C, out->sets,
                                out->used_w, tdp, out->status, r.vprev, st));
    }
    ProfScope ps(KK_TPT, st, 0.0, (double)C * 12.0);
    KS_TRY(launch_tpt(out->values, tdp, C, s.t_target, params->gamma_max, params->alpha_lo,
                      params->alpha_scale, params->alpha_max, out->tpt, out->best, out->best_tpt,
                      st));
  }
  return KS_OK;
}

ks_status ks_solve(const ks_model_desc* model, const ks_layer_weights* layers,
                   const ks_cache_desc* cache, int32_t T, const float* x0, const float* ref,
                   const int32_t* w, const double* t, const ks_params* params, void* workspace,
                   size_t workspace_bytes, ks_result* out, ks_stream_t stream) {
  KS_TRY(check_model(model));
  KS_TRY(check_params(params));
  SolveCtx s;
  KS_TRY(prepare_context(model, w, t, params, x0, ref, out, &s));
  KS_TRY(make_ctx(model, layers, cache, T, s.C + 1, workspace, workspace_bytes,
                  (cudaStream_t)stream, &s.c));
  return solve_run(model, layers, 1, &s, params);
}

ks_status ks_workspace_size_contexts(const ks_model_desc* model, int32_t n_ctx,
                                     const int32_t* n_cells, int32_t T, size_t* bytes) {
  KS_TRY(check_model(model));
  KS_TRY(check_T(T));
  if (!bytes || !n_cells) return fail(KS_ERR_INVALID_ARG, "workspace_size_contexts: NULL pointer");
  if (n_ctx < 1 || n_ctx > kGemmMaxGroups)
    return fail(KS_ERR_INVALID_ARG, "workspace_size_contexts: n_ctx must be in 1..4");
  size_t total = 0;
  for (int j = 0; j < n_ctx; ++j) {
    if (n_cells[j] < 1) return fail(KS_ERR_INVALID_ARG, "n_cells must be >= 1");
    total += align_up(carve(model, (long long)n_cells[j] + 1, T, nullptr).total);
  }
  *bytes = total;
  return KS_OK;
}

ks_status ks_solve_contexts(const ks_model_desc* model, const ks_layer_weights* layers,
                            int32_t n_ctx, const ks_cache_desc* caches, int32_t T,
                            const float* const* x0, const int32_t* const* w,
                            const double* const* t, const ks_params* params, void* workspace,
                            size_t workspace_bytes, ks_result* outs, ks_stream_t stream) {
  KS_TRY(check_model(model));
  KS_TRY(check_params(params));
  if (n_ctx < 1 || n_ctx > kGemmMaxGroups)
    return fail(KS_ERR_INVALID_ARG, "solve_contexts: n_ctx must be in 1..4");
  if (!caches || !x0 || !t || !outs) return fail(KS_ERR_INVALID_ARG, "solve_contexts: NULL argument");
  if (params->dedup && n_ctx > 1)
    return fail(KS_ERR_UNSUPPORTED, "solve_contexts: distinct-state execution runs one context at a time");
  if (!workspace) return fail(KS_ERR_INVALID_ARG, "workspace is NULL");
  std::vector<SolveCtx> ss(n_ctx);
  size_t off = 0;
  for (int j = 0; j < n_ctx; ++j) {
    if (caches[j].kv_mode != caches[0].kv_mode)
      return fail(KS_ERR_INVALID_ARG, "solve_contexts: every context needs the same kv_mode");
    KS_TRY(prepare_context(model, w ? w[j] : nullptr, t[j], params, x0[j], nullptr, &outs[j],
                           &ss[j]));
    const size_t need = align_up(carve(model, (long long)ss[j].C + 1, T, nullptr).total);
    if (off + need > workspace_bytes)
      return fail(KS_ERR_WORKSPACE, "workspace too small for the contexts (see ks_workspace_size_contexts)");
    KS_TRY(make_ctx(model, layers, &caches[j], T, ss[j].C + 1, (char*)workspace + off, need,
                    (cudaStream_t)stream, &ss[j].c));
    off += need;
  }
  return solve_run(model, layers, n_ctx, ss.data(), params);
}

ks_status ks_eval_set(const ks_model_desc* model, const ks_layer_weights* layers,
                      const ks_cache_desc* cache, int32_t T, const float* x0, const float* target,
                      const uint64_t* set, float* value_out, float* state_out, void* workspace,
                      size_t workspace_bytes, ks_stream_t stream) {
  Ctx c;
  KS_TRY(make_ctx(model, layers, cache, T, 1, workspace, workspace_bytes, (cudaStream_t)stream, &c));
  if (!x0 || !target || !set || !value_out) return fail(KS_ERR_INVALID_ARG, "eval_set: NULL argument");
  KS_TRY(check_aligned16({x0, target}, "eval_set"));
  const int n_items = 2 * model->n_layers;
  const int words = (n_items + 63) / 64;
  if (n_items % 64 && (set[words - 1] >> (n_items % 64)) != 0)
    return fail(KS_ERR_INVALID_ARG, "eval_set: the set has bits at or above n_items");
  const long long cell = (long long)T * model->d_model;
  KS_CUDA_TRY(cudaMemsetAsync(c.status, 0, sizeof(int32_t), c.st));
  KS_TRY(launch_rope_table(c.ws.rope, T, model->head_dim, cache->ctx, model->rope_base, c.st));
  // the set's items in increasing order on x0, each exactly as ks_sublayer_forward runs it
  float* a = c.ws.prev;
  float* b = c.ws.cur;
  KS_CUDA_TRY(cudaMemcpyAsync(a, x0, cell * sizeof(float), cudaMemcpyDeviceToDevice, c.st));
  for (int k = 0; k < n_items; ++k) {
    if (!((set[k >> 6] >> (k & 63)) & 1)) continue;
    KS_TRY(sublayer(c, k, a, 1, b));
    std::swap(a, b);
  }
  // value: the select step's skip score of one cell (C = 1 < w, so no execute
  // candidate is read); the copy of the kept state goes to scratch
  KS_TRY(launch_select(a, a, target, 1, T, model->d_model, 1, c.ws.exec, value_out, c.ws.bp,
                       nullptr, nullptr, c.st));
  if (state_out)
    KS_CUDA_TRY(cudaMemcpyAsync(state_out, a, cell * sizeof(float), cudaMemcpyDeviceToDevice, c.st));
  return KS_OK;
}

ks_status ks_reference_forward_noalloc(const ks_model_desc* model,
                                       const ks_layer_weights* layers,
                                       const ks_cache_desc* cache, int32_t T, const float* x0,
                                       float* ref_out, ks_stream_t stream) {
  KS_TRY(check_model(model));
  KS_TRY(check_T(T));
  KS_TRY(check_cache(model, cache, T));
  KS_TRY(check_layers(model, layers, cache));
  if (!x0 || !ref_out) return fail(KS_ERR_INVALID_ARG, "x0 / ref_out is NULL");
  KS_TRY(check_aligned16({x0, ref_out}, "reference_forward_noalloc"));
  if (cache->kv_mode != KS_KV_CACHE)
    return fail(KS_ERR_UNSUPPORTED,
                "reference_forward_noalloc: only KS_KV_CACHE (use ks_reference_forward)");
  Workspace w;
  const size_t need = carve_sublayer_only(model, T, nullptr, &w);
  if (need > kStaticScratchBytes)
    return fail(KS_ERR_UNSUPPORTED,
                "reference_forward_noalloc: this model and T need " + std::to_string(need) +
                    " bytes of scratch, above the fixed " + std::to_string(kStaticScratchBytes) +
                    "; use ks_reference_forward with a workspace");
  char* base = nullptr;
  KS_TRY(static_scratch(&base));
  Ctx c;
  c.m = model;
  c.layers = layers;
  c.cache = cache;
  c.T = T;
  c.act = model->wdtype == KS_F32 ? ACT_F32 : ACT_BF16;
  carve_sublayer_only(model, T, base, &c.ws);
  c.status = nullptr;
  c.st = (cudaStream_t)stream;
  KS_TRY(launch_rope_table(c.ws.rope, T, model->head_dim, cache->ctx, model->rope_base, c.st));
  return reference_chain(c, x0, ref_out);
}

ks_status ks_gemm_bf16(const void* A, const void* B, float* C, const float* resid, int32_t M,
                       int32_t N, int32_t K, int32_t* status, ks_stream_t stream) {
  if (!A || !B || !C) return fail(KS_ERR_INVALID_ARG, "gemm: NULL pointer");
  if (M < 0 || N < 1 || K < 1) return fail(KS_ERR_INVALID_ARG, "gemm: bad size");
  KS_TRY(check_aligned16({A, B, C, resid}, "gemm"));
  return tc_gemm(A, B, nullptr, C, resid, M, N, K, resid ? EPI_RESID_F32 : EPI_STORE_F32, nullptr,
                 1, 64, status, (cudaStream_t)stream);
}

ks_status ks_workspace_status(const void* workspace, int32_t* host_status, ks_stream_t stream) {
  if (!workspace || !host_status) return fail(KS_ERR_INVALID_ARG, "workspace_status: NULL pointer");
  KS_CUDA_TRY(cudaMemcpyAsync(host_status, workspace, sizeof(int32_t), cudaMemcpyDeviceToHost,
                              (cudaStream_t)stream));
  KS_CUDA_TRY(cudaStreamSynchronize((cudaStream_t)stream));
  return KS_OK;
}

ks_status ks_attention_bf16(const void* q, const void* k_layer, const void* v_layer,
                            int64_t cache_rows, int32_t R, int32_t T, int32_t Hq, int32_t Hkv,
                            int32_t head_dim, int32_t ctx, void* out, int32_t* status,
                            ks_stream_t stream) {
  if (!q || !k_layer || !v_layer || !out) return fail(KS_ERR_INVALID_ARG, "attention: NULL pointer");
  if (R < 0 || T < 1 || Hq < 1 || Hkv < 1 || ctx < 0) return fail(KS_ERR_INVALID_ARG, "attention: bad size");
  KS_TRY(check_aligned16({q, k_layer, v_layer, out}, "attention"));
  return tc_attention(q, k_layer, v_layer, cache_rows, R, T, Hq, Hkv, head_dim, ctx, out, status,
                      (cudaStream_t)stream);
}

}  // extern "C"
