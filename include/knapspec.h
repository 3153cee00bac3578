/*
 * knapspec.h -- C ABI of the B200 (sm_100a) KnapSpec knapsack layer-selection DP.
 *
 * Method: "KnapSpec: Self-Speculative Decoding via Adaptive Layer Selection as a
 * Knapsack Problem" (arXiv 2602.20217), as the Pith review page of the paper
 * describes it.  Every Attention and every MLP sublayer of a decoder is one
 * knapsack item whose integer weight is its latency (review, "What carries the
 * argument"; referee major 4 on §3.6).  For every latency-budget cell b the DP
 * keeps whichever of "skip item i" (carry cell b) and "execute item i" (run the
 * sublayer on cell b - w_i) scores higher, the score being the cosine with the
 * state X^(i) the unpruned model reaches at that depth (Eq. 6-8, Algorithm 1;
 * referee major 1), stores a backpointer, reads one layer set per budget back
 * (Algorithm 2; referee minor 4) and grid-searches the draft length gamma for
 * the largest Tokens-per-Time
 * TPT(S, gamma) = ((1 - a^(gamma+1)) / (1 - a)) / (gamma t_Draft(S) + t_Target)
 * (Eq. 4, Eq. 5).
 *
 * Conventions shared by every call:
 *  - The comments below label the steps of the solve a0 .. a6: a0 item weights
 *    and the budget grid, a1 the full model's reference states, a2 / a3 the
 *    Attention / MLP item on a batch of states, a4 the select with its
 *    backpointer, a5 the set reconstruction, a6 the TPT grid search.
 *  - Items are numbered k = 0 .. 2L-1: item 2l is the Attention sublayer of
 *    layer l, item 2l+1 its MLP sublayer.  X^(0) is the T evaluation tokens'
 *    input state, X^(k+1) = item_k(X^(k)).
 *  - Budget cells b = 0 .. C-1 with C = K + 1 and K = sum of the item weights.
 *    A cell holds the best state that uses at most b weight units; every cell
 *    starts from X^(0).  Execute reads cell b - w_k and wins only when its
 *    value is strictly larger.
 *  - The value of a state H [T][d] is the mean over tokens of the per-token
 *    cosine with the target state.
 *  - Pointers named "device" are CUDA device pointers (cudaMalloc or a
 *    torch CUDA tensor); "host" pointers are ordinary host memory.  The caller
 *    owns every buffer; the library allocates nothing.  All dense arrays are
 *    row-major and contiguous.  Device arrays of weights, caches and states
 *    (and the GEMM / attention utilities' operands and outputs) must start on
 *    a 16-byte boundary: the kernels move them 16 bytes at a time.  A
 *    misaligned pointer is KS_ERR_INVALID_ARG, before anything is enqueued.
 *  - Calls that take a stream are asynchronous on it: they validate their
 *    arguments on the host, enqueue kernels and return.  Results are valid
 *    once the stream has been synchronised.  Host-side argument errors return
 *    a ks_status before anything is enqueued; the text is in ks_last_error().
 *    A kernel that gives up a bounded wait writes KS_ERR_TIMEOUT into the
 *    caller's device status word (ks_result.status) and returns; kernels never
 *    trap.
 *  - Linear weights are stored [out_features][in_features] (the layout of
 *    torch.nn.Linear.weight).  Weights and the KV cache are bf16 (KS_BF16) or
 *    fp32 (KS_F32); hidden states are always fp32.
 */
#ifndef KNAPSPEC_H
#define KNAPSPEC_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define KS_API __attribute__((visibility("default")))
#else
#define KS_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* A CUDA stream (cudaStream_t); NULL is the legacy default stream. */
typedef void* ks_stream_t;

typedef enum {
  KS_OK = 0,
  KS_ERR_INVALID_ARG = 1,   /* bad pointer, size or shape */
  KS_ERR_UNSUPPORTED = 2,   /* shape or dtype the kernels do not handle */
  KS_ERR_WORKSPACE = 3,     /* workspace smaller than ks_workspace_size() */
  KS_ERR_CUDA = 4,          /* a CUDA runtime call failed */
  KS_ERR_TIMEOUT = 5,       /* device side: a bounded wait expired */
  KS_ERR_INTERNAL = 6
} ks_status;

typedef enum { KS_F32 = 0, KS_BF16 = 1 } ks_dtype;

/* Decoder shape.  head_dim must be 64 or 128; n_q_heads a multiple of
 * n_kv_heads; d_model a multiple of 64; ffn a multiple of 16.  bf16 weights
 * run on the tensor-core GEMM, whose output tiles are 256 columns wide (128
 * for the SwiGLU gate/up pair): there d_model and n_q_heads * head_dim must
 * be multiples of 256 and ffn of 128 (else KS_ERR_UNSUPPORTED, before any
 * launch). */
typedef struct {
  int32_t n_layers;
  int32_t d_model;
  int32_t n_q_heads;
  int32_t n_kv_heads;
  int32_t head_dim;
  int32_t ffn;
  float rms_eps;       /* RMSNorm: x / sqrt(mean(x^2) + eps) * gain */
  double rope_base;    /* rotate-half RoPE, theta_j = base^(-2j/head_dim) */
  int32_t wdtype;      /* ks_dtype of the weights and the KV cache */
} ks_model_desc;

/* Device pointers to one layer's weights (dtype = ks_model_desc.wdtype):
 * attn_norm [d], wq [Hq*hd][d], wo [d][Hq*hd], mlp_norm [d],
 * w_gate [ffn][d], w_up [ffn][d], w_down [d][ffn]; wk, wv [Hkv*hd][d].
 * wk and wv are read only under KS_KV_WINDOW (they may be NULL otherwise):
 * with the default KS_KV_CACHE every key and value comes from the cache. */
typedef struct {
  const void* attn_norm;
  const void* wq;
  const void* wo;
  const void* mlp_norm;
  const void* w_gate;
  const void* w_up;
  const void* w_down;
  const void* wk;
  const void* wv;
} ks_layer_weights;

/* Where an Attention item's keys and values come from.  The review leaves the
 * attention of a pruned draft's evaluation tokens open ("What carries the
 * argument": the value compares a draft state with the full model's state,
 * Eq. 6); two readings are offered:
 *  KS_KV_CACHE  -- every position 0 .. ctx+T-1 from the full model's cache
 *                  (the evaluation tokens are already verified tokens);
 *  KS_KV_WINDOW -- positions 0 .. ctx-1 from the cache, and the T window
 *                  positions' keys and values recomputed from the candidate
 *                  state itself: k = RoPE(x^ Wk^T) at position ctx + t,
 *                  v = x^ Wv^T, with x^ the item's normalised input.  Token t
 *                  sees the context and window tokens 0 .. t of its own state.
 * With bf16 weights (tensor-core kernels) KS_KV_WINDOW needs T to divide 128,
 * so that a 128-row tile of the batch holds whole states. */
typedef enum { KS_KV_CACHE = 0, KS_KV_WINDOW = 1 } ks_kv_mode;

/* The full model's KV cache (device, dtype = wdtype), laid out
 * [n_layers][cache_rows][n_kv_heads][head_dim] for K and for V, keys already
 * rotated.  Evaluation token t (0 .. T-1) sits at position ctx + t and attends
 * to positions 0 .. ctx + t, so cache_rows >= ctx + T.  With fp32 weights
 * (SIMT kernels) ctx + T + head_dim must be at most 51200, else
 * KS_ERR_UNSUPPORTED before any launch.  kv_mode is a ks_kv_mode; under
 * KS_KV_WINDOW the cache rows ctx .. ctx+T-1 are not read. */
typedef struct {
  const void* k_cache;
  const void* v_cache;
  int64_t cache_rows;
  int32_t ctx;
  int32_t kv_mode;
} ks_cache_desc;

/* Budget semantics of a cell b (the review notes the paper's main text and
 * appendix initialise the table differently, referee major 1). */
typedef enum {
  KS_BUDGET_AT_MOST = 0,   /* b caps the used weight; every cell starts from X^(0) */
  KS_BUDGET_EXACT = 1      /* b is the used weight exactly; only cell 0 starts valid, a
                              cell no subset fills stays invalid (value NaN) */
} ks_budget_mode;

/* Selection parameters.  alpha(b) = clamp((value_b - alpha_lo) / alpha_scale,
 * 0, alpha_max) is the acceptance-rate stand-in; gamma runs 1 .. gamma_max. */
typedef struct {
  int32_t gamma_max;
  int32_t n_bins;      /* budget-grid bins for ks_quantize_weights (ks_solve
                          uses it when no weights are passed) */
  int32_t budget_mode; /* ks_budget_mode */
  double alpha_lo;
  double alpha_scale;
  double alpha_max;
  /* Optional pruning (review: tau = 0.5 cosine threshold, K/2 skipped-weight
   * cap; "Assumptions & free parameters", "Reading between the lines").  After
   * item k a cell is dropped (invalid: value NaN, never read again, no set) if
   * its kept value is below prune_tau, or if its budget b < W_k - skip_cap with
   * W_k = w_0 + .. + w_k.  prune_tau = -INFINITY and skip_cap < 0 turn them off. */
  double prune_tau;
  int32_t skip_cap;
  /* Distinct-state execution: before each item, budget cells whose states are
   * bit-for-bit equal (and valid) are folded together and the item runs once
   * per distinct state.  Candidates are found by a 64-bit fingerprint of each
   * state and every fold is then confirmed by comparing the two states' bytes;
   * a state whose bytes differ from its representative's runs on its own.
   * Results are therefore identical to the dense solve (every row's arithmetic
   * is independent of its batch); only the work shrinks.  0 = off, 1 = on,
   * 2 = on with the fingerprints cut to 8 bits, so that unequal states collide
   * often and the byte comparison must separate them (a self-test mode). */
  int32_t dedup;
} ks_params;

/* Outputs of ks_solve: caller-allocated DEVICE buffers.  C = K + 1 cells,
 * words = ceil(n_items / 64).  Optional buffers may be NULL. */
typedef struct {
  int32_t* status;     /* [1] required: 0, or a ks_status a kernel wrote */
  float* values;       /* [C] required: final-row value of every cell */
  uint64_t* sets;      /* [C][words] required: bit k set = item k executed */
  int32_t* used_w;     /* [C] optional: sum of the executed items' weights (-1: invalid cell) */
  double* t_draft;     /* [C] optional: sum of the executed items' latencies (NaN: invalid) */
  uint8_t* bp;         /* [n_items][C] optional: 1 = execute won */
  float* cos_skip;     /* [n_items][C] optional: skip candidate's value */
  float* cos_exec;     /* [n_items][C] optional: execute candidate's value (NaN if b < w) */
  double* tpt;         /* [C][gamma_max] optional: the TPT grid */
  int32_t* best;       /* [2] required: best cell b*, best gamma* */
  double* best_tpt;    /* [1] optional: TPT(b*, gamma*) */
  float* ref_states;   /* [n_items+1][T][d] optional: the full model's states X^(k)
                          the solve computed (they ride along in each item's batch) */
  int32_t* exec_counts; /* [n_items] optional: states item k ran on (with dedup: the
                           distinct ones, the reference included) */
  float* final_states;  /* [C][T][d] optional: every cell's state after the last item */
  int32_t* dedup_rejected; /* [n_items] optional, distinct-state execution only: the
                              fingerprint matches item k's byte comparison rejected */
} ks_result;

/* Library version string (static storage). */
KS_API const char* ks_version(void);

/* Text of the last host-side error of the calling thread ("" if none). */
KS_API const char* ks_last_error(void);

/* Static text naming a status code. */
KS_API const char* ks_status_string(ks_status s);

/*
 * a0 -- latency weights (review, referee major 4 on §3.6: w_Attn ~ t_Attn/Delta).
 * Host only.  t: host [n_items] positive latencies; w_out: host [n_items].
 * Delta = sum(t) / n_bins (summed in item order), w_k = max(1, floor(t_k/Delta + 1/2)).
 * Errors: KS_ERR_INVALID_ARG for NULL pointers, n_items < 1, n_bins < 1 or a
 * latency that is not positive.
 */
KS_API ks_status ks_quantize_weights(const double* t, int32_t n_items, int32_t n_bins, int32_t* w_out);

/*
 * Workspace bytes ks_solve / ks_reference_forward / ks_sublayer_forward need
 * for a model, a batch of up to n_cells budget cells and T evaluation tokens.
 * Host only.  The workspace is a caller-owned device buffer, 256-byte aligned,
 * used as scratch; one workspace must not be shared by calls that overlap.
 */
KS_API ks_status ks_workspace_size(const ks_model_desc* model, int32_t n_cells, int32_t T, size_t* bytes);

/*
 * Device status of the last ks_sublayer_forward / ks_reference_forward call
 * that used this workspace: its first 4 bytes hold 0, or the ks_status a
 * kernel reported (KS_ERR_TIMEOUT when a bounded wait gave up).  Copies them
 * to *host_status and synchronises the stream.
 */
KS_API ks_status ks_workspace_status(const void* workspace, int32_t* host_status, ks_stream_t stream);

/*
 * Utility -- the tensor-core GEMM the sublayers are built on:
 * C[M][N] = A[M][K] . B[N][K]^T (+ resid[M][N]).  A, B: device bf16
 * row-major; C, resid: device fp32 [M][N]; resid may be NULL.  K must be a
 * multiple of 64 and N of 256 (else KS_ERR_UNSUPPORTED).  status: device [1]
 * word for a timed-out wait, or NULL.  Exposed for testing and reuse.
 */
KS_API ks_status ks_gemm_bf16(const void* A, const void* B, float* C, const float* resid,
                              int32_t M, int32_t N, int32_t K, int32_t* status, ks_stream_t stream);

/*
 * Utility -- the tensor-core attention the Attention sublayer is built on:
 * out[r][h] = softmax(q[r][h] . K[0 .. ctx+t]^T / sqrt(hd)) . V[0 .. ctx+t]
 * with t = r % T and kv head h / (Hq / Hkv).  q, out: device bf16
 * [R][Hq][head_dim]; k_layer, v_layer: device bf16 [cache_rows][Hkv][head_dim]
 * (one layer of the cache); head_dim 64 or 128; cache_rows >= ctx + T.
 * status: device [1] word for a timed-out wait, or NULL.  KS_ERR_INTERNAL if
 * the library was built with a register count the kernel's warpgroup register
 * split does not expect (the launch is refused rather than left to wait).
 */
KS_API ks_status ks_attention_bf16(const void* q, const void* k_layer, const void* v_layer,
                                   int64_t cache_rows, int32_t R, int32_t T, int32_t Hq,
                                   int32_t Hkv, int32_t head_dim, int32_t ctx, void* out,
                                   int32_t* status, ks_stream_t stream);

/*
 * a2 / a3 -- one sublayer on a batch of E states (Eq. 7's "execute" branch).
 * Attention (item 2l): H + Wo . Attn(RoPE(Wq . RMSNorm(H))) with causal GQA
 * over the cache; MLP (item 2l+1): H + W_down (silu(W_gate x) * W_up x),
 * x = RMSNorm(H).
 * states_in, states_out: device [E][T][d] fp32 (must not overlap).
 * Errors: KS_ERR_INVALID_ARG / KS_ERR_UNSUPPORTED / KS_ERR_WORKSPACE on the host.
 */
KS_API ks_status ks_sublayer_forward(const ks_model_desc* model, const ks_layer_weights* layers,
                              const ks_cache_desc* cache, int32_t T, int32_t item,
                              const float* states_in, int32_t E, float* states_out,
                              void* workspace, size_t workspace_bytes, ks_stream_t stream);

/*
 * a1 -- the full model's reference states (the X^(i) of Eq. 6/7):
 * ref_out[0] = x0, ref_out[k+1] = item_k(ref_out[k]).
 * layers: HOST array [n_layers] of device weight pointers.  x0: device [T][d]
 * fp32.  ref_out: device [n_items+1][T][d] fp32.
 */
KS_API ks_status ks_reference_forward(const ks_model_desc* model, const ks_layer_weights* layers,
                               const ks_cache_desc* cache, int32_t T, const float* x0,
                               float* ref_out, void* workspace, size_t workspace_bytes,
                               ks_stream_t stream);

/*
 * ks_reference_forward without a workspace argument (the paper has no
 * counterpart; this is a deployment convenience).  Same inputs, outputs and
 * arithmetic as ks_reference_forward, for callers that cannot allocate device
 * memory at the point where they need the reference states -- for example a
 * serving loop that refreshes X^(i) between decode steps while its memory
 * pool forbids new device allocations, or a plugin host that hands out only
 * input and output buffers.  The library allocates nothing here either: the
 * scratch is one fixed 8 MiB device array inside the library, which every GPU
 * that loads the library holds until the process exits.
 *  - The first call on a device looks up that array's device address (with
 *    that device current); make that first call before any stream capture.
 *    The address is then kept for the life of the process, so it belongs to
 *    the device's primary context: do not call this entry point after a
 *    cudaDeviceReset of that device, nor with a different context current.
 *  - Sizes whose scratch exceeds 8 MiB are rejected with KS_ERR_UNSUPPORTED.
 *    The scratch is T * (d_model + 2 Hq hd + 2 ffn) * bytes-per-element
 *    (4 for fp32 weights, 2 for bf16) for the operands plus T * head_dim * 4
 *    bytes for the RoPE table, each of the six pieces rounded up to 256 bytes.
 *  - All calls on a device share the array and it keeps the last call's
 *    contents; every byte a call reads it has written first, so nothing needs
 *    clearing.  Calls that overlap on the GPU (other streams, other threads)
 *    race on the array: serialise them.
 *  - This path has no status word: a bounded device wait that gives up is not
 *    reported here (use ks_reference_forward to see it).
 */
KS_API ks_status ks_reference_forward_noalloc(const ks_model_desc* model,
                                              const ks_layer_weights* layers,
                                              const ks_cache_desc* cache, int32_t T,
                                              const float* x0, float* ref_out,
                                              ks_stream_t stream);

/*
 * a4 -- one DP row's select step (Eq. 7/8): for every cell b in 0 .. C-1,
 *   s = meancos(prev[b], target), e = meancos(exec[b - w], target) if b >= w,
 *   cur[b] = exec[b - w] if e > s else prev[b];  val[b], bp[b] record the choice.
 * prev, cur: device [C][T][d] fp32 (must not overlap); exec: device [C-w][T][d]
 * fp32 (exec[e] belongs to cell e + w); target: device [T][d] fp32.
 * val: device [C] fp32; bp: device [C] u8; cos_skip / cos_exec: device [C] fp32
 * or NULL.  Cosines are accumulated in fp64.  w >= 1.
 */
KS_API ks_status ks_select_step(const float* prev, const float* exec, const float* target,
                         int32_t C, int32_t T, int32_t d, int32_t w, float* cur, float* val,
                         uint8_t* bp, float* cos_skip, float* cos_exec, ks_stream_t stream);

/*
 * a5 -- set reconstruction (Algorithm 2 with stored backpointers): for every
 * cell b, walk j = b from the last item down; item k is in the set when
 * bp[k][j] = 1, and then j -= w[k].
 * bp: device [n_items][C] u8; w: device [n_items] int32; t: device [n_items]
 * fp64.  sets: device [C][words]; used_w: device [C] int32 (or NULL); t_draft:
 * device [C] fp64 (or NULL), summed over the set in increasing item order.
 * A walk that would leave the grid writes KS_ERR_INTERNAL to status (device [1]).
 */
KS_API ks_status ks_reconstruct(const uint8_t* bp, const int32_t* w, const double* t, int32_t n_items,
                         int32_t C, uint64_t* sets, int32_t* used_w, double* t_draft,
                         int32_t* status, ks_stream_t stream);

/*
 * a6 -- TPT grid search (Eq. 4, Eq. 5) in fp64: for every cell b and gamma in
 * 1 .. gamma_max, TPT = (sum_{k=0..gamma} a_b^k) / (gamma t_draft[b] + t_target)
 * with a_b = clamp((values[b] - alpha_lo)/alpha_scale, 0, alpha_max); the
 * geometric sum is taken term by term.  The best pair is the largest TPT, ties
 * to the smaller b, then the smaller gamma.
 * values: device [C] fp32; t_draft: device [C] fp64; tpt: device
 * [C][gamma_max] fp64 or NULL; best: device [2] int32 (b*, gamma*);
 * best_tpt: device [1] fp64 or NULL.
 */
KS_API ks_status ks_tpt_argmax(const float* values, const double* t_draft, int32_t C, double t_target,
                        const ks_params* params, double* tpt, int32_t* best, double* best_tpt,
                        ks_stream_t stream);

/*
 * a0-a6 -- the whole DP on one GPU (the library's main entry).
 * layers: HOST array [n_layers] of device weight pointers; cache: the full
 * model's KV cache; x0: device [T][d] fp32; ref: device [n_items+1][T][d] fp32
 * reference states to compare against, or NULL to use the ones the solve
 * computes itself (X^(k) is carried as one extra state through every item's
 * batch, with the cells' arithmetic); w: HOST [n_items] item weights, or NULL
 * to quantise t with params->n_bins; t: HOST [n_items] latencies (t_Target =
 * their sum).
 * The number of cells is C = sum(w) + 1; out's buffers must be sized for it
 * (ks_solve_cells() returns C).  The workspace must hold
 * ks_workspace_size(model, C, T).  Nothing is copied back to the host.
 */
KS_API ks_status ks_solve(const ks_model_desc* model, const ks_layer_weights* layers,
                   const ks_cache_desc* cache, int32_t T, const float* x0, const float* ref,
                   const int32_t* w, const double* t, const ks_params* params,
                   void* workspace, size_t workspace_bytes, ks_result* out, ks_stream_t stream);

/*
 * The DP re-solved at several contexts in one pass (up to 4).  The review notes
 * that the layer set is re-optimised every T = 64 / 128 decoding steps while the
 * context grows ("Assumptions & free parameters") and that Attention latency
 * grows with the context (Figure 4 caption), so each context has its own item
 * weights and budget grid, its own reference states and its own attention
 * window, while the model's weights are the same.  Each item's GEMMs run once
 * over all contexts' batches, so every weight tile is read once for all of
 * them; attention and the select run per context.  Context j's results equal
 * those of ks_solve(model, layers, &caches[j], T, x0[j], NULL, w[j], t[j], ...)
 * bit for bit (every row's arithmetic is independent of its batch).
 * caches: HOST [n_ctx] (ctx per context; every kv_mode alike); x0: HOST [n_ctx]
 * of device [T][d] fp32 pointers; w: HOST [n_ctx] of HOST [n_items] weights (w
 * or w[j] NULL: quantise t[j] with params->n_bins); t: HOST [n_ctx] of HOST
 * [n_items] latencies; outs: HOST [n_ctx] results, each sized for its own C.
 * The workspace must hold ks_workspace_size_contexts(model, n_ctx, C[], T).
 * Distinct-state execution (params->dedup) is refused with n_ctx > 1.
 */
KS_API ks_status ks_workspace_size_contexts(const ks_model_desc* model, int32_t n_ctx,
                                            const int32_t* n_cells, int32_t T, size_t* bytes);
KS_API ks_status ks_solve_contexts(const ks_model_desc* model, const ks_layer_weights* layers,
                                   int32_t n_ctx, const ks_cache_desc* caches, int32_t T,
                                   const float* const* x0, const int32_t* const* w,
                                   const double* const* t, const ks_params* params,
                                   void* workspace, size_t workspace_bytes, ks_result* outs,
                                   ks_stream_t stream);

/*
 * Re-run check of one layer set (review: the DP keeps a single state per cell
 * with no optimality proof, referee major 1 on Eq. 8 / Algorithm 1 -- so a
 * chosen set is worth checking from scratch): the set's items run on x0 in
 * increasing item order, each exactly as ks_sublayer_forward runs it on one
 * state, and the result is scored against target:
 *   value = meancos(state, target), as ks_select_step scores a skip candidate.
 * With target = X^(2L) (ks_result.ref_states row n_items) and the set of cell
 * b, value reproduces ks_result.values[b] up to the rounding of the
 * normalised operand (the solve fuses that RMSNorm into its select step).
 * set: HOST [words] bitmask, bit k = item k runs (bits >= n_items must be 0).
 * x0, target: device [T][d] fp32.  value_out: device [1] fp32.  state_out:
 * device [T][d] fp32 (the set's final state) or NULL.  The workspace must hold
 * ks_workspace_size(model, 1, T); its status word reports a timed-out wait
 * (ks_workspace_status).  Errors: as ks_sublayer_forward, and
 * KS_ERR_INVALID_ARG for a NULL argument or a bit at or above n_items.
 */
KS_API ks_status ks_eval_set(const ks_model_desc* model, const ks_layer_weights* layers,
                             const ks_cache_desc* cache, int32_t T, const float* x0,
                             const float* target, const uint64_t* set, float* value_out,
                             float* state_out, void* workspace, size_t workspace_bytes,
                             ks_stream_t stream);

/* C = sum(w) + 1 for the weights ks_solve would use (w, or t quantised with
 * params->n_bins when w is NULL).  Host only. */
KS_API ks_status ks_solve_cells(int32_t n_items, const int32_t* w, const double* t,
                         const ks_params* params, int32_t* n_cells);

/*
 * Diagnostics of the device-side failure handling (the paper has no
 * counterpart).  Launches one kernel whose mbarrier wait nothing completes,
 * bounded by the routine every tensor-core kernel's waits use, with a limit of
 * limit_us microseconds (1 .. 2,000,000).  When the bound works the kernel
 * returns on its own and writes KS_ERR_TIMEOUT into *status (device int32,
 * which the caller zeroes first) and the nanoseconds it waited into *waited_ns
 * (device uint64, or NULL); the CUDA context stays usable.
 */
KS_API ks_status ks_check_bounded_wait(uint32_t limit_us, int32_t* status, uint64_t* waited_ns,
                                       ks_stream_t stream);

/*
 * Lemma 4.1 checker (review page: §4 Lemma 4.1, referee major 2, "What would
 * settle it").  For N states [N][T][d] (e.g. ks_result.final_states) and the
 * full model's final state ref [T][d] (ks_result.ref_states row n_items):
 * h = RMSNorm(ref_t) * g, h' = RMSNorm(state_t) * g rescaled to ||h|| (equal
 * norms, the lemma's premise), logits through lm_head W [V][d] bf16:
 * i*_t = argmax W h (first on ties), margin_t = z_i* - max_{j != i*} z_j,
 * dist_t = max_j ||w_i* - w_j||.  bound[n][t] = (||h - h'|| * dist < margin),
 * the lemma's sufficient condition for argmax W h' = i*; agree[n][t] = (argmax
 * W h' = i*).  counts = {#bound, #agree, #bound-and-not-agree}.  Operands of
 * the logits are rounded to bf16 (fp32 accumulation); the norms and cosines
 * are fp64 sums.  final_norm: bf16 [d] gain or NULL (gain 1).  d a multiple of
 * 64, V of 256.  All buffers are device memory.
 */
typedef struct {
  int32_t* istar;      /* [T] */
  float* margin;       /* [T] */
  float* dist;         /* [T] */
  float* cos;          /* [N][T] cosine of h' with h */
  uint8_t* bound;      /* [N][T] */
  uint8_t* agree;      /* [N][T] */
  int32_t* counts;     /* [3] */
} ks_lemma_result;

KS_API ks_status ks_lemma_workspace_size(int32_t N, int32_t T, int32_t d, int32_t V, size_t* bytes);
KS_API ks_status ks_lemma_check(const float* states, int32_t N, const float* ref, int32_t T,
                                int32_t d, const void* final_norm, float eps, const void* lm_head,
                                int32_t V, void* workspace, size_t workspace_bytes,
                                ks_lemma_result* out, int32_t* status, ks_stream_t stream);

/*
 * Launch accounting.  Between ks_profile_start and ks_profile_stop the library
 * counts the kernels it enqueues per kind, adds up their algorithmic FLOPs and
 * bytes (the work the DP defines, not what the hardware moved) and, when
 * timing != 0, records a CUDA event pair on the launching stream around each
 * kind's launches (not while the stream is being captured into a graph).
 * ks_profile_stop waits for those events, fills up to `capacity` entries (one
 * per kind that launched) and reports the number of kinds in *n_kinds.
 * Process-wide state; calls from several threads are serialised.
 */
typedef struct {
  char name[32];
  int64_t launches;
  double total_ms;     /* summed event time (0 when timing was off) */
  double flops;        /* algorithmic floating-point operations */
  double bytes;        /* algorithmic HBM bytes */
} ks_kernel_stat;

KS_API ks_status ks_profile_start(int32_t timing);
KS_API ks_status ks_profile_stop(ks_kernel_stat* stats, int32_t capacity, int32_t* n_kinds);

#ifdef __cplusplus
}
#endif

#endif /* KNAPSPEC_H */
