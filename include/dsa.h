/*
 * dsa.h — C ABI of libdsa, a B200 (sm_100a) implementation of the
 * DeepSeek-Sparse-Attention (DSA) layer compute:
 *
 *   (1) lightning-indexer scores   I[t,s] = sum_h w[t,h] * relu(scale * q[t,h,:] . k[s,:])
 *   (2) deterministic top-k        higher score first, then smaller key index
 *   (3) sparse MLA attention       softmax(scale * q . K[i]) V[i] over the selected keys only
 *   (+) kpool variant              pooled indexer keys, pool selection expanded to tokens
 *   (+) indexer q/k preparation    key LayerNorm, NEOX RoPE, Walsh-Hadamard rotation, cache store
 *
 * Sources: the fak note "GLM-5.2: the DSA sparse attention moves onto the pure
 * fak kernel" (score formula in section 3, the sparse attend in "What
 * changed"); ik_llama.cpp PR #2063 "Another DSA attempt" with the commit
 * messages of PR #2045 (indexer with one shared MQA key head, causal mask,
 * per-sequence visibility); the metrale docs page of module glm5next_dsa_ref
 * (index_scores, topk_pools, pool_states, kept_pools, expand_selection,
 * topk_to_mask, mla_masked_attention, DsaDims with no defaults, INVALID).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Ownership: every pointer argument is caller-owned memory.  Array arguments
 *   are DEVICE pointers on the current CUDA device unless stated otherwise; the
 *   library never allocates device memory and never frees anything.
 * - Execution: work is enqueued on `stream` (may be 0, the legacy default
 *   stream) and the call returns without synchronizing.  Outputs are valid
 *   once the stream has reached the enqueued work.
 * - Layouts: all tensors are dense, row-major (C order) unless a stride
 *   argument says otherwise.  B = dims->batch, T = dims->n_q, S = dims->n_kv.
 * - Visibility (step S1): key row s of sequence b is visible to the query at
 *   absolute position p = q_pos[b*T+t] iff kv_start[b] <= s <= p and
 *   s < kv_len[b].  A query with p < kv_start[b] is a padded row and sees
 *   nothing.  In pool mode (dims->kpool >= 1) the keys are pools: pool j
 *   covers tokens kv_start[b] + j*kpool ... + kpool-1 and is visible iff its
 *   last token is <= p and < kv_len[b].  q_pos/kv_start/kv_len are int32
 *   device arrays of B*T, B and B entries.
 * - Index rows are int32 with DSA_INVALID (-1) in every slot that holds no key.
 * - Errors: argument and shape errors are reported synchronously, before any
 *   launch, as DSA_ERR_INVALID_ARGUMENT; shapes or dtypes this build does not
 *   implement give DSA_ERR_UNSUPPORTED (there is no fallback of any kind);
 *   a failed launch gives DSA_ERR_CUDA.  Every bounded device-side wait that
 *   expires records DSA_ERR_TIMEOUT, read by dsa_get_device_status().
 *   dsa_last_error() returns a message describing the most recent failure on
 *   the calling host thread.
 * - Thread safety: entry points may be called from several host threads; the
 *   device status word is shared by all calls on a device.
 */
#ifndef DSA_H_
#define DSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* dsa_stream_t; /* identical to cudaStream_t */

typedef enum {
  DSA_OK = 0,
  DSA_ERR_INVALID_ARGUMENT = 1,
  DSA_ERR_UNSUPPORTED = 2,
  DSA_ERR_WORKSPACE = 3,
  DSA_ERR_CUDA = 4,
  DSA_ERR_TIMEOUT = 5
} dsa_status;

typedef enum { DSA_F32 = 0, DSA_BF16 = 1 } dsa_dtype;

#define DSA_INVALID (-1)

/* Geometry of one call.  Every field is read explicitly; there are no
 * defaults (metrale glm5next_dsa_ref, struct DsaDims: "No field has a
 * default").  Each entry point lists the fields it reads; the others are
 * ignored. */
typedef struct dsa_dims {
  int32_t batch;     /* B: independent sequences                               */
  int32_t n_q;       /* T: query rows per sequence                             */
  int32_t n_kv;      /* S: key rows per sequence (pools in pool mode)          */
  int32_t idx_heads; /* H_I: indexer query heads                               */
  int32_t idx_dim;   /* D_I: indexer head width (shared MQA key width)         */
  int32_t top_k;     /* k: keys (or pools) selected per query                  */
  int32_t heads;     /* H: attention query heads                               */
  int32_t kv_heads;  /* Hk: key/value heads, 1 (shared latent) or divides H    */
  int32_t kd;        /* key width (q and K)                                    */
  int32_t vd;        /* value width (V and out)                                */
  int32_t kpool;     /* 0: keys are tokens; >= 1: keys are pools of kpool tokens */
  int32_t out_width; /* expand_selection row width                             */
  int32_t dtype;     /* dsa_dtype of q_idx, k_idx, q, K, V, pooled and out     */
} dsa_dims;

enum { DSA_OP_TOPK = 1, DSA_OP_LAYER_FORWARD = 2 };

/* Human-readable name of a status code (static storage). */
const char* dsa_status_string(dsa_status s);

/* Message for the most recent failure on this host thread ("" if none). */
const char* dsa_last_error(void);

/* Library version string (static storage). */
const char* dsa_version(void);

/* Kernels launched by the most recent top-level entry point call on this host
 * thread, comma-separated in launch order, e.g. "index_tc,topk_set,attend_tc"
 * for a fused layer on the tensor cores; "" if that call launched nothing.
 * Family names: index_tc / index_simt / index_tc_fp8 and fp8_quantize (S2),
 * topk_ranked / topk_set (S3), index_topk / index_topk_fp8 (S2 + S3 fused),
 * attend_tc / attend_simt (S4), pool_states, expand_selection, head_gemm_tc /
 * head_gemm_simt (S8), index_rotate, wait_selftest.  Shows which kernel served a
 * shape that more than one kernel implements (see dsa_sparse_attend).  Thread-local
 * storage, valid until the next entry point call on the same thread. */
const char* dsa_last_kernels(void);

/* Kernel family for shapes that both the tensor-core and the CUDA-core
 * kernels implement: 0 (default) selects the tensor-core kernels, 1 the
 * CUDA-core kernels (to compare the two on the same inputs).  Process-wide;
 * returns the previous setting.  Shapes only one family implements always use
 * that family; there is no fallback on failure. */
int dsa_set_kernel_policy(int policy);

/* Bytes of caller workspace an entry point needs for `dims`.
 * op = DSA_OP_TOPK:          workspace of dsa_topk (0 in this build).
 * op = DSA_OP_LAYER_FORWARD: the fp32 score matrix [B,T,S] plus, when the
 *                            caller passes no idx_out, the int32 index rows
 *                            [B,T,top_k]; each region 256-byte aligned.
 * Returns 0 for an unknown op or invalid dims. */
size_t dsa_workspace_size(const dsa_dims* dims, int op);

/* S2 — lightning-indexer scores.
 * Defines: I[b,t,s] = sum_{h<H_I} w[b,t,h] * relu(scale * sum_d q_idx[b,t,h,d]*k_idx[b,s,d])
 * for visible s, and -inf for every key that is not visible (fak note, section
 * 3; metrale index_scores; ik_llama.cpp #2045 "scores = relu(indexer_k .
 * indexer_q), scaled per-head weights, summed over heads, + base causal
 * mask").  A signed-zero score is written as +0.
 * Reads dims: batch, n_q, n_kv, idx_heads, idx_dim, kpool, dtype.
 * q_idx  [B,T,H_I,D_I] dtype     k_idx [B,S,D_I] dtype (one shared key per row)
 * w      [B,T,H_I] fp32          scores [B,T,S] fp32 (written for every s)
 * bf16 inputs with D_I = 128 run on the tensor cores with fp32 accumulation;
 * fp32 inputs accumulate in fp32 on the CUDA cores. */
dsa_status dsa_index_scores(const dsa_dims* dims, const void* q_idx, const void* k_idx,
                            const float* w, float scale, const int32_t* q_pos,
                            const int32_t* kv_start, const int32_t* kv_len, float* scores,
                            dsa_stream_t stream);

/* S2 with FP8 operands, step 1: per-vector e4m3 quantisation.
 * ik_llama.cpp PR #2063 (commit messages of #2045) ships the indexer tensors in
 * F8_E4M3; the per-vector scaling is this library's reading of it.  Row r of x
 * (dim values) gets scale s[r] = amax/448 (amax = max |x[r,:]|; 1 for a zero
 * row) and codes[r,:] = e4m3(x[r,:] * fl(448/amax)), where fl() and the
 * product round to fp32 and e4m3() rounds to nearest even (saturating at 448),
 * so that x ~= codes * s.  Quantise queries as n_vectors = B*T*H_I rows of
 * q_idx and keys as B*S rows of k_idx (once, when they enter the cache).
 * x: n_vectors rows of dim values of in_dtype, x_row_stride values apart,
 * aligned to 4 values.  codes: [n_vectors, dim] e4m3 bytes (dense), 4-byte
 * aligned; scales: [n_vectors] fp32.  dim must be 128 (else DSA_ERR_UNSUPPORTED). */
dsa_status dsa_fp8_quantize(int64_t n_vectors, int32_t dim, dsa_dtype in_dtype, const void* x,
                            int64_t x_row_stride, void* codes, float* scales, dsa_stream_t stream);

/* S2 with FP8 operands, step 2: lightning-indexer scores from e4m3 codes.
 * I[b,t,s] = sum_h w[b,t,h] * relu(scale * sq[b,t,h] * sk[b,s] * (qc[b,t,h,:] . kc[b,s,:]))
 * for visible s, -inf otherwise (the score of dsa_index_scores, fak note section 3,
 * with the operands of dsa_fp8_quantize).  The code products accumulate in fp32 on
 * the tensor cores (tcgen05 kind::f8f6f4).  A signed-zero score is written as +0.
 * Reads dims: batch, n_q, n_kv, idx_heads, idx_dim, kpool.
 * q_codes [B,T,H_I,128] e4m3, q_scales [B,T,H_I] fp32, k_codes [B,S,128] e4m3,
 * k_scales [B,S] fp32, w [B,T,H_I] fp32, scores [B,T,S] fp32.  Codes 16-byte aligned.
 * idx_dim must be 128 and idx_heads 32, 64 or 128, with batch*n_kv >= 128
 * (else DSA_ERR_UNSUPPORTED).  The selection then runs on these scores with
 * dsa_topk / dsa_topk_set as usual. */
dsa_status dsa_index_scores_fp8(const dsa_dims* dims, const void* q_codes, const float* q_scales,
                                const void* k_codes, const float* k_scales, const float* w, float scale,
                                const int32_t* q_pos, const int32_t* kv_start, const int32_t* kv_len,
                                float* scores, dsa_stream_t stream);

/* S3 — deterministic top-k.
 * For each row (b,t): the min(k, n_visible) visible keys with the highest
 * score, ordered by higher score and then smaller key index, so ties resolve
 * identically on every run (metrale topk_pools; ik_llama.cpp #2045
 * ggml_top_k(min(top_k, n_tokens))).  Slots past the selection hold
 * DSA_INVALID.  Only visible keys are candidates, whatever their score;
 * -0.0 and +0.0 compare equal.  Scores must be finite (NaN order undefined).
 * Reads dims: batch, n_q, n_kv, kpool.
 * scores [B,T,S] fp32   idx [B,T,k] int32   vals [B,T,k] fp32 or NULL (score of
 * each selected key, -inf in INVALID slots).  1 <= k <= 4096.
 * ws/ws_bytes: workspace of dsa_workspace_size(dims, DSA_OP_TOPK) bytes. */
dsa_status dsa_topk(const dsa_dims* dims, const float* scores, const int32_t* q_pos,
                    const int32_t* kv_start, const int32_t* kv_len, int32_t k, int32_t* idx,
                    float* vals, void* ws, size_t ws_bytes, dsa_stream_t stream);

/* S3' — the same selection as a set.
 * Selects exactly the keys dsa_topk(k) selects (same scores, same visibility,
 * same tie rule) and lists them in ascending key order, DSA_INVALID after
 * them; vals (or NULL) holds each listed key's score, -inf in INVALID slots.
 * The attention reads a selection as a set, so this is the form the fused
 * layer uses: it needs no rank sort.  Arguments as in dsa_topk (no workspace).
 * (The pages define the selection as a set; dsa_topk's rank order is this
 * library's deterministic listing of it.) */
dsa_status dsa_topk_set(const dsa_dims* dims, const float* scores, const int32_t* q_pos,
                        const int32_t* kv_start, const int32_t* kv_len, int32_t k, int32_t* idx,
                        float* vals, dsa_stream_t stream);

/* S2 + S3 fused — the selection straight from the indexer inputs, without a
 * score matrix in memory.  Selects exactly what dsa_index_scores followed by
 * dsa_topk_set(k) select (the same scores, visibility and tie rule: fak note
 * section 3, the selection is score dots plus a top-k; metrale topk_pools) and
 * lists the keys in ascending key order, DSA_INVALID after them.  One cluster of
 * up to 8 CTAs scores a query row on the tensor cores, keeps the scores in shared
 * memory and selects them there (radix select over distributed shared memory), so
 * only the index rows are written.  Meant for rows with few queries per sequence
 * (decode): every query row reads its sequence's keys once.
 * Reads dims: batch, n_q, n_kv, idx_heads, idx_dim, kpool (must be 0), dtype.
 * q_idx [B,T,H_I,128] bf16, k_idx [B,S,128] bf16, w [B,T,H_I] fp32, idx [B,T,k]
 * int32, 1 <= k <= 4096.  Requires bf16, idx_dim 128, idx_heads 32, 64 or 128
 * and n_kv <= 131072 (else DSA_ERR_UNSUPPORTED). */
dsa_status dsa_index_topk(const dsa_dims* dims, const void* q_idx, const void* k_idx, const float* w,
                          float scale, const int32_t* q_pos, const int32_t* kv_start, const int32_t* kv_len,
                          int32_t k, int32_t* idx, dsa_stream_t stream);

/* S2 + S3 fused with FP8 operands: the selection dsa_index_scores_fp8 followed by
 * dsa_topk_set(k) gives, computed as dsa_index_topk computes it (no score matrix
 * in memory).  Arguments as in dsa_index_scores_fp8 (codes and scales of
 * dsa_fp8_quantize, 16-byte aligned codes) plus k and idx [B,T,k] as in
 * dsa_index_topk; the same requirements as dsa_index_topk. */
dsa_status dsa_index_topk_fp8(const dsa_dims* dims, const void* q_codes, const float* q_scales,
                              const void* k_codes, const float* k_scales, const float* w, float scale,
                              const int32_t* q_pos, const int32_t* kv_start, const int32_t* kv_len,
                              int32_t k, int32_t* idx, dsa_stream_t stream);

/* S4 — sparse attention over the selected keys.
 * For every (b,t,h): U = the set of distinct entries i of idx[b,t,:] with
 * 0 <= i < S (duplicates collapse, DSA_INVALID and out-of-range entries are
 * dropped: metrale topk_to_mask), and
 *   out[b,t,h,:] = sum_{i in U} softmax_i(scale * q[b,t,h,:] . K(b,i,g)) V(b,i,g)
 *   lse[b,t,h]   = log sum_{i in U} exp(scale * q . K(b,i,g))
 * with g = h / (H/Hk) (fak note, "What changed": dot*scale, softmax, weighted
 * sum of V, separate key width kd and value width vd; metrale
 * mla_masked_attention).  An empty U gives out = 0 and lse = -inf.
 * K(b,i,g)[d] = k[(b*S + i)*k_row_stride + g*kd + d]   (element strides)
 * V(b,i,g)[d] = v[(b*S + i)*v_row_stride + g*vd + d]
 * so a shared MLA latent row of kd columns whose first vd columns are the
 * value is passed as v = k, k_row_stride = v_row_stride = kd, kv_heads = 1.
 * Reads dims: batch, n_q, n_kv, heads, kv_heads, kd, vd, dtype.
 * q [B,T,H,kd] dtype   idx [B,T,width] int32   out [B,T,H,vd] dtype
 * lse [B,T,H] fp32 or NULL.  Softmax and accumulation are fp32.
 * bf16 with kv_heads = 1 (V = the first vd columns of the K rows, same pointer and
 * stride), kd in {512, 576}, vd = 512, H in {64, 128}, n_kv <= 294912 (with
 * batch*n_kv < 2^31) and width up to about 3400 (2200 when n_kv > 65536) runs on
 * the tensor cores; other shapes run on the CUDA cores, which dsa_last_kernels()
 * reports as "attend_simt". */
dsa_status dsa_sparse_attend(const dsa_dims* dims, const void* q, const void* k,
                             int64_t k_row_stride, const void* v, int64_t v_row_stride,
                             const int32_t* idx, int32_t width, float scale, void* out,
                             float* lse, dsa_stream_t stream);

/* S5 — the fused layer: dsa_index_scores -> dsa_topk(top_k) -> dsa_sparse_attend
 * on one stream with one caller workspace (fak note, sections "The selection
 * stays host-side" and 3: index dots and top-k choose the keys the sparse
 * attend reads).  idx_in != NULL skips S2/S3 and attends over the caller's
 * rows [B,T,top_k] (reuse of an earlier layer's selection); otherwise the
 * selection is written to idx_out [B,T,top_k] when idx_out != NULL, or kept in
 * the workspace.  The selection is the set dsa_topk(top_k) picks (same
 * scores, same tie rule) listed in ascending key order, DSA_INVALID after it:
 * the attention reads it as a set, so no rank sort is spent on it.  With one
 * query per sequence (n_q = 1, decode) and a shape dsa_index_topk takes, the
 * selection comes from dsa_index_topk (the same keys; the scores stay on chip
 * and the workspace's score region is not written); otherwise from
 * dsa_index_scores into the workspace and dsa_topk_set.  All other arguments are
 * as in the three calls above.
 * Reads dims: every field of the three calls; kpool must be 0. */
dsa_status dsa_layer_forward(const dsa_dims* dims, const void* q_idx, const void* k_idx,
                             const float* w, float idx_scale, const int32_t* q_pos,
                             const int32_t* kv_start, const int32_t* kv_len, const void* q,
                             const void* k, int64_t k_row_stride, const void* v,
                             int64_t v_row_stride, float attn_scale, const int32_t* idx_in,
                             int32_t* idx_out, void* out, float* lse, void* ws, size_t ws_bytes,
                             dsa_stream_t stream);

/* S6 — kpool: k_norm LayerNorm and gated pooling (metrale pool_states,
 * kept_pools, layer_norm; invariants: the pool softmax runs over the slot axis
 * separately for each channel; pooling starts at the first valid token; a
 * trailing partial pool is not a pool).  For sequence b with f = kv_start[b]:
 *   n_pools[b] = max(0, (kv_len[b] - f) / kpool)     (the kept pool ids are 0..n_pools-1)
 *   kn[s,:]    = (k[b,s,:] - mean) / sqrt(var + ln_eps) * ln_w + ln_b   (biased var)
 *   pooled[b,j,c] = sum_{r<kpool} softmax_r(gate[b,f+j*kpool+r,c]) * kn[f+j*kpool+r,c]
 * and pooled rows j >= n_pools[b] are zero.
 * Reads dims: batch, n_kv (tokens), idx_dim, kpool, dtype.  P = n_kv / kpool.
 * k, gate [B,S,D_I] dtype   ln_w, ln_b [D_I] fp32 or NULL (1 and 0)
 * pooled [B,P,D_I] dtype    n_pools [B] int32.   ln_eps must be > 0
 * (ik_llama.cpp #2045: eps 0 aborts LayerNorm). */
dsa_status dsa_pool_states(const dsa_dims* dims, const void* k, const void* gate, const float* ln_w,
                           const float* ln_b, float ln_eps, const int32_t* kv_start,
                           const int32_t* kv_len, void* pooled, int32_t* n_pools,
                           dsa_stream_t stream);

/* S7 — kpool: expand selected pools to token indices (metrale
 * expand_selection: every row is written for all out_width entries, INVALID in
 * every slot that holds no token, a padded query row stays all INVALID; the
 * tail append covers the trailing partial pool).  Row (b,t) with p = q_pos,
 * f = kv_start[b]: the tokens f+j*kpool .. f+j*kpool+kpool-1 of each selected
 * pool j (entries outside [0, n_pools) are skipped) in rank order, then the
 * visible tail f + V*kpool .. min(p, kv_len-1) with V = min((p-f+1)/kpool,
 * n_pools), then DSA_INVALID.
 * Reads dims: batch, n_q, top_k (pool_idx width), kpool, out_width.
 * pool_idx [B,T,top_k] int32   n_pools [B] int32 (from dsa_pool_states)
 * tok_idx [B,T,out_width] int32; out_width >= top_k*kpool + kpool - 1. */
dsa_status dsa_expand_selection(const dsa_dims* dims, const int32_t* pool_idx,
                                const int32_t* q_pos, const int32_t* kv_start,
                                const int32_t* kv_len, const int32_t* n_pools, int32_t* tok_idx,
                                dsa_stream_t stream);

/* S8 — NoPE MLA absorption (metrale expand_kv: K_h = W_UK,h c, V_h = W_UV,h c
 * from the latent c; absorbing the up-projections into the query and the
 * output is algebraically the same attention):
 *   dsa_absorb_q:   q_lat[n,h,l] = sum_d q[n,h,d] * w_uk[h,d,l]
 *   dsa_absorb_out: out[n,h,e]   = sum_l o_lat[n,h,l] * w_uv[h,e,l]
 * n runs over the B*T query rows.  Reads dims: batch, n_q, heads, dtype (bf16).
 * q [n,H,d] bf16, w_uk [H,d,L] bf16, q_lat [n,H,L] bf16;
 * o_lat [n,H,L] bf16, w_uv [H,e,L] bf16, out [n,H,e] bf16; fp32 accumulation.
 * d, L, e are given explicitly. */
dsa_status dsa_absorb_q(const dsa_dims* dims, const void* q, int32_t d, const void* w_uk,
                        int32_t L, void* q_lat, dsa_stream_t stream);
dsa_status dsa_absorb_out(const dsa_dims* dims, const void* o_lat, int32_t L, const void* w_uv,
                          int32_t e, void* out, dsa_stream_t stream);

/* S9 — indexer query / key preparation, the step that produces q_idx and the
 * k_idx cache rows the indexer reads (ik_llama.cpp PR #2063 with the PR #2045
 * commit messages: "What it does" splits the indexer query and key into a rope
 * part and a nope part, gives the rope part NEOX RoPE and concatenates; the key
 * is LayerNorm-ed with bias first; the decode-cache commit rotates both by the
 * Walsh-Hadamard matrix and writes the keys into the indexer cache at their
 * slot; the K-shift commit states the cached key as H * concat(RoPE(k_pe, pos),
 * k_nope) with NEOX RoPE unscaled).  For row r < n_rows and head h < heads,
 * with x = in[r, h, 0:dim]:
 *   y = layer_norm ? (x - mean) / sqrt(var + ln_eps) * ln_w + ln_b : x   (biased var)
 *   for i < n_rope/2, a = pos[r] * rope_theta^(-2i/n_rope):
 *     y'[i]            = y[i] cos a - y[i + n_rope/2] sin a
 *     y'[i + n_rope/2] = y[i + n_rope/2] cos a + y[i] sin a
 *   (values from n_rope on are unchanged: the rope part is the first n_rope)
 *   z = hadamard ? H y' / sqrt(dim) : y',   H[i][j] = (-1)^popcount(i & j)
 *   out[dst, h, 0:dim] = z,   dst = out_rows ? out_rows[r] : r
 * A row whose dst lies outside [0, out_capacity) is not written (a padded token
 * can carry slot -1).  The angles are evaluated in double precision, the rest
 * in fp32; the store rounds to out_dtype (round to nearest even for bf16).
 * The Hadamard rotation leaves every q.k unchanged, so queries and keys must
 * both be rotated or both not.
 * in:  n_rows rows of heads*dim values of in_dtype, in_row_stride values apart.
 * out: out_capacity rows of heads*dim values of out_dtype, out_row_stride apart
 *      (a key cache [B, n_kv, dim] written at slots b*n_kv + position, say).
 * pos [n_rows] int32 positions (may be NULL when n_rope == 0);
 * out_rows [n_rows] int32 or NULL; ln_w, ln_b [dim] fp32 or NULL (1 and 0).
 * Requirements (else DSA_ERR_INVALID_ARGUMENT): n_rows >= 0, heads >= 1,
 * dim in {32, 64, 128}, n_rope even with 0 <= n_rope <= dim and (n_rope/2) a
 * multiple of dim/32, rope_theta > 0 when n_rope > 0, ln_eps > 0 with
 * layer_norm, strides >= heads*dim and multiples of dim/32, in and out aligned
 * to dim/32 values, out_capacity >= n_rows when out_rows is NULL.  in and out
 * must not overlap unless the call is exactly in place (same pointer, stride and
 * dtype, out_rows NULL). */
dsa_status dsa_index_rotate(int32_t n_rows, int32_t heads, int32_t dim, int32_t n_rope, float rope_theta,
                            int32_t layer_norm, const float* ln_w, const float* ln_b, float ln_eps,
                            int32_t hadamard, const int32_t* pos, dsa_dtype in_dtype, const void* in,
                            int64_t in_row_stride, dsa_dtype out_dtype, void* out, int64_t out_row_stride,
                            const int32_t* out_rows, int64_t out_capacity, dsa_stream_t stream);

/* Allocation-free variant of dsa_layer_forward, for callers that cannot
 * allocate device memory where they run the layer (a serving engine that plans
 * all memory up front and forbids allocation on its decode path, code running
 * inside an allocator callback, a runtime handed a fixed memory budget).  The
 * DSA pages have no counterpart: this is a library convenience, not part of the
 * method.  Same arguments and result as dsa_layer_forward without ws/ws_bytes:
 * the score matrix and index rows live in one fixed 16 MiB array inside the
 * library's device memory, held by every GPU that loads the library until the
 * process exits.  Calls whose workspace need (dsa_workspace_size) exceeds
 * 16 MiB return DSA_ERR_WORKSPACE with a message.  The first call on a device
 * looks up the array's device address with that device current, so make it
 * before any stream capture.  All calls share the array and it keeps the last
 * call's contents; calls that overlap on the GPU race on it.  No part of the
 * array needs to start at zero.  The address is remembered with the context it
 * was read in: after a cudaDeviceReset the next call on that device looks it up
 * again (also outside any stream capture). */
dsa_status dsa_layer_forward_static(const dsa_dims* dims, const void* q_idx, const void* k_idx,
                                    const float* w, float idx_scale, const int32_t* q_pos,
                                    const int32_t* kv_start, const int32_t* kv_len, const void* q,
                                    const void* k, int64_t k_row_stride, const void* v,
                                    int64_t v_row_stride, float attn_scale, const int32_t* idx_in,
                                    int32_t* idx_out, void* out, float* lse, dsa_stream_t stream);

/* Synchronize `stream`, then return and clear the device status word:
 * DSA_ERR_TIMEOUT if any bounded device-side wait expired since the last
 * call, DSA_ERR_CUDA if the stream reports an error, DSA_OK otherwise. */
dsa_status dsa_get_device_status(dsa_stream_t stream);

/* Self-test of the bounded-wait machinery: launches one block that waits on
 * a shared-memory barrier nothing arrives on, with a limit of `timeout_ns`
 * nanoseconds (1e3 .. 1e10).  The wait must expire, record DSA_ERR_TIMEOUT in
 * the device status word and return; dsa_get_device_status() then reports it. */
dsa_status dsa_selftest_wait_timeout(int64_t timeout_ns, dsa_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* DSA_H_ */
