/*
 * dsa.h - C ABI of the B200 (sm_100a) DeepSeek Sparse Attention forward path.
 *
 * The method ("DeepSeek-V3.2: Pushing the Frontier of Open Large Language
 * Models", bud-325 paper digest, "Key claims", section 2.1 Eq. 1-2, Fig. 2, and
 * "Method"):
 *   1. a lightning indexer scores every causal key s of query token t as
 *        I[t,s] = sum_j w[t,j] * ReLU(q^I[t,j] . k^I[s])   over H_I heads, in FP8;
 *   2. the top-k keys by I[t,:] are selected (k = 2048 in the paper);
 *   3. MLA attention in MQA mode runs over only those k latent rows, one latent
 *      row shared by all query heads of the token.
 *
 * Conventions shared by every entry point
 *   - All tensor pointers are DEVICE pointers owned by the caller, except in
 *     dsa_forward_host. The library never allocates device memory; scratch
 *     space comes from the caller's workspace. Pointers must be 16-byte aligned.
 *   - All tensors are dense, row-major, contiguous, with the shapes given below.
 *     FP8 e4m3 (OCP "fn" encoding) is passed as uint8_t, bf16 as uint16_t bits.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *     Work is enqueued asynchronously; a call returns once it is enqueued.
 *   - Query row t of a sequence sits at absolute position p = q_pos0 + t and its
 *     candidate keys are s = 0..p (requires q_pos0 + Lq <= Lk). Prefill uses
 *     q_pos0 = 0, Lq = Lk; decode uses q_pos0 = Lk - Lq.
 *   - Every call validates all arguments before launching anything. On failure
 *     it returns a negative DSA_ERR_* code, launches nothing, and records a
 *     message readable with dsa_last_error() from the same thread.
 *   - Supported shapes: indexer (H_I, d_I) in {(4, 32), (64, 128)};
 *     attention (H, Dqk, Dv) in {(8, 80, 64), (128, 576, 512)}; k a multiple of 32,
 *     1 <= k <= 4096 for selection (k <= 2048 when selection and attention are
 *     fused in dsa_forward).
 *   - Device-side waits are bounded. A wait that runs out sets a device status
 *     word that dsa_check_status() reads; the kernel then returns early, leaving
 *     its outputs undefined. It never traps.
 */
#ifndef DSA_H_
#define DSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Status codes. */
#define DSA_OK 0
#define DSA_ERR_INVALID_ARG (-1)       /* null pointer, bad size, misalignment */
#define DSA_ERR_UNSUPPORTED_SHAPE (-2) /* valid but not one of the supported shapes */
#define DSA_ERR_WORKSPACE_TOO_SMALL (-3)
#define DSA_ERR_CUDA (-4)              /* a CUDA runtime/driver call failed */
#define DSA_ERR_TIMEOUT (-5)           /* a bounded device wait ran out */

/* Element type of the index weights w. */
#define DSA_DTYPE_F32 0
#define DSA_DTYPE_BF16 1

#define DSA_MODE_PREFILL 0
#define DSA_MODE_DECODE 1

/* Message describing the last failure on the calling thread ("" if none). */
const char* dsa_last_error(void);

/* Library version string. */
const char* dsa_version(void);

/*
 * dsa_indexer_scores - lightning-indexer scores, materialised (Eq. 1).
 *   qI        [B, Lq, H_I, d_I] e4m3 codes of the indexer queries
 *   qI_scale  [B, Lq, H_I] fp32, > 0: dequantised q^I[t,j] = code * qI_scale[t,j]
 *   kI        [B, Lk, d_I] e4m3 codes of the indexer keys
 *   kI_scale  [B, Lk] fp32, > 0: dequantised k^I[s] = code * kI_scale[s]
 *   w         [B, Lq, H_I], fp32 or bf16 (w_dtype); any sign
 *   scores    [B, Lq, Lk] fp32 output:
 *               scores[b,t,s] = kI_scale[s] * sum_j w[t,j] * qI_scale[t,j]
 *                               * max(0, qhat[t,j] . khat[s])     for s <= q_pos0+t
 *               scores[b,t,s] = -INFINITY                          for s >  q_pos0+t
 * The whole [Lq, Lk] matrix is written; dsa_forward never materialises it.
 */
int dsa_indexer_scores(const uint8_t* qI, const float* qI_scale, const uint8_t* kI,
                       const float* kI_scale, const void* w, int w_dtype, float* scores,
                       int B, int Lq, int Lk, int q_pos0, int H_I, int d_I, void* stream);

/*
 * dsa_topk_select - fine-grained token selection ("Key claims", section 2.1;
 * "Method": k = 2048).
 *   scores [B, Lq, Lk] fp32 (row (b,t) reads only s <= q_pos0 + t; NaN not allowed)
 *   idx    [B, Lq, k] int32 output: the k keys with the largest score, ties to the
 *          lowest key index, written in ascending key order; when a row has
 *          fewer than k candidates it selects all of them and pads with -1.
 *          -0.0 and +0.0 compare equal.
 */
int dsa_topk_select(const float* scores, int32_t* idx, int B, int Lq, int Lk, int q_pos0,
                    int k, void* stream);

/*
 * dsa_sparse_mla_workspace_size - bytes of workspace dsa_sparse_mla_fwd needs for
 * this shape (0 when it runs without key splitting).
 */
size_t dsa_sparse_mla_workspace_size(int B, int Lq, int Lk, int H, int Dqk, int Dv, int k);

/*
 * dsa_sparse_mla_fwd - MLA attention in MQA mode over the selected latent rows
 * ("Key claims", section 2.1 Eq. 2 / Fig. 2; "Method": the latent vector is shared
 * by all query heads of a token).
 *   q    [B, Lq, H, Dqk] bf16 queries
 *   kv   [B, Lk, Dqk] bf16 latent rows c_s; the values are c_s[0:Dv]
 *   idx  [B, Lq, k] int32 selected keys; entries < 0 or >= Lk are skipped
 *   out  [B, Lq, H, Dv] bf16 output (round to nearest even from fp32):
 *          out[h] = sum_s softmax_s(sm_scale * q[h] . c_s) * c_s[0:Dv]
 *   lse  [B, Lq, H] fp32 natural-log log-sum-exp of the scaled logits, or NULL.
 *        A row with no valid key gets out = 0 and lse = -INFINITY.
 *   ws   workspace of at least dsa_sparse_mla_workspace_size(...) bytes.
 */
int dsa_sparse_mla_fwd(const uint16_t* q, const uint16_t* kv, const int32_t* idx, uint16_t* out,
                       float* lse, int B, int Lq, int Lk, int H, int Dqk, int Dv, int k,
                       float sm_scale, void* ws, size_t ws_bytes, void* stream);

/*
 * dsa_sparse_mla_fwd_noalloc - dsa_sparse_mla_fwd for callers that cannot
 * allocate device memory. (The paper has no counterpart: this is a deployment
 * convenience of this library.) Some callers cannot call cudaMalloc or hand
 * over a workspace: plugins running inside a host framework that reserves all
 * device memory up front, or code paths where the implicit synchronisation of
 * an allocation is not acceptable. This entry point takes the same inputs and
 * outputs as dsa_sparse_mla_fwd and calls no allocator: the key-split partial
 * results live in a 16 MiB array compiled into the library, which every GPU
 * that loads the library holds until the process exits.
 *   - When the partials of the recommended number of key splits (the one
 *     dsa_sparse_mla_workspace_size sizes for) need more than 16 MiB, the
 *     largest number of splits whose partials fit is used instead (one split
 *     needs none), so every shape dsa_sparse_mla_fwd accepts is accepted.
 *   - The first call on a device looks up the array's device address with the
 *     device current; make that first call before any stream capture.
 *   - That address is kept for the life of the process. cudaDeviceReset
 *     unloads the library's device code, so after a reset the kept address is
 *     stale: do not call this entry point again in that process.
 *   - All calls share the one array and every call fully overwrites the part it
 *     uses (nothing needs clearing), so calls that overlap on the GPU (other
 *     streams, other host threads) race with each other: serialise them.
 *   - Results equal dsa_sparse_mla_fwd's for the same shape when the
 *     recommended splits fit, and otherwise differ from them only by the
 *     rounding of a different merge order.
 */
int dsa_sparse_mla_fwd_noalloc(const uint16_t* q, const uint16_t* kv, const int32_t* idx,
                               uint16_t* out, float* lse, int B, int Lq, int Lk, int H, int Dqk,
                               int Dv, int k, float sm_scale, void* stream);

/*
 * dsa_indexer_kl - the indexer alignment target, forward only: for every query
 * token, KL(p || r) between the main attention aggregated over heads and the
 * lightning indexer's distribution, both over the token's key set.
 * ("DeepSeek-V3.2: Pushing the Frontier of Open Large Language Models", bud-325
 * paper digest: "Key claims", paper section 2.1.1 Eq. 3-4, given in words - a
 * KL-divergence loss aligns the indexer output with the main attention
 * aggregated over heads, in the dense warm-up; "Method" - in the sparse stage
 * the KL is taken on the selected tokens. The equations are not printed; this is
 * the plain reading.) For token t with key set S = the valid entries of idx[t,:]:
 *     a[h,s] = exp(sm_scale * q[t,h] . kv[s] - lse[t,h])   (attention of head h)
 *     p_s    = sum_h a[h,s] / H                           (L1-normalised aggregate)
 *     r_s    = exp(sel[t,s]) / sum_{s' in S} exp(sel[t,s'])
 *     KL_t   = sum_{s in S} p_s (ln p_s - ln r_s)          (terms with p_s = 0 are 0)
 * For the dense warm-up pass every causal key in idx (k >= the token's position
 * + 1); for the sparse stage pass the top-k set of dsa_forward.
 *   q          [B, Lq, H, Dqk] bf16                  (as dsa_sparse_mla_fwd)
 *   kv         [B, Lk, Dqk] bf16 latent rows
 *   idx        [B, Lq, k] int32; entries < 0 or >= Lk are not in the set
 *   lse        [B, Lq, H] fp32: natural-log log-sum-exp over S of the scaled
 *              logits, as dsa_sparse_mla_fwd / dsa_forward return it for the
 *              same idx (it makes each head's a[h,:] sum to 1)
 *   sel_scores [B, Lq, k] fp32: index scores I[t, idx[t,j]], aligned with idx
 *              (entries outside the set are ignored)
 *   p_out      [B, Lq, k] fp32 or NULL: p at each slot of idx, 0 outside the set
 *   kl_out     [B, Lq] fp32: KL_t (0 for a token with an empty set)
 *   (H, Dqk) in {(128, 576), (8, 80)}; k a multiple of 32 in [32, 4096].
 * All pointers are caller-owned device memory, 16-byte aligned; nothing is
 * allocated. Errors: DSA_ERR_INVALID_ARG (null or misaligned pointer, bad
 * sm_scale), DSA_ERR_UNSUPPORTED_SHAPE, DSA_ERR_CUDA (launch), and a device
 * wait that ran out is reported by dsa_check_status.
 */
int dsa_indexer_kl(const uint16_t* q, const uint16_t* kv, const int32_t* idx, const float* lse,
                   const float* sel_scores, float* p_out, float* kl_out, int B, int Lq, int Lk,
                   int H, int Dqk, int k, float sm_scale, void* stream);

/*
 * Sparse training stage: gradients. ("DeepSeek-V3.2: Pushing the Frontier of
 * Open Large Language Models", bud-325 paper digest, "Method": in the sparse
 * stage the main model is trained through attention over the top-k selected
 * entries, and the indexer keeps training on the KL over the selected tokens with
 * its input detached from the main model's graph.) The contractions run as
 * batched bf16 GEMMs on the tensor cores (tcgen05, fp32 accumulation) over the
 * selected rows, gathered per chunk of up to 64 tokens into the workspace; the
 * gathers, the softmax / ReLU gradients and the scatter-add of key gradients are
 * kernels of this library too, and nothing is allocated. Key gradients are
 * accumulated with atomics, so their last bits may differ from run to run. All
 * pointers are caller-owned device memory, 16-byte aligned.
 * Errors: DSA_ERR_INVALID_ARG (null or misaligned pointer, bad scalar),
 * DSA_ERR_UNSUPPORTED_SHAPE, DSA_ERR_WORKSPACE_TOO_SMALL (below one token's
 * share), DSA_ERR_CUDA (a launch failed); a device wait that ran out is reported
 * by dsa_check_status.
 *
 * dsa_sparse_mla_bwd - gradients of the sparse attention (dsa_sparse_mla_fwd)
 * with respect to q and the latent rows, given dout = dL/d(out). With
 * z[h,s] = sm_scale q[h].c_s over the valid slots s of idx[t,:], P = exp(z - lse)
 * and dP[h,s] = dout[h] . c_s[:Dv]:
 *     D[h]    = sum_s P[h,s] dP[h,s] / sum_s P[h,s]    (= dout[h] . out[h])
 *     dz[h,s] = sm_scale P[h,s] (dP[h,s] - D[h])
 *     dq[h]   = sum_s dz[h,s] c_s                      (all Dqk columns)
 *     dkv[s] += sum_h dz[h,s] q[h]   and, on columns < Dv, sum_h P[h,s] dout[h]
 *   D is formed from the recomputed fp32 P and dP rather than from the forward's
 *   bf16 output, whose bf16-rounded P would dominate dP - D on short sets.
 *   q [B, Lq, H, Dqk], kv [B, Lk, Dqk], dout [B, Lq, H, Dv]: bf16; idx [B, Lq, k]
 *   int32 (slots < 0 or >= Lk skipped); lse [B, Lq, H] fp32 as the forward
 *   returned it; dq [B, Lq, H, Dqk] fp32 (overwritten);
 *   dkv [B, Lk, Dqk] fp32, zeroed first unless accumulate_dkv != 0.
 *   (H, Dqk, Dv) in {(8, 80, 64), (128, 576, 512)}; k a multiple of 32 in
 *   [32, 4096]. P and dz enter their GEMMs rounded to bf16.
 *   ws: dsa_sparse_mla_bwd_workspace_size(...) bytes (about 10 MB per token of a
 *   chunk at H = 128, k = 2048); less makes smaller chunks.
 */
size_t dsa_sparse_mla_bwd_workspace_size(int B, int Lq, int H, int Dqk, int Dv, int k);
int dsa_sparse_mla_bwd(const uint16_t* q, const uint16_t* kv, const int32_t* idx,
                       const float* lse, const uint16_t* dout, float* dq, float* dkv,
                       int accumulate_dkv, int B, int Lq, int Lk, int H, int Dqk, int Dv, int k,
                       float sm_scale, void* ws, size_t ws_bytes, void* stream);

/*
 * dsa_indexer_kl_grad - dI = loss_scale * (r - p): the gradient of
 * loss_scale * KL(p || r) (dsa_indexer_kl) with respect to the selected index
 * scores, p held fixed (the indexer's input is detached), r = softmax over the
 * set of sel_scores. sel_scores, p (dsa_indexer_kl's p_out), dI: [B, Lq, k] fp32;
 * idx [B, Lq, k] int32, slots < 0 or >= Lk get 0. k a multiple of 32 in
 * [32, 4096]; loss_scale finite.
 */
int dsa_indexer_kl_grad(const float* sel_scores, const float* p, const int32_t* idx, float* dI,
                        int B, int Lq, int Lk, int k, float loss_scale, void* stream);

/*
 * dsa_indexer_bwd - gradients of L = sum_{t,j} dI[t,j] I[t, idx[t,j]] (Eq. 1) with
 * respect to the dequantised indexer inputs q^I = s^q qhat, k^I = s^k khat and
 * the weights w; the FP8 rounding is passed through as the identity. With
 * x[j,s] = q^I[t,j] . k^I[s]:
 *     dw[t,j]   = sum_s dI[t,s] max(x[j,s], 0)
 *     g[j,s]    = dI[t,s] w[t,j] [x[j,s] > 0]
 *     dqI[t,j]  = sum_s g[j,s] k^I[s]
 *     dkI[s]   += sum_{t,j} g[j,s] q^I[t,j]
 *   qI [B, Lq, H_I, d_I] and kI [B, Lk, d_I] e4m3 codes, qI_scale [B, Lq, H_I],
 *   kI_scale [B, Lk], w [B, Lq, H_I] (w_dtype) as for dsa_indexer_scores;
 *   idx, dI [B, Lq, k] aligned (slots < 0 or >= Lk skipped); dqI
 *   [B, Lq, H_I, d_I], dw [B, Lq, H_I] fp32 (overwritten); dkI [B, Lk, d_I] fp32,
 *   zeroed first unless accumulate_dkI != 0. The code dots qhat . khat run on
 *   the tensor cores with fp32 accumulation (every product of two e4m3 codes is
 *   exact); wherever their rounding could flip the sign (|X| within 2^-12
 *   |qhat| |khat| of zero) the dot is recomputed exactly in fp64, so the ReLU mask
 *   is the exact code dot's. The gradient factors g enter the two remaining
 *   products as three bf16 terms each (24 significant bits).
 *   ws: dsa_indexer_bwd_workspace_size(...) bytes; less makes smaller chunks.
 */
size_t dsa_indexer_bwd_workspace_size(int B, int Lq, int H_I, int d_I, int k);
int dsa_indexer_bwd(const uint8_t* qI, const float* qI_scale, const uint8_t* kI,
                    const float* kI_scale, const void* w, int w_dtype, const int32_t* idx,
                    const float* dI, float* dqI, float* dkI, float* dw, int accumulate_dkI, int B,
                    int Lq, int Lk, int H_I, int d_I, int k, void* ws, size_t ws_bytes,
                    void* stream);

/*
 * Decode with one sequence's key cache split over G devices ("Key claims",
 * section 2.1: the top-k over I[t,:] and attention over the selected entries).
 * Shard g holds keys [shard_lo[g], shard_lo[g] + len_g) of every sequence, the
 * shards in key order. Per step:
 *   1. each device selects the top-k of its shard: dsa_forward on its shard as a
 *      decode problem (Lk = len_g, q_pos0 = len_g - 1) with out = NULL, idx_out
 *      and sel_scores_out;
 *   2. the candidates (sel_scores_out, idx_out) of all shards are all-gathered
 *      (a collective of the caller's) and merged: dsa_topk_merge;
 *   3. each device takes its view of the merged selection (dsa_index_localize)
 *      and attends over it with dsa_sparse_mla_fwd on its shard, giving out_g
 *      and lse_g (zeros and -inf where the shard holds none of the keys);
 *   4. the pairs (out_g, lse_g) are all-gathered and combined: dsa_attn_combine.
 * The merged selection equals the unsplit one bit for bit: a key among the k
 * largest overall is among the k largest of its shard under the same tie rule,
 * and the merge keeps (score descending, lower global index first). The output
 * is the lse-weighted mean of the partial outputs, each rounded to bf16 once.
 *
 * dsa_topk_merge - the top-k of G shards' candidate lists.
 *   cand_scores [G, R, k] fp32 and cand_idx [G, R, k] int32 (shard-local key
 *   indices, ascending, < 0 for no candidate), device; shard_lo [G] int64, host:
 *   first key of each shard, increasing; G in [1, 16]; k a multiple of 32 in
 *   [32, 4096]. idx_out [R, k] int32: the k best candidates by (score
 *   descending, global index ascending), as global indices in ascending order,
 *   -1 padded when fewer than k candidates exist; sel_out [R, k] fp32 or NULL:
 *   their scores (0 at padding). ws: dsa_topk_merge_workspace_size(G, R, k)
 *   bytes, caller-owned device memory.
 * dsa_index_localize - idx_local[i] = idx[i] - lo for lo <= idx[i] < lo + len,
 *   else -1 (n int32 entries, device).
 * dsa_attn_combine - out[r, h, :] = sum_g exp(lse_g - L) out_g[r, h, :] with
 *   L = ln sum_g exp(lse_g) (lse_out, optional): part_out [G, R, H, Dv] bf16 and
 *   part_lse [G, R, H] fp32 as dsa_sparse_mla_fwd returns them; out [R, H, Dv]
 *   bf16 (round to nearest even). A row with every lse_g = -inf gives zeros and
 *   L = -inf.
 * All pointers 16-byte aligned; nothing is allocated. Errors as for the other
 * calls (DSA_ERR_INVALID_ARG, DSA_ERR_UNSUPPORTED_SHAPE,
 * DSA_ERR_WORKSPACE_TOO_SMALL, DSA_ERR_CUDA).
 */
size_t dsa_topk_merge_workspace_size(int G, int R, int k);
int dsa_topk_merge(const float* cand_scores, const int32_t* cand_idx, const long long* shard_lo,
                   int G, int R, int k, int32_t* idx_out, float* sel_out, void* ws,
                   size_t ws_bytes, void* stream);
int dsa_index_localize(const int32_t* idx, int32_t* idx_local, long long n, int lo, int len,
                       void* stream);
int dsa_attn_combine(const uint16_t* part_out, const float* part_lse, int G, int R, int H, int Dv,
                     uint16_t* out, float* lse_out, void* stream);

/*
 * dsa_last_launch_count - number of kernel launches that the calling thread's
 * last dsa_forward, dsa_forward_host, dsa_forward_profiled, dsa_sparse_mla_bwd,
 * dsa_indexer_bwd or dsa_indexer_kl_grad call enqueued (all of this library's
 * kernels, on the caller's stream and on the library's internal side stream).
 * 0 before the first call. For benchmarks that report how many
 * of the library's kernels ran in a timed region.
 */
int dsa_last_launch_count(void);

/* Whole-path problem description for dsa_forward. */
typedef struct dsa_problem {
  int mode;        /* DSA_MODE_PREFILL or DSA_MODE_DECODE (informational; the
                      shape decides the schedule) */
  int B, Lq, Lk, q_pos0;
  int H_I, d_I;    /* indexer heads, head dim */
  int H, Dqk, Dv;  /* attention heads, latent key width, value width */
  int k;           /* top-k */
  float sm_scale;
  int w_dtype;     /* DSA_DTYPE_F32 or DSA_DTYPE_BF16 */
} dsa_problem;

/* Tensors of one dsa_forward call; shapes as in the calls above. */
typedef struct dsa_tensors {
  const uint8_t* qI;
  const float* qI_scale;
  const uint8_t* kI;
  const float* kI_scale;
  const void* w;
  const uint16_t* q;
  const uint16_t* kv;
  uint16_t* out;    /* [B, Lq, H, Dv] bf16; NULL for a selection-only call, which
                       stops after the top-k (idx_out then required; q, kv and lse
                       are not read) */
  float* lse;       /* [B, Lq, H] fp32, optional (NULL) */
  int32_t* idx_out; /* [B, Lq, k] int32, optional: the selected set */
  float* sel_scores_out; /* [B, Lq, k] fp32, optional: the index score I[t, idx_out[t, j]]
                            of every selected key, aligned with idx_out (0 at the -1
                            padding); what dsa_indexer_kl takes as sel_scores. When
                            given, rows with p + 1 <= k are scored too. Needs idx_out. */
} dsa_tensors;

/* Bytes of workspace dsa_forward needs for problem p (scores are streamed in
 * query chunks, so this is far below B*Lq*Lk*4). */
size_t dsa_forward_workspace_size(const dsa_problem* p);

/*
 * dsa_forward - the hot path: indexer -> top-k -> sparse MLA, for prefill
 * (q_pos0 = 0) and decode (q_pos0 = Lk - Lq). Query rows with p + 1 <= k select
 * every causal key without scoring (the top-k of at most k candidates is all of
 * them). The score matrix is produced and consumed one query chunk at a time in
 * the workspace (a chunk stays in L2): the indexer scores a half-chunk while the
 * top-k of the previous one runs on a library-owned stream. Results equal
 * dsa_indexer_scores + dsa_topk_select + dsa_sparse_mla_fwd.
 */
int dsa_forward(const dsa_problem* p, const dsa_tensors* t, void* ws, size_t ws_bytes,
                void* stream);

/*
 * dsa_forward_fused - dsa_forward with the top-k selection inside the indexer
 * kernel: selector warps of each persistent indexer CTA pick a row's top-k from
 * the score chunk (in L2) as soon as every piece of the row is scored, while the
 * CTA's other warps score further rows. One cooperative launch per chunk (every
 * CTA resident at once, so the waits between CTAs always end; they are bounded
 * as well). Same arguments, workspace (dsa_forward_workspace_size) and results,
 * bit for bit, as dsa_forward; sel_scores_out is supported. On B200 it is slower
 * than dsa_forward: the few selector threads that fit beside the indexer's warps
 * take longer to select than the separate top-k kernel needs.
 */
int dsa_forward_fused(const dsa_problem* p, const dsa_tensors* t, void* ws, size_t ws_bytes,
                      void* stream);

/*
 * Paged, variable-length caches (a serving layout; the pages describe the method
 * only, so this is a plain reading: each sequence's keys are the tokens of its
 * own cache, "Key claims" section 2.1, and the query rows are its newest tokens).
 * The latent rows kv, index keys kI and key scales kI_scale of every sequence live
 * in shared pools of num_pages pages of page_size tokens. Logical key s of sequence
 * b is pool row block_table[b][s / page_size] * page_size + s % page_size.
 */
typedef struct dsa_paged_cache {
  const int32_t* block_table; /* [B, max_blocks] device: pool page of each logical block */
  const int32_t* seq_lens;    /* [B] device: tokens in each sequence's cache, its Lq query
                                 rows included (query row t sits at seq_lens[b] - Lq + t) */
  int max_blocks;             /* logical blocks per sequence; Lk = max_blocks * page_size */
  int page_size;              /* tokens per page: a positive multiple of 128 */
  int num_pages;              /* pages in each pool */
} dsa_paged_cache;

/*
 * dsa_forward_paged - dsa_forward over a paged cache with per-sequence lengths.
 * p: as for dsa_forward with Lk = max_blocks * page_size (the capacity of one
 * sequence); q_pos0 is ignored (the positions come from seq_lens). t: qI,
 * qI_scale, w, q as for dsa_forward ([B, Lq, ...]); kv [num_pages * page_size,
 * Dqk], kI [num_pages * page_size, d_I] and kI_scale [num_pages * page_size] are
 * the pools. Each row's candidates are keys 0 .. seq_lens[b] - Lq + t of its own
 * sequence, selected by the same top-k rule; idx_out holds logical key positions.
 * ws: at least dsa_forward_paged_workspace_size(p) bytes. Device-side contents are
 * not validated: seq_lens outside [Lq, Lk] or page numbers outside [0, num_pages)
 * give unspecified results but never an out-of-bounds access (a page number
 * outside the pool reads pool row 0 or zeros). Errors as for dsa_forward, plus
 * DSA_ERR_INVALID_ARG / DSA_ERR_UNSUPPORTED_SHAPE for the cache description.
 */
size_t dsa_forward_paged_workspace_size(const dsa_problem* p);
int dsa_forward_paged(const dsa_problem* p, const dsa_tensors* t, const dsa_paged_cache* c,
                      void* ws, size_t ws_bytes, void* stream);

/*
 * dsa_forward_host - dsa_forward on HOST tensors: copies every input from host
 * memory (pinned for asynchronous copies) into the caller's device staging
 * buffers `dev` (same layout as dsa_tensors, all device pointers), runs
 * dsa_forward, copies out (and lse/idx_out when both host and device pointers are
 * given) back to host, and waits for the stream. `host` holds host pointers.
 * With Lq >= 1024 the call is pipelined per sequence in blocks of 4096 query rows
 * (a remainder under 1024 rows joins the block before it): a block's query rows
 * and the keys it newly needs are copied in on a library-owned stream while the
 * previous block computes on `stream`, and its results are copied out on a second
 * library-owned stream while later blocks compute. Rows are independent, so the
 * results equal one dsa_forward over all rows. The copies begin after the work
 * already queued on `stream`; the call returns when all of them are done. ws:
 * as for dsa_forward over the whole problem. Errors as for dsa_forward; a failed
 * copy returns DSA_ERR_CUDA.
 */
int dsa_forward_host(const dsa_problem* p, const dsa_tensors* host, const dsa_tensors* dev,
                     void* ws, size_t ws_bytes, void* stream);

/* Kernel kinds reported by dsa_forward_profiled. */
#define DSA_KIND_INDEXER 1
#define DSA_KIND_TOPK 2
#define DSA_KIND_SPARSE_MLA 3
#define DSA_KIND_COMBINE 4
#define DSA_KIND_INDEXER_TOPK 5   /* the fused indexer + top-k launch */

/*
 * dsa_forward_profiled - dsa_forward that also records a CUDA event around each
 * kernel launch, for per-kernel timing on the launching stream.
 *   events        max_launches + 1 caller-created cudaEvent_t (as void*): events[0]
 *                 is recorded before the first launch, events[i + 1] after launch i
 *   kinds         [max_launches] out: DSA_KIND_* of launch i
 *   n_launches    out: number of kernel launches made
 * Fails with DSA_ERR_INVALID_ARG (after enqueueing part of the work) if the call
 * needs more than max_launches launches; results are otherwise identical to
 * dsa_forward.
 */
int dsa_forward_profiled(const dsa_problem* p, const dsa_tensors* t, void* ws, size_t ws_bytes,
                         void* stream, void* const* events, int* kinds, int max_launches,
                         int* n_launches);

/*
 * dsa_check_status - wait for `stream`, then read and clear the device status
 * word. Returns DSA_OK, DSA_ERR_TIMEOUT (a bounded wait ran out; the message names
 * the kernel) or DSA_ERR_CUDA (a launch or execution error).
 */
int dsa_check_status(void* stream);

/*
 * dsa_set_wait_limit_ns - bound on every device-side wait, in nanoseconds
 * (default 2e9). Used by tests to make a wait run out on purpose.
 */
int dsa_set_wait_limit_ns(unsigned long long ns);

/*
 * dsa_debug_wait_timeout - launch one small kernel that waits on an mbarrier no
 * one arrives at, bounded by the current wait limit, so that tests can check the
 * timeout path: afterwards dsa_check_status() returns DSA_ERR_TIMEOUT.
 */
int dsa_debug_wait_timeout(void* stream);

#ifdef __cplusplus
}
#endif

#endif /* DSA_H_ */
