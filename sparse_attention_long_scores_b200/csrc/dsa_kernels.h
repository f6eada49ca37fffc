// dsa_kernels.h - host-side launch interface of the DSA kernels (internal).
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "dsa_common.cuh"

namespace dsa {

// ---------------- lightning indexer (Eq. 1) ----------------
struct IndexerArgs {
  const float* qI_scale;  // [B, Lq, H_I]
  const void* w;          // [B, Lq, H_I] fp32 or bf16
  int w_bf16;
  const float* kI_scale;  // [B, Lk]
  float* scores;          // row (b, t) at scores + (b * sc_bstride + t - sc_t0) * sc_ld
  long long sc_ld;
  long long sc_bstride;
  int sc_t0;
  int B, Lq, Lk, q_pos0;
  int t_lo, t_hi;    // query rows [t_lo, t_hi) of every sequence are scored
  int piece_keys;    // keys per work unit (multiple of 128)
  // optional paged cache (see key_row / seq_pos0): kI and kI_scale are then pools of
  // num_pages * page_size rows, and sequence b's rows sit at seq_lens[b] - Lq + t
  const int32_t* seq_lens;
  const int32_t* block_table;
  int max_blocks, page_size, num_pages;
  // Fused top-k selection (select != 0): selector warps of the same kernel pick the
  // k largest scores of every row of rows [sel_t0, sel_t1) of each sequence once all
  // pieces of the row are scored (rows of at most k candidates select every key);
  // the scored rows [t_lo, t_hi) lie inside that range.
  int select;
  int k;
  int sel_t0, sel_t1;
  int32_t* idx;          // [B, Lq, k] selected keys, ascending, -1 padded
  float* sel_scores;     // [B, Lq, k] or null: the index score of each selected key (0 at padding)
  int* row_cnt;          // [B * (sel_t1 - sel_t0)] pieces scored per row; zero on entry, left zero
  DevCtl ctl;
};

// Launch the tcgen05 FP8 indexer for (H_I, d_I) in {(4,32), (64,128)}. With
// a.select set the launch is cooperative (every CTA resident at once).
// `decode_like` selects the one-token-per-block variant (Lq == 1).
cudaError_t launch_indexer(const CUtensorMap& tmap_q, const CUtensorMap& tmap_k,
                           const IndexerArgs& a, int H_I, int d_I, int num_sms,
                           cudaStream_t stream);

// scores[b,t,s] = -inf for s > q_pos0 + t (public score matrix only).
cudaError_t launch_fill_noncausal(float* scores, int B, int Lq, int Lk, int q_pos0,
                                  cudaStream_t stream);

// ---------------- top-k selection ----------------
struct TopkArgs {
  const float* scores;  // row (b, t) at scores + (b * sc_bstride + t - sc_t0) * sc_ld
  long long sc_ld;
  long long sc_bstride;
  int sc_t0;
  int32_t* idx;  // [B, Lq, k]
  int B, Lq, Lk, q_pos0, k;
  int t_lo, t_hi;  // rows [t_lo, t_hi) of every sequence
  int vec4;        // rows are 16-byte aligned (sc_ld % 4 == 0, aligned base)
  const int32_t* seq_lens;   // [B] or null: per-sequence lengths (row t at seq_lens[b] - Lq + t)
  float* sel;      // [B, Lq, k] or null: score of each selected key (0 at padding); rows with
                   // at most k candidates then read their scores too
  DevCtl ctl;
};
cudaError_t launch_topk(const TopkArgs& a, int num_sms, cudaStream_t stream);

// ---------------- sparse MLA (MQA mode) ----------------
struct MlaArgs {
  const uint16_t* q;   // [B, Lq, H, Dqk] bf16
  const int32_t* idx;  // [B, Lq, k]
  uint16_t* out;       // [B, Lq, H, Dv] bf16
  float* lse;          // [B, Lq, H] or null
  float* part_o;       // [tokens, splits, H, Dv] fp32 (splits > 1)
  float* part_ml;      // [tokens, splits, H, 2]   (splits > 1)
  int B, Lq, Lk, H, Dqk, Dv, k;
  float scale_log2;    // sm_scale * log2(e)
  int n_dv;            // value chunks per token
  int splits;          // key splits per token
  int wave;            // CTAs resident at once (one per SM): the next CTA an SM runs
                       // is about this many block indices further on
  // optional paged latent cache (see key_row): kv is then a pool of
  // num_pages * page_size rows
  const int32_t* block_table;
  int max_blocks, page_size, num_pages;
  DevCtl ctl;
};
// (H, Dqk, Dv) in {(8,80,64), (128,576,512)}.
cudaError_t launch_sparse_mla(const CUtensorMap& tmap_q, const uint16_t* kv, const MlaArgs& a,
                              cudaStream_t stream);
cudaError_t launch_mla_combine(const MlaArgs& a, cudaStream_t stream);

// ---------------- indexer alignment target (KL, forward) ----------------
struct KlArgs {
  const uint16_t* q;   // [B, Lq, H, Dqk] bf16
  const int32_t* idx;  // [B, Lq, k] key set of each query token (entries < 0 are not in it)
  const float* lse;    // [B, Lq, H] natural-log log-sum-exp of the scaled logits over the set
  const float* sel;    // [B, Lq, k] index scores of the selected keys, aligned with idx
  float* p_out;        // [B, Lq, k] or null: aggregated attention target (0 outside the set)
  float* kl_out;       // [B, Lq]
  int B, Lq, Lk, H, Dqk, k;
  float scale_log2;    // sm_scale * log2(e)
  DevCtl ctl;
};
// (H, Dqk) in {(8, 80), (128, 576)}.
cudaError_t launch_indexer_kl(const uint16_t* kv, const KlArgs& a, cudaStream_t stream);

// ---------------- sparse-stage gradients (backward.cu) ----------------
// Chunk of T tokens starting at flattened token tok0 (sequence tok / Lq); slot j
// of token tok is key idx[tok * k + j], skipped outside [0, Lk).
// out [T, k, D] bf16 = the selected rows of kv [B, Lk, D] (zeros for skipped
// slots); D % 8 == 0.
cudaError_t launch_gather_rows_bf16(const uint16_t* kv, const int32_t* idx, uint16_t* out,
                                    long long tok0, int T, int Lq, int Lk, int k, int D,
                                    int num_sms, cudaStream_t stream);
// qo [T, 2H, Dqk] bf16 = per token the H rows of q [B*Lq, H, Dqk] and the H rows of
// dout [B*Lq, H, Dv] padded with zeros to Dqk columns; Dqk % 8 == 0, Dv % 8 == 0.
cudaError_t launch_pack_qo(const uint16_t* q, const uint16_t* dout, uint16_t* qo, long long tok0,
                           int T, int H, int Dqk, int Dv, int num_sms, cudaStream_t stream);
// PZ [T, 2H, k] bf16 (rows of dz, then rows of P) from SP [T, 2H, k] fp32 (rows of
// raw q.c, then rows of dout.c[:Dv]) and lse [B*Lq, H].
cudaError_t launch_mla_bwd_softmax(const float* SP, const float* lse, const int32_t* idx,
                                   uint16_t* PZ, long long tok0, int T, int H, int k, int Lk,
                                   float sm_scale, int num_sms, cudaStream_t stream);
// out [T, k, d_I] bf16 = the selected e4m3 rows of kI [B, Lk, d_I] (codes, exact).
cudaError_t launch_gather_e4m3_rows_bf16(const uint8_t* kI, const int32_t* idx, uint16_t* out,
                                         long long tok0, int T, int Lq, int Lk, int k, int d_I,
                                         int num_sms, cudaStream_t stream);
// out [n] bf16 = e4m3 codes [n] (exact).
cudaError_t launch_decode_e4m3_bf16(const uint8_t* codes, uint16_t* out, long long n, int num_sms,
                                    cudaStream_t stream);
// ReLU gradient of the indexer from the tensor-core code dots XT [T, k, H_I] fp32:
// G1s [T, H_I, 3 kp] and G2s [T, 3 hp, k] bf16 (three-term splits of G1 / G2, zero
// padded), dw [B*Lq, H_I] += the weight gradient (zeroed by the caller). The ReLU
// mask is the sign of the exact code dot. H_I <= 64, d_I <= 128.
cudaError_t launch_indexer_bwd_relu_tc(const float* XT, const uint16_t* Kb, const uint16_t* Qb,
                                       const int32_t* idx, const float* dI,
                                       const float* qI_scale, const float* kI_scale,
                                       const void* w, int w_bf16, uint16_t* G1s, uint16_t* G2s,
                                       float* dw, long long tok0, int T, int Lq, int Lk, int H_I,
                                       int d_I, int k, int kp, int hp, cudaStream_t stream);
// dI [rows, k] = loss_scale (softmax over the set of sel - p).
cudaError_t launch_kl_score_grad(const float* sel, const float* p, const int32_t* idx, float* dI,
                                 long long rows, int k, int Lk, float loss_scale, int num_sms,
                                 cudaStream_t stream);

// ---------------- batched tensor-core GEMM (sparse-stage gradients) ----------------
// C[z] (fp32) = A[z] B[z]^T for z < batch: A is M x K, B is N x K, bf16, each
// K-major (stored [M][K] / [N][K]) or MN-major (stored [K][M] / [K][N]) as given
// by a_mn / b_mn; the tensor maps (built by the caller) are 3-D {inner, rows, z}
// with 128-byte swizzle and boxes {64, 128} (A, K-major), {64, bn} (B, K-major)
// or {64, 64} (MN-major). K tile kt of A reads A's tile kt % a_kt (B likewise).
struct BgemmArgs {
  int M, N, K;
  int a_kt, b_kt;
  float* C;                  // element (z, m, n) at C + z * sC + m * c_sm + n * c_sn
  long long c_sm, c_sn, sC;
  // Scatter-add mode (sidx != null, c_sn == 1): row m of batch z is added with fp32
  // atomics into row s = sidx[(s_tok0 + z) * s_k + m] of sequence (s_tok0 + z) / s_Lq,
  // i.e. at C + (((s_tok0 + z) / s_Lq) * s_Lk + s) * c_sm; rows with s outside
  // [0, s_Lk) are dropped (sC is unused).
  const int32_t* sidx;
  long long s_tok0;
  int s_k, s_Lq, s_Lk;
  DevCtl ctl;
};
// Tile width (N) used for an N-column product: 64, 128, 192 or 256.
int bgemm_tile_n(int N);
cudaError_t launch_bgemm(const CUtensorMap& ta, const CUtensorMap& tb, const BgemmArgs& a,
                         int batch, bool a_mn, bool b_mn, int bn, cudaStream_t stream);

// ---------------- split key cache (decode over G devices) ----------------
struct ShardOffsets {
  long long v[16];   // first key of shard g
};
// ext_scores / ext_idx [R][G k] from the shards' candidates [G][R][k] (score and
// shard-local index, < 0 none): -inf and -1 where there is no candidate.
cudaError_t launch_cp_pack(const float* cand_scores, const int32_t* cand_idx,
                           const ShardOffsets& lo, int G, long long R, int k, float* ext_scores,
                           int32_t* ext_idx, int num_sms, cudaStream_t stream);
// idx_out [R][k] = global indices of the selected positions pos [R][k], keyless
// ones dropped, ascending then -1; sel [R][k] (optional) compacted alongside.
cudaError_t launch_cp_map_compact(const int32_t* pos, const int32_t* ext_idx, long long R, int n,
                                  int k, int32_t* idx_out, float* sel, int num_sms,
                                  cudaStream_t stream);
cudaError_t launch_cp_localize(const int32_t* idx, int32_t* out, long long n, int lo, int len,
                               int num_sms, cudaStream_t stream);
// out [rows][Dv] bf16 (and lse_out [rows], optional) from G partial pairs
// part_out [G][rows][Dv] bf16, part_lse [G][rows].
cudaError_t launch_cp_combine(const uint16_t* part_out, const float* part_lse, int G,
                              long long rows, int Dv, uint16_t* out, float* lse_out, int num_sms,
                              cudaStream_t stream);

// ---------------- debug ----------------
cudaError_t launch_debug_wait(DevCtl ctl, cudaStream_t stream);

}  // namespace dsa
