// context_parallel.cu - decode with one sequence's key cache split over G
// devices: shard g holds keys [lo_g, lo_g + len_g) of every sequence. Each
// device selects the top-k of its own shard, the (score, index) candidates of
// all shards are gathered and merged into the global top-k, each device attends
// over the selected keys that lie in its shard, and the partial (out, lse) pairs
// are combined with log-sum-exp weights. The global selection is the top-k of
// the union of the shards' top-k sets (a key among the k largest overall is
// among the k largest of its shard, ties going to the lower index in both), and
// attention over a union of disjoint key sets is the lse-weighted mean of the
// per-set attentions ("DeepSeek-V3.2: Pushing the Frontier of Open Large
// Language Models", bud-325 paper digest, "Key claims", section 2.1 and Eq. 2).
//
// The merge runs the library's exact top-k on the concatenated candidates:
// shards are concatenated in key order and each shard's list is ascending, so a
// candidate's position orders it exactly as its global index does.
#include <cuda_bf16.h>

#include "dsa_kernels.h"

namespace dsa {
namespace {

constexpr int kCpThreads = 256;

// ext_scores / ext_idx [R][G k]: row r, position g k + j = candidate j of shard g
// (score, global index); candidates without a key get -inf and -1.
__global__ void cp_pack_kernel(const float* __restrict__ cs, const int32_t* __restrict__ ci,
                               ShardOffsets lo, int G, long long R, int k,
                               float* __restrict__ ext_scores, int32_t* __restrict__ ext_idx) {
  const long long n = (long long)G * R * k;
  for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < n;
       e += (long long)gridDim.x * blockDim.x) {
    const int j = (int)(e % k);
    const long long r = (e / k) % R;
    const int g = (int)(e / ((long long)k * R));
    const int32_t s = ci[e];
    const long long dst = r * (long long)G * k + (long long)g * k + j;
    ext_scores[dst] = s >= 0 ? cs[e] : -INFINITY;
    ext_idx[dst] = s >= 0 ? (int32_t)(lo.v[g] + s) : -1;
  }
}

// Row r: positions pos[r][0..k) chosen by the top-k (ascending, -1 padded) ->
// global indices, the ones without a key dropped and the rest moved to the
// front in order, -1 behind; the selected scores (sel, optional) move along,
// 0 at padding. One warp per row, 32 slots at a time (a slot is written only
// after the warp has read it).
__global__ void cp_map_compact_kernel(const int32_t* __restrict__ pos,
                                      const int32_t* __restrict__ ext_idx, long long R, int n,
                                      int k, int32_t* __restrict__ idx_out, float* sel) {
  const int lane = threadIdx.x & 31;
  const long long warps = (long long)gridDim.x * blockDim.x / 32;
  for (long long r = ((long long)blockIdx.x * blockDim.x + threadIdx.x) / 32; r < R; r += warps) {
    const int32_t* prow = pos + r * k;
    const int32_t* xrow = ext_idx + r * (long long)n;
    int32_t* orow = idx_out + r * k;
    float* srow = sel != nullptr ? sel + r * k : nullptr;
    int w = 0;   // write cursor (warp-uniform)
    for (int j0 = 0; j0 < k; j0 += 32) {
      const int j = j0 + lane;
      int32_t gidx = -1;
      float sc = 0.f;
      if (j < k) {
        const int32_t p = prow[j];
        gidx = p >= 0 ? xrow[p] : -1;
        if (srow != nullptr) sc = srow[j];
      }
      const unsigned m = __ballot_sync(0xffffffffu, gidx >= 0);
      __syncwarp();
      if (gidx >= 0) {
        const int o = w + __popc(m & ((1u << lane) - 1u));
        orow[o] = gidx;
        if (srow != nullptr) srow[o] = sc;
      }
      w += __popc(m);
    }
    __syncwarp();
    for (int j = w + lane; j < k; j += 32) {
      orow[j] = -1;
      if (srow != nullptr) srow[j] = 0.f;
    }
  }
}

// idx_local[i] = idx[i] - lo for lo <= idx[i] < lo + len, else -1.
__global__ void cp_localize_kernel(const int32_t* __restrict__ idx, int32_t* __restrict__ out,
                                   long long n, int lo, int len) {
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x) {
    const int32_t s = idx[i];
    out[i] = (s >= lo && s < lo + len) ? s - lo : -1;
  }
}

__device__ __forceinline__ float bf16_to_f(uint16_t u) { return __uint_as_float((uint32_t)u << 16); }

// One warp per (row, head): L = ln sum_g exp(lse_g), out = sum_g exp(lse_g - L) out_g
// (a shard with lse = -inf has weight 0; all -inf gives zeros and L = -inf).
__global__ void cp_combine_kernel(const uint16_t* __restrict__ part_out,
                                  const float* __restrict__ part_lse, int G, long long rows,
                                  int Dv, uint16_t* __restrict__ out, float* __restrict__ lse_out) {
  const int lane = threadIdx.x & 31;
  const long long warps = (long long)gridDim.x * blockDim.x / 32;
  for (long long r = ((long long)blockIdx.x * blockDim.x + threadIdx.x) / 32; r < rows; r += warps) {
    float M = -INFINITY;
    for (int g = 0; g < G; ++g) M = fmaxf(M, part_lse[(long long)g * rows + r]);
    float sum = 0.f;
    if (M != -INFINITY)
      for (int g = 0; g < G; ++g) sum += __expf(part_lse[(long long)g * rows + r] - M);
    const float L = M != -INFINITY ? M + __logf(sum) : -INFINITY;
    if (lane == 0 && lse_out != nullptr) lse_out[r] = L;
    for (int d = lane; d < Dv; d += 32) {
      float acc = 0.f;
      if (M != -INFINITY) {
        for (int g = 0; g < G; ++g) {
          const float l = part_lse[(long long)g * rows + r];
          if (l != -INFINITY)
            acc += __expf(l - L) * bf16_to_f(part_out[((long long)g * rows + r) * Dv + d]);
        }
      }
      out[r * Dv + d] = __bfloat16_as_ushort(__float2bfloat16_rn(acc));
    }
  }
}

int grid_for(long long work, int per_block, int num_sms) {
  long long b = (work + per_block - 1) / per_block;
  const long long cap = (long long)(num_sms > 0 ? num_sms : 148) * 16;
  if (b > cap) b = cap;
  return (int)(b < 1 ? 1 : b);
}

}  // namespace

cudaError_t launch_cp_pack(const float* cand_scores, const int32_t* cand_idx,
                           const ShardOffsets& lo, int G, long long R, int k, float* ext_scores,
                           int32_t* ext_idx, int num_sms, cudaStream_t stream) {
  cp_pack_kernel<<<grid_for((long long)G * R * k, kCpThreads, num_sms), kCpThreads, 0, stream>>>(
      cand_scores, cand_idx, lo, G, R, k, ext_scores, ext_idx);
  return cudaGetLastError();
}

cudaError_t launch_cp_map_compact(const int32_t* pos, const int32_t* ext_idx, long long R, int n,
                                  int k, int32_t* idx_out, float* sel, int num_sms,
                                  cudaStream_t stream) {
  cp_map_compact_kernel<<<grid_for(R * 32, kCpThreads, num_sms), kCpThreads, 0, stream>>>(
      pos, ext_idx, R, n, k, idx_out, sel);
  return cudaGetLastError();
}

cudaError_t launch_cp_localize(const int32_t* idx, int32_t* out, long long n, int lo, int len,
                               int num_sms, cudaStream_t stream) {
  cp_localize_kernel<<<grid_for(n, kCpThreads, num_sms), kCpThreads, 0, stream>>>(idx, out, n, lo,
                                                                                 len);
  return cudaGetLastError();
}

cudaError_t launch_cp_combine(const uint16_t* part_out, const float* part_lse, int G,
                              long long rows, int Dv, uint16_t* out, float* lse_out, int num_sms,
                              cudaStream_t stream) {
  cp_combine_kernel<<<grid_for(rows * 32, kCpThreads, num_sms), kCpThreads, 0, stream>>>(
      part_out, part_lse, G, rows, Dv, out, lse_out);
  return cudaGetLastError();
}

}  // namespace dsa
