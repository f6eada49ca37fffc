// backward.cu - the memory-bound kernels of the sparse training stage's
// gradients ("DeepSeek-V3.2: Pushing the Frontier of Open Large Language
// Models", bud-325 paper digest, "Method": in the sparse stage the main model
// learns through attention over the selected entries, and the indexer through
// its own detached inputs with the KL on the selected tokens).
//
// The contractions of both gradients run as batched tensor-core GEMMs
// (bgemm.cu) over the selected rows gathered here into a dense per-token block;
// these kernels do the gathers and the softmax / ReLU gradient in between (the
// GEMMs add the key gradients into the shared rows themselves). The row kernels
// are grid-stride loops with one warp per row, so any grid size is correct.
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "dsa_kernels.h"

namespace dsa {
namespace {

constexpr int kRowThreads = 256;   // 8 warps per block, one row per warp

__device__ __forceinline__ float bf16_bits_to_float(uint16_t u) {
  return __uint_as_float(static_cast<uint32_t>(u) << 16);
}

__device__ __forceinline__ uint16_t float_to_bf16_bits(float f) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}

__device__ __forceinline__ float e4m3_to_float(uint8_t code) {
  __nv_fp8_e4m3 x;
  x.__x = code;
  return static_cast<float>(x);
}

__device__ __forceinline__ float warp_sum(float v) {
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float warp_max(float v) {
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__device__ __forceinline__ long long warp_id_global() {
  return (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
}

__device__ __forceinline__ long long warps_in_grid() {
  return (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
}

// Rows (tt, j) of a chunk of T tokens starting at token tok0: the selected key
// s = idx[tok][j] of sequence b = tok / Lq, or none when s is outside [0, Lk).
__device__ __forceinline__ int selected_key(const int32_t* idx, long long tok, int j, int k,
                                            int Lk) {
  const int s = idx[tok * k + j];
  return (s >= 0 && s < Lk) ? s : -1;
}

// out[tt][j][:] = kv[b][idx[tok][j]][:] (bf16 rows of V 16-byte vectors), zeros
// for a slot without a valid key.
__global__ void gather_rows_bf16_kernel(const uint4* __restrict__ kv,
                                        const int32_t* __restrict__ idx, uint4* __restrict__ out,
                                        long long tok0, int T, int Lq, int Lk, int k, int V) {
  const int lane = threadIdx.x & 31;
  const long long rows = static_cast<long long>(T) * k;
  for (long long r = warp_id_global(); r < rows; r += warps_in_grid()) {
    const long long tok = tok0 + r / k;
    const int j = static_cast<int>(r % k);
    const int s = selected_key(idx, tok, j, k, Lk);
    const long long b = tok / Lq;
    uint4* dst = out + r * V;
    if (s < 0) {
      for (int v = lane; v < V; v += 32) dst[v] = make_uint4(0u, 0u, 0u, 0u);
    } else {
      const uint4* src = kv + (b * Lk + s) * V;
      for (int v = lane; v < V; v += 32) dst[v] = src[v];
    }
  }
}

// QO[tt] = [q[tok] (H rows); dout[tok] padded with zeros to Dqk columns (H rows)],
// bf16 rows of V 16-byte vectors (Vd of them hold dout).
__global__ void pack_qo_kernel(const uint4* __restrict__ q, const uint4* __restrict__ dout,
                               uint4* __restrict__ qo, long long tok0, int T, int H, int V,
                               int Vd) {
  const int lane = threadIdx.x & 31;
  const long long rows = static_cast<long long>(T) * 2 * H;
  for (long long r = warp_id_global(); r < rows; r += warps_in_grid()) {
    const long long tok = tok0 + r / (2 * H);
    const int hh = static_cast<int>(r % (2 * H));
    uint4* dst = qo + r * V;
    if (hh < H) {
      const uint4* src = q + (tok * H + hh) * V;
      for (int v = lane; v < V; v += 32) dst[v] = src[v];
    } else {
      const uint4* src = dout + (tok * H + (hh - H)) * Vd;
      for (int v = lane; v < V; v += 32) dst[v] = v < Vd ? src[v] : make_uint4(0u, 0u, 0u, 0u);
    }
  }
}

// Softmax gradient of one (token, head) row over its k slots, with S and dP the
// raw q.c_s and dout.c_s[:Dv] of the batched GEMM (per token, SP holds the H rows
// of S and then the H rows of dP):
//   P_s  = exp(sm_scale S_s - lse)
//   D    = sum_s P_s dP_s / sum_s P_s       (= dout . out; from the fp32 P and dP,
//                                             so that sum_s dz_s vanishes up to fp32
//                                             rounding, also for short sets)
//   dz_s = sm_scale P_s (dP_s - D)
// dz and P are written as bf16 for the GEMMs that follow, per token the H rows of dz
// and then the H rows of P (PZ); slots without a valid key get 0.
__global__ void mla_bwd_softmax_kernel(const float* __restrict__ SP,
                                       const float* __restrict__ lse,
                                       const int32_t* __restrict__ idx, uint16_t* __restrict__ PZ,
                                       long long tok0, int T, int H, int k, int Lk,
                                       float sm_scale) {
  const int lane = threadIdx.x & 31;
  const long long rows = static_cast<long long>(T) * H;
  for (long long r = warp_id_global(); r < rows; r += warps_in_grid()) {
    const long long tt = r / H;
    const long long tok = tok0 + tt;
    const int h = static_cast<int>(r % H);
    const float l = lse[tok * H + h];
    const long long zrow = (tt * 2 * H + h) * k;        // row h of the token's block
    const long long prow_off = zrow + static_cast<long long>(H) * k;   // row H + h
    const float* srow = SP + zrow;
    const float* prow = SP + prow_off;
    // four consecutive slots per lane per step (k % 32 == 0: rows are 16-byte aligned)
    const int4* irow = reinterpret_cast<const int4*>(idx + tok * k);
    float sp = 0.f, spd = 0.f;
    for (int j = lane * 4; j < k; j += 128) {
      const int4 iv = irow[j >> 2];
      const float4 sv = *reinterpret_cast<const float4*>(srow + j);
      const float4 dv = *reinterpret_cast<const float4*>(prow + j);
      const int ii[4] = {iv.x, iv.y, iv.z, iv.w};
      const float ss[4] = {sv.x, sv.y, sv.z, sv.w}, dd[4] = {dv.x, dv.y, dv.z, dv.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        if (ii[q] >= 0 && ii[q] < Lk) {
          const float p = expf(ss[q] * sm_scale - l);
          sp += p;
          spd += p * dd[q];
        }
      }
    }
    sp = warp_sum(sp);
    spd = warp_sum(spd);
    const float d = sp > 0.f ? spd / sp : 0.f;
    uint16_t* z_out = PZ + zrow;
    uint16_t* p_out = PZ + prow_off;
    for (int j = lane * 4; j < k; j += 128) {
      const int4 iv = irow[j >> 2];
      const float4 sv = *reinterpret_cast<const float4*>(srow + j);
      const float4 dv = *reinterpret_cast<const float4*>(prow + j);
      const int ii[4] = {iv.x, iv.y, iv.z, iv.w};
      const float ss[4] = {sv.x, sv.y, sv.z, sv.w}, dd[4] = {dv.x, dv.y, dv.z, dv.w};
      uint16_t pb[4], zb[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        float p = 0.f, z = 0.f;
        if (ii[q] >= 0 && ii[q] < Lk) {
          p = expf(ss[q] * sm_scale - l);
          z = sm_scale * p * (dd[q] - d);
        }
        pb[q] = float_to_bf16_bits(p);
        zb[q] = float_to_bf16_bits(z);
      }
      *reinterpret_cast<uint2*>(p_out + j) = make_uint2(pb[0] | (uint32_t(pb[1]) << 16), pb[2] | (uint32_t(pb[3]) << 16));
      *reinterpret_cast<uint2*>(z_out + j) = make_uint2(zb[0] | (uint32_t(zb[1]) << 16), zb[2] | (uint32_t(zb[3]) << 16));
    }
  }
}

// out[tt][j][:] = khat[b][idx[tok][j]][:] as bf16 for e4m3 rows of d_I bytes (the
// unscaled codes, which bf16 holds exactly), zeros for a slot without a valid key.
__global__ void gather_e4m3_rows_bf16_kernel(const uint8_t* __restrict__ kI,
                                             const int32_t* __restrict__ idx,
                                             uint16_t* __restrict__ out, long long tok0, int T,
                                             int Lq, int Lk, int k, int d_I) {
  const int lane = threadIdx.x & 31;
  const long long rows = static_cast<long long>(T) * k;
  // whole 4-code words when the rows allow it (the codes come from the caller)
  const bool vec = (d_I & 3) == 0 && (reinterpret_cast<uintptr_t>(kI) & 3u) == 0 &&
                   (reinterpret_cast<uintptr_t>(out) & 7u) == 0;
  for (long long r = warp_id_global(); r < rows; r += warps_in_grid()) {
    const long long tok = tok0 + r / k;
    const int j = static_cast<int>(r % k);
    const int s = selected_key(idx, tok, j, k, Lk);
    const long long b = tok / Lq;
    uint16_t* dst = out + r * d_I;
    const uint8_t* src = kI + (b * Lk + (s < 0 ? 0 : s)) * d_I;
    if (vec) {
      // four codes per lane: one 4-byte load, one 8-byte store
      for (int c = 4 * lane; c < d_I; c += 128) {
        uint32_t w = s < 0 ? 0u : *reinterpret_cast<const uint32_t*>(src + c);
        uint32_t lo = 0u, hi = 0u;
        if (s >= 0) {
          lo = (uint32_t)float_to_bf16_bits(e4m3_to_float((uint8_t)(w & 0xFFu))) |
               ((uint32_t)float_to_bf16_bits(e4m3_to_float((uint8_t)((w >> 8) & 0xFFu))) << 16);
          hi = (uint32_t)float_to_bf16_bits(e4m3_to_float((uint8_t)((w >> 16) & 0xFFu))) |
               ((uint32_t)float_to_bf16_bits(e4m3_to_float((uint8_t)(w >> 24))) << 16);
        }
        *reinterpret_cast<uint2*>(dst + c) = make_uint2(lo, hi);
      }
    } else {
      for (int c = lane; c < d_I; c += 32)
        dst[c] = s < 0 ? uint16_t(0) : float_to_bf16_bits(e4m3_to_float(src[c]));
    }
  }
}

// out[i] = codes[i] as bf16 (exact) for n e4m3 codes.
__global__ void decode_e4m3_bf16_kernel(const uint8_t* __restrict__ codes,
                                        uint16_t* __restrict__ out, long long n) {
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<long long>(gridDim.x) * blockDim.x)
    out[i] = float_to_bf16_bits(e4m3_to_float(codes[i]));
}

// Three bf16 terms whose sum is v to 24 significant bits: each residual
// v - hi is exact in fp32, so the terms carry 8 + 8 + 8 bits.
__device__ __forceinline__ void split3(float v, uint16_t& a, uint16_t& b, uint16_t& c) {
  a = float_to_bf16_bits(v);
  const float r1 = v - bf16_bits_to_float(a);
  b = float_to_bf16_bits(r1);
  const float r2 = r1 - bf16_bits_to_float(b);
  c = float_to_bf16_bits(r2);
}

// The code dots X = qhat_j . khat_s come from a tensor-core product with fp32
// accumulation; an fp32 sum of d_I <= 128 exact products, each addition off by
// at most 2^-23 relative (rounded or truncated), is within
// d_I 2^-23 sum_i |qhat_ji khat_si| <= 2^-16 |qhat_j| |khat_s| of the exact dot.
// Where |X| is within kDotBand |qhat_j| |khat_s| of zero (four times that bound)
// the dot is recomputed exactly in fp64, so the ReLU mask is the exact code
// dot's sign.
constexpr float kDotBand = 1.0f / 16384.0f;
constexpr int kReluThreads = 256;
constexpr int kReluMaxHeads = 64;
constexpr int kReluMaxDim = 128;

// ReLU gradient for token tt of the chunk and 256 of its slots (one thread per
// slot), from XT [T][k][H_I] (fp32 code dots), the gathered key codes Kb
// [T][k][d_I] and the query codes Qb [T][H_I][d_I] (bf16). With the dequantised
// dot x = s^q_j s^k_s X:
//   dw_j    += sum_s dI_s max(x, 0)                     (dw zeroed by the caller)
//   g       = dI_s w_j [X > 0]
//   G1[j,s] = g s^k_s   -> G1s [T][H_I][3 kp]: part p at columns p kp + s
//   G2[j,s] = g s^q_j   -> G2s [T][3 hp][k]:  part p at rows p hp + j
// (three bf16 parts each, see split3), so that dq^I_j = sum_s G1[j,s] khat_s and
// dk^I_s = sum_j G2[j,s] qhat_j run as bf16 tensor-core products with fp32-level
// accuracy. Columns k..kp-1 of G1s and rows H_I..hp-1 of G2s are written as zeros.
__global__ void __launch_bounds__(kReluThreads) indexer_bwd_relu_tc_kernel(
    const float* __restrict__ XT, const uint16_t* __restrict__ Kb,
    const uint16_t* __restrict__ Qb, const int32_t* __restrict__ idx,
    const float* __restrict__ dI, const float* __restrict__ qI_scale,
    const float* __restrict__ kI_scale, const void* __restrict__ w, int w_bf16,
    uint16_t* __restrict__ G1s, uint16_t* __restrict__ G2s, float* __restrict__ dw,
    long long tok0, int Lq, int Lk, int H_I, int d_I, int k, int kp, int hp) {
  __shared__ float s_q[kReluMaxHeads * kReluMaxDim];
  __shared__ float s_sq[kReluMaxHeads], s_w[kReluMaxHeads], s_qn[kReluMaxHeads];
  __shared__ float s_dw[kReluMaxHeads];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int tt = blockIdx.y;
  const long long tok = tok0 + tt;
  const long long b = tok / Lq;
  for (int i = threadIdx.x; i < H_I * d_I; i += kReluThreads)
    s_q[i] = bf16_bits_to_float(Qb[static_cast<long long>(tt) * H_I * d_I + i]);
  for (int j = threadIdx.x; j < H_I; j += kReluThreads) {
    const long long qrow = tok * H_I + j;
    s_sq[j] = qI_scale[qrow];
    s_w[j] = w_bf16 ? bf16_bits_to_float(static_cast<const uint16_t*>(w)[qrow])
                    : static_cast<const float*>(w)[qrow];
    s_dw[j] = 0.f;
  }
  __syncthreads();
  for (int j = warp; j < H_I; j += kReluThreads / 32) {
    float acc = 0.f;
    for (int c = lane; c < d_I; c += 32) acc += s_q[j * d_I + c] * s_q[j * d_I + c];
    acc = warp_sum(acc);
    if (lane == 0) s_qn[j] = sqrtf(acc);
  }
  __syncthreads();

  const int slot = blockIdx.x * kReluThreads + threadIdx.x;
  const bool in_row = slot < k;
  const uint16_t* krow = Kb + (static_cast<long long>(tt) * k + slot) * d_I;
  int s = -1;
  float d = 0.f, sk = 0.f, kn = 0.f;
  if (in_row) {
    s = selected_key(idx, tok, slot, k, Lk);
    if (s >= 0) {
      d = dI[tok * k + slot];
      sk = kI_scale[b * Lk + s];
      float acc = 0.f;
      const uint4* k8 = reinterpret_cast<const uint4*>(krow);
      for (int c8 = 0; c8 < d_I / 8; ++c8) {
        const uint4 v = k8[c8];
        const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          const float lo = __uint_as_float(wv[h] << 16), hi = __uint_as_float(wv[h] & 0xFFFF0000u);
          acc += lo * lo + hi * hi;
        }
      }
      kn = sqrtf(acc);
    }
  }
  const float* xrow = XT + (static_cast<long long>(tt) * k + slot) * H_I;
  uint16_t* g1row = G1s + static_cast<long long>(tt) * H_I * 3 * kp + slot;
  uint16_t* g2col = G2s + static_cast<long long>(tt) * 3 * hp * k + slot;
  float4 x4 = make_float4(0.f, 0.f, 0.f, 0.f);   // four heads' dots per load (H_I % 4 == 0)
  for (int j = 0; j < hp; ++j) {
    float g1 = 0.f, g2 = 0.f, contrib = 0.f;
    if (s >= 0 && j < H_I) {
      if ((j & 3) == 0) x4 = *reinterpret_cast<const float4*>(xrow + j);
      const float x = (j & 3) == 0 ? x4.x : (j & 3) == 1 ? x4.y : (j & 3) == 2 ? x4.z : x4.w;
      double xe = x;
      if (fabsf(x) <= kDotBand * kn * s_qn[j]) {
        // exact: products of codes need <= 8 bits, sums stay on a 2^-18 grid below 2^25
        double e = 0.0;
        const uint4* k8 = reinterpret_cast<const uint4*>(krow);
        const float* qj = s_q + j * d_I;
        for (int c8 = 0; c8 < d_I / 8; ++c8) {
          const uint4 v = k8[c8];
          const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            e += static_cast<double>(qj[c8 * 8 + 2 * h]) * static_cast<double>(__uint_as_float(wv[h] << 16));
            e += static_cast<double>(qj[c8 * 8 + 2 * h + 1]) *
                 static_cast<double>(__uint_as_float(wv[h] & 0xFFFF0000u));
          }
        }
        xe = e;
      }
      if (xe > 0.0) {
        const float g = d * s_w[j];
        g1 = g * sk;
        g2 = g * s_sq[j];
        contrib = static_cast<float>(static_cast<double>(d) *
                                     (static_cast<double>(s_sq[j]) * static_cast<double>(sk) * xe));
      }
    }
    const float wsum = warp_sum(contrib);
    if (lane == 0 && j < H_I && wsum != 0.f) atomicAdd(&s_dw[j], wsum);
    if (j < H_I && slot < kp) {
      uint16_t a0, a1, a2;
      split3(g1, a0, a1, a2);
      uint16_t* g1p = g1row + static_cast<long long>(j) * 3 * kp;
      g1p[0] = a0;
      g1p[kp] = a1;
      g1p[2 * kp] = a2;
    }
    if (in_row) {
      uint16_t c0, c1, c2;
      split3(g2, c0, c1, c2);
      g2col[static_cast<long long>(j) * k] = c0;
      g2col[static_cast<long long>(hp + j) * k] = c1;
      g2col[static_cast<long long>(2 * hp + j) * k] = c2;
    }
  }
  __syncthreads();
  for (int j = threadIdx.x; j < H_I; j += kReluThreads)
    if (s_dw[j] != 0.f) atomicAdd(&dw[tok * H_I + j], s_dw[j]);
}

// dI = loss_scale (softmax(sel over the set) - p) per row of k slots; 0 outside
// the set (and everywhere for a row with an empty set).
__global__ void kl_score_grad_kernel(const float* __restrict__ sel, const float* __restrict__ p,
                                     const int32_t* __restrict__ idx, float* __restrict__ dI,
                                     long long rows, int k, int Lk, float loss_scale) {
  const int lane = threadIdx.x & 31;
  for (long long r = warp_id_global(); r < rows; r += warps_in_grid()) {
    const float* srow = sel + r * k;
    float m = -INFINITY;
    for (int j = lane; j < k; j += 32)
      if (selected_key(idx, r, j, k, Lk) >= 0) m = fmaxf(m, srow[j]);
    m = warp_max(m);
    float sum = 0.f;
    if (m != -INFINITY)
      for (int j = lane; j < k; j += 32)
        if (selected_key(idx, r, j, k, Lk) >= 0) sum += expf(srow[j] - m);
    sum = warp_sum(sum);
    const float inv = sum > 0.f ? 1.f / sum : 0.f;
    for (int j = lane; j < k; j += 32) {
      float g = 0.f;
      if (selected_key(idx, r, j, k, Lk) >= 0)
        g = loss_scale * (expf(srow[j] - m) * inv - p[r * k + j]);
      dI[r * k + j] = g;
    }
  }
}

// Blocks for a warp-per-row loop: enough to fill the GPU, never more than rows.
int row_blocks(long long rows, int num_sms) {
  const long long per_block = kRowThreads / 32;
  long long want = (rows + per_block - 1) / per_block;
  const long long cap = static_cast<long long>(num_sms > 0 ? num_sms : 148) * 16;
  if (want > cap) want = cap;
  return static_cast<int>(want < 1 ? 1 : want);
}

// Blocks for a flat element loop.
int flat_blocks(long long n, int num_sms) {
  long long blocks = (n + kRowThreads - 1) / kRowThreads;
  const long long cap = static_cast<long long>(num_sms > 0 ? num_sms : 148) * 16;
  if (blocks > cap) blocks = cap;
  return static_cast<int>(blocks < 1 ? 1 : blocks);
}

}  // namespace

cudaError_t launch_gather_rows_bf16(const uint16_t* kv, const int32_t* idx, uint16_t* out,
                                    long long tok0, int T, int Lq, int Lk, int k, int D,
                                    int num_sms, cudaStream_t stream) {
  const long long rows = static_cast<long long>(T) * k;
  gather_rows_bf16_kernel<<<row_blocks(rows, num_sms), kRowThreads, 0, stream>>>(
      reinterpret_cast<const uint4*>(kv), idx, reinterpret_cast<uint4*>(out), tok0, T, Lq, Lk, k,
      D / 8);
  return cudaGetLastError();
}

cudaError_t launch_pack_qo(const uint16_t* q, const uint16_t* dout, uint16_t* qo, long long tok0,
                           int T, int H, int Dqk, int Dv, int num_sms, cudaStream_t stream) {
  const long long rows = static_cast<long long>(T) * 2 * H;
  pack_qo_kernel<<<row_blocks(rows, num_sms), kRowThreads, 0, stream>>>(
      reinterpret_cast<const uint4*>(q), reinterpret_cast<const uint4*>(dout),
      reinterpret_cast<uint4*>(qo), tok0, T, H, Dqk / 8, Dv / 8);
  return cudaGetLastError();
}

cudaError_t launch_mla_bwd_softmax(const float* SP, const float* lse, const int32_t* idx,
                                   uint16_t* PZ, long long tok0, int T, int H, int k, int Lk,
                                   float sm_scale, int num_sms, cudaStream_t stream) {
  if (k % 4 != 0) return cudaErrorInvalidValue;
  const long long rows = static_cast<long long>(T) * H;
  mla_bwd_softmax_kernel<<<row_blocks(rows, num_sms), kRowThreads, 0, stream>>>(
      SP, lse, idx, PZ, tok0, T, H, k, Lk, sm_scale);
  return cudaGetLastError();
}

cudaError_t launch_gather_e4m3_rows_bf16(const uint8_t* kI, const int32_t* idx, uint16_t* out,
                                         long long tok0, int T, int Lq, int Lk, int k, int d_I,
                                         int num_sms, cudaStream_t stream) {
  const long long rows = static_cast<long long>(T) * k;
  gather_e4m3_rows_bf16_kernel<<<row_blocks(rows, num_sms), kRowThreads, 0, stream>>>(
      kI, idx, out, tok0, T, Lq, Lk, k, d_I);
  return cudaGetLastError();
}

cudaError_t launch_decode_e4m3_bf16(const uint8_t* codes, uint16_t* out, long long n, int num_sms,
                                    cudaStream_t stream) {
  decode_e4m3_bf16_kernel<<<flat_blocks(n, num_sms), kRowThreads, 0, stream>>>(codes, out, n);
  return cudaGetLastError();
}

cudaError_t launch_indexer_bwd_relu_tc(const float* XT, const uint16_t* Kb, const uint16_t* Qb,
                                       const int32_t* idx, const float* dI,
                                       const float* qI_scale, const float* kI_scale,
                                       const void* w, int w_bf16, uint16_t* G1s, uint16_t* G2s,
                                       float* dw, long long tok0, int T, int Lq, int Lk, int H_I,
                                       int d_I, int k, int kp, int hp, cudaStream_t stream) {
  if (H_I > kReluMaxHeads || H_I % 4 != 0 || d_I > kReluMaxDim || d_I % 8 != 0 || T > 65535)
    return cudaErrorInvalidValue;
  const dim3 grid(static_cast<unsigned>((kp + kReluThreads - 1) / kReluThreads),
                  static_cast<unsigned>(T));
  indexer_bwd_relu_tc_kernel<<<grid, kReluThreads, 0, stream>>>(
      XT, Kb, Qb, idx, dI, qI_scale, kI_scale, w, w_bf16, G1s, G2s, dw, tok0, Lq, Lk, H_I, d_I,
      k, kp, hp);
  return cudaGetLastError();
}

cudaError_t launch_kl_score_grad(const float* sel, const float* p, const int32_t* idx, float* dI,
                                 long long rows, int k, int Lk, float loss_scale, int num_sms,
                                 cudaStream_t stream) {
  kl_score_grad_kernel<<<row_blocks(rows, num_sms), kRowThreads, 0, stream>>>(
      sel, p, idx, dI, rows, k, Lk, loss_scale);
  return cudaGetLastError();
}

}  // namespace dsa
