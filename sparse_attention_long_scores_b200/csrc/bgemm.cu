// bgemm.cu - batched bf16 GEMM on the 5th-generation tensor cores for the
// contractions of the sparse-stage gradients ("DeepSeek-V3.2: Pushing the
// Frontier of Open Large Language Models", bud-325 paper digest, "Method": the
// main model learns through the attention over the selected entries, the
// indexer through its own detached inputs).
//
//   C[z] (fp32) = A[z] B[z]^T     for z < batch,   A: M x K,  B: N x K
//
// Each operand is K-major (K contiguous: A stored [M][K], B stored [N][K]) or
// MN-major (M or N contiguous: A stored [K][M], B stored [K][N]); a batch is a
// third tensor-map dimension, so rows, columns and K beyond an operand's extent
// arrive as zeros. A K-period (in 64-element tiles) lets one operand repeat
// along K, which the split-precision products use (A [a0|a1|a2] times B
// [b|b|b]). C is written with arbitrary element strides for m and n, so a
// transposed result needs no separate pass, or added row by row with fp32
// atomics into rows chosen by an index list (the key gradients of the selected
// rows go straight into the shared key rows).
//
// One CTA computes one 128 x BN tile: thread 0 streams 64-deep K tiles of A and
// B with TMA (128-byte swizzle) through a ring of 2 to 4 stages, thread 32 issues
// tcgen05.mma (M = 128, N = BN, K = 16) into a TMEM accumulator, and the four
// warps then read their 32 TMEM lanes each and store the rows (transposed through
// shared memory into full-row stores); two CTAs share an SM, so one's stores
// overlap the other's main loop. Every wait is bounded (site kSiteGemm).
#include <cuda_bf16.h>

#include "dsa_kernels.h"

namespace dsa {
namespace {

constexpr int BG_BM = 128;
constexpr int BG_BK = 64;          // K elements per tile: 128 bytes of bf16
constexpr int BG_THREADS = 128;

template <int BN, bool A_MN, bool B_MN>
struct BgTraits {
  static_assert(BN % 64 == 0 && BN >= 64 && BN <= 256, "BN");
  // as many stages as leave room for two CTAs per SM: one CTA's epilogue then
  // overlaps the other's loads and MMAs
  static constexpr int STAGES = BN >= 192 ? 2 : BN == 128 ? 3 : 4;
  static constexpr int A_BYTES = BG_BM * 128;   // K-major: 128 rows x 128 B; MN-major: 2 boxes of 64 x 64
  static constexpr int B_BYTES = BN * 128;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int OFF_BAR = STAGES * STAGE_BYTES;
  // full[STAGES], empty[STAGES], done; then the TMEM base and the abort flag
  static constexpr int SMEM_BYTES = OFF_BAR + (2 * STAGES + 1) * 8 + 16 + 1024;
  static_assert(2 * SMEM_BYTES <= 232448, "two CTAs per SM");
  static constexpr int TMEM_COLS = BN <= 64 ? 64 : BN <= 128 ? 128 : 256;
  static constexpr uint32_t IDESC = make_idesc(1, 1, A_MN ? 1 : 0, B_MN ? 1 : 0, BN, 128);
  // MN-major operands: 64-element column blocks of BG_BK rows x 128 B each
  static constexpr uint32_t MN_LBO = BG_BK * 128;
};

template <int BN, bool A_MN, bool B_MN>
__global__ void __launch_bounds__(BG_THREADS, 2)
    bgemm_kernel(const __grid_constant__ CUtensorMap tmap_a,
                 const __grid_constant__ CUtensorMap tmap_b, const BgemmArgs a) {
  using Tr = BgTraits<BN, A_MN, B_MN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + Tr::OFF_BAR);
  uint64_t* empty = full + Tr::STAGES;
  uint64_t* done = empty + Tr::STAGES;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * BN, m0 = blockIdx.y * BG_BM, z = blockIdx.z;
  const int KT = (a.K + BG_BK - 1) / BG_BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < Tr::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_map(&tmap_a);
    tma_prefetch_map(&tmap_b);
  }
  if (warp == 1) tmem_alloc(tmem_slot, Tr::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;

  if (threadIdx.x == 0) {
    // producer: K tile kt of A is tile kt % a_kt of its own K extent (likewise B)
    for (int kt = 0; kt < KT; ++kt) {
      const int st = kt % Tr::STAGES;
      if (kt >= Tr::STAGES &&
          !mbar_wait(&empty[st], (uint32_t)((kt / Tr::STAGES) - 1) & 1u, a.ctl, abort_flag, kSiteGemm, 1))
        break;
      uint8_t* sa = smem + st * Tr::STAGE_BYTES;
      uint8_t* sb = sa + Tr::A_BYTES;
      mbar_arrive_expect_tx(&full[st], Tr::STAGE_BYTES);
      const int ka = (kt % a.a_kt) * BG_BK, kb = (kt % a.b_kt) * BG_BK;
      if constexpr (A_MN) {
        tma_load_3d(sa, &tmap_a, m0, ka, z, &full[st]);
        tma_load_3d(sa + Tr::MN_LBO, &tmap_a, m0 + 64, ka, z, &full[st]);
      } else {
        tma_load_3d(sa, &tmap_a, ka, m0, z, &full[st]);
      }
      if constexpr (B_MN) {
#pragma unroll
        for (int j = 0; j < BN / 64; ++j) tma_load_3d(sb + j * Tr::MN_LBO, &tmap_b, n0 + 64 * j, kb, z, &full[st]);
      } else {
        tma_load_3d(sb, &tmap_b, kb, n0, z, &full[st]);
      }
    }
  } else if (threadIdx.x == 32) {
    // MMA issuer: four K = 16 steps per tile; a K-major step advances 32 bytes
    // along the swizzled row, an MN-major step 16 rows of 128 bytes
    bool ok = true;
    for (int kt = 0; kt < KT && ok; ++kt) {
      const int st = kt % Tr::STAGES;
      if (!mbar_wait(&full[st], (uint32_t)(kt / Tr::STAGES) & 1u, a.ctl, abort_flag, kSiteGemm, 2)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t sa = smem_u32(smem + st * Tr::STAGE_BYTES);
      const uint32_t sb = sa + Tr::A_BYTES;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint64_t ad = A_MN ? make_sdesc(sa + kk * 2048, Tr::MN_LBO, 1024, 2)
                                 : make_sdesc(sa + kk * 32, 16, 1024, 2);
        const uint64_t bd = B_MN ? make_sdesc(sb + kk * 2048, Tr::MN_LBO, 1024, 2)
                                 : make_sdesc(sb + kk * 32, 16, 1024, 2);
        mma_f16_ss(tbase, ad, bd, Tr::IDESC, (kt | kk) ? 1u : 0u);
      }
      mma_commit(&empty[st]);
    }
    if (ok) mma_commit(done);
  }
  __syncwarp();

  // epilogue: warp w holds rows m0 + 32 w .. + 31 in TMEM lanes 32 w ..
  const bool have = mbar_wait(done, 0u, a.ctl, abort_flag, kSiteGemm, 3);
  tc_fence_after();
  fence_proxy_async_smem();   // the stages' TMA data is consumed; their space is reused below
  if (have) {
    // Row-major C (c_sn == 1): each 32 x 32 block goes through shared memory (the
    // drained pipeline stages), so that a store instruction writes 32 consecutive
    // columns of one row instead of one column of 32 rows.
    float* tile = reinterpret_cast<float*>(smem) + warp * (32 * 33);
    const int m_lane = m0 + warp * 32 + lane;
#pragma unroll 1
    for (int c0 = 0; c0 < BN; c0 += 32) {
      if (n0 + c0 >= a.N) break;   // uniform across the CTA
      uint32_t r[32];
      tmem_ld32(tbase + ((uint32_t)(warp * 32) << 16) + (uint32_t)c0, r);
      tmem_wait_ld();
      const int n = n0 + c0;
      if (a.c_sn == 1) {
#pragma unroll
        for (int j = 0; j < 32; ++j) tile[lane * 33 + j] = __uint_as_float(r[j]);
        __syncwarp();
        const bool col_ok = n + lane < a.N;
        if (a.sidx != nullptr) {
          // scatter-add: each row goes to its key's row of the sequence
          const long long tok = a.s_tok0 + z;
          float* cseq = a.C + (tok / a.s_Lq) * (long long)a.s_Lk * a.c_sm;
          const int32_t* srow = a.sidx + tok * a.s_k;
#pragma unroll 4
          for (int rr = 0; rr < 32; ++rr) {
            const int m = m0 + warp * 32 + rr;
            const int key = m < a.M ? srow[m] : -1;
            if (key >= 0 && key < a.s_Lk && col_ok)
              atomicAdd(cseq + (long long)key * a.c_sm + n + lane, tile[rr * 33 + lane]);
          }
        } else {
#pragma unroll 4
          for (int rr = 0; rr < 32; ++rr) {
            const int m = m0 + warp * 32 + rr;
            if (m < a.M && col_ok)
              a.C[(long long)z * a.sC + (long long)m * a.c_sm + n + lane] = tile[rr * 33 + lane];
          }
        }
        __syncwarp();
      } else if (m_lane < a.M) {
        // column-strided C: consecutive lanes (rows) are consecutive when c_sm == 1
        float* crow = a.C + (long long)z * a.sC + (long long)m_lane * a.c_sm;
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (n + j < a.N) crow[(long long)(n + j) * a.c_sn] = __uint_as_float(r[j]);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tbase, Tr::TMEM_COLS);
}

template <int BN, bool A_MN, bool B_MN>
cudaError_t launch_bgemm_t(const CUtensorMap& ta, const CUtensorMap& tb, const BgemmArgs& a,
                           int batch, cudaStream_t stream) {
  using Tr = BgTraits<BN, A_MN, B_MN>;
  auto kern = bgemm_kernel<BN, A_MN, B_MN>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Tr::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  const dim3 grid((unsigned)((a.N + BN - 1) / BN), (unsigned)((a.M + BG_BM - 1) / BG_BM), (unsigned)batch);
  kern<<<grid, BG_THREADS, Tr::SMEM_BYTES, stream>>>(ta, tb, a);
  return cudaGetLastError();
}

template <bool A_MN, bool B_MN>
cudaError_t launch_bgemm_bn(const CUtensorMap& ta, const CUtensorMap& tb, const BgemmArgs& a,
                            int batch, int bn, cudaStream_t stream) {
  switch (bn) {
    case 64: return launch_bgemm_t<64, A_MN, B_MN>(ta, tb, a, batch, stream);
    case 128: return launch_bgemm_t<128, A_MN, B_MN>(ta, tb, a, batch, stream);
    case 192: return launch_bgemm_t<192, A_MN, B_MN>(ta, tb, a, batch, stream);
    case 256: return launch_bgemm_t<256, A_MN, B_MN>(ta, tb, a, batch, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

int bgemm_tile_n(int N) {
  if (N <= 64) return 64;
  if (N <= 128) return 128;
  if (N % 256 == 0) return 256;
  if (N <= 192 || N % 192 == 0) return 192;
  return 256;
}

cudaError_t launch_bgemm(const CUtensorMap& ta, const CUtensorMap& tb, const BgemmArgs& a,
                         int batch, bool a_mn, bool b_mn, int bn, cudaStream_t stream) {
  if (batch < 1 || batch > 65535 || a.M < 1 || a.N < 1 || a.K < 1 || a.a_kt < 1 || a.b_kt < 1)
    return cudaErrorInvalidValue;
  if (a.sidx != nullptr && (a.c_sn != 1 || a.s_k < a.M || a.s_Lq < 1 || a.s_Lk < 1))
    return cudaErrorInvalidValue;
  if (a_mn) {
    return b_mn ? launch_bgemm_bn<true, true>(ta, tb, a, batch, bn, stream)
                : launch_bgemm_bn<true, false>(ta, tb, a, batch, bn, stream);
  }
  return b_mn ? launch_bgemm_bn<false, true>(ta, tb, a, batch, bn, stream)
              : launch_bgemm_bn<false, false>(ta, tb, a, batch, bn, stream);
}

}  // namespace dsa
