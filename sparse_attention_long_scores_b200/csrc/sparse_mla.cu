// sparse_mla.cu - MLA attention in MQA mode over the selected latent rows
// ("DeepSeek-V3.2: Pushing the Frontier of Open Large Language Models", bud-325
// paper digest, "Key claims", section 2.1 Eq. 2 / Fig. 2: attention only on the
// top-k key-value entries; "Method": the latent vector of a token is shared by
// all query heads, so one gathered KV row serves every head).
//
// One CTA computes, for one query token and one chunk of DVC value columns:
//     z[h,s] = sm_scale * q[h] . c_s        (tcgen05, M = 128 heads, N = 32 keys,
//                                            K = Dqk in 16-wide steps)
//     online softmax over the key tiles     (base 2, lazy rescale of O)
//     O[h, chunk] += P[h,s] . c_s[chunk]    (tcgen05, M = 128, N = DVC, K = 32 keys)
// Layout of the work:
//   warp 0      producer: Q once (TMA tiles), then the selected latent rows of each
//               32-key tile with TMA gather4 (4 rows per instruction, 64-column
//               128-byte-swizzled boxes) into a 2-stage ring;
//   warp 1      tcgen05 issuer: S_i = Q K_i^T into one of two TMEM buffers,
//               then O += P_{i-1} V_{i-1};
//   warps 2..5  softmax: one head (TMEM lane) per thread. Writes P (bf16) to
//               shared memory in the 64-byte-swizzled K-major layout, rescales O
//               in TMEM only when the running max grew by more than 2^8, and
//               normalises at the end.
// O for 128 heads x 512 values in fp32 would fill all of TMEM, so the value
// columns are split over CTAs (DVC = 256): each CTA recomputes S for its token.
// With several key splits (decode) each CTA writes an unnormalised partial
// (O, running max, sum) and a combine kernel merges them.
#include "dsa_kernels.h"

namespace dsa {
namespace {

constexpr int MLA_THREADS = 192;
constexpr int KEYS = 32;                       // keys per tile

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

template <int NKB, int DVC>
struct MlaTraits {
  static constexpr int QBLK = 128 * 128;            // one 64-column block of Q: 128 rows x 128 B
  static constexpr int KVBLK = KEYS * 128;          // one 64-column block of a KV tile
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_KV = OFF_Q + NKB * QBLK;
  static constexpr int OFF_P = OFF_KV + 2 * NKB * KVBLK;
  static constexpr int OFF_BAR = OFF_P + 128 * 64;
  static constexpr int NUM_BARS = 1 + 2 + 2 + 2 + 2 + 1 + 1 + 1;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 32 + 1024;
  static constexpr int TMEM_COLS = (DVC + 2 * KEYS) <= 128 ? 128 : (DVC + 2 * KEYS) <= 256 ? 256 : 512;
  static constexpr uint32_t IDESC_S = make_idesc(1, 1, 0, 0, KEYS, 128);   // bf16, K-major both
  static constexpr uint32_t IDESC_PV = make_idesc(1, 1, 0, 1, DVC, 128);   // B (values) MN-major
  static_assert(DVC % 64 == 0 && DVC <= 256, "DVC");
  static_assert(SMEM_BYTES <= 232448, "shared memory");
};

template <int NKB, int DVC>
__global__ void __launch_bounds__(MLA_THREADS, 1)
    sparse_mla_kernel(const __grid_constant__ CUtensorMap tmap_q,
                      const __grid_constant__ CUtensorMap tmap_kv, const MlaArgs a) {
  using Tr = MlaTraits<NKB, DVC>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  uint8_t* q_smem = smem + Tr::OFF_Q;
  uint8_t* kv_smem = smem + Tr::OFF_KV;
  uint8_t* p_smem = smem + Tr::OFF_P;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Tr::OFF_BAR);
  uint64_t* q_full = bars;
  uint64_t* kv_full = bars + 1;
  uint64_t* kv_empty = bars + 3;
  uint64_t* s_full = bars + 5;
  uint64_t* s_empty = bars + 7;
  uint64_t* p_full = bars + 9;
  uint64_t* o_done = bars + 10;
  uint64_t* done_bar = bars + 11;
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + Tr::OFF_MISC);
  uint32_t* tmem_slot = misc;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
  volatile uint32_t* masks = misc + 2;   // [2]
  volatile int* ntiles_slot = reinterpret_cast<volatile int*>(misc + 4);

  const int warp = warp_id();
  const int lane = lane_id();
  const int per_token = a.n_dv * a.splits;
  const long long token = blockIdx.x / per_token;
  const int rem = blockIdx.x % per_token;
  const int dvc = rem / a.splits;
  const int split = rem % a.splits;
  const int b = (int)(token / a.Lq);
  const int32_t* idx_row = a.idx + token * a.k;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_empty[i], 1);
      mbar_init(&s_full[i], 1);
      mbar_init(&s_empty[i], 128);
    }
    mbar_init(p_full, 128);
    mbar_init(o_done, 1);
    mbar_init(done_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_map(&tmap_q);
    tma_prefetch_map(&tmap_kv);
  }
  if (warp == 0) {
    // number of 32-key tiles this CTA covers: trailing invalid entries are trimmed
    int last = -1;
    for (int base = ((a.k - 1) / 32) * 32; base >= 0 && last < 0; base -= 32) {
      int pos = base + lane;
      int v = pos < a.k ? idx_row[pos] : -1;
      unsigned m = __ballot_sync(0xffffffffu, v >= 0 && v < a.Lk);
      if (m) last = base + 31 - __clz((int)m);
    }
    int tiles_all = (last + 1 + KEYS - 1) / KEYS;
    int per_split = (tiles_all + a.splits - 1) / a.splits;
    int t_lo = split * per_split;
    int t_hi = min(tiles_all, t_lo + per_split);
    if (lane == 0) {
      ntiles_slot[0] = max(0, t_hi - t_lo);
      ntiles_slot[1] = t_lo;
    }
  }
  if (warp == 1) tmem_alloc(tmem_slot, Tr::TMEM_COLS);
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;
  const int ntiles = ntiles_slot[0];
  const int tile0 = ntiles_slot[1];
  const uint32_t o_tmem = tbase;
  const uint32_t s_tmem = tbase + DVC;

  if (warp == 0) {
    // ------------------------------------------------ producer
    bool ok = true;
    int kv_pending[2] = {-1, -1};
    int q_pending = -1;
    if (ntiles > 0 && lane == 0) {
      mbar_arrive_expect_tx(q_full, NKB * Tr::QBLK);
      for (int kb = 0; kb < NKB; ++kb)
        tma_load_2d(q_smem + kb * Tr::QBLK, &tmap_q, kb * 64, (int)(token * a.H), q_full);
      q_pending = 0;
    }
    for (int i = 0; i < ntiles && ok; ++i) {
      const int st = i & 1;
      const int ph = (i >> 1) & 1;
      const int pos = (tile0 + i) * KEYS + lane;
      const int v = pos < a.k ? idx_row[pos] : -1;
      const bool valid = v >= 0 && v < a.Lk;
      const int row = b * a.Lk + (valid ? v : 0);
      const unsigned m = __ballot_sync(0xffffffffu, valid);
      int rows[KEYS];
#pragma unroll
      for (int j = 0; j < KEYS; ++j) rows[j] = __shfl_sync(0xffffffffu, row, j);
      if (lane == 0) {
        if (!mbar_wait(&kv_empty[st], ph ^ 1, a.ctl, abort_flag, kSiteMla, 1)) {
          ok = false;
        } else {
          kv_pending[st] = -1;
          masks[st] = m;
          mbar_arrive_expect_tx(&kv_full[st], NKB * Tr::KVBLK);
          uint8_t* dst = kv_smem + st * NKB * Tr::KVBLK;
#pragma unroll
          for (int g = 0; g < KEYS / 4; ++g)
#pragma unroll
            for (int kb = 0; kb < NKB; ++kb)
              tma_gather4(dst + kb * Tr::KVBLK + g * 512, &tmap_kv, kb * 64, rows[4 * g],
                          rows[4 * g + 1], rows[4 * g + 2], rows[4 * g + 3], &kv_full[st]);
          kv_pending[st] = ph;
        }
      }
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
    }
    if (lane == 0 && *abort_flag) {
      DevCtl drain = a.ctl;
      volatile int never = 0;
      for (int i = 0; i < 2; ++i)
        if (kv_pending[i] >= 0) mbar_wait(&kv_full[i], kv_pending[i], drain, &never, kSiteMla, 2);
      if (q_pending >= 0) mbar_wait(q_full, 0, drain, &never, kSiteMla, 2);
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = ntiles == 0 || mbar_wait(q_full, 0, a.ctl, abort_flag, kSiteMla, 3);
      const uint32_t q_addr = smem_u32(q_smem);
      const uint32_t p_addr = smem_u32(p_smem);
      const uint32_t v_off = (uint32_t)(dvc * (DVC / 64)) * Tr::KVBLK;
      auto issue_pv = [&](int j) -> bool {
        if (!mbar_wait(p_full, j & 1, a.ctl, abort_flag, kSiteMla, 4)) return false;
        tc_fence_after();
        const int stj = j & 1;
        const uint32_t kv_addr = smem_u32(kv_smem + stj * NKB * Tr::KVBLK);
#pragma unroll
        for (int kk = 0; kk < KEYS / 16; ++kk) {
          uint64_t ad = make_sdesc(p_addr + kk * 32, 16, 512, 4);
          uint64_t bd = make_sdesc(kv_addr + v_off + kk * 2048, Tr::KVBLK, 1024, 2);
          mma_f16_ss(o_tmem, ad, bd, Tr::IDESC_PV, (j > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(&kv_empty[stj]);
        mma_commit(o_done);
        return true;
      };
      for (int i = 0; i < ntiles && ok; ++i) {
        const int st = i & 1;
        const int ph = (i >> 1) & 1;
        if (!mbar_wait(&kv_full[st], ph, a.ctl, abort_flag, kSiteMla, 5)) { ok = false; break; }
        if (!mbar_wait(&s_empty[st], ph ^ 1, a.ctl, abort_flag, kSiteMla, 6)) { ok = false; break; }
        tc_fence_after();
        const uint32_t kv_addr = smem_u32(kv_smem + st * NKB * Tr::KVBLK);
        const uint32_t d = s_tmem + st * KEYS;
#pragma unroll
        for (int kb = 0; kb < NKB; ++kb) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            uint64_t ad = make_sdesc(q_addr + kb * Tr::QBLK + kk * 32, 16, 1024, 2);
            uint64_t bd = make_sdesc(kv_addr + kb * Tr::KVBLK + kk * 32, 16, 1024, 2);
            mma_f16_ss(d, ad, bd, Tr::IDESC_S, (kb | kk) ? 1u : 0u);
          }
        }
        mma_commit(&s_full[st]);
        if (i > 0 && !issue_pv(i - 1)) { ok = false; break; }
      }
      if (ok && ntiles > 0) issue_pv(ntiles - 1);
      mma_commit(done_bar);
      DevCtl drain = a.ctl;
      volatile int never = 0;
      mbar_wait(done_bar, 0, drain, &never, kSiteMla, 7);
    }
  } else {
    // ------------------------------------------------ softmax / epilogue
    const int quad = warp & 3;
    const int h = quad * 32 + lane;  // head = TMEM lane
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    float m_used = -INFINITY;  // running max (log2 domain) that P is relative to
    float l = 0.f;
    bool ok = true;
    for (int i = 0; i < ntiles; ++i) {
      const int st = i & 1;
      const int ph = (i >> 1) & 1;
      if (!mbar_wait(&s_full[st], ph, a.ctl, abort_flag, kSiteMla, 8)) { ok = false; break; }
      if (!mbar_wait(&kv_full[st], ph, a.ctl, abort_flag, kSiteMla, 9)) { ok = false; break; }
      tc_fence_after();
      uint32_t r[32];
      tmem_ld32(s_tmem + lane_off + st * KEYS, r);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(&s_empty[st]);
      const uint32_t m = masks[st];
      float x[32];
      float tmax = -INFINITY;
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        x[j] = ((m >> j) & 1u) ? __uint_as_float(r[j]) * a.scale_log2 : -INFINITY;
        tmax = fmaxf(tmax, x[j]);
      }
      if (i > 0) {
        if (!mbar_wait(o_done, (i - 1) & 1, a.ctl, abort_flag, kSiteMla, 10)) { ok = false; break; }
        tc_fence_after();
      }
      const bool grow = tmax > m_used + 8.0f;
      const float m_new = grow ? tmax : m_used;
      const bool need_o = grow && m_used != -INFINITY;
      if (__any_sync(0xffffffffu, need_o)) {
        const float alpha = need_o ? ex2(m_used - m_new) : 1.f;
#pragma unroll 1
        for (int c0 = 0; c0 < DVC; c0 += 32) {
          uint32_t o[32];
          tmem_ld32(o_tmem + lane_off + c0, o);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 32; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * alpha);
          tmem_st32(o_tmem + lane_off + c0, o);
        }
        tmem_wait_st();
        l *= alpha;
      }
      m_used = m_new;
      uint32_t pk[16];
      float psum = 0.f;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        float p0 = ex2(x[2 * j] - m_used);
        float p1 = ex2(x[2 * j + 1] - m_used);
        if (m_used == -INFINITY) { p0 = 0.f; p1 = 0.f; }
        psum += p0 + p1;
        pk[j] = pack_bf16x2(p0, p1);
      }
      l += psum;
      // P row h: 32 bf16 = four 16-byte chunks, 64-byte swizzle (chunk ^= (h >> 1) & 3)
      uint8_t* prow = p_smem + h * 64;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int pc = c ^ ((h >> 1) & 3);
        *reinterpret_cast<uint4*>(prow + pc * 16) = make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(p_full);
    }
    if (ok && ntiles > 0) {
      ok = mbar_wait(o_done, (ntiles - 1) & 1, a.ctl, abort_flag, kSiteMla, 11);
      tc_fence_after();
    }
    if (ok) {
      const bool row_ok = h < a.H;
      const bool empty = !(l > 0.f);
      if (a.splits == 1) {
        const float inv = empty ? 0.f : 1.f / l;
        uint16_t* orow = a.out + (token * a.H + h) * (long long)a.Dv + dvc * DVC;
#pragma unroll 1
        for (int c0 = 0; c0 < DVC; c0 += 32) {
          uint32_t o[32];
          if (ntiles > 0) {
            tmem_ld32(o_tmem + lane_off + c0, o);
            tmem_wait_ld();
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) o[j] = 0u;
          }
          uint32_t pk[16];
#pragma unroll
          for (int j = 0; j < 16; ++j)
            pk[j] = pack_bf16x2(__uint_as_float(o[2 * j]) * inv, __uint_as_float(o[2 * j + 1]) * inv);
          if (row_ok) {
            uint4* d4 = reinterpret_cast<uint4*>(orow + c0);
#pragma unroll
            for (int c = 0; c < 4; ++c) d4[c] = make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
          }
        }
        if (row_ok && dvc == 0 && a.lse != nullptr)
          a.lse[token * a.H + h] = empty ? -INFINITY : (m_used + __log2f(l)) * 0.69314718055994531f;
      } else {
        const long long prow_i = (token * a.splits + split) * a.H + h;
        float* po = a.part_o + prow_i * a.Dv + dvc * DVC;
#pragma unroll 1
        for (int c0 = 0; c0 < DVC; c0 += 32) {
          uint32_t o[32];
          if (ntiles > 0) {
            tmem_ld32(o_tmem + lane_off + c0, o);
            tmem_wait_ld();
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) o[j] = 0u;
          }
          if (row_ok) {
            float4* d4 = reinterpret_cast<float4*>(po + c0);
#pragma unroll
            for (int c = 0; c < 8; ++c)
              d4[c] = make_float4(__uint_as_float(o[4 * c]), __uint_as_float(o[4 * c + 1]),
                                  __uint_as_float(o[4 * c + 2]), __uint_as_float(o[4 * c + 3]));
          }
        }
        if (row_ok && dvc == 0) {
          a.part_ml[prow_i * 2 + 0] = empty ? -INFINITY : m_used;
          a.part_ml[prow_i * 2 + 1] = empty ? 0.f : l;
        }
      }
    }
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, Tr::TMEM_COLS);
  }
}

// Merge key-split partials: out = sum_s 2^(m_s - M) O_s / sum_s 2^(m_s - M) l_s.
__global__ void mla_combine_kernel(const MlaArgs a) {
  const long long row = blockIdx.x;  // token * H + h
  const long long token = row / a.H;
  const int h = (int)(row % a.H);
  float M = -INFINITY;
  for (int s = 0; s < a.splits; ++s) {
    const float* ml = a.part_ml + ((token * a.splits + s) * a.H + h) * 2;
    if (ml[1] > 0.f) M = fmaxf(M, ml[0]);
  }
  float L = 0.f;
  for (int s = 0; s < a.splits; ++s) {
    const float* ml = a.part_ml + ((token * a.splits + s) * a.H + h) * 2;
    if (ml[1] > 0.f) L += ml[1] * ex2(ml[0] - M);
  }
  const float inv = L > 0.f ? 1.f / L : 0.f;
  uint16_t* orow = a.out + row * (long long)a.Dv;
  for (int c = threadIdx.x * 2; c < a.Dv; c += blockDim.x * 2) {
    float acc0 = 0.f, acc1 = 0.f;
    for (int s = 0; s < a.splits; ++s) {
      const long long pr = (token * a.splits + s) * a.H + h;
      const float* ml = a.part_ml + pr * 2;
      if (!(ml[1] > 0.f)) continue;
      const float f = ex2(ml[0] - M);
      const float2 v = *reinterpret_cast<const float2*>(a.part_o + pr * a.Dv + c);
      acc0 = fmaf(v.x, f, acc0);
      acc1 = fmaf(v.y, f, acc1);
    }
    *reinterpret_cast<uint32_t*>(orow + c) = pack_bf16x2(acc0 * inv, acc1 * inv);
  }
  if (threadIdx.x == 0 && a.lse != nullptr)
    a.lse[row] = L > 0.f ? (M + __log2f(L)) * 0.69314718055994531f : -INFINITY;
}

template <int NKB, int DVC>
cudaError_t launch_mla_variant(const CUtensorMap& tq, const CUtensorMap& tkv, const MlaArgs& a,
                               cudaStream_t stream) {
  using Tr = MlaTraits<NKB, DVC>;
  auto kern = sparse_mla_kernel<NKB, DVC>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       Tr::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  long long grid = (long long)a.B * a.Lq * a.n_dv * a.splits;
  if (grid <= 0) return cudaSuccess;
  kern<<<(unsigned)grid, MLA_THREADS, Tr::SMEM_BYTES, stream>>>(tq, tkv, a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_sparse_mla(const CUtensorMap& tmap_q, const CUtensorMap& tmap_kv,
                              const MlaArgs& a, cudaStream_t stream) {
  if (a.H == 128 && a.Dqk == 576 && a.Dv == 512) return launch_mla_variant<9, 256>(tmap_q, tmap_kv, a, stream);
  if (a.H == 8 && a.Dqk == 80 && a.Dv == 64) return launch_mla_variant<2, 64>(tmap_q, tmap_kv, a, stream);
  return cudaErrorInvalidValue;
}

cudaError_t launch_mla_combine(const MlaArgs& a, cudaStream_t stream) {
  long long rows = (long long)a.B * a.Lq * a.H;
  if (rows <= 0) return cudaSuccess;
  mla_combine_kernel<<<(unsigned)rows, 128, 0, stream>>>(a);
  return cudaGetLastError();
}

// A kernel that waits on an mbarrier nobody arrives at: exercises the bounded
// wait and the status word without faulting or hanging the GPU.
__global__ void debug_wait_kernel(DevCtl ctl) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, ctl, &abort_flag, kSiteDebug, 1);
  __syncthreads();
}

cudaError_t launch_debug_wait(DevCtl ctl, cudaStream_t stream) {
  debug_wait_kernel<<<1, 32, 0, stream>>>(ctl);
  return cudaGetLastError();
}

}  // namespace dsa
