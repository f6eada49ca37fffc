// indexer_kl.cu - the indexer alignment target, forward only: KL between the
// head-aggregated main attention over a query token's key set and the softmax of
// the index scores over the same set
// ("DeepSeek-V3.2: Pushing the Frontier of Open Large Language Models", bud-325
// paper digest: "Key claims", paper section 2.1.1 Eq. 3-4, given in words: a KL
// loss aligns the indexer output with the main attention aggregated over heads;
// "Method": in the sparse stage the KL is taken on the selected tokens. The
// eu.36kr.com article, section 02: the indexer learns to mimic the original
// attention's distribution).
//
// For query token t with key set S (the valid entries of idx[t,:]):
//     a[h,s] = exp(sm_scale q[h].c_s - lse[h])   (the forward's per-head lse over S)
//     p_s    = sum_h a[h,s] / H                  (each head sums to 1 over S)
//     r_s    = softmax over S of the index scores sel[t,:]
//     KL_t   = sum_s p_s (ln p_s - ln r_s)
// One CTA per query token:
//   warp 0      tcgen05 issuer: S_i = Q K_i^T of each 64-key tile into one of two
//               TMEM buffers; Q lives entirely in TMEM (there is no output
//               accumulator here), so shared memory holds three KV stages;
//   warps 5..12 gather producers: each warp owns 8 rows of every tile, loads their
//               indices once and copies the rows 16 bytes per thread per cp.async
//               into the 128-byte-swizzled K-major layout;
//   warps 1..4  one head per thread (TMEM lane): a[h,s] for the tile's 64 keys,
//               summed over the warp's 32 heads by a butterfly reduce-scatter (each
//               lane ends with two keys), then over the four warps in shared
//               memory; warp 1 forms p_s and the KL terms and writes p.
#include "dsa_kernels.h"

namespace dsa {
namespace {

constexpr int KEYS = 64;
constexpr int PROD_WARPS = 8;
constexpr int KL_THREADS = 32 + 128 + PROD_WARPS * 32;
constexpr int PROD_T0 = 160;
constexpr float kLog2e = 1.4426950408889634f;

template <int NKB>
struct KlTraits {
  static constexpr int KVBLK = KEYS * 128;          // one 64-column block of a KV tile
  static constexpr int STAGES = 3;
  static constexpr int NP = PROD_WARPS * 32;
  static constexpr int OFF_KV = 0;
  static constexpr int OFF_RED = OFF_KV + STAGES * NKB * KVBLK;   // [2][4 warps][KEYS] fp32
  static constexpr int OFF_BAR = OFF_RED + 2 * 4 * KEYS * 4;
  static constexpr int BAR_QT = 0;                       // Q in TMEM written
  static constexpr int BAR_KV_FULL = 1;                  // [STAGES]
  static constexpr int BAR_KV_EMPTY = BAR_KV_FULL + STAGES;
  static constexpr int BAR_S_FULL = BAR_KV_EMPTY + STAGES;   // [2]
  static constexpr int BAR_S_FREE = BAR_S_FULL + 2;          // [2] S buffer read
  static constexpr int BAR_RED_FULL = BAR_S_FREE + 2;        // [2] per-warp head sums written
  static constexpr int BAR_RED_FREE = BAR_RED_FULL + 2;      // [2] head sums read by warp 1
  static constexpr int BAR_DONE = BAR_RED_FREE + 2;
  static constexpr int NUM_BARS = BAR_DONE + 1;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 32 + 1024;
  // TMEM columns: two S buffers [0, 2 KEYS), Q [2 KEYS, 2 KEYS + 32 NKB)
  static constexpr int COL_Q = 2 * KEYS;
  static constexpr int COLS_USED = COL_Q + 32 * NKB;
  static constexpr int TMEM_COLS = COLS_USED <= 128 ? 128 : COLS_USED <= 256 ? 256 : 512;
  static constexpr uint32_t IDESC_S = make_idesc(1, 1, 0, 0, KEYS, 128);   // bf16, K-major both
  static_assert(COLS_USED <= 512, "TMEM");
  static_assert(SMEM_BYTES <= 232448, "shared memory");
};

// S = Q K^T for one tile: every column block of Q from TMEM (TS form), fully
// unrolled so that every offset is a compile-time constant.
template <int NKB>
__device__ __forceinline__ void issue_s_tile(uint32_t s_tmem, uint32_t qt_tmem, uint64_t kd0) {
  using Tr = KlTraits<NKB>;
#pragma unroll
  for (int kb = 0; kb < NKB; ++kb) {
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
      mma_f16_ts(s_tmem, qt_tmem + kb * 32 + kk * 8,
                 kd0 + (uint64_t)((kb * Tr::KVBLK + kk * 32) >> 4), Tr::IDESC_S, (kb | kk) ? 1u : 0u);
  }
}

// One halving step of the butterfly reduce-scatter over the warp: lanes whose
// `o` bit is set keep the upper half of their N values, the others the lower
// half, each adding its partner's copy of the half it keeps.
template <int N>
__device__ __forceinline__ void reduce_half(const float (&in)[N], float (&out)[N / 2], int o, bool upper) {
#pragma unroll
  for (int j = 0; j < N / 2; ++j) {
    const float keep = upper ? in[j + N / 2] : in[j];
    const float send = upper ? in[j] : in[j + N / 2];
    out[j] = keep + __shfl_xor_sync(0xffffffffu, send, o);
  }
}

template <int NKB>
__global__ void __launch_bounds__(KL_THREADS, 1)
    indexer_kl_kernel(const uint16_t* __restrict__ kv, const KlArgs a) {
  using Tr = KlTraits<NKB>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  uint8_t* kv_smem = smem + Tr::OFF_KV;
  float* red = reinterpret_cast<float*>(smem + Tr::OFF_RED);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Tr::OFF_BAR);
  uint64_t* qt_full = bars + Tr::BAR_QT;
  uint64_t* kv_full = bars + Tr::BAR_KV_FULL;     // [STAGES]
  uint64_t* kv_empty = bars + Tr::BAR_KV_EMPTY;   // [STAGES]
  uint64_t* s_full = bars + Tr::BAR_S_FULL;       // [2]
  uint64_t* s_free = bars + Tr::BAR_S_FREE;       // [2]
  uint64_t* red_full = bars + Tr::BAR_RED_FULL;   // [2]
  uint64_t* red_free = bars + Tr::BAR_RED_FREE;   // [2]
  uint64_t* done_bar = bars + Tr::BAR_DONE;
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + Tr::OFF_MISC);
  uint32_t* tmem_slot = misc;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
  volatile int* ntiles_slot = reinterpret_cast<volatile int*>(misc + 2);

  const int warp = warp_id();
  const int lane = lane_id();
  const long long token = blockIdx.x;
  const int b = (int)(token / a.Lq);
  const int32_t* idx_row = a.idx + token * a.k;

  if (threadIdx.x == 0) {
    mbar_init(qt_full, 128);
    for (int i = 0; i < Tr::STAGES; ++i) {
      mbar_init(&kv_full[i], Tr::NP);
      mbar_init(&kv_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], 128);
      mbar_init(&red_full[i], 128);
      mbar_init(&red_free[i], 32);
    }
    mbar_init(done_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    // tiles up to the last valid key: trailing invalid entries are not visited
    int last = -1;
    for (int base = ((a.k - 1) / 32) * 32; base >= 0 && last < 0; base -= 32) {
      const int pos = base + lane;
      const int v = pos < a.k ? idx_row[pos] : -1;
      const unsigned m = __ballot_sync(0xffffffffu, v >= 0 && v < a.Lk);
      if (m) last = base + 31 - __clz((int)m);
    }
    if (lane == 0) ntiles_slot[0] = (last + 1 + KEYS - 1) / KEYS;
  }
  if (warp == 0) tmem_alloc(tmem_slot, Tr::TMEM_COLS);
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;
  const int ntiles = ntiles_slot[0];
  const uint32_t s_tmem = tbase;
  const uint32_t qt_tmem = tbase + Tr::COL_Q;

  if (warp == 0) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = ntiles == 0 || mbar_wait(qt_full, 0, a.ctl, abort_flag, kSiteKl, 1);
      for (int i = 0; ok && i < ntiles; ++i) {
        const int st = i % Tr::STAGES;
        if (!mbar_wait(&kv_full[st], (i / Tr::STAGES) & 1, a.ctl, abort_flag, kSiteKl, 2)) break;
        // S buffer i % 2 was last read for tile i - 2
        if (i >= 2 && !mbar_wait(&s_free[i & 1], ((i >> 1) & 1) ^ 1, a.ctl, abort_flag, kSiteKl, 3)) break;
        tc_fence_after();
        const uint64_t kd0 = make_sdesc(smem_u32(kv_smem + st * NKB * Tr::KVBLK), 16, 1024, 2);
        issue_s_tile<NKB>(s_tmem + (uint32_t)((i & 1) * KEYS), qt_tmem, kd0);
        mma_commit(&kv_empty[st]);
        mma_commit(&s_full[i & 1]);
      }
      mma_commit(done_bar);
      DevCtl drain = a.ctl;
      volatile int never = 0;
      mbar_wait(done_bar, 0, drain, &never, kSiteKl, 4);
    }
  } else if (warp >= PROD_T0 / 32) {
    // ------------------------------------------------ gather producers
    // Chunk c of a tile is 16 bytes: row r = c / (8 NKB), 16-byte chunk q of that
    // row, stored at column block q / 8, row r, slot (q % 8) ^ (r % 8) of the
    // 128-byte-swizzled K-major layout. Chunks past the end of a row are zeros.
    const int pw = warp - PROD_T0 / 32;   // this warp owns rows 8 pw .. 8 pw + 7 of every tile
    const int row_bytes = a.Dqk * 2;
    const uint8_t* kv_b = reinterpret_cast<const uint8_t*>(kv) + (size_t)b * a.Lk * row_bytes;
    const uint32_t kv_base = smem_u32(kv_smem);
    constexpr int CHUNKS = 8 * NKB * 8;   // 16-byte chunks of the warp's 8 rows
    static_assert(CHUNKS % 32 == 0 && PROD_WARPS * 8 == KEYS, "producer mapping");
    for (int i = 0; i < ntiles; ++i) {
      const int st = i % Tr::STAGES;
      // the rows' indices once per tile (lanes 0..7); invalid keys read row 0, masked later
      const int pos = i * KEYS + pw * 8 + lane;
      int v = -1;
      if (lane < 8 && pos < a.k) v = __ldg(idx_row + pos);
      const int row = (v >= 0 && v < a.Lk) ? v : 0;
      const uint8_t* src_row = kv_b + (size_t)row * row_bytes;
      if (!mbar_wait(&kv_empty[st], ((i / Tr::STAGES) & 1) ^ 1, a.ctl, abort_flag, kSiteKl, 5)) break;
      const uint32_t stage = kv_base + st * NKB * Tr::KVBLK;
#pragma unroll
      for (int jj = 0; jj < CHUNKS / 32; ++jj) {
        const int q = lane + jj * 32;
        const int rr = q / (NKB * 8);
        const int rem = q - rr * NKB * 8;
        const int kb = rem >> 3, q8 = rem & 7;
        const uint8_t* src = reinterpret_cast<const uint8_t*>(
            __shfl_sync(0xffffffffu, reinterpret_cast<uintptr_t>(src_row), rr));
        const int r = pw * 8 + rr;
        const int qc = kb * 8 + q8;   // 16-byte chunk within the row
        const bool in_row = qc * 16 < row_bytes;
        cp_async16(stage + kb * Tr::KVBLK + r * 128 + ((q8 ^ (r & 7)) << 4), src + (in_row ? qc * 16 : 0),
                   in_row ? 16u : 0u);
      }
      cp_async_commit();
      cp_async_wait<0>();
      fence_proxy_async_smem();
      mbar_arrive(&kv_full[st]);
    }
    cp_async_wait_all();
  } else {
    // ------------------------------------------------ head warps (1..4)
    const int quad = warp & 3;
    const int h = quad * 32 + lane;   // head = TMEM lane
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const bool head_ok = h < a.H;
    if (ntiles > 0) {
      // all of this head's query row into TMEM (lane = head, 32-bit column = two
      // consecutive bf16); bytes past the end of the row are zeros
      const long long qrow = token * a.H + h;
      const int row_bytes = a.Dqk * 2;
      const uint8_t* qsrc = reinterpret_cast<const uint8_t*>(a.q) + (head_ok ? qrow : 0) * (long long)row_bytes;
#pragma unroll 1
      for (int kb = 0; kb < NKB; ++kb) {
        uint32_t qv[32];
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const int off = kb * 128 + c * 16;
          const uint4 u = (head_ok && off < row_bytes) ? *reinterpret_cast<const uint4*>(qsrc + off)
                                                       : make_uint4(0u, 0u, 0u, 0u);
          qv[4 * c] = u.x; qv[4 * c + 1] = u.y; qv[4 * c + 2] = u.z; qv[4 * c + 3] = u.w;
        }
        tmem_st32(qt_tmem + lane_off + kb * 32, qv);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(qt_full);
    }
    // a[h,s] = 2^(z * log2 e - lse[h] * log2 e); heads past H contribute nothing
    const float lse2 = head_ok ? a.lse[token * a.H + h] * kLog2e : 0.f;
    // warp 1: log-sum-exp of the index scores over the key set (ln r_s = sel_s - lse_I)
    float lse_i = 0.f;
    const float* sel_row = a.sel + token * a.k;
    if (warp == 1) {
      float mx = -INFINITY;
      for (int j = lane; j < a.k; j += 32) {
        const int v = idx_row[j];
        if (v >= 0 && v < a.Lk) mx = fmaxf(mx, sel_row[j]);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      float sum = 0.f;
      if (mx != -INFINITY) {
        for (int j = lane; j < a.k; j += 32) {
          const int v = idx_row[j];
          if (v >= 0 && v < a.Lk) sum += ex2((sel_row[j] - mx) * kLog2e);
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      lse_i = mx + logf(sum);
    }
    float kl_acc = 0.f;
    bool ok = true;
    for (int i = 0; i < ntiles; ++i) {
      if (!mbar_wait(&s_full[i & 1], (i >> 1) & 1, a.ctl, abort_flag, kSiteKl, 6)) { ok = false; break; }
      tc_fence_after();
      uint32_t mk[2];
#pragma unroll
      for (int hw = 0; hw < 2; ++hw) {
        const int pos = i * KEYS + hw * 32 + lane;
        const int v = pos < a.k ? idx_row[pos] : -1;
        mk[hw] = __ballot_sync(0xffffffffu, v >= 0 && v < a.Lk);
      }
      const uint32_t sbuf = s_tmem + (uint32_t)((i & 1) * KEYS) + lane_off;
      float x[KEYS];
#pragma unroll
      for (int hw = 0; hw < 2; ++hw) {
        uint32_t r[32];
        tmem_ld32(sbuf + hw * 32, r);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 32; ++j)
          x[hw * 32 + j] = (head_ok && ((mk[hw] >> j) & 1u))
                               ? ex2(__uint_as_float(r[j]) * a.scale_log2 - lse2) : 0.f;
      }
      tc_fence_before();
      mbar_arrive(&s_free[i & 1]);   // S values are in registers
      // sum over the warp's 32 heads: lane l ends with keys 2l and 2l + 1
      float w32[32], w16[16], w8[8], w4[4], w2[2];
      reduce_half<64>(x, w32, 16, (lane & 16) != 0);
      reduce_half<32>(w32, w16, 8, (lane & 8) != 0);
      reduce_half<16>(w16, w8, 4, (lane & 4) != 0);
      reduce_half<8>(w8, w4, 2, (lane & 2) != 0);
      reduce_half<4>(w4, w2, 1, (lane & 1) != 0);
      float* rb = red + (i & 1) * 4 * KEYS;
      if (i >= 2 && !mbar_wait(&red_free[i & 1], ((i >> 1) & 1) ^ 1, a.ctl, abort_flag, kSiteKl, 7)) { ok = false; break; }
      *reinterpret_cast<float2*>(rb + quad * KEYS + 2 * lane) = make_float2(w2[0], w2[1]);
      mbar_arrive(&red_full[i & 1]);
      if (warp == 1) {
        if (!mbar_wait(&red_full[i & 1], (i >> 1) & 1, a.ctl, abort_flag, kSiteKl, 8)) { ok = false; break; }
        float psum[2];
#pragma unroll
        for (int j = 0; j < 2; ++j)
          psum[j] = rb[2 * lane + j] + rb[KEYS + 2 * lane + j] + rb[2 * KEYS + 2 * lane + j] +
                    rb[3 * KEYS + 2 * lane + j];
        mbar_arrive(&red_free[i & 1]);
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int key = 2 * lane + j;
          const int pos = i * KEYS + key;
          if (pos < a.k) {
            const bool valid = (mk[key >> 5] >> (key & 31)) & 1u;
            const float p = valid ? psum[j] / (float)a.H : 0.f;
            if (a.p_out != nullptr) a.p_out[token * a.k + pos] = p;
            if (p > 0.f) kl_acc += p * (logf(p) - (sel_row[pos] - lse_i));
          }
        }
      }
    }
    if (warp == 1) {
      // slots past the last visited tile are outside the key set
      if (a.p_out != nullptr)
        for (int pos = ntiles * KEYS + lane; pos < a.k; pos += 32) a.p_out[token * a.k + pos] = 0.f;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) kl_acc += __shfl_xor_sync(0xffffffffu, kl_acc, o);
      if (lane == 0 && ok) a.kl_out[token] = kl_acc;
    }
  }

  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tbase, Tr::TMEM_COLS);
  }
}

template <int NKB>
cudaError_t launch_kl_variant(const uint16_t* kv, const KlArgs& a, cudaStream_t stream) {
  using Tr = KlTraits<NKB>;
  auto kern = indexer_kl_kernel<NKB>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       Tr::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  const long long grid = (long long)a.B * a.Lq;
  if (grid <= 0) return cudaSuccess;
  kern<<<(unsigned)grid, KL_THREADS, Tr::SMEM_BYTES, stream>>>(kv, a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_indexer_kl(const uint16_t* kv, const KlArgs& a, cudaStream_t stream) {
  if (a.H == 128 && a.Dqk == 576) return launch_kl_variant<9>(kv, a, stream);
  if (a.H == 8 && a.Dqk == 80) return launch_kl_variant<2>(kv, a, stream);
  return cudaErrorInvalidValue;
}

}  // namespace dsa
