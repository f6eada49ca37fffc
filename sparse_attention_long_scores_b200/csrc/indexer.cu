// indexer.cu - the lightning indexer on sm_100a tensor cores.
//
// Computes, for query rows t of every sequence and their causal keys s <= q_pos0+t,
//     I[t,s] = kI_scale[s] * sum_j (w[t,j] * qI_scale[t,j]) * max(0, qhat[t,j] . khat[s])
// which is the index score of "DeepSeek-V3.2: Pushing the Frontier of Open Large
// Language Models" (bud-325 paper digest, "Key claims", section 2.1 Eq. 1) with
// FP8 e4m3 inputs dequantised by positive per-row scales (a positive scale
// commutes with ReLU, so both scales move outside it exactly).
//
// Design (one persistent CTA per SM):
//   * The GEMM is transposed so the head reduction needs no cross-thread
//     traffic: A = 128 indexer keys (M, one TMEM lane each), B = T_BLK query
//     tokens x H_I heads (N = 256, or 64 for single-token decode blocks),
//     K = d_I. One tcgen05.mma kind::f8f6f4 per 32 bytes of K.
//   * Warp 0 streams key tiles with TMA into a STAGES-deep ring; warp 1 issues
//     the MMAs into two TMEM accumulators; warps 2.. are the epilogue (four per
//     TMEM lane quadrant at N = 256, one token each): each
//     thread owns one key, reads its accumulator row with tcgen05.ld, applies
//     ReLU and the folded weight w*s^q per column, reduces over heads in
//     registers and writes one fp32 score per (token, key). The L x L score
//     matrix never exists in full: the caller picks the rows and key range.
//   * Work unit = (sequence, token block, piece of `piece_keys` keys); units are
//     dealt to CTAs round robin.
#include "dsa_kernels.h"

namespace dsa {
namespace {

// ---------------------------------------------------------------------------
// Fused top-k: exact selection of the k largest scores of a row by a group of NT
// selector threads (bar.sync 1 among them), reading the row from L2 where the
// epilogue left it. Scores map to order-preserving 32-bit keys (-0.0 folded onto
// +0.0); a three-digit radix select (11 + 11 + 10 bits, most significant first)
// finds the exact k-th largest key T, each pass histogramming the keys that match
// the prefix chosen so far; a final pass in index order writes every key > T and
// the first (k - #{key > T}) keys == T, so ties go to the lowest index and the
// output is ascending ("DeepSeek-V3.2: Pushing the Frontier of Open Large Language
// Models", bud-325 paper digest, "Key claims", section 2.1: attention reads the
// top-k entries of I[t,:]; "Method": k = 2048).
// ---------------------------------------------------------------------------
struct SelShared {
  uint32_t hist[2048];
  uint32_t tmp[32];
  uint32_t sel[2];
  uint32_t ucnt[4];   // epilogue threads done with the CTA's recent units (ring of 4)
  int go;             // the row's scores are complete (set by selector thread 0)
};

template <int NT>
__device__ __forceinline__ void sel_bar() {
  asm volatile("bar.sync 1, %0;" ::"n"(NT) : "memory");
}

__device__ __forceinline__ uint32_t sel_key(float x) {
  uint32_t u = __float_as_uint(x);
  if (u == 0x80000000u) u = 0u;   // -0.0 == +0.0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ uint32_t ld_acquire_u32(const int* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Exclusive scan of one value per selector thread; also returns the total.
template <int NT>
__device__ __forceinline__ uint32_t sel_scan(uint32_t v, SelShared& sh, int tid, uint32_t& total) {
  const int lane = tid & 31, wid = tid >> 5;
  uint32_t incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t n = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += n;
  }
  if (lane == 31) sh.tmp[wid] = incl;
  sel_bar<NT>();
  uint32_t off = 0, tot = 0;
#pragma unroll
  for (int w = 0; w < NT / 32; ++w) {
    const uint32_t x = sh.tmp[w];
    off += w < wid ? x : 0u;
    tot += x;
  }
  sel_bar<NT>();
  total = tot;
  return off + incl - v;
}

// From the histogram of the current digit, the digit holding the need-th largest
// key: extends prefix by it and makes need the rank within that digit.
template <int NT, int BITS>
__device__ __forceinline__ void sel_find(SelShared& sh, int tid, bool first, uint32_t& prefix,
                                         uint32_t& need) {
  constexpr int BPT = (1 << BITS) / NT;
  static_assert(BPT >= 1, "bins per thread");
  const int b0 = tid * BPT;
  uint32_t local = 0;
#pragma unroll
  for (int j = 0; j < BPT; ++j) local += sh.hist[b0 + j];
  uint32_t total;
  const uint32_t before = sel_scan<NT>(local, sh, tid, total);
  uint32_t above = total - before - local;   // keys in the bins of higher-numbered threads
#pragma unroll
  for (int j = BPT - 1; j >= 0; --j) {
    const uint32_t h = sh.hist[b0 + j];
    if (above < need && need <= above + h) {
      sh.sel[0] = (uint32_t)(b0 + j);
      sh.sel[1] = need - above;
    }
    above += h;
  }
  sel_bar<NT>();
  prefix = first ? sh.sel[0] : ((prefix << BITS) | sh.sel[0]);
  need = sh.sel[1];
  sel_bar<NT>();
}

// One radix pass over the row: histogram of digit (key >> shift) of the keys whose
// higher bits equal prefix, then the digit that holds the need-th largest key.
template <int NT, int BITS>
__device__ __forceinline__ void sel_pass(const float* src, int n, int shift, bool first,
                                         uint32_t& prefix, uint32_t& need, SelShared& sh, int tid) {
  constexpr int NB = 1 << BITS;
  for (int i = tid; i < NB; i += NT) sh.hist[i] = 0u;
  sel_bar<NT>();
  const int hi = shift + BITS;
  auto count = [&](float x) {
    const uint32_t key = sel_key(x);
    if (first || (key >> hi) == prefix) atomicAdd(&sh.hist[(key >> shift) & (NB - 1)], 1u);
  };
  const int n4 = n & ~3;
  for (int i = tid * 4; i < n4; i += NT * 4) {
    const float4 v = __ldcg(reinterpret_cast<const float4*>(src + i));
    count(v.x);
    count(v.y);
    count(v.z);
    count(v.w);
  }
  for (int i = n4 + tid; i < n; i += NT) count(__ldcg(src + i));
  sel_bar<NT>();
  sel_find<NT, BITS>(sh, tid, first, prefix, need);
}

// The top-k of the n scores at src (16-byte aligned): indices ascending into dst
// [k] (-1 padded when n < k) and, if dsc is not null, their scores into dsc.
template <int NT>
__device__ void select_row(const float* src, int n, int k, int32_t* dst, float* dsc, SelShared& sh,
                           int tid) {
  if (n <= k) {
    for (int i = tid; i < k; i += NT) {
      dst[i] = i < n ? i : -1;
      if (dsc != nullptr) dsc[i] = i < n ? __ldcg(src + i) : 0.f;
    }
    return;
  }
  uint32_t prefix = 0, need = (uint32_t)k;
  sel_pass<NT, 11>(src, n, 21, true, prefix, need, sh, tid);
  sel_pass<NT, 11>(src, n, 10, false, prefix, need, sh, tid);
  sel_pass<NT, 10>(src, n, 0, false, prefix, need, sh, tid);
  const uint32_t T = prefix;
  const uint32_t need_eq = need;   // keys equal to T that are selected, lowest indices first
  constexpr int ITEMS = 8;
  uint32_t g_run = 0, e_run = 0;
  for (int base = 0; base < n; base += NT * ITEMS) {
    const int i0 = base + tid * ITEMS;
    float x[ITEMS];
    if (i0 + ITEMS <= n) {
      const float4 v0 = __ldcg(reinterpret_cast<const float4*>(src + i0));
      const float4 v1 = __ldcg(reinterpret_cast<const float4*>(src + i0 + 4));
      x[0] = v0.x; x[1] = v0.y; x[2] = v0.z; x[3] = v0.w;
      x[4] = v1.x; x[5] = v1.y; x[6] = v1.z; x[7] = v1.w;
    } else {
#pragma unroll
      for (int j = 0; j < ITEMS; ++j) x[j] = i0 + j < n ? __ldcg(src + i0 + j) : 0.f;
    }
    uint32_t g = 0, e = 0;
#pragma unroll
    for (int j = 0; j < ITEMS; ++j) {
      const uint32_t key = sel_key(x[j]);
      if (i0 + j < n) {
        g += key > T;
        e += key == T;
      }
    }
    uint32_t total;
    const uint32_t excl = sel_scan<NT>((e << 16) | g, sh, tid, total);
    uint32_t G = g_run + (excl & 0xFFFFu);
    uint32_t E = e_run + (excl >> 16);
#pragma unroll
    for (int j = 0; j < ITEMS; ++j) {
      if (i0 + j < n) {
        const uint32_t key = sel_key(x[j]);
        if (key > T) {
          const uint32_t pos = G + min(E, need_eq);
          dst[pos] = i0 + j;
          if (dsc != nullptr) dsc[pos] = x[j];
          ++G;
        } else if (key == T) {
          if (E < need_eq) {
            dst[G + E] = i0 + j;
            if (dsc != nullptr) dsc[G + E] = x[j];
          }
          ++E;
        }
      }
    }
    g_run += total & 0xFFFFu;
    e_run += total >> 16;
  }
}

template <int D_I, int H_I, int N, bool SEL = false>
struct IdxTraits {
  static constexpr int T_BLK = N / H_I;
  static constexpr int KT = 128;
  static constexpr int KTILE_BYTES = KT * D_I;
  static constexpr int QBLK_BYTES = N * D_I;
  // key-tile ring depth; the single-token variant keeps two CTAs per SM in smem
  static constexpr int STAGES = (D_I == 128) ? (N == 64 ? 5 : 6) : 8;
  static constexpr int ACC = 2;
  static constexpr int TMEM_COLS = (ACC * N <= 32) ? 32 : (ACC * N <= 64) ? 64
                                   : (ACC * N <= 128) ? 128 : (ACC * N <= 256) ? 256 : 512;
  // epilogue warps: four per TMEM lane quadrant with one token each at N = 256 (the
  // epilogue is latency-bound; with the fused selectors' threads the registers
  // allow two per quadrant)
  static constexpr int EPI_WARPS = (T_BLK >= 4 && !SEL) ? 16 : (T_BLK >= 2) ? 8 : 4;
  static constexpr int MIN_CTAS = (N == 64) ? 2 : 1;        // CTAs per SM the registers must allow
  static constexpr int EPI_THREADS = EPI_WARPS * 32;
  // selector warps of the fused top-k (two beside the single-token epilogue, so two
  // CTAs still share an SM)
  static constexpr int SEL_WARPS = SEL ? (N == 64 ? 2 : 4) : 0;
  static constexpr int SEL_THREADS = SEL_WARPS * 32;
  static constexpr int THREADS = 64 + EPI_THREADS + SEL_THREADS;
  static constexpr uint32_t SWZ = (D_I == 128) ? 2u : 6u;   // 128B / 32B swizzle
  static constexpr uint32_t SBO = 8u * D_I;                  // bytes per 8-row group
  static constexpr uint32_t IDESC = make_idesc(0, 0, 0, 0, N, 128);
  // shared memory layout (offsets from a 1024-aligned base)
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + 2 * QBLK_BYTES;
  static constexpr int OFF_W = OFF_K + STAGES * KTILE_BYTES;
  static constexpr int OFF_BAR = OFF_W + 4 * N * 4;  // EPI_WARPS x (N / HALVES) floats
  static constexpr int NUM_BARS = 2 + 2 + 2 * STAGES + 2 * ACC + 1;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr int OFF_SEL = OFF_MISC + 16;             // selector state (fused top-k)
  static constexpr int SMEM_BYTES = OFF_SEL + (SEL ? (int)sizeof(SelShared) : 0) + 1024;  // + alignment slack
  static_assert(N % 16 == 0 && N <= 256, "N");
  static_assert(ACC * N <= 512, "TMEM");
  static_assert(H_I == 64 || (H_I < 32 && 32 % H_I == 0), "heads per chunk");
};

struct Unit {
  int b, t_a, t_b, s_lo, s_hi;
};

template <int T_BLK, bool PAGED>
__device__ __forceinline__ int unit_count(const IndexerArgs& a, int& nblk, int& maxp) {
  nblk = (a.t_hi - a.t_lo + T_BLK - 1) / T_BLK;
  // with per-sequence lengths every sequence may use the whole capacity
  int keys_max = PAGED ? a.Lk : min(a.Lk, a.q_pos0 + a.t_hi);
  maxp = (keys_max + a.piece_keys - 1) / a.piece_keys;
  return a.B * nblk * maxp;
}

template <int T_BLK, bool PAGED>
__device__ __forceinline__ bool get_unit(const IndexerArgs& a, int u, int nblk, int maxp,
                                         Unit& o) {
  int piece = u % maxp;
  int rest = u / maxp;
  int blk = rest % nblk;
  o.b = rest / nblk;
  o.t_a = a.t_lo + blk * T_BLK;
  o.t_b = min(o.t_a + T_BLK, a.t_hi);
  const int qp = PAGED ? seq_pos0(a.seq_lens, a.q_pos0, a.Lq, o.b) : a.q_pos0;
  int keys = min(a.Lk, qp + o.t_b);  // keys 0 .. q_pos0 + t_b - 1
  o.s_lo = piece * a.piece_keys;
  o.s_hi = min(keys, o.s_lo + a.piece_keys);
  return o.s_lo < o.s_hi;
}

// PAGED: keys, key scales and causal bounds come through the paged-cache fields
// (block table, per-sequence lengths); the unpaged instantiation has none of it.
// SEL: fused top-k; selector warps (after the epilogue warps) select rows once the
// pieces of every unit of the row have been scored, from the same score chunk.
template <int D_I, int H_I, int N, bool PAGED, bool SEL>
__global__ void __launch_bounds__(IdxTraits<D_I, H_I, N, SEL>::THREADS, IdxTraits<D_I, H_I, N, SEL>::MIN_CTAS)
    indexer_kernel(const __grid_constant__ CUtensorMap tmap_q,
                   const __grid_constant__ CUtensorMap tmap_k, const IndexerArgs a) {
  using Tr = IdxTraits<D_I, H_I, N, SEL>;
  constexpr int T_BLK = Tr::T_BLK;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);

  uint8_t* q_smem = smem + Tr::OFF_Q;
  uint8_t* k_smem = smem + Tr::OFF_K;
  float* wq = reinterpret_cast<float*>(smem + Tr::OFF_W);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Tr::OFF_BAR);
  uint64_t* q_full = bars;
  uint64_t* q_empty = bars + 2;
  uint64_t* k_full = bars + 4;
  uint64_t* k_empty = k_full + Tr::STAGES;
  uint64_t* acc_full = k_empty + Tr::STAGES;
  uint64_t* acc_empty = acc_full + Tr::ACC;
  uint64_t* done_bar = acc_empty + Tr::ACC;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Tr::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Tr::OFF_MISC + 4);

  const int warp = warp_id();
  const int lane = lane_id();

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 1);
    }
    for (int i = 0; i < Tr::STAGES; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
    }
    for (int i = 0; i < Tr::ACC; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], Tr::EPI_THREADS);
    }
    mbar_init(done_bar, 1);
    *abort_flag = 0;
    if constexpr (SEL) {
      SelShared* sh = reinterpret_cast<SelShared*>(smem + Tr::OFF_SEL);
      for (int i = 0; i < 4; ++i) sh->ucnt[i] = 0u;
    }
    fence_barrier_init();
    tma_prefetch_map(&tmap_q);
    tma_prefetch_map(&tmap_k);
  }
  if (warp == 1) tmem_alloc(tmem_slot, Tr::TMEM_COLS);
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;

  int nblk, maxp;
  const int total = unit_count<T_BLK, PAGED>(a, nblk, maxp);

  if (warp == 0) {
    // ------------------------------------------------ TMA producer
    if (lane == 0) {
      int kst = 0, kph = 0, qb = 0, qph = 0;
      int k_pending[Tr::STAGES];
      for (int i = 0; i < Tr::STAGES; ++i) k_pending[i] = -1;
      int q_pending[2] = {-1, -1};
      bool ok = true;
      for (int u = blockIdx.x; u < total && ok; u += gridDim.x) {
        Unit un;
        if (!get_unit<T_BLK, PAGED>(a, u, nblk, maxp, un)) continue;
        if (!mbar_wait(&q_empty[qb], qph ^ 1, a.ctl, abort_flag, kSiteIndexer, 1)) { ok = false; break; }
        q_pending[qb] = -1;
        mbar_arrive_expect_tx(&q_full[qb], Tr::QBLK_BYTES);
        tma_load_2d(q_smem + qb * Tr::QBLK_BYTES, &tmap_q, 0,
                    (un.b * a.Lq + un.t_a) * H_I, &q_full[qb]);
        q_pending[qb] = qph;
        if (++qb == 2) { qb = 0; qph ^= 1; }
        for (int s0 = un.s_lo; s0 < un.s_hi; s0 += Tr::KT) {
          if (!mbar_wait(&k_empty[kst], kph ^ 1, a.ctl, abort_flag, kSiteIndexer, 2)) { ok = false; break; }
          k_pending[kst] = -1;
          mbar_arrive_expect_tx(&k_full[kst], Tr::KTILE_BYTES);
          // a tile of 128 keys never crosses a page (page_size is a multiple of 128); a
          // page number outside the pool points past the tensor map: the tile reads zeros
          long long krow = (long long)un.b * a.Lk + s0;
          if constexpr (PAGED) {
            krow = key_row(a.block_table, a.max_blocks, a.page_size, a.num_pages, un.b, a.Lk, s0);
            if (krow < 0) krow = (long long)a.num_pages * a.page_size;
          }
          tma_load_2d(k_smem + kst * Tr::KTILE_BYTES, &tmap_k, 0, (int)krow, &k_full[kst]);
          k_pending[kst] = kph;
          if (++kst == Tr::STAGES) { kst = 0; kph ^= 1; }
        }
      }
      if (*abort_flag) {
        // Let copies that are still in flight land before the CTA exits.
        DevCtl drain = a.ctl;
        volatile int never = 0;
        for (int i = 0; i < Tr::STAGES; ++i)
          if (k_pending[i] >= 0) mbar_wait(&k_full[i], k_pending[i], drain, &never, kSiteIndexer, 3);
        for (int i = 0; i < 2; ++i)
          if (q_pending[i] >= 0) mbar_wait(&q_full[i], q_pending[i], drain, &never, kSiteIndexer, 3);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      int kst = 0, kph = 0, qb = 0, qph = 0, ac = 0, aph = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < total && ok; u += gridDim.x) {
        Unit un;
        if (!get_unit<T_BLK, PAGED>(a, u, nblk, maxp, un)) continue;
        if (!mbar_wait(&q_full[qb], qph, a.ctl, abort_flag, kSiteIndexer, 4)) { ok = false; break; }
        const uint32_t q_addr = smem_u32(q_smem + qb * Tr::QBLK_BYTES);
        for (int s0 = un.s_lo; s0 < un.s_hi; s0 += Tr::KT) {
          if (!mbar_wait(&k_full[kst], kph, a.ctl, abort_flag, kSiteIndexer, 5)) { ok = false; break; }
          if (!mbar_wait(&acc_empty[ac], aph ^ 1, a.ctl, abort_flag, kSiteIndexer, 6)) { ok = false; break; }
          tc_fence_after();
          const uint32_t k_addr = smem_u32(k_smem + kst * Tr::KTILE_BYTES);
          const uint32_t d_tmem = tbase + (uint32_t)(ac * N);
#pragma unroll
          for (int kk = 0; kk < D_I / 32; ++kk) {
            uint64_t ad = make_sdesc(k_addr + kk * 32, 16, Tr::SBO, Tr::SWZ);
            uint64_t bd = make_sdesc(q_addr + kk * 32, 16, Tr::SBO, Tr::SWZ);
            mma_f8_ss(d_tmem, ad, bd, Tr::IDESC, kk > 0 ? 1u : 0u);
          }
          mma_commit(&k_empty[kst]);
          mma_commit(&acc_full[ac]);
          if (++kst == Tr::STAGES) { kst = 0; kph ^= 1; }
          if (++ac == Tr::ACC) { ac = 0; aph ^= 1; }
        }
        if (!ok) break;
        mma_commit(&q_empty[qb]);
        if (++qb == 2) { qb = 0; qph ^= 1; }
      }
      // every MMA issued by this thread has completed once done_bar flips
      mma_commit(done_bar);
      DevCtl drain = a.ctl;
      volatile int never = 0;
      mbar_wait(done_bar, 0, drain, &never, kSiteIndexer, 7);
    }
  } else if (warp < 2 + Tr::EPI_WARPS) {
    // ------------------------------------------------ epilogue
    const int ew = warp - 2;                 // 0 .. EPI_WARPS-1
    const int quad = warp & 3;               // TMEM lane quadrant this warp may access
    constexpr int HALVES = Tr::EPI_WARPS / 4;
    const int half = ew / 4;
    constexpr int COLS = N / HALVES;         // columns (token x head) handled by this warp
    const int c_begin = half * COLS;
    const int key_in_tile = quad * 32 + lane;
    float* wbuf = wq + ew * COLS;           // this warp's folded weights
    const uint32_t t_lane = tbase + ((uint32_t)(quad * 32) << 16);
    int ac = 0, aph = 0;
    bool ok = true;
    uint32_t ul = 0;   // units of this CTA done so far
    for (int u = blockIdx.x; u < total && ok; u += gridDim.x) {
      Unit un;
      if (!get_unit<T_BLK, PAGED>(a, u, nblk, maxp, un)) continue;
      // folded per-(token, head) weight w * s^q of this warp's columns, in a
      // buffer private to the warp (no cross-warp barrier)
      __syncwarp();
      for (int c = c_begin + lane; c < c_begin + COLS; c += 32) {
        int t = un.t_a + c / H_I;
        float v = 0.f;
        if (t < un.t_b) {
          size_t off = ((size_t)un.b * a.Lq + t) * H_I + (c % H_I);
          float wv = a.w_bf16 ? __uint_as_float(((uint32_t)reinterpret_cast<const uint16_t*>(a.w)[off]) << 16)
                              : reinterpret_cast<const float*>(a.w)[off];
          v = wv * a.qI_scale[off];
        }
        wbuf[c - c_begin] = v;
      }
      __syncwarp();
      // single-token blocks (decode): this unit's 64 folded weights stay in registers
      float wr[(T_BLK == 1 && H_I == 64) ? 64 : 1];
      if constexpr (T_BLK == 1 && H_I == 64) {
#pragma unroll
        for (int j = 0; j < 64; ++j) wr[j] = wbuf[j];
      }
      // key scales are fetched one tile ahead so their latency hides behind a tile
      const float* ks_row = a.kI_scale + (size_t)un.b * a.Lk;
      auto ks_at = [&](int s) -> float {   // scale of logical key s of this unit's sequence
        if constexpr (PAGED) {
          const long long r = key_row(a.block_table, a.max_blocks, a.page_size, a.num_pages, un.b, a.Lk, s);
          return r >= 0 ? __ldg(a.kI_scale + r) : 0.f;
        } else {
          return __ldg(ks_row + s);
        }
      };
      const int qp = PAGED ? seq_pos0(a.seq_lens, a.q_pos0, a.Lq, un.b) : a.q_pos0;
      float ks_next = (un.s_lo + key_in_tile < un.s_hi) ? ks_at(un.s_lo + key_in_tile) : 0.f;
      for (int s0 = un.s_lo; s0 < un.s_hi; s0 += Tr::KT) {
        const int s = s0 + key_in_tile;
        const bool key_ok = s < un.s_hi;
        const float ks = ks_next;
        ks_next = (s + Tr::KT < un.s_hi) ? ks_at(s + Tr::KT) : 0.f;
        if (!mbar_wait(&acc_full[ac], aph, a.ctl, abort_flag, kSiteIndexer, 8)) { ok = false; break; }
        tc_fence_after();
        if constexpr (H_I == 64) {
          // all of this warp's columns (one token of 64 heads per 64 columns) are
          // loaded with one wait, and the accumulator goes back to the MMA issuer
          // before the head reduction runs from registers
          // (with the fused selectors' threads the registers allow one token per wait)
          constexpr int NTOK = COLS / 64;
          constexpr int G = SEL ? 1 : NTOK;   // tokens per wait
#pragma unroll
          for (int tg = 0; tg < NTOK; tg += G) {
          uint32_t rr[G][64];
#pragma unroll
          for (int tk = 0; tk < G; ++tk) {
            tmem_ld32(t_lane + (uint32_t)(ac * N + c_begin + 64 * (tg + tk)),
                      *reinterpret_cast<uint32_t(*)[32]>(rr[tk]));
            tmem_ld32(t_lane + (uint32_t)(ac * N + c_begin + 64 * (tg + tk) + 32),
                      *reinterpret_cast<uint32_t(*)[32]>(rr[tk] + 32));
          }
          tmem_wait_ld();
          if (tg + G >= NTOK) {
            tc_fence_before();
            mbar_arrive(&acc_empty[ac]);
          }
#pragma unroll
          for (int tk = 0; tk < G; ++tk) {
            const int c0 = c_begin + 64 * (tg + tk);
            const uint32_t* r = rr[tk];
            // four independent packed partial sums: no serial FMA chain
            float2 acc2[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                              make_float2(0.f, 0.f)};
#pragma unroll
            for (int g = 0; g < 16; ++g) {
              float4 wv;
              if constexpr (T_BLK == 1) {
                wv = make_float4(wr[4 * g], wr[4 * g + 1], wr[4 * g + 2], wr[4 * g + 3]);
              } else {
                wv = reinterpret_cast<const float4*>(wbuf + (c0 - c_begin))[g];
              }
              const float2 x01 = make_float2(fmaxf(__uint_as_float(r[4 * g + 0]), 0.f),
                                             fmaxf(__uint_as_float(r[4 * g + 1]), 0.f));
              const float2 x23 = make_float2(fmaxf(__uint_as_float(r[4 * g + 2]), 0.f),
                                             fmaxf(__uint_as_float(r[4 * g + 3]), 0.f));
              ffma2(acc2[(2 * g) & 3], make_float2(wv.x, wv.y), x01);
              ffma2(acc2[(2 * g + 1) & 3], make_float2(wv.z, wv.w), x23);
            }
            const float part = ((acc2[0].x + acc2[0].y) + (acc2[1].x + acc2[1].y)) +
                               ((acc2[2].x + acc2[2].y) + (acc2[3].x + acc2[3].y));
            const int t = un.t_a + c0 / 64;
            if (key_ok && t < un.t_b && s <= qp + t)
              a.scores[((long long)un.b * a.sc_bstride + (t - a.sc_t0)) * a.sc_ld + s] = part * ks;
          }
          }
        } else {
#pragma unroll 1
          for (int c0 = c_begin; c0 < c_begin + COLS; c0 += 32) {
            uint32_t r[32];
            tmem_ld32(t_lane + (uint32_t)(ac * N + c0), r);
            tmem_wait_ld();
            constexpr int TPC = 32 / H_I;  // tokens per 32-column chunk
            const float* wv = wbuf + (c0 - c_begin);
#pragma unroll
            for (int g = 0; g < TPC; ++g) {
              float acc = 0.f;
#pragma unroll
              for (int j = 0; j < H_I; ++j)
                acc = fmaf(wv[g * H_I + j], fmaxf(__uint_as_float(r[g * H_I + j]), 0.f), acc);
              const int t = un.t_a + c0 / H_I + g;
              if (key_ok && t < un.t_b && s <= qp + t) {
                a.scores[((long long)un.b * a.sc_bstride + (t - a.sc_t0)) * a.sc_ld + s] = acc * ks;
              }
            }
          }
          tc_fence_before();
          mbar_arrive(&acc_empty[ac]);
        }
        if (++ac == Tr::ACC) { ac = 0; aph ^= 1; }
      }
      if constexpr (SEL) {
        // The unit's scores are written. The last epilogue thread of the CTA to get
        // here counts the unit as one scored piece of each of its rows: every
        // thread fences its own score stores before its count, and the last one
        // fences again before publishing, so a selector that reads the row's
        // count with acquire semantics sees every score of the row.
        if (ok) {
          SelShared* sh = reinterpret_cast<SelShared*>(smem + Tr::OFF_SEL);
          __threadfence();
          const uint32_t old = atomicAdd(&sh->ucnt[ul & 3u], 1u);
          if (old + 1u == (uint32_t)Tr::EPI_THREADS * ((ul >> 2) + 1u)) {
            __threadfence();
            const int rows = a.sel_t1 - a.sel_t0;
            for (int t = un.t_a; t < un.t_b; ++t)
              atomicAdd(a.row_cnt + (long long)un.b * rows + (t - a.sel_t0), 1);
          }
          ++ul;
        }
      }
    }
  } else if constexpr (SEL) {
    // ------------------------------------------------ selectors (fused top-k)
    // Row r of the launch (sequence b, query row t in [sel_t0, sel_t1)) belongs to
    // CTA r % gridDim.x. Scored rows wait until all pieces of their unit are
    // counted; rows with at most k candidates select every key.
    SelShared& sh = *reinterpret_cast<SelShared*>(smem + Tr::OFF_SEL);
    constexpr int NT = Tr::SEL_THREADS;
    const int tid = threadIdx.x - (64 + Tr::EPI_THREADS);
    const int rows_per_b = a.sel_t1 - a.sel_t0;
    const long long nrows = (long long)a.B * rows_per_b;
    for (long long r = blockIdx.x; r < nrows; r += gridDim.x) {
      const int b = (int)(r / rows_per_b);
      const int t = a.sel_t0 + (int)(r % rows_per_b);
      const int qp = PAGED ? seq_pos0(a.seq_lens, a.q_pos0, a.Lq, b) : a.q_pos0;
      const int n = min(a.Lk, qp + t + 1);
      const bool scored = t >= a.t_lo && t < a.t_hi;
      if (tid == 0) {
        int go = 1;
        if (scored) {
          // pieces of the row's unit: as many as get_unit gives its token block
          const int blk = (t - a.t_lo) / T_BLK;
          const int t_b = min(a.t_lo + (blk + 1) * T_BLK, a.t_hi);
          const int keys = min(a.Lk, qp + t_b);
          const uint32_t pieces = (uint32_t)((keys + a.piece_keys - 1) / a.piece_keys);
          const int* cnt = a.row_cnt + r;
          const uint64_t t0 = globaltimer_ns();
          while (ld_acquire_u32(cnt) < pieces) {
            if (*abort_flag || *reinterpret_cast<volatile int*>(a.ctl.status) != 0) { go = 0; break; }
            if (globaltimer_ns() - t0 > a.ctl.wait_ns) {
              report_timeout(a.ctl, kSiteIndexer, 20);
              go = 0;
              break;
            }
            __nanosleep(256);
          }
          if (go) a.row_cnt[r] = 0;   // counted out: zero again for the next launch
        }
        sh.go = go;
      }
      sel_bar<NT>();
      const int go = sh.go;
      sel_bar<NT>();
      if (!go) {
        if (tid == 0) *abort_flag = 1;
        break;
      }
      const float* src = a.scores + ((long long)b * a.sc_bstride + (t - a.sc_t0)) * a.sc_ld;
      const long long orow = ((long long)b * a.Lq + t) * a.k;
      select_row<NT>(src, scored ? n : min(n, a.k), a.k, a.idx + orow,
                     a.sel_scores != nullptr && scored ? a.sel_scores + orow : nullptr, sh, tid);
      sel_bar<NT>();
    }
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, Tr::TMEM_COLS);
  }
}

template <int D_I, int H_I, int N, bool SEL>
cudaError_t launch_variant(const CUtensorMap& tq, const CUtensorMap& tk, const IndexerArgs& a,
                           int num_sms, cudaStream_t stream) {
  using Tr = IdxTraits<D_I, H_I, N, SEL>;
  const bool paged = a.block_table != nullptr || a.seq_lens != nullptr;
  auto kern = paged ? indexer_kernel<D_I, H_I, N, true, SEL> : indexer_kernel<D_I, H_I, N, false, SEL>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       Tr::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  int nblk = (a.t_hi - a.t_lo + Tr::T_BLK - 1) / Tr::T_BLK;
  if (nblk < 0) nblk = 0;
  int keys_max = a.seq_lens != nullptr ? a.Lk : (a.q_pos0 + a.t_hi < a.Lk ? a.q_pos0 + a.t_hi : a.Lk);
  long long maxp = (keys_max + a.piece_keys - 1) / a.piece_keys;
  long long units = (long long)a.B * nblk * maxp;
  // fused top-k: CTAs without units still select rows
  const long long work = SEL ? (units > (long long)a.B * (a.sel_t1 - a.sel_t0) ? units
                                                                             : (long long)a.B * (a.sel_t1 - a.sel_t0))
                             : units;
  if (work <= 0) return cudaSuccess;
  // persistent CTAs: as many as fit on the SMs at once (smem and TMEM allow two
  // of the single-token variant per SM)
  int per_sm = (2 * Tr::SMEM_BYTES <= 227 * 1024 && 2 * Tr::TMEM_COLS <= 512) ? 2 : 1;
  if (SEL) {
    // the selectors wait on rows other CTAs score: every CTA must be resident at
    // once, which the cooperative launch guarantees for a grid within occupancy
    int occ = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, Tr::THREADS, Tr::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    if (occ < per_sm) per_sm = occ;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
  }
  const int grid = (int)(work < (long long)per_sm * num_sms ? work : (long long)per_sm * num_sms);
  if (!SEL) {
    kern<<<grid, Tr::THREADS, Tr::SMEM_BYTES, stream>>>(tq, tk, a);
    return cudaGetLastError();
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(Tr::THREADS);
  cfg.dynamicSmemBytes = Tr::SMEM_BYTES;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, tq, tk, a);
}

__global__ void fill_noncausal_kernel(float* scores, int B, int Lq, int Lk, int q_pos0) {
  const long long row = blockIdx.x;  // b * Lq + t
  const int t = (int)(row % Lq);
  const int first = q_pos0 + t + 1;
  float* dst = scores + row * Lk;
  for (int s = first + (int)threadIdx.x; s < Lk; s += blockDim.x) dst[s] = -__int_as_float(0x7f800000);
}


template <bool SEL>
cudaError_t launch_indexer_sel(const CUtensorMap& tmap_q, const CUtensorMap& tmap_k,
                               const IndexerArgs& a, int H_I, int d_I, int num_sms,
                               cudaStream_t stream) {
  if (H_I == 64 && d_I == 128) {
    if (a.t_hi - a.t_lo <= 1) return launch_variant<128, 64, 64, SEL>(tmap_q, tmap_k, a, num_sms, stream);
    return launch_variant<128, 64, 256, SEL>(tmap_q, tmap_k, a, num_sms, stream);
  }
  if (H_I == 4 && d_I == 32) return launch_variant<32, 4, 256, SEL>(tmap_q, tmap_k, a, num_sms, stream);
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_indexer(const CUtensorMap& tmap_q, const CUtensorMap& tmap_k,
                           const IndexerArgs& a, int H_I, int d_I, int num_sms,
                           cudaStream_t stream) {
  if (a.select) {
    if (a.sel_t1 <= a.sel_t0) return cudaSuccess;
    return launch_indexer_sel<true>(tmap_q, tmap_k, a, H_I, d_I, num_sms, stream);
  }
  if (a.t_hi <= a.t_lo) return cudaSuccess;
  return launch_indexer_sel<false>(tmap_q, tmap_k, a, H_I, d_I, num_sms, stream);
}


cudaError_t launch_fill_noncausal(float* scores, int B, int Lq, int Lk, int q_pos0,
                                  cudaStream_t stream) {
  long long rows = (long long)B * Lq;
  if (rows == 0) return cudaSuccess;
  fill_noncausal_kernel<<<(unsigned)rows, 256, 0, stream>>>(scores, B, Lq, Lk, q_pos0);
  return cudaGetLastError();
}

}  // namespace dsa
