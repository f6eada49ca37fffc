// topk.cu - fine-grained token selection: the k largest index scores of each
// query row ("DeepSeek-V3.2: Pushing the Frontier of Open Large Language Models",
// bud-325 paper digest, "Key claims", section 2.1, and "Method": k = 2048 key-value
// entries per query token).
//
// One CTA per query row. Scores are mapped to order-preserving 32-bit keys
// (-0.0 folded onto +0.0) and the exact k-th largest key T is found by a
// three-digit radix select (11 + 11 + 10 bits, most significant first): each
// pass histograms the keys that still match the selected prefix in shared
// memory (the first while the row is staged) and a block scan picks the digit
// where the running count from the top crosses k. A final ordered pass writes
// every key > T and the first (k - #{key > T}) keys == T, in ascending index
// order: each warp owns a contiguous run of the row, counts its (greater,
// equal) keys, and after one block-wide exchange of those counts writes its run
// with warp scans of 128 keys at a time. Ties therefore go to the lowest index
// and the output is sorted. Shared-memory sweeps read four keys per thread per
// load.
// Rows of up to 48K candidates are staged once in shared memory as keys. Longer
// rows, or launches with fewer rows than SMs, spread each row over a cluster of
// 8 CTAs (topk_cluster_kernel); rows beyond 8 x 48K are re-read from global
// memory (L2) on each pass.
// Rows with at most k candidates select all of them and pad with -1.
#include <type_traits>

#include "dsa_kernels.h"

namespace dsa {
namespace {

constexpr int TK_THREADS = 512;                   // a CTA of the cluster kernel (rows split over 8)
constexpr int TK1_THREADS = 1024;                 // a CTA of the single-CTA kernel on long rows
constexpr int TK_MAX_WARPS = TK1_THREADS / 32;
// Rows staged in more shared memory than two CTAs of an SM can hold run with
// TK1_THREADS threads per CTA (one row per SM: more warps hide the passes'
// latency); shorter rows run with TK_THREADS, several CTAs per SM.
constexpr int TK_WIDE_KEYS = 26 * 1024;
constexpr int TK_SMEM_MAX = 48 * 1024;            // candidates staged in shared memory
constexpr int TK_STEP = 128;                      // keys per warp step of the output pass

__device__ __forceinline__ uint32_t score_key(float x) {
  uint32_t u = __float_as_uint(x);
  if (u == 0x80000000u) u = 0u;                   // -0.0 == +0.0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// The score of an order-preserving key (-0.0 comes back as +0.0).
__device__ __forceinline__ float key_score(uint32_t key) {
  return __uint_as_float((key & 0x80000000u) ? (key & 0x7FFFFFFFu) : ~key);
}

__device__ __forceinline__ uint32_t warp_sum_u32(uint32_t v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Exclusive block scan of one int per thread; also returns the block total.
template <int NT>
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t* tmp, uint32_t& total) {
  constexpr int NW = NT / 32;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  uint32_t incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    uint32_t n = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += n;
  }
  if (lane == 31) tmp[wid] = incl;
  __syncthreads();
  if (wid == 0) {
    uint32_t x = lane < NW ? tmp[lane] : 0u;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      uint32_t n = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += n;
    }
    if (lane < NW) tmp[lane] = x;
  }
  __syncthreads();
  uint32_t off = wid > 0 ? tmp[wid - 1] : 0u;
  total = tmp[NW - 1];
  __syncthreads();
  return off + incl - v;
}

// Given a histogram of the candidate digits, pick the digit holding the
// `need`-th largest key; extend `prefix` by it and make `need` the rank within
// that digit (uniform across the block).
template <int BITS, int NT>
__device__ __forceinline__ void find_bin(const uint32_t* hist, bool first, uint32_t& prefix,
                                         uint32_t& need, uint32_t* tmp, uint32_t* sel) {
  constexpr int BPT = (1 << BITS) / NT;
  uint32_t local = 0;
  const int b0 = threadIdx.x * BPT;
#pragma unroll
  for (int j = 0; j < BPT; ++j) local += hist[b0 + j];
  uint32_t total;
  uint32_t before = block_excl_scan<NT>(local, tmp, total);
  uint32_t above = total - before - local;  // keys in bins of higher-numbered threads
#pragma unroll
  for (int j = BPT - 1; j >= 0; --j) {
    uint32_t h = hist[b0 + j];
    if (above < need && need <= above + h) {
      sel[0] = (uint32_t)(b0 + j);
      sel[1] = need - above;
    }
    above += h;
  }
  __syncthreads();
  prefix = first ? sel[0] : ((prefix << BITS) | sel[0]);
  need = sel[1];
  __syncthreads();
}

// Keys staged in shared memory. The staging buffer holds a multiple of four
// words, so a 16-byte load at any i % 4 == 0 with i < m stays inside it; the
// words past m are never counted (callers pass validity separately).
struct SmemKeys {
  const uint32_t* keys;
  __device__ __forceinline__ uint4 load4(int i, int) const {
    return *reinterpret_cast<const uint4*>(keys + i);
  }
};

// Keys computed from global (L2-resident) scores on every read.
struct GlobalKeys {
  const float* src;
  bool vec;   // 16-byte aligned row
  __device__ __forceinline__ uint4 load4(int i, int m) const {
    if (vec && i + 3 < m) {
      const float4 v = __ldg(reinterpret_cast<const float4*>(src + i));
      return make_uint4(score_key(v.x), score_key(v.y), score_key(v.z), score_key(v.w));
    }
    uint4 r;
    r.x = i < m ? score_key(__ldg(src + i)) : 0u;
    r.y = i + 1 < m ? score_key(__ldg(src + i + 1)) : 0u;
    r.z = i + 2 < m ? score_key(__ldg(src + i + 2)) : 0u;
    r.w = i + 3 < m ? score_key(__ldg(src + i + 3)) : 0u;
    return r;
  }
};

// Histogram (into `hist`, already cleared) the digit (key >> shift) of the keys
// of [0, m) whose bits above `shift + BITS` equal `prefix`.
template <int BITS, int NT, class Keys>
__device__ __forceinline__ void histogram_digit(const Keys& keys, int m, int shift, bool first,
                                                uint32_t prefix, uint32_t* hist) {
  constexpr uint32_t MASK = (1u << BITS) - 1u;
  const int hi_shift = shift + BITS;
  auto count = [&](uint32_t key, bool valid) {
    if (valid && (first || (key >> hi_shift) == prefix)) atomicAdd(&hist[(key >> shift) & MASK], 1u);
  };
  const int groups = (m + 3) >> 2;
#pragma unroll 4
  for (int g = threadIdx.x; g < groups; g += NT) {
    const int i = g << 2;
    const uint4 v = keys.load4(i, m);
    count(v.x, true);
    count(v.y, i + 1 < m);
    count(v.z, i + 2 < m);
    count(v.w, i + 3 < m);
  }
}

// One radix pass of the single-CTA kernel: histogram, then find the digit
// holding the `need`-th largest key. Updates prefix/need in place.
template <int BITS, int NT, class Keys>
__device__ __forceinline__ void radix_pass(const Keys& keys, int n, int shift, bool first,
                                           uint32_t& prefix, uint32_t& need, uint32_t* hist,
                                           uint32_t* tmp, uint32_t* sel) {
  constexpr int NB = 1 << BITS;
  static_assert(NB / NT >= 1, "bins");
  for (int i = threadIdx.x; i < NB; i += NT) hist[i] = 0u;
  __syncthreads();
  histogram_digit<BITS, NT>(keys, n, shift, first, prefix, hist);
  __syncthreads();
  find_bin<BITS, NT>(hist, first, prefix, need, tmp, sel);
}

// ---------------------------------------------------------------------------
// The ordered output pass. Warp w owns the 128-key steps [s0, s1) of [0, m).
// ---------------------------------------------------------------------------
struct Run {
  int s0, s1;
};

template <int NT>
__device__ __forceinline__ Run warp_run(int m) {
  constexpr int NW = NT / 32;
  const int steps = (m + TK_STEP - 1) / TK_STEP;
  const int per = (steps + NW - 1) / NW;
  const int s0 = min(steps, (int)(threadIdx.x >> 5) * per);
  return Run{s0, min(steps, s0 + per)};
}

// (greater, equal) of one key against T, packed as equal << 16 | greater.
__device__ __forceinline__ uint32_t ge_bits(uint32_t key, bool valid, uint32_t T) {
  return (uint32_t)(valid && key > T) | ((uint32_t)(valid && key == T) << 16);
}

// Counts of keys > T and == T in this warp's run (warp-uniform results).
template <class Keys>
__device__ __forceinline__ void run_counts(const Keys& keys, int m, uint32_t T, Run run,
                                           uint32_t& g, uint32_t& e) {
  const int lane = threadIdx.x & 31;
  uint32_t gl = 0, el = 0;
  for (int s = run.s0; s < run.s1; ++s) {
    const int i = s * TK_STEP + lane * 4;
    if (i < m) {
      const uint4 v = keys.load4(i, m);
      const uint32_t c = ge_bits(v.x, true, T) + ge_bits(v.y, i + 1 < m, T) +
                         ge_bits(v.z, i + 2 < m, T) + ge_bits(v.w, i + 3 < m, T);
      gl += c & 0xFFFFu;
      el += c >> 16;
    }
  }
  g = warp_sum_u32(gl);
  e = warp_sum_u32(el);
}

// Write the selected keys of this warp's run. G and E are the numbers of keys
// > T and == T before the run (in index order, over the whole row); the output
// index of key i is base + i.
template <class Keys>
__device__ __forceinline__ void write_run(const Keys& keys, int m, uint32_t T, uint32_t need_eq,
                                          uint32_t G, uint32_t E, int base, Run run,
                                          int32_t* dst, float* dsc) {
  const int lane = threadIdx.x & 31;
  for (int s = run.s0; s < run.s1; ++s) {
    const int i = s * TK_STEP + lane * 4;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (i < m) v = keys.load4(i, m);
    const uint32_t kk[4] = {v.x, v.y, v.z, v.w};
    uint32_t own = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) own += ge_bits(kk[j], i + j < m, T);
    uint32_t incl = own;   // a step holds at most 128 keys: the packed halves cannot carry
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t x = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += x;
    }
    const uint32_t ex = incl - own;
    uint32_t Gl = G + (ex & 0xFFFFu), El = E + (ex >> 16);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const bool valid = i + j < m;
      const bool gt = valid && kk[j] > T, eq = valid && kk[j] == T;
      // a key > T goes after the selected equal keys before it; an equal key is
      // selected while fewer than need_eq equal keys precede it
      const uint32_t slot = Gl + (gt ? min(El, need_eq) : El);
      if (gt || (eq && El < need_eq)) {
        dst[slot] = base + i + j;
        if (dsc != nullptr) dsc[slot] = key_score(kk[j]);
      }
      Gl += gt;
      El += eq;
    }
    const uint32_t tot = __shfl_sync(0xffffffffu, incl, 31);
    G += tot & 0xFFFFu;
    E += tot >> 16;
  }
}

// Per-warp counts of the run into tmp[wid] / tmp[NT / 32 + wid], then this
// warp's (G, E) offsets within the block and the block totals.
template <int NT, class Keys>
__device__ __forceinline__ void block_run_offsets(const Keys& keys, int m, uint32_t T, Run run,
                                                  uint32_t* tmp, uint32_t& G, uint32_t& E,
                                                  uint32_t& g_tot, uint32_t& e_tot) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  uint32_t g, e;
  run_counts(keys, m, T, run, g, e);
  if (lane == 0) {
    tmp[wid] = g;
    tmp[(NT / 32) + wid] = e;
  }
  __syncthreads();
  G = 0;
  E = 0;
  g_tot = 0;
  e_tot = 0;
#pragma unroll
  for (int w = 0; w < (NT / 32); ++w) {
    const uint32_t gw = tmp[w], ew = tmp[(NT / 32) + w];
    if (w < wid) {
      G += gw;
      E += ew;
    }
    g_tot += gw;
    e_tot += ew;
  }
}

// Stage scores [0, m) as keys in shared memory and histogram their top 11 bits
// (hist already cleared). The caller synchronises.
template <int NT>
__device__ __forceinline__ void stage_keys(const float* src, int m, uint32_t* keys, uint32_t* hist) {
  auto put = [&](int i, uint32_t key) {
    keys[i] = key;
    atomicAdd(&hist[key >> 21], 1u);
  };
  if ((reinterpret_cast<uintptr_t>(src) & 15u) == 0) {
    const int m4 = m >> 2;
    const float4* s4 = reinterpret_cast<const float4*>(src);
    uint4* k4 = reinterpret_cast<uint4*>(keys);
#pragma unroll 4
    for (int i = threadIdx.x; i < m4; i += NT) {
      const float4 v = __ldg(s4 + i);
      const uint4 kk = make_uint4(score_key(v.x), score_key(v.y), score_key(v.z), score_key(v.w));
      k4[i] = kk;
      atomicAdd(&hist[kk.x >> 21], 1u);
      atomicAdd(&hist[kk.y >> 21], 1u);
      atomicAdd(&hist[kk.z >> 21], 1u);
      atomicAdd(&hist[kk.w >> 21], 1u);
    }
    for (int i = (m4 << 2) + threadIdx.x; i < m; i += NT) put(i, score_key(__ldg(src + i)));
  } else {
    for (int i = threadIdx.x; i < m; i += NT) put(i, score_key(__ldg(src + i)));
  }
}

template <bool SMEM_ROW, int NT>
__global__ void __launch_bounds__(NT) topk_kernel(const TopkArgs a) {
  extern __shared__ __align__(16) uint32_t row_keys[];
  __shared__ uint32_t hist[2048];
  __shared__ uint32_t tmp[2 * TK_MAX_WARPS];
  __shared__ uint32_t sel[2];
  using Keys = typename std::conditional<SMEM_ROW, SmemKeys, GlobalKeys>::type;
  const int rows_per_b = a.t_hi - a.t_lo;
  const long long nrows = (long long)a.B * rows_per_b;
  for (long long r = blockIdx.x; r < nrows; r += gridDim.x) {
    const int b = (int)(r / rows_per_b);
    const int t = a.t_lo + (int)(r % rows_per_b);
    const int n = min(a.Lk, seq_pos0(a.seq_lens, a.q_pos0, a.Lq, b) + t + 1);
    int32_t* dst = a.idx + ((long long)b * a.Lq + t) * a.k;
    float* dsc = a.sel != nullptr ? a.sel + ((long long)b * a.Lq + t) * a.k : nullptr;
    const float* src = a.scores + ((long long)b * a.sc_bstride + (t - a.sc_t0)) * a.sc_ld;
    if (n <= a.k) {
      for (int i = threadIdx.x; i < a.k; i += NT) {
        dst[i] = i < n ? i : -1;
        if (dsc != nullptr) dsc[i] = i < n ? src[i] : 0.f;
      }
      continue;
    }
    Keys keys;
    uint32_t prefix = 0, need = (uint32_t)a.k;
    if constexpr (SMEM_ROW) {
      // staging builds the first digit's histogram on the way
      for (int i = threadIdx.x; i < 2048; i += NT) hist[i] = 0u;
      __syncthreads();
      stage_keys<NT>(src, n, row_keys, hist);
      __syncthreads();
      find_bin<11, NT>(hist, true, prefix, need, tmp, sel);
      keys = SmemKeys{row_keys};
    } else {
      keys = GlobalKeys{src, a.vec4 != 0};
      radix_pass<11, NT>(keys, n, 21, true, prefix, need, hist, tmp, sel);
    }
    radix_pass<11, NT>(keys, n, 10, false, prefix, need, hist, tmp, sel);
    radix_pass<10, NT>(keys, n, 0, false, prefix, need, hist, tmp, sel);
    const uint32_t T = prefix;
    const uint32_t need_eq = need;  // keys equal to T that are selected (lowest indices first)

    const Run run = warp_run<NT>(n);
    uint32_t G, E, g_tot, e_tot;
    block_run_offsets<NT>(keys, n, T, run, tmp, G, E, g_tot, e_tot);
    write_run(keys, n, T, need_eq, G, E, 0, run, dst, dsc);
    __syncthreads();   // tmp, hist and the staged row are reused by the next row
  }
}

// ---------------------------------------------------------------------------
// Long rows, or few rows: a cluster of TKC CTAs shares one row. Each CTA stages
// 1/TKC of the row in shared memory; the per-pass histograms are summed over
// the cluster through distributed shared memory, so every CTA picks the same
// digits; the output slots of each CTA follow from a cluster-wide prefix of the
// (greater, equal) counts of the CTAs before it. Same result as topk_kernel.
// ---------------------------------------------------------------------------
constexpr int TKC = 8;

// Sum the CTAs' histograms of one digit over the cluster and pick the digit, as a
// reduce-scatter: CTA r sums bins [r SL, (r + 1) SL) over the cluster into its own
// `ghist` slice and publishes the slice total; then every CTA reads the TKC totals,
// picks the slice that holds the need-th largest key, and finds the bin inside it
// from that slice's sums (read from the CTA that holds them). Every CTA reaches the
// same digit from the same sums. Each CTA reads 1/TKC of the bins from each peer
// instead of all of them.
template <int BITS>
__device__ __forceinline__ void cluster_find(bool first, uint32_t& prefix, uint32_t& need,
                                             uint32_t* hist, uint32_t* ghist, uint32_t* tmp,
                                             uint32_t* sel, uint32_t* stot) {
  constexpr int NB = 1 << BITS;
  constexpr int SL = NB / TKC;        // bins per slice
  constexpr int G4 = SL / 4;          // threads summing a slice, four bins each
  constexpr int PER = SL / 32;        // bins per lane when one warp searches a slice
  static_assert(G4 % 32 == 0 && G4 <= TK_THREADS && PER >= 1, "slice shape");
  const uint32_t rank = cluster_ctarank();
  const int tid = threadIdx.x, lane = tid & 31;
  cluster_sync();   // every CTA's histogram is complete and visible
  if (tid < G4) {
    const uint32_t h0 = smem_u32(hist) + (uint32_t)(rank * SL + 4 * tid) * 4u;
    uint4 v[TKC];
#pragma unroll
    for (int p = 0; p < TKC; ++p) v[p] = ld_cluster_v4(mapa_shared(h0, p));
    uint4 acc = v[0];
#pragma unroll
    for (int p = 1; p < TKC; ++p) {
      acc.x += v[p].x;
      acc.y += v[p].y;
      acc.z += v[p].z;
      acc.w += v[p].w;
    }
    reinterpret_cast<uint4*>(ghist + rank * SL)[tid] = acc;
    const uint32_t part = warp_sum_u32(acc.x + acc.y + acc.z + acc.w);
    if (lane == 0) tmp[tid >> 5] = part;
  }
  __syncthreads();
  if (tid == 0) {
    uint32_t t = 0;
#pragma unroll
    for (int w = 0; w < G4 / 32; ++w) t += tmp[w];
    *stot = t;
  }
  cluster_sync();   // slices and totals are published; peers are done reading `hist`
  if (tid < 32) {
    // the slice: above(s) = keys in the slices above s (higher digits hold larger keys)
    const uint32_t tot = lane < TKC ? ld_cluster_u32(mapa_shared(smem_u32(stot), (uint32_t)lane)) : 0u;
    uint32_t above = 0;
#pragma unroll
    for (int q = TKC - 1; q > 0; --q) {
      const uint32_t tq = __shfl_sync(0xffffffffu, tot, q);
      if (q > lane) above += tq;
    }
    const bool hit = lane < TKC && above < need && need <= above + tot;
    const uint32_t hits = __ballot_sync(0xffffffffu, hit);   // exactly one slice holds it
    const int s_sel = hits != 0u ? __ffs(hits) - 1 : 0;
    const uint32_t need_s = need - __shfl_sync(0xffffffffu, above, s_sel);
    // the bin inside slice s_sel: lane l holds bins [l PER, (l + 1) PER) of it
    const uint32_t g0 = mapa_shared(smem_u32(ghist) + (uint32_t)(s_sel * SL + lane * PER) * 4u, (uint32_t)s_sel);
    uint32_t h[PER];
    uint32_t mine = 0;
#pragma unroll
    for (int j = 0; j < PER; ++j) {
      h[j] = ld_cluster_u32(g0 + 4u * (uint32_t)j);
      mine += h[j];
    }
    // keys in the bins of higher lanes
    uint32_t incl = mine;   // inclusive suffix sum over lanes >= this one
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t x = __shfl_down_sync(0xffffffffu, incl, o);
      if (lane + o < 32) incl += x;
    }
    uint32_t ab = incl - mine;
#pragma unroll
    for (int j = PER - 1; j >= 0; --j) {
      if (ab < need_s && need_s <= ab + h[j]) {
        sel[0] = (uint32_t)(s_sel * SL + lane * PER + j);
        sel[1] = need_s - ab;
      }
      ab += h[j];
    }
  }
  __syncthreads();
  prefix = first ? sel[0] : ((prefix << BITS) | sel[0]);
  need = sel[1];
  __syncthreads();
}

template <int BITS>
__device__ __forceinline__ void cluster_pass(const SmemKeys& keys, int m, int shift,
                                             uint32_t& prefix, uint32_t& need, uint32_t* hist,
                                             uint32_t* ghist, uint32_t* tmp, uint32_t* sel,
                                             uint32_t* stot) {
  constexpr int NB = 1 << BITS;
  for (int i = threadIdx.x; i < NB; i += TK_THREADS) hist[i] = 0u;
  __syncthreads();
  histogram_digit<BITS, TK_THREADS>(keys, m, shift, false, prefix, hist);
  cluster_find<BITS>(false, prefix, need, hist, ghist, tmp, sel, stot);
}

__global__ void __cluster_dims__(TKC, 1, 1) __launch_bounds__(TK_THREADS)
    topk_cluster_kernel(const TopkArgs a) {
  extern __shared__ __align__(16) uint32_t seg_keys[];
  __shared__ __align__(16) uint32_t hist[2048];
  __shared__ __align__(16) uint32_t ghist[2048];
  __shared__ uint32_t tmp[2 * (TK_THREADS / 32)];
  __shared__ uint32_t sel[2];
  __shared__ uint32_t counts[2];
  __shared__ uint32_t stot;   // this CTA's slice total of the current digit
  const uint32_t rank = cluster_ctarank();
  const int rows_per_b = a.t_hi - a.t_lo;
  const long long r = blockIdx.x / TKC;
  const int b = (int)(r / rows_per_b);
  const int t = a.t_lo + (int)(r % rows_per_b);
  const int n = min(a.Lk, seq_pos0(a.seq_lens, a.q_pos0, a.Lq, b) + t + 1);
  int32_t* dst = a.idx + ((long long)b * a.Lq + t) * a.k;
  float* dsc = a.sel != nullptr ? a.sel + ((long long)b * a.Lq + t) * a.k : nullptr;
  if (n <= a.k) {   // the same decision in every CTA of the cluster: no shared traffic below
    if (rank == 0) {
      const float* row = a.scores + ((long long)b * a.sc_bstride + (t - a.sc_t0)) * a.sc_ld;
      for (int i = threadIdx.x; i < a.k; i += TK_THREADS) {
        dst[i] = i < n ? i : -1;
        if (dsc != nullptr) dsc[i] = i < n ? row[i] : 0.f;
      }
    }
    return;
  }
  const int seg = (((n + TKC - 1) / TKC) + 3) & ~3;
  const int lo = (int)rank * seg;
  const int m = max(0, min(n - lo, seg));
  const float* src = a.scores + ((long long)b * a.sc_bstride + (t - a.sc_t0)) * a.sc_ld + lo;
  for (int i = threadIdx.x; i < 2048; i += TK_THREADS) hist[i] = 0u;
  __syncthreads();
  stage_keys<TK_THREADS>(src, m, seg_keys, hist);   // with the first digit's histogram
  const SmemKeys keys{seg_keys};
  uint32_t prefix = 0, need = (uint32_t)a.k;
  cluster_find<11>(true, prefix, need, hist, ghist, tmp, sel, &stot);   // its cluster barrier publishes the keys
  cluster_pass<11>(keys, m, 10, prefix, need, hist, ghist, tmp, sel, &stot);
  cluster_pass<10>(keys, m, 0, prefix, need, hist, ghist, tmp, sel, &stot);
  const uint32_t T = prefix;
  const uint32_t need_eq = need;

  // this CTA's counts, then the counts of the segments before it
  const Run run = warp_run<TK_THREADS>(m);
  uint32_t G, E, g_tot, e_tot;
  block_run_offsets<TK_THREADS>(keys, m, T, run, tmp, G, E, g_tot, e_tot);
  if (threadIdx.x == 0) {
    counts[0] = g_tot;
    counts[1] = e_tot;
  }
  cluster_sync();
  const uint32_t c0 = smem_u32(counts);
  for (uint32_t p = 0; p < rank; ++p) {
    G += ld_cluster_u32(mapa_shared(c0, p));
    E += ld_cluster_u32(mapa_shared(c0 + 4u, p));
  }
  write_run(keys, m, T, need_eq, G, E, lo, run, dst, dsc);
  cluster_sync();   // peers are done reading `counts` before this CTA exits
}

}  // namespace

cudaError_t launch_topk(const TopkArgs& a, int num_sms, cudaStream_t stream) {
  const int rows_per_b = a.t_hi - a.t_lo;
  if (rows_per_b <= 0 || a.B <= 0) return cudaSuccess;
  long long nrows = (long long)a.B * rows_per_b;
  const int n_max = a.seq_lens != nullptr ? a.Lk : (a.q_pos0 + a.t_hi < a.Lk ? a.q_pos0 + a.t_hi : a.Lk);
  unsigned grid = (unsigned)(nrows < (1LL << 30) ? nrows : (1LL << 30));
  const bool cluster = n_max <= TKC * TK_SMEM_MAX &&
                       (n_max > TK_SMEM_MAX || (nrows < num_sms && n_max > 4096));
  if (cluster && nrows * TKC < (1LL << 31)) {
    const size_t smem = (size_t)((((n_max + TKC - 1) / TKC) + 3) & ~3) * 4;
    cudaError_t e = cudaFuncSetAttribute(topk_cluster_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    topk_cluster_kernel<<<(unsigned)(nrows * TKC), TK_THREADS, smem, stream>>>(a);
  } else if (n_max <= TK_SMEM_MAX) {
    size_t smem = (size_t)((n_max + 3) & ~3) * 4;
    const bool wide = n_max > TK_WIDE_KEYS;
    auto kern = wide ? topk_kernel<true, TK1_THREADS> : topk_kernel<true, TK_THREADS>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<grid, wide ? TK1_THREADS : TK_THREADS, smem, stream>>>(a);
  } else {
    topk_kernel<false, TK1_THREADS><<<grid, TK1_THREADS, 0, stream>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace dsa
