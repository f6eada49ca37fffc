// topk.cu - fine-grained token selection: the k largest index scores of each
// query row ("DeepSeek-V3.2: Pushing the Frontier of Open Large Language Models",
// bud-325 paper digest, "Key claims", section 2.1, and "Method": k = 2048 key-value
// entries per query token).
//
// One CTA per query row. Scores are mapped to order-preserving 32-bit keys
// (-0.0 folded onto +0.0) and the exact k-th largest key T is found by a
// three-digit radix select (11 + 11 + 10 bits, most significant first): each
// pass histograms the keys that still match the selected prefix in shared
// memory and a block scan picks the digit where the running count from the top
// crosses k. A final ordered pass writes every key > T and the first
// (k - #{key > T}) keys == T, in ascending index order: one block-wide scan of
// packed (greater, equal) counts per 4096 candidates gives every element its
// output slot. Ties therefore go to the lowest index and the output is sorted.
// Rows of up to 48K candidates are staged once in shared memory as keys. Longer
// rows, or launches with fewer rows than SMs, spread each row over a cluster of
// 8 CTAs (topk_cluster_kernel); rows beyond 8 x 48K are re-read from global
// memory (L2) on each pass.
// Rows with at most k candidates select all of them and pad with -1.
#include "dsa_kernels.h"

namespace dsa {
namespace {

constexpr int TK_THREADS = 512;
constexpr int TK_WARPS = TK_THREADS / 32;
constexpr int TK_ITEMS = 8;                       // contiguous elements per thread, output pass
constexpr int TK_SMEM_MAX = 48 * 1024;            // candidates staged in shared memory

__device__ __forceinline__ uint32_t score_key(float x) {
  uint32_t u = __float_as_uint(x);
  if (u == 0x80000000u) u = 0u;                   // -0.0 == +0.0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// The score of an order-preserving key (-0.0 comes back as +0.0).
__device__ __forceinline__ float key_score(uint32_t key) {
  return __uint_as_float((key & 0x80000000u) ? (key & 0x7FFFFFFFu) : ~key);
}

// Exclusive block scan of one int per thread; also returns the block total.
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t* tmp, uint32_t& total) {
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
    uint32_t x = lane < TK_WARPS ? tmp[lane] : 0u;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      uint32_t n = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += n;
    }
    if (lane < TK_WARPS) tmp[lane] = x;
  }
  __syncthreads();
  uint32_t off = wid > 0 ? tmp[wid - 1] : 0u;
  total = tmp[TK_WARPS - 1];
  __syncthreads();
  return off + incl - v;
}

// Given a histogram of the candidate digits, pick the digit holding the
// `need`-th largest key; extend `prefix` by it and make `need` the rank within
// that digit (uniform across the block).
template <int BITS>
__device__ __forceinline__ void find_bin(const uint32_t* hist, bool first, uint32_t& prefix,
                                         uint32_t& need, uint32_t* tmp, uint32_t* sel) {
  constexpr int BPT = (1 << BITS) / TK_THREADS;
  uint32_t local = 0;
  const int b0 = threadIdx.x * BPT;
#pragma unroll
  for (int j = 0; j < BPT; ++j) local += hist[b0 + j];
  uint32_t total;
  uint32_t before = block_excl_scan(local, tmp, total);
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

template <bool SMEM_ROW>
struct RowSrc {
  const uint32_t* keys;  // shared-memory keys (SMEM_ROW)
  const float* src;      // global scores
  __device__ __forceinline__ uint32_t operator()(int i) const {
    if constexpr (SMEM_ROW) return keys[i];
    else return score_key(__ldg(src + i));
  }
};

// One radix pass: histogram digit (key >> shift) & (nbins-1) of keys whose bits
// above `shift + bits` equal `prefix`; then find the digit holding the `need`-th
// largest key. Updates prefix/need in place (uniform across the block).
template <bool SMEM_ROW, int BITS>
__device__ __forceinline__ void radix_pass(const RowSrc<SMEM_ROW>& row, int n, int shift,
                                           bool first, uint32_t& prefix, uint32_t& need,
                                           uint32_t* hist, uint32_t* tmp, uint32_t* sel) {
  constexpr int NB = 1 << BITS;
  constexpr int BPT = NB / TK_THREADS;  // bins per thread
  static_assert(BPT >= 1, "bins");
  for (int i = threadIdx.x; i < NB; i += TK_THREADS) hist[i] = 0u;
  __syncthreads();
  const int hi_shift = shift + BITS;
  const int lane = threadIdx.x & 31;
  auto count = [&](uint32_t key, bool valid) {
    if (valid && (first || (key >> hi_shift) == prefix))
      atomicAdd(&hist[(key >> shift) & (NB - 1)], 1u);
  };
  if constexpr (SMEM_ROW) {
    for (int i = threadIdx.x; i < n; i += TK_THREADS) count(row.keys[i], true);
  } else {
    // eight consecutive scores per thread per step (two 16-byte loads in flight)
    const bool vec = (reinterpret_cast<uintptr_t>(row.src) & 15u) == 0;
    for (int base = (threadIdx.x & ~31) * 8; base < n; base += TK_THREADS * 8) {
      const int i0 = base + lane * 8;
      float4 v0, v1;
      if (vec && i0 + 7 < n) {
        v0 = __ldg(reinterpret_cast<const float4*>(row.src + i0));
        v1 = __ldg(reinterpret_cast<const float4*>(row.src + i0 + 4));
      } else {
        float t[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) t[j] = i0 + j < n ? __ldg(row.src + i0 + j) : 0.f;
        v0 = make_float4(t[0], t[1], t[2], t[3]);
        v1 = make_float4(t[4], t[5], t[6], t[7]);
      }
      count(score_key(v0.x), i0 < n);
      count(score_key(v0.y), i0 + 1 < n);
      count(score_key(v0.z), i0 + 2 < n);
      count(score_key(v0.w), i0 + 3 < n);
      count(score_key(v1.x), i0 + 4 < n);
      count(score_key(v1.y), i0 + 5 < n);
      count(score_key(v1.z), i0 + 6 < n);
      count(score_key(v1.w), i0 + 7 < n);
    }
  }
  __syncthreads();
  find_bin<BITS>(hist, first, prefix, need, tmp, sel);
}

template <bool SMEM_ROW>
__global__ void __launch_bounds__(TK_THREADS) topk_kernel(const TopkArgs a) {
  extern __shared__ uint32_t row_keys[];
  __shared__ uint32_t hist[2048];
  __shared__ uint32_t tmp[32];
  __shared__ uint32_t sel[2];
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
      for (int i = threadIdx.x; i < a.k; i += TK_THREADS) {
        dst[i] = i < n ? i : -1;
        if (dsc != nullptr) dsc[i] = i < n ? src[i] : 0.f;
      }
      continue;
    }
    if constexpr (SMEM_ROW) {
      if ((reinterpret_cast<uintptr_t>(src) & 15u) == 0) {
        const int n4 = n >> 2;
        const float4* s4 = reinterpret_cast<const float4*>(src);
        uint4* k4 = reinterpret_cast<uint4*>(row_keys);
        for (int i = threadIdx.x; i < n4; i += TK_THREADS) {
          const float4 v = __ldg(s4 + i);
          k4[i] = make_uint4(score_key(v.x), score_key(v.y), score_key(v.z), score_key(v.w));
        }
        for (int i = (n4 << 2) + threadIdx.x; i < n; i += TK_THREADS) row_keys[i] = score_key(__ldg(src + i));
      } else {
        for (int i = threadIdx.x; i < n; i += TK_THREADS) row_keys[i] = score_key(__ldg(src + i));
      }
      __syncthreads();
    }
    RowSrc<SMEM_ROW> row{row_keys, src};
    uint32_t prefix = 0, need = (uint32_t)a.k;
    radix_pass<SMEM_ROW, 11>(row, n, 21, true, prefix, need, hist, tmp, sel);
    radix_pass<SMEM_ROW, 11>(row, n, 10, false, prefix, need, hist, tmp, sel);
    radix_pass<SMEM_ROW, 10>(row, n, 0, false, prefix, need, hist, tmp, sel);
    const uint32_t T = prefix;
    const uint32_t need_eq = need;  // keys equal to T that are selected (lowest indices first)

    uint32_t g_run = 0, e_run = 0;
    for (int base = 0; base < n; base += TK_THREADS * TK_ITEMS) {
      const int i0 = base + threadIdx.x * TK_ITEMS;
      uint32_t keys[TK_ITEMS];
      bool full = i0 + TK_ITEMS <= n;
      if constexpr (!SMEM_ROW) {
        if (full && a.vec4) {
          float4 v0 = __ldg(reinterpret_cast<const float4*>(src + i0));
          float4 v1 = __ldg(reinterpret_cast<const float4*>(src + i0 + 4));
          keys[0] = score_key(v0.x); keys[1] = score_key(v0.y);
          keys[2] = score_key(v0.z); keys[3] = score_key(v0.w);
          keys[4] = score_key(v1.x); keys[5] = score_key(v1.y);
          keys[6] = score_key(v1.z); keys[7] = score_key(v1.w);
        } else {
#pragma unroll
          for (int j = 0; j < TK_ITEMS; ++j) keys[j] = (i0 + j < n) ? row(i0 + j) : 0u;
        }
      } else {
#pragma unroll
        for (int j = 0; j < TK_ITEMS; ++j) keys[j] = (i0 + j < n) ? row_keys[i0 + j] : 0u;
      }
      uint32_t g = 0, e = 0;
#pragma unroll
      for (int j = 0; j < TK_ITEMS; ++j) {
        if (i0 + j < n) {
          g += keys[j] > T;
          e += keys[j] == T;
        }
      }
      uint32_t total;
      uint32_t excl = block_excl_scan((e << 16) | g, tmp, total);
      uint32_t G = g_run + (excl & 0xFFFFu);
      uint32_t E = e_run + (excl >> 16);
#pragma unroll
      for (int j = 0; j < TK_ITEMS; ++j) {
        if (i0 + j < n) {
          if (keys[j] > T) {
            dst[G + min(E, need_eq)] = i0 + j;
            if (dsc != nullptr) dsc[G + min(E, need_eq)] = key_score(keys[j]);
            ++G;
          } else if (keys[j] == T) {
            if (E < need_eq) {
              dst[G + E] = i0 + j;
              if (dsc != nullptr) dsc[G + E] = key_score(keys[j]);
            }
            ++E;
          }
        }
      }
      g_run += total & 0xFFFFu;
      e_run += total >> 16;
    }
    __syncthreads();
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

template <int BITS>
__device__ __forceinline__ void cluster_pass(const uint32_t* keys, int m, int shift, bool first,
                                             uint32_t& prefix, uint32_t& need, uint32_t* hist,
                                             uint32_t* ghist, uint32_t* tmp, uint32_t* sel) {
  constexpr int NB = 1 << BITS;
  for (int i = threadIdx.x; i < NB; i += TK_THREADS) hist[i] = 0u;
  __syncthreads();
  const int hi_shift = shift + BITS;
  for (int i = threadIdx.x; i < m; i += TK_THREADS) {
    const uint32_t key = keys[i];
    if (first || (key >> hi_shift) == prefix) atomicAdd(&hist[(key >> shift) & (NB - 1)], 1u);
  }
  cluster_sync();   // every CTA's histogram is complete and visible
  const uint32_t h0 = smem_u32(hist);
  for (int i = threadIdx.x; i < NB; i += TK_THREADS) {
    uint32_t sum = 0;
#pragma unroll
    for (int p = 0; p < TKC; ++p) sum += ld_cluster_u32(mapa_shared(h0 + 4u * i, p));
    ghist[i] = sum;
  }
  cluster_sync();   // peers are done reading `hist` before it is cleared again
  find_bin<BITS>(ghist, first, prefix, need, tmp, sel);
}

__global__ void __cluster_dims__(TKC, 1, 1) __launch_bounds__(TK_THREADS)
    topk_cluster_kernel(const TopkArgs a) {
  extern __shared__ uint32_t seg_keys[];
  __shared__ uint32_t hist[2048];
  __shared__ uint32_t ghist[2048];
  __shared__ uint32_t tmp[32];
  __shared__ uint32_t sel[2];
  __shared__ uint32_t counts[2];
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
  if ((reinterpret_cast<uintptr_t>(src) & 15u) == 0) {
    const int m4 = m >> 2;
    for (int i = threadIdx.x; i < m4; i += TK_THREADS) {
      const float4 v = __ldg(reinterpret_cast<const float4*>(src) + i);
      reinterpret_cast<uint4*>(seg_keys)[i] =
          make_uint4(score_key(v.x), score_key(v.y), score_key(v.z), score_key(v.w));
    }
    for (int i = (m4 << 2) + threadIdx.x; i < m; i += TK_THREADS) seg_keys[i] = score_key(__ldg(src + i));
  } else {
    for (int i = threadIdx.x; i < m; i += TK_THREADS) seg_keys[i] = score_key(__ldg(src + i));
  }
  __syncthreads();
  uint32_t prefix = 0, need = (uint32_t)a.k;
  cluster_pass<11>(seg_keys, m, 21, true, prefix, need, hist, ghist, tmp, sel);
  cluster_pass<11>(seg_keys, m, 10, false, prefix, need, hist, ghist, tmp, sel);
  cluster_pass<10>(seg_keys, m, 0, false, prefix, need, hist, ghist, tmp, sel);
  const uint32_t T = prefix;
  const uint32_t need_eq = need;

  // counts of this segment, then the counts of the segments before it
  uint32_t g = 0, e = 0;
  for (int i = threadIdx.x; i < m; i += TK_THREADS) {
    g += seg_keys[i] > T;
    e += seg_keys[i] == T;
  }
  uint32_t total;
  block_excl_scan((e << 16) | g, tmp, total);   // segment of <= 48K keys: counts fit 16 bits
  if (threadIdx.x == 0) {
    counts[0] = total & 0xFFFFu;
    counts[1] = total >> 16;
  }
  cluster_sync();
  uint32_t g_run = 0, e_run = 0;
  const uint32_t c0 = smem_u32(counts);
  for (uint32_t p = 0; p < rank; ++p) {
    g_run += ld_cluster_u32(mapa_shared(c0, p));
    e_run += ld_cluster_u32(mapa_shared(c0 + 4u, p));
  }
  for (int base = 0; base < m; base += TK_THREADS * TK_ITEMS) {
    const int i0 = base + threadIdx.x * TK_ITEMS;
    uint32_t keys[TK_ITEMS];
#pragma unroll
    for (int j = 0; j < TK_ITEMS; ++j) keys[j] = (i0 + j < m) ? seg_keys[i0 + j] : 0u;
    uint32_t gl = 0, el = 0;
#pragma unroll
    for (int j = 0; j < TK_ITEMS; ++j) {
      if (i0 + j < m) {
        gl += keys[j] > T;
        el += keys[j] == T;
      }
    }
    uint32_t tot;
    const uint32_t excl = block_excl_scan((el << 16) | gl, tmp, tot);
    uint32_t G = g_run + (excl & 0xFFFFu);
    uint32_t E = e_run + (excl >> 16);
#pragma unroll
    for (int j = 0; j < TK_ITEMS; ++j) {
      if (i0 + j < m) {
        if (keys[j] > T) {
          dst[G + min(E, need_eq)] = lo + i0 + j;
          if (dsc != nullptr) dsc[G + min(E, need_eq)] = key_score(keys[j]);
          ++G;
        } else if (keys[j] == T) {
          if (E < need_eq) {
            dst[G + E] = lo + i0 + j;
            if (dsc != nullptr) dsc[G + E] = key_score(keys[j]);
          }
          ++E;
        }
      }
    }
    g_run += tot & 0xFFFFu;
    e_run += tot >> 16;
  }
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
    cudaError_t e = cudaFuncSetAttribute(topk_kernel<true>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    topk_kernel<true><<<grid, TK_THREADS, smem, stream>>>(a);
  } else {
    topk_kernel<false><<<grid, TK_THREADS, 0, stream>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace dsa
