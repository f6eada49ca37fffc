// sparse_mla.cu - MLA attention in MQA mode over the selected latent rows
// ("DeepSeek-V3.2: Pushing the Frontier of Open Large Language Models", bud-325
// paper digest, "Key claims", section 2.1 Eq. 2 / Fig. 2: attention only on the
// top-k key-value entries; "Method": the latent vector of a token is shared by
// all query heads, so one gathered KV row serves every head).
//
// One CTA computes, for one query token and one chunk of DVC value columns:
//     z[h,s] = sm_scale * q[h] . c_s        (tcgen05, M = 128 heads, N = 64 keys,
//                                            K = Dqk in 16-wide steps)
//     online softmax over the key tiles     (base 2, lazy rescale of O)
//     O[h, chunk] += P[h,s] . c_s[chunk]    (tcgen05, M = 128, N = DVC, K = 64 keys)
// Layout of the work:
//   warp 0      tcgen05 issuer: for each 64-key tile, in a fixed order, S_i =
//               Q K_i^T into one of two TMEM buffers (part A of the columns, then
//               part B) and, between the two parts as soon as P_{i-1} is ready,
//               O += P_{i-1} V_{i-1} with P read from TMEM. One lane runs the loop
//               when each sequence has one query row (decode); with several rows
//               (prefill) the whole warp runs it and one elected lane issues;
//   warps 1..8  softmax, two warps per TMEM lane quadrant: a thread owns one head
//               (TMEM lane) and 32 of the tile's 64 keys. The two threads of a head
//               exchange their maxima through shared memory, write P_i (bf16) over
//               the first half of S_i's own TMEM buffer, rescale their half of O in
//               TMEM only when the running max grew by more than 2^8, and
//               normalise at the end;
//   warps 9..16 gather producers: each warp owns 8 rows of every tile, loads their
//               indices once and copies the rows 16 bytes per thread per cp.async,
//               straight into the 128-byte-swizzled K-major layout the tensor core
//               reads, into a 2-stage ring. A TMA gather4 costs about as much issue
//               time per 512 bytes as these warps need for a whole tile, so
//               threads gather the rows.
// O for 128 heads x 512 values in fp32 would fill all of TMEM, so the value
// columns are split over CTAs (DVC = 256): each CTA recomputes S for its token.
// With several key splits (decode) each CTA writes an unnormalised partial
// (O, running max, sum) and a combine kernel merges them.
#include <type_traits>

#include "dsa_kernels.h"

namespace dsa {
namespace {

constexpr int KEYS = 64;                       // keys per tile (N of the S MMA)
constexpr int SMX_WARPS = 8;                   // softmax warps (two per lane quadrant)
constexpr int PROD_WARPS = 8;                  // gather warps
constexpr int ROWS_PER_PROD = KEYS / PROD_WARPS;
constexpr int MLA_THREADS = 32 + SMX_WARPS * 32 + PROD_WARPS * 32;
constexpr int SMX_T0 = 32;                     // first softmax thread
constexpr int PROD_T0 = SMX_T0 + SMX_WARPS * 32;   // first producer thread
static_assert(KEYS % PROD_WARPS == 0 && ROWS_PER_PROD <= 32, "rows per producer warp");

template <int NKB, int DVC>
struct MlaTraits {
  static constexpr int QBLK = 128 * 128;            // one 64-column block of Q: 128 rows x 128 B
  static constexpr int KVBLK = KEYS * 128;          // one 64-column block of a KV tile
  static constexpr int QT_KB = (NKB == 9) ? 4 : 1;  // Q column blocks held in TMEM
  static constexpr int QS_KB = NKB - QT_KB;         // Q column blocks held in shared memory
  static constexpr int STAGES = 2;                  // KV ring depth
  // A tile's column blocks come in two parts: part B = the DVC / 64 value blocks
  // this CTA multiplies with P (read by S and by PV), part A = the others (read
  // by S only). Part A of a stage is refilled as soon as S of its tile is done.
  static constexpr int NB_B = DVC / 64;
  static constexpr int NB_A = NKB - NB_B;
  static constexpr int NP = PROD_WARPS * 32;
  // 16-byte chunks per producer lane and part: 8 rows x NB blocks x 8 chunks / 32
  static constexpr int CPL_A = ROWS_PER_PROD * NB_A * 8 / 32;
  static constexpr int CPL_B = ROWS_PER_PROD * NB_B * 8 / 32;
  static_assert(ROWS_PER_PROD * NB_A * 8 % 32 == 0 && ROWS_PER_PROD * NB_B * 8 % 32 == 0, "chunks");
  static_assert(NB_A >= 1 && NB_B >= 1, "both parts must be non-empty");
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_KV = OFF_Q + QS_KB * QBLK;
  static constexpr int OFF_BAR = OFF_KV + STAGES * NKB * KVBLK;
  // mbarrier slots (8 bytes each), in this order
  static constexpr int BAR_Q = 0;                     // Q part in shared memory landed
  static constexpr int BAR_QT = 1;                    // Q part in TMEM written
  static constexpr int BAR_KV_FULL = 2;               // [2 parts][STAGES]
  static constexpr int BAR_KV_EMPTY = BAR_KV_FULL + 2 * STAGES;   // [2 parts][STAGES]
  static constexpr int BAR_S_FULL = BAR_KV_EMPTY + 2 * STAGES;   // [2] S buffer computed
  static constexpr int BAR_P_FULL = BAR_S_FULL + 2;   // [2] P written over its S buffer
  static constexpr int BAR_PV_DONE = BAR_P_FULL + 2;  // [2] PV of a tile of that parity done
  static constexpr int BAR_XMAX = BAR_PV_DONE + 2;    // [2] both halves' tile maxima written
  static constexpr int BAR_XL = BAR_XMAX + 2;         // both halves' sums written (end)
  static constexpr int BAR_DONE = BAR_XL + 1;
  static constexpr int NUM_BARS = BAR_DONE + 1;
  // exchange area of the two softmax halves: tile maxima as bf16 [2 tiles][2 halves]
  // [128 heads], and at the end the row sums as fp32 [2 halves][128 heads]
  static constexpr int OFF_XMAX = OFF_BAR + NUM_BARS * 8;
  static constexpr int OFF_MISC = OFF_XMAX + 2 * 2 * 128 * 2;
  static constexpr int SMEM_BYTES = OFF_MISC + 48 + 1024;
  // TMEM columns: O [0, DVC), two S buffers [DVC, DVC + 2 KEYS) (P_i, bf16, is
  // written over the first KEYS / 2 columns of S_i's buffer), Q part after them
  static constexpr int COL_S = DVC;
  static constexpr int COL_Q = DVC + 2 * KEYS;
  static constexpr int COLS_USED = COL_Q + 32 * QT_KB;
  static constexpr int TMEM_COLS = COLS_USED <= 128 ? 128 : COLS_USED <= 256 ? 256 : 512;
  static constexpr uint32_t IDESC_S = make_idesc(1, 1, 0, 0, KEYS, 128);   // bf16, K-major both
  static_assert(KEYS == 64, "masks hold two 32-key words per tile");
  // PV: A = P from TMEM, B = values MN-major
  static constexpr uint32_t IDESC_PV = make_idesc(1, 1, 0, 1, DVC, 128);
  static_assert(DVC % 64 == 0 && DVC <= 256, "DVC");
  static_assert(QT_KB % 2 == 0 || QT_KB == 1, "Q blocks in TMEM split over the two halves");
  static_assert(COLS_USED <= 512, "TMEM");
  static_assert(SMEM_BYTES <= 232448, "shared memory");
};

// One part of S = Q K^T for a tile whose stage starts at descriptor kd0: part
// A (PART = 0, the column blocks only S reads) or part B (PART = 1, the value
// blocks of the CTA's slice DVCI of the output columns).
// Block order, offsets and the operand form of every MMA are compile-time
// constants: Q's first QT_KB column blocks are read from TMEM, the rest from
// shared memory. Issue from a fully unrolled sequence costs about as much as
// the MMAs take to run; the same sequence built from a runtime block index
// costs up to twice as much per MMA.
template <int NKB, int DVC, int DVCI, int PART>
__device__ __forceinline__ void issue_s_part(uint32_t s_tmem, uint32_t qt_tmem, uint64_t qd0, uint64_t kd0) {
  using Tr = MlaTraits<NKB, DVC>;
  constexpr int VB0 = DVCI * Tr::NB_B;
  constexpr int NB = PART ? Tr::NB_B : Tr::NB_A;
  static_assert(VB0 + Tr::NB_B <= NKB, "value blocks of the slice");
#pragma unroll
  for (int j = 0; j < NB; ++j) {
    const int kb = PART ? VB0 + j : (j < VB0 ? j : j + Tr::NB_B);
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      const uint32_t acc = (PART | j | kk) ? 1u : 0u;   // the first MMA of part A overwrites S
      const uint64_t kdesc = kd0 + (uint64_t)((kb * Tr::KVBLK + kk * 32) >> 4);
      if (kb < Tr::QT_KB)
        mma_f16_ts(s_tmem, qt_tmem + kb * 32 + kk * 8, kdesc, Tr::IDESC_S, acc);
      else
        mma_f16_ss(s_tmem, qd0 + (uint64_t)(((kb - Tr::QT_KB) * Tr::QBLK + kk * 32) >> 4), kdesc,
                   Tr::IDESC_S, acc);
    }
  }
}

// PV for one tile: O += P V, P = the bf16 probabilities over the first KEYS / 2
// columns of the tile's S buffer, V = this CTA's value blocks of the stage (bd0).
template <int NKB, int DVC>
__device__ __forceinline__ void issue_pv(uint32_t o_tmem, uint32_t pt, uint64_t bd0, bool first) {
  using Tr = MlaTraits<NKB, DVC>;
#pragma unroll
  for (int kk = 0; kk < KEYS / 16; ++kk)
    mma_f16_ts(o_tmem, pt + kk * 8, bd0 + (uint64_t)(kk * 16 * 128 >> 4), Tr::IDESC_PV,
               (!first || kk > 0) ? 1u : 0u);
}

// The issuer's loop over the CTA's tiles, for output-column slice DVCI. Per tile
// i, in this order: part A of S_i (its stage's part-A blocks have landed; its S
// buffer was last read by PV_{i-2}, issued before), then PV_{i-1} if P_{i-1} is
// already written, part B of S_i once the value blocks have landed, and PV_{i-1}
// if it was not issued yet. The tensor pipe runs MMAs in issue order, which
// orders every buffer reuse. Returns false if a wait gave up.
template <int NKB, int DVC, int DVCI>
__device__ __noinline__ bool mla_issue_tiles(int ntiles, uint32_t tbase, uint32_t kv_base, uint64_t qd0,
                                             uint64_t* bars, const DevCtl& ctl, volatile int* abort_flag) {
  using Tr = MlaTraits<NKB, DVC>;
  uint64_t* kvA_full = bars + Tr::BAR_KV_FULL;
  uint64_t* kvB_full = bars + Tr::BAR_KV_FULL + Tr::STAGES;
  uint64_t* kvA_empty = bars + Tr::BAR_KV_EMPTY;
  uint64_t* kvB_empty = bars + Tr::BAR_KV_EMPTY + Tr::STAGES;
  uint64_t* s_full = bars + Tr::BAR_S_FULL;
  uint64_t* p_full = bars + Tr::BAR_P_FULL;
  uint64_t* pv_done = bars + Tr::BAR_PV_DONE;
  const uint32_t o_tmem = tbase, s_tmem = tbase + Tr::COL_S, qt_tmem = tbase + Tr::COL_Q;
  // stage descriptors: K-major for S, and this slice's value blocks MN-major for PV.
  // They are chosen per stage with selects, not indexed from an array: an array
  // indexed at run time lives in local memory, and every MMA's memory clobber
  // would then reload it, putting a local-memory round trip in front of each
  // MMA issue.
  const uint64_t kd0 = make_sdesc(kv_base, 16, 1024, 2);
  const uint64_t kd1 = make_sdesc(kv_base + NKB * Tr::KVBLK, 16, 1024, 2);
  constexpr uint32_t v_off = (uint32_t)(DVCI * Tr::NB_B) * Tr::KVBLK;
  const uint64_t bd0 = make_sdesc(kv_base + v_off, Tr::KVBLK, 1024, 2);
  const uint64_t bd1 = make_sdesc(kv_base + NKB * Tr::KVBLK + v_off, Tr::KVBLK, 1024, 2);
  auto pv = [&](int j) {
    issue_pv<NKB, DVC>(o_tmem, s_tmem + (uint32_t)((j & 1) * KEYS), (j & 1) ? bd1 : bd0, j == 0);
    mma_commit(&kvB_empty[j & 1]);
    mma_commit(&pv_done[j & 1]);
  };
  for (int i = 0; i < ntiles; ++i) {
    const int st = i & 1;   // STAGES == 2
    const uint32_t ph = (uint32_t)(i >> 1) & 1u;
    const uint32_t sb = s_tmem + (uint32_t)(st * KEYS);
    if (!mbar_wait(&kvA_full[st], ph, ctl, abort_flag, kSiteMla, 3)) return false;
    tc_fence_after();
    const uint64_t kds = st ? kd1 : kd0;
    issue_s_part<NKB, DVC, DVCI, 0>(sb, qt_tmem, qd0, kds);
    mma_commit(&kvA_empty[st]);
    bool pv_pending = i > 0;
    if (pv_pending && mbar_test_wait(smem_u32(&p_full[(i - 1) & 1]), (uint32_t)((i - 1) >> 1) & 1u)) {
      tc_fence_after();
      pv(i - 1);
      pv_pending = false;
    }
    if (!mbar_wait(&kvB_full[st], ph, ctl, abort_flag, kSiteMla, 4)) return false;
    tc_fence_after();
    issue_s_part<NKB, DVC, DVCI, 1>(sb, qt_tmem, qd0, kds);
    mma_commit(&s_full[st]);
    if (pv_pending) {
      if (!mbar_wait(&p_full[(i - 1) & 1], (uint32_t)((i - 1) >> 1) & 1u, ctl, abort_flag, kSiteMla, 5))
        return false;
      tc_fence_after();
      pv(i - 1);
    }
  }
  if (ntiles > 0) {
    const int j = ntiles - 1;
    if (!mbar_wait(&p_full[j & 1], (uint32_t)(j >> 1) & 1u, ctl, abort_flag, kSiteMla, 6)) return false;
    tc_fence_after();
    pv(j);
  }
  return true;
}

// elect.sync over the full warp: true in exactly one lane (the same one every time).
__device__ __forceinline__ bool elect_one_lane() {
  uint32_t pred = 0;
  asm volatile("{\n\t.reg .pred P;\n\telect.sync _|P, 0xffffffff;\n\tselp.u32 %0, 1, 0, P;\n\t}" : "=r"(pred));
  return pred != 0;
}

// The same issue order run by the whole issuer warp: every lane computes the
// descriptors (warp-uniform values), one elected lane issues the MMAs and the
// commits, lane 0 waits on the barriers and passes the outcome on by shuffle.
// Issuing is faster this way, the barrier hand-offs slower: it pays where the
// tensor pipe is the limit (many query rows per sequence, gathers mostly from
// L2), not where the gathers' latency is (one decode row per sequence).
template <int NKB, int DVC, int DVCI>
__device__ __noinline__ bool mla_issue_tiles_warp(int ntiles, uint32_t tbase, uint32_t kv_base, uint64_t qd0,
                                             uint64_t* bars, const DevCtl& ctl, volatile int* abort_flag) {
  using Tr = MlaTraits<NKB, DVC>;
  const int lane = lane_id();
  uint64_t* kvA_full = bars + Tr::BAR_KV_FULL;
  uint64_t* kvB_full = bars + Tr::BAR_KV_FULL + Tr::STAGES;
  uint64_t* kvA_empty = bars + Tr::BAR_KV_EMPTY;
  uint64_t* kvB_empty = bars + Tr::BAR_KV_EMPTY + Tr::STAGES;
  uint64_t* s_full = bars + Tr::BAR_S_FULL;
  uint64_t* p_full = bars + Tr::BAR_P_FULL;
  uint64_t* pv_done = bars + Tr::BAR_PV_DONE;
  const uint32_t o_tmem = tbase, s_tmem = tbase + Tr::COL_S, qt_tmem = tbase + Tr::COL_Q;
  const uint64_t kd0 = make_sdesc(kv_base, 16, 1024, 2);
  const uint64_t kd1 = make_sdesc(kv_base + NKB * Tr::KVBLK, 16, 1024, 2);
  constexpr uint32_t v_off = (uint32_t)(DVCI * Tr::NB_B) * Tr::KVBLK;
  const uint64_t bd0 = make_sdesc(kv_base + v_off, Tr::KVBLK, 1024, 2);
  const uint64_t bd1 = make_sdesc(kv_base + NKB * Tr::KVBLK + v_off, Tr::KVBLK, 1024, 2);
  auto wait_w = [&](uint64_t* bar, uint32_t par, int id) -> bool {
    int r = 1;
    if (lane == 0) r = mbar_wait(bar, par, ctl, abort_flag, kSiteMla, id) ? 1 : 0;
    return __shfl_sync(0xffffffffu, r, 0) != 0;
  };
  auto pv = [&](int j) {
    if (elect_one_lane()) {
      issue_pv<NKB, DVC>(o_tmem, s_tmem + (uint32_t)((j & 1) * KEYS), (j & 1) ? bd1 : bd0, j == 0);
      mma_commit(&kvB_empty[j & 1]);
      mma_commit(&pv_done[j & 1]);
    }
    __syncwarp();
  };
  for (int i = 0; i < ntiles; ++i) {
    const int st = i & 1;   // STAGES == 2
    const uint32_t ph = (uint32_t)(i >> 1) & 1u;
    const uint32_t sb = s_tmem + (uint32_t)(st * KEYS);
    const uint64_t kds = st ? kd1 : kd0;
    if (!wait_w(&kvA_full[st], ph, 3)) return false;
    tc_fence_after();
    if (elect_one_lane()) {
      issue_s_part<NKB, DVC, DVCI, 0>(sb, qt_tmem, qd0, kds);
      mma_commit(&kvA_empty[st]);
    }
    __syncwarp();
    bool pv_pending = i > 0;
    if (pv_pending) {
      int ready = 0;
      if (lane == 0) ready = mbar_test_wait(smem_u32(&p_full[(i - 1) & 1]), (uint32_t)((i - 1) >> 1) & 1u) ? 1 : 0;
      if (__shfl_sync(0xffffffffu, ready, 0)) {
        tc_fence_after();
        pv(i - 1);
        pv_pending = false;
      }
    }
    if (!wait_w(&kvB_full[st], ph, 4)) return false;
    tc_fence_after();
    if (elect_one_lane()) {
      issue_s_part<NKB, DVC, DVCI, 1>(sb, qt_tmem, qd0, kds);
      mma_commit(&s_full[st]);
    }
    __syncwarp();
    if (pv_pending) {
      if (!wait_w(&p_full[(i - 1) & 1], (uint32_t)((i - 1) >> 1) & 1u, 5)) return false;
      tc_fence_after();
      pv(i - 1);
    }
  }
  if (ntiles > 0) {
    const int j = ntiles - 1;
    if (!wait_w(&p_full[j & 1], (uint32_t)(j >> 1) & 1u, 6)) return false;
    tc_fence_after();
    pv(j);
  }
  return true;
}

// The smallest bf16 value >= x (x not NaN), as its bit pattern. Both softmax
// halves of a head derive the running max from the same two such values, so they
// agree on it exactly; an upper bound of the tile max serves the online softmax as
// well as the max itself (P and the row sum use the same reference).
__device__ __forceinline__ uint16_t bf16_at_least(float x) {
  const uint32_t u = __float_as_uint(x);
  uint32_t hi = u >> 16;
  if ((u & 0xffffu) != 0u && (u & 0x80000000u) == 0u) ++hi;   // positive: round up
  return (uint16_t)hi;                                         // negative: truncation rounds up
}
__device__ __forceinline__ float bf16_bits_to_float(uint16_t v) { return __uint_as_float((uint32_t)v << 16); }

// 16 consecutive 32-bit TMEM columns of this warp's 32 lanes from registers.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15])
      : "memory");
}

// PAGED: latent rows are gathered through the block table (pool rows); the
// unpaged instantiation reads sequence b's rows directly.
template <int NKB, int DVC, bool PAGED, bool WARP_ISSUE>
__global__ void __launch_bounds__(MLA_THREADS, 1)
    sparse_mla_kernel(const __grid_constant__ CUtensorMap tmap_q, const uint16_t* __restrict__ kv,
                      const MlaArgs a) {
  using Tr = MlaTraits<NKB, DVC>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  uint8_t* q_smem = smem + Tr::OFF_Q;
  uint8_t* kv_smem = smem + Tr::OFF_KV;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Tr::OFF_BAR);
  uint64_t* q_full = bars + Tr::BAR_Q;          // Q part in shared memory (TMA)
  uint64_t* qt_full = bars + Tr::BAR_QT;        // Q part in TMEM (softmax warps)
  uint64_t* kvA_full = bars + Tr::BAR_KV_FULL;                  // [STAGES]
  uint64_t* kvB_full = bars + Tr::BAR_KV_FULL + Tr::STAGES;     // [STAGES]
  uint64_t* kvA_empty = bars + Tr::BAR_KV_EMPTY;                // [STAGES]
  uint64_t* kvB_empty = bars + Tr::BAR_KV_EMPTY + Tr::STAGES;   // [STAGES]
  uint64_t* s_full = bars + Tr::BAR_S_FULL;     // [2] S_i computed (buffer i % 2)
  uint64_t* p_full = bars + Tr::BAR_P_FULL;     // [2] P_i written over S_i
  uint64_t* pv_done = bars + Tr::BAR_PV_DONE;   // [2] PV_i done (tile parity)
  uint64_t* xmax_bar = bars + Tr::BAR_XMAX;     // [2] tile maxima of both halves written
  uint64_t* xl_bar = bars + Tr::BAR_XL;         // row sums of both halves written
  uint64_t* done_bar = bars + Tr::BAR_DONE;
  uint16_t* xmax = reinterpret_cast<uint16_t*>(smem + Tr::OFF_XMAX);   // [tile parity][half][head]
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + Tr::OFF_MISC);
  uint32_t* tmem_slot = misc;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
  volatile int* ntiles_slot = reinterpret_cast<volatile int*>(misc + 2);   // [2]
  // valid-key bits of the tile in each stage: [STAGES][8 producer warps] bytes, read
  // as [STAGES][2] 32-key words
  volatile uint8_t* mask8 = reinterpret_cast<volatile uint8_t*>(misc + 4);
  const volatile uint32_t* masks = misc + 4;

  const int warp = warp_id();
  const int lane = lane_id();
  const int per_token = a.n_dv * a.splits;
  const long long token = blockIdx.x / per_token;
  const int rem = blockIdx.x % per_token;
  const int dvc = rem / a.splits;
  const int split = rem % a.splits;
  const int b = (int)(token / a.Lq);
  const int32_t* idx_row = a.idx + token * a.k;

  // Warm L2 for the Q and index rows of the CTA that will probably run next on
  // this SM (one wave of block indices further on): its prologue waits on them.
  if (warp == PROD_T0 / 32 && lane == 0) {
    const long long nb = (long long)blockIdx.x + a.wave;
    if (nb < (long long)gridDim.x) {
      const long long ntok = nb / per_token;
      const uint8_t* qn = reinterpret_cast<const uint8_t*>(a.q) + ntok * a.H * (long long)a.Dqk * 2;
      const uint32_t qbytes = (uint32_t)(a.H * a.Dqk * 2);
      if ((reinterpret_cast<uintptr_t>(qn) & 15) == 0 && (qbytes & 15) == 0) bulk_prefetch_l2(qn, qbytes);
      const int32_t* in = a.idx + ntok * a.k;
      const uint32_t ibytes = (uint32_t)a.k * 4u;
      if ((reinterpret_cast<uintptr_t>(in) & 15) == 0 && (ibytes & 15) == 0) bulk_prefetch_l2(in, ibytes);
    }
  }
  if (threadIdx.x == 0) {
    // All of the token's Q rows are requested first, before anything else of the
    // prologue (they are its longest wait): the blocks read from shared memory to
    // their place, and the blocks that go to TMEM into the second KV stage, which
    // no tile uses before the softmax warps have moved them on (qt_full).
    tma_prefetch_map(&tmap_q);
    mbar_init(q_full, 1);
    fence_barrier_init();
    mbar_arrive_expect_tx(q_full, NKB * Tr::QBLK);
    for (int kb = 0; kb < Tr::QS_KB; ++kb)
      tma_load_2d(q_smem + kb * Tr::QBLK, &tmap_q, (Tr::QT_KB + kb) * 64, (int)(token * a.H), q_full);
    for (int kb = 0; kb < Tr::QT_KB; ++kb)
      tma_load_2d(kv_smem + NKB * Tr::KVBLK + kb * Tr::QBLK, &tmap_q, kb * 64, (int)(token * a.H), q_full);
    mbar_init(qt_full, SMX_WARPS * 32);
    for (int i = 0; i < Tr::STAGES; ++i) {
      mbar_init(&kvA_full[i], Tr::NP);
      mbar_init(&kvB_full[i], Tr::NP);
      mbar_init(&kvA_empty[i], 1);
      mbar_init(&kvB_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], SMX_WARPS * 32);
      mbar_init(&pv_done[i], 1);
      mbar_init(&xmax_bar[i], SMX_WARPS * 32);
    }
    mbar_init(xl_bar, SMX_WARPS * 32);
    mbar_init(done_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
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
  // TMEM comes from a warp that has nothing else to do before the barrier
  if (warp == 2) tmem_alloc(tmem_slot, Tr::TMEM_COLS);
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;
  const int ntiles = ntiles_slot[0];
  const int tile0 = ntiles_slot[1];
  const uint32_t o_tmem = tbase;
  const uint32_t s_tmem = tbase + Tr::COL_S;
  const uint32_t qt_tmem = tbase + Tr::COL_Q;

  if (warp == 0) {
    // ------------------------------------------------ MMA issuer (Q was requested at CTA start)
    if constexpr (WARP_ISSUE) {
      int okl = 1;
      if (lane == 0) {
        bool ok0 = mbar_wait(q_full, 0, a.ctl, abort_flag, kSiteMla, 1);
        if (!ok0) {
          DevCtl drain = a.ctl;
          volatile int never = 0;
          mbar_wait(q_full, 0, drain, &never, kSiteMla, 2);
        }
        if (ntiles > 0) ok0 = ok0 && mbar_wait(qt_full, 0, a.ctl, abort_flag, kSiteMla, 12);
        okl = ok0 ? 1 : 0;
      }
      bool ok = __shfl_sync(0xffffffffu, okl, 0) != 0;
      const uint64_t qd0 = make_sdesc(smem_u32(q_smem), 16, 1024, 2);
      if (ok && ntiles > 0) {
        if (Tr::NB_B * 2 <= NKB && dvc != 0)
          ok = mla_issue_tiles_warp<NKB, DVC, 1>(ntiles, tbase, smem_u32(kv_smem), qd0, bars, a.ctl, abort_flag);
        else
          ok = mla_issue_tiles_warp<NKB, DVC, 0>(ntiles, tbase, smem_u32(kv_smem), qd0, bars, a.ctl, abort_flag);
      }
      if (elect_one_lane()) {
        if (!ok) *abort_flag = 1;
        mma_commit(done_bar);
        DevCtl drain = a.ctl;
        volatile int never = 0;
        mbar_wait(done_bar, 0, drain, &never, kSiteMla, 7);
      }
      __syncwarp();
    } else {
      if (lane == 0) {
        // Q's copies land even when the CTA has no tile (they were issued before
        // the tile count was known) and must not be in flight when it exits
        bool ok = mbar_wait(q_full, 0, a.ctl, abort_flag, kSiteMla, 1);
        if (!ok) {
          DevCtl drain = a.ctl;
          volatile int never = 0;
          mbar_wait(q_full, 0, drain, &never, kSiteMla, 2);
        }
        if (ntiles > 0) ok = ok && mbar_wait(qt_full, 0, a.ctl, abort_flag, kSiteMla, 12);
        // Descriptors are built once; per MMA only the start-address field moves
        // (byte offset / 16 added to the low bits, which never carry: smem < 256 KB).
        const uint64_t qd0 = make_sdesc(smem_u32(q_smem), 16, 1024, 2);
        if (ok && ntiles > 0) {
          if (Tr::NB_B * 2 <= NKB && dvc != 0)
            ok = mla_issue_tiles<NKB, DVC, 1>(ntiles, tbase, smem_u32(kv_smem), qd0, bars, a.ctl, abort_flag);
          else
            ok = mla_issue_tiles<NKB, DVC, 0>(ntiles, tbase, smem_u32(kv_smem), qd0, bars, a.ctl, abort_flag);
        }
        if (!ok) *abort_flag = 1;
        mma_commit(done_bar);
        DevCtl drain = a.ctl;
        volatile int never = 0;
        mbar_wait(done_bar, 0, drain, &never, kSiteMla, 7);
      }
    }
  } else if (warp >= PROD_T0 / 32) {
    // ------------------------------------------------ gather producers
    // Producer warp pw owns rows 8 pw .. 8 pw + 7 of every tile. Lanes 0..7 load
    // the rows' indices once per tile; the row offsets are broadcast by shuffle.
    // A part's chunks are 16 bytes: chunk q of the warp = row q / (8 NB), column
    // block q / 8 % NB of the part, 16-byte slot q % 8; consecutive lanes copy
    // consecutive 16 bytes of a row. A chunk lands in the 128-byte-swizzled
    // K-major layout the tensor core reads: column block kb, row r, 16-byte slot
    // q8 ^ (r % 8). Chunks past the end of a row (padding up to the 64-column
    // block) are zeros. Once its copies of a part have landed, a thread makes them
    // visible to the tensor core (proxy fence) and arrives on that part's full
    // barrier.
    const int pw = warp - PROD_T0 / 32;
    const int row_bytes = a.Dqk * 2;
    const uint8_t* kv_g = reinterpret_cast<const uint8_t*>(kv);
    const uint8_t* kv_b = kv_g + (size_t)b * a.Lk * row_bytes;   // unpaged: sequence b's rows
    const uint32_t kv_base = smem_u32(kv_smem);
    const int vb0 = dvc * Tr::NB_B;
    auto gather_part = [&](int i, const uint8_t* src_row, auto part_c) {
      constexpr int PART = decltype(part_c)::value;
      constexpr int NB = PART ? Tr::NB_B : Tr::NB_A;
      constexpr int CPL = PART ? Tr::CPL_B : Tr::CPL_A;
      const uint32_t stage = kv_base + (i % Tr::STAGES) * NKB * Tr::KVBLK;
#pragma unroll
      for (int jj = 0; jj < CPL; ++jj) {
        const int q = lane + jj * 32;
        const int rr = q / (NB * 8);             // row within the warp's 8
        const int rem = q - rr * NB * 8;
        const int j = rem >> 3, q8 = rem & 7;
        const int kb = PART ? vb0 + j : (j < vb0 ? j : j + Tr::NB_B);
        const int qc = kb * 8 + q8;               // 16-byte chunk within the row
        const uint8_t* src = reinterpret_cast<const uint8_t*>(
            __shfl_sync(0xffffffffu, reinterpret_cast<uintptr_t>(src_row), rr));
        const int r = pw * ROWS_PER_PROD + rr;
        const bool in_row = qc * 16 < row_bytes;
        cp_async16(stage + kb * Tr::KVBLK + r * 128 + ((q8 ^ (r & 7)) << 4), src + (in_row ? qc * 16 : 0),
                   in_row ? 16u : 0u);
      }
      cp_async_commit();
    };
    for (int i = 0; i < ntiles; ++i) {
      const int st = i % Tr::STAGES;
      const uint32_t ph = ((i / Tr::STAGES) & 1) ^ 1;
      // the second stage first holds Q's TMEM blocks
      if (i == 1 && !mbar_wait(qt_full, 0, a.ctl, abort_flag, kSiteMla, 18)) break;
      // this warp's rows: index, validity and source row (invalid keys read row 0
      // and are masked later; paged: the key's pool row, a page outside the pool
      // reads pool row 0)
      const int pos = (tile0 + i) * KEYS + pw * ROWS_PER_PROD + lane;
      int v = -1;
      if (lane < ROWS_PER_PROD && pos < a.k) v = __ldg(idx_row + pos);
      const bool valid = lane < ROWS_PER_PROD && v >= 0 && v < a.Lk;
      const uint8_t* src_row;
      if constexpr (PAGED) {
        long long prow = valid ? key_row(a.block_table, a.max_blocks, a.page_size, a.num_pages, b, a.Lk, v) : 0;
        if (prow < 0) prow = 0;
        src_row = kv_g + (size_t)prow * row_bytes;
      } else {
        src_row = kv_b + (size_t)(valid ? v : 0) * row_bytes;
      }
      const unsigned vmask = __ballot_sync(0xffffffffu, valid);
      // part A is free once S of the tile that last used this stage is done ...
      if (!mbar_wait(&kvA_empty[st], ph, a.ctl, abort_flag, kSiteMla, 8)) break;
      gather_part(i, src_row, std::integral_constant<int, 0>{});
      cp_async_wait<0>();
      fence_proxy_async_smem();
      mbar_arrive(&kvA_full[st]);
      // ... part B (the values) once PV of that tile is done
      if (!mbar_wait(&kvB_empty[st], ph, a.ctl, abort_flag, kSiteMla, 9)) break;
      gather_part(i, src_row, std::integral_constant<int, 1>{});
      if (lane == 0) mask8[st * PROD_WARPS + pw] = (uint8_t)(vmask & ((1u << ROWS_PER_PROD) - 1u));
      cp_async_wait<0>();
      fence_proxy_async_smem();
      mbar_arrive(&kvB_full[st]);
    }
    cp_async_wait_all();
  } else {
    // ------------------------------------------------ softmax / epilogue (warps 1..8)
    const int sw = warp - SMX_T0 / 32;       // 0 .. 7
    const int quad = warp & 3;               // TMEM lane quadrant this warp may access
    const int hf = sw / 4;                   // which 32 keys of each tile, which half of O
    const int h = quad * 32 + lane;          // head = TMEM lane
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    constexpr int OCOLS = DVC / 2;           // O columns this thread rescales and writes
    // this head's first QT_KB * 64 query columns go to TMEM (the MMA's A operand:
    // lane = head, 32-bit column = two consecutive bf16 of the row), read from the
    // 128-byte-swizzled rows the TMA put into the second KV stage; each half
    // writes its share of the blocks
    bool ok = true;
    if (ntiles > 0) {
      ok = mbar_wait(q_full, 0, a.ctl, abort_flag, kSiteMla, 17);
      if (ok) {
        const uint32_t qrow = smem_u32(kv_smem + NKB * Tr::KVBLK) + (uint32_t)h * 128u;
#pragma unroll 1
        for (int kb = hf; kb < Tr::QT_KB; kb += 2) {
          uint32_t qv[32];
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const uint4 u = ld_shared_v4(qrow + (uint32_t)(kb * Tr::QBLK) + ((uint32_t)(c ^ (h & 7)) << 4));
            qv[4 * c] = u.x; qv[4 * c + 1] = u.y; qv[4 * c + 2] = u.z; qv[4 * c + 3] = u.w;
          }
          tmem_st32(qt_tmem + lane_off + kb * 32, qv);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(qt_full);
      }
    }
    float m_used = -INFINITY;  // running max (log2 domain) that P is relative to
    float l = 0.f;             // this thread's 32-key share of the row sum
    for (int i = 0; ok && i < ntiles; ++i) {
      const int st = i % Tr::STAGES;
      if (!mbar_wait(&s_full[i & 1], (i >> 1) & 1, a.ctl, abort_flag, kSiteMla, 10)) { ok = false; break; }
      if (!mbar_wait(&kvB_full[st], (i / Tr::STAGES) & 1, a.ctl, abort_flag, kSiteMla, 11)) { ok = false; break; }
      tc_fence_after();
      const uint32_t sbuf = s_tmem + (uint32_t)((i & 1) * KEYS) + lane_off;   // this head's S_i
      uint32_t r[32];
      tmem_ld32(sbuf + hf * 32, r);
      tmem_wait_ld();
      const uint32_t m = masks[st * 2 + hf];
      float x[32];
      float tmax = -INFINITY;
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        x[j] = ((m >> j) & 1u) ? __uint_as_float(r[j]) * a.scale_log2 : -INFINITY;
        tmax = fmaxf(tmax, x[j]);
      }
      // both halves' maxima: S_i has been read into registers by both threads of
      // the head once this barrier completes, so P may be written over it
      volatile uint16_t* xm = xmax + (i & 1) * 256;
      const uint16_t mine = bf16_at_least(tmax);
      xm[hf * 128 + h] = mine;
      mbar_arrive(&xmax_bar[i & 1]);
      if (!mbar_wait(&xmax_bar[i & 1], (i >> 1) & 1, a.ctl, abort_flag, kSiteMla, 13)) { ok = false; break; }
      tmax = fmaxf(bf16_bits_to_float(mine), bf16_bits_to_float(xm[(hf ^ 1) * 128 + h]));
      const bool grow = tmax > m_used + 8.0f;
      const float m_new = grow ? tmax : m_used;
      const bool need_o = grow && m_used != -INFINITY;
      if (__any_sync(0xffffffffu, need_o)) {
        // O is rescaled in place: PV_{i-1} (the last one issued) must be done
        if (!mbar_wait(&pv_done[(i - 1) & 1], ((i - 1) >> 1) & 1, a.ctl, abort_flag, kSiteMla, 14)) { ok = false; break; }
        tc_fence_after();
        const float alpha = need_o ? ex2(m_used - m_new) : 1.f;
#pragma unroll 1
        for (int c0 = hf * OCOLS; c0 < (hf + 1) * OCOLS; c0 += 32) {
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
      float psum0 = 0.f, psum1 = 0.f;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        float p0 = ex2(x[2 * j] - m_used);
        float p1 = ex2(x[2 * j + 1] - m_used);
        if (m_used == -INFINITY) { p0 = 0.f; p1 = 0.f; }
        psum0 += p0;
        psum1 += p1;
        pk[j] = pack_bf16x2(p0, p1);
      }
      l += psum0 + psum1;
      // P_i for this thread's 32 keys over columns 16 hf .. 16 hf + 15 of S_i's buffer
      tmem_st16(sbuf + hf * 16, pk);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&p_full[i & 1]);
    }
    if (ok && ntiles > 0) {
      ok = mbar_wait(&pv_done[(ntiles - 1) & 1], ((ntiles - 1) >> 1) & 1, a.ctl, abort_flag, kSiteMla, 15);
      tc_fence_after();
    }
    if (ok) {
      // the head's row sum over both halves of every tile
      volatile float* xl = reinterpret_cast<volatile float*>(xmax);   // the maxima are no longer read
      xl[hf * 128 + h] = l;
      mbar_arrive(xl_bar);
      ok = mbar_wait(xl_bar, 0, a.ctl, abort_flag, kSiteMla, 16);
      if (ok) l += xl[(hf ^ 1) * 128 + h];
    }
    ok = __all_sync(0xffffffffu, ok);   // the epilogue below synchronises the warp
    if (ok) {
      const bool row_ok = h < a.H;
      const bool empty = !(l > 0.f);
      if (a.splits == 1) {
        const float inv = empty ? 0.f : 1.f / l;
        // The warp's 32 rows of OCOLS bf16 go through shared memory (the KV stages:
        // every MMA is done) so that the global stores are row-contiguous: written
        // one row per lane with the 16-byte chunks rotated by the row (no bank
        // conflicts), read back NCH lanes per row.
        constexpr int NCH = OCOLS * 2 / 16;            // 16-byte chunks per row
        const uint32_t stg = smem_u32(kv_smem) + (uint32_t)(sw * 32 * OCOLS * 2);
        const uint32_t my_row = stg + (uint32_t)(lane * OCOLS * 2);
#pragma unroll 1
        for (int c0 = 0; c0 < OCOLS; c0 += 32) {
          uint32_t o[32];
          if (ntiles > 0) {
            tmem_ld32(o_tmem + lane_off + hf * OCOLS + c0, o);
            tmem_wait_ld();
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) o[j] = 0u;
          }
          uint32_t pk[16];
#pragma unroll
          for (int j = 0; j < 16; ++j)
            pk[j] = pack_bf16x2(__uint_as_float(o[2 * j]) * inv, __uint_as_float(o[2 * j + 1]) * inv);
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const int ch = c0 / 8 + c;
            st_shared_v4(my_row + (uint32_t)(((ch + lane) % NCH) * 16),
                         make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]));
          }
        }
        __syncwarp();
        uint16_t* obase = a.out + token * a.H * (long long)a.Dv + dvc * DVC + hf * OCOLS;
#pragma unroll 4
        for (int e = lane; e < 32 * NCH; e += 32) {
          const int r = e / NCH, ch = e % NCH;
          const uint4 v = ld_shared_v4(stg + (uint32_t)(r * OCOLS * 2 + ((ch + r) % NCH) * 16));
          const int hr = quad * 32 + r;
          if (hr < a.H) *reinterpret_cast<uint4*>(obase + (long long)hr * a.Dv + ch * 8) = v;
        }
        if (row_ok && hf == 0 && dvc == 0 && a.lse != nullptr)
          a.lse[token * a.H + h] = empty ? -INFINITY : (m_used + __log2f(l)) * 0.69314718055994531f;
      } else {
        const long long prow_i = (token * a.splits + split) * a.H + h;
        float* po = a.part_o + prow_i * a.Dv + dvc * DVC;
#pragma unroll 1
        for (int c0 = hf * OCOLS; c0 < (hf + 1) * OCOLS; c0 += 32) {
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
        if (row_ok && hf == 0 && dvc == 0) {
          a.part_ml[prow_i * 2 + 0] = empty ? -INFINITY : m_used;
          a.part_ml[prow_i * 2 + 1] = empty ? 0.f : l;
        }
      }
    }
  }

  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tbase, Tr::TMEM_COLS);
  }
}

// Merge key-split partials: out = sum_s 2^(m_s - M) O_s / sum_s 2^(m_s - M) l_s.
// One CTA per (token, head) row, four value columns per thread; the weights of
// the (at most kMaxSplits) partials are computed once and all partial loads of a
// thread are issued before any is used. Dv is a multiple of 4 (512 or 64).
constexpr int kMaxSplits = 16;
constexpr int kCombineThreads = 128;
__global__ void __launch_bounds__(kCombineThreads) mla_combine_kernel(const MlaArgs a) {
  const long long row = blockIdx.x;  // token * H + h
  const long long token = row / a.H;
  const int h = (int)(row % a.H);
  const float* ml0 = a.part_ml + (token * a.splits * a.H + h) * 2;
  const long long ml_stride = (long long)a.H * 2;
  float M = -INFINITY;
#pragma unroll
  for (int s = 0; s < kMaxSplits; ++s)
    if (s < a.splits && ml0[s * ml_stride + 1] > 0.f) M = fmaxf(M, ml0[s * ml_stride]);
  float f[kMaxSplits];
  float L = 0.f;
#pragma unroll
  for (int s = 0; s < kMaxSplits; ++s) {
    f[s] = 0.f;
    if (s < a.splits && ml0[s * ml_stride + 1] > 0.f) {
      f[s] = ex2(ml0[s * ml_stride] - M);
      L += ml0[s * ml_stride + 1] * f[s];
    }
  }
  const float inv = L > 0.f ? 1.f / L : 0.f;
  const float* o0 = a.part_o + (token * a.splits * a.H + h) * (long long)a.Dv;
  const long long o_stride = (long long)a.H * a.Dv;
  uint16_t* orow = a.out + row * (long long)a.Dv;
  for (int c = threadIdx.x * 4; c < a.Dv; c += kCombineThreads * 4) {
    float4 v[kMaxSplits];
#pragma unroll
    for (int s = 0; s < kMaxSplits; ++s)
      v[s] = f[s] != 0.f ? __ldcs(reinterpret_cast<const float4*>(o0 + s * o_stride + c))
                         : make_float4(0.f, 0.f, 0.f, 0.f);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int s = 0; s < kMaxSplits; ++s) {
      acc.x = fmaf(v[s].x, f[s], acc.x);
      acc.y = fmaf(v[s].y, f[s], acc.y);
      acc.z = fmaf(v[s].z, f[s], acc.z);
      acc.w = fmaf(v[s].w, f[s], acc.w);
    }
    uint2 packed;
    packed.x = pack_bf16x2(acc.x * inv, acc.y * inv);
    packed.y = pack_bf16x2(acc.z * inv, acc.w * inv);
    *reinterpret_cast<uint2*>(orow + c) = packed;
  }
  if (threadIdx.x == 0 && a.lse != nullptr)
    a.lse[row] = L > 0.f ? (M + __log2f(L)) * 0.69314718055994531f : -INFINITY;
}

template <int NKB, int DVC>
cudaError_t launch_mla_variant(const CUtensorMap& tq, const uint16_t* kv, const MlaArgs& a,
                               cudaStream_t stream) {
  using Tr = MlaTraits<NKB, DVC>;
  // several query rows per sequence (prefill): the warp-wide issuer
  const bool warp_issue = a.Lq > 1;
  auto kern = a.block_table != nullptr
                  ? (warp_issue ? sparse_mla_kernel<NKB, DVC, true, true> : sparse_mla_kernel<NKB, DVC, true, false>)
                  : (warp_issue ? sparse_mla_kernel<NKB, DVC, false, true> : sparse_mla_kernel<NKB, DVC, false, false>);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       Tr::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  long long grid = (long long)a.B * a.Lq * a.n_dv * a.splits;
  if (grid <= 0) return cudaSuccess;
  kern<<<(unsigned)grid, MLA_THREADS, Tr::SMEM_BYTES, stream>>>(tq, kv, a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_sparse_mla(const CUtensorMap& tmap_q, const uint16_t* kv, const MlaArgs& a,
                              cudaStream_t stream) {
  if (a.H == 128 && a.Dqk == 576 && a.Dv == 512) return launch_mla_variant<9, 256>(tmap_q, kv, a, stream);
  if (a.H == 8 && a.Dqk == 80 && a.Dv == 64) return launch_mla_variant<2, 64>(tmap_q, kv, a, stream);
  return cudaErrorInvalidValue;
}

cudaError_t launch_mla_combine(const MlaArgs& a, cudaStream_t stream) {
  long long rows = (long long)a.B * a.Lq * a.H;
  if (rows <= 0) return cudaSuccess;
  mla_combine_kernel<<<(unsigned)rows, kCombineThreads, 0, stream>>>(a);
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
