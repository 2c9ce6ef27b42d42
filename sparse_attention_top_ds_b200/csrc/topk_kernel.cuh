// topk_kernel.cuh -- row-wise top-k with one thread-block cluster per row.
//
// What it computes: for each row, the k largest of the first L = valid_len
// scores, ties to the lower position (DeepSelect hub page, use-case
// paragraphs: top-k of a bfloat16 indexer score row, and of a float32 logit
// row over a ~129K vocabulary; options sorted_index and return_value).
//
// How (B200 design, not the pages' design):
//  * A row is split into C contiguous slices, one per CTA of a cluster.  Pass 0
//    streams the slice from HBM with 128-bit loads straight into registers,
//    turns each score into an order-preserving unsigned key and builds a
//    4096-bin shared-memory histogram of its top 12 bits.  No score is kept on
//    chip: shared memory holds only histograms and a candidate buffer, so
//    several CTAs fit on an SM and the load phase of one overlaps the
//    synchronisation of the others.
//  * The histograms are added into the leader CTA through distributed shared
//    memory; the leader finds the bin b0 that holds the k-th key.
//  * Pass 1 re-reads the slice (now resident in the 126 MB L2): keys above b0
//    are final and are written out at once (output slots from an atomic counter
//    in the leader); keys inside b0 are appended to a candidate buffer in the
//    leader's shared memory.  The leader then finishes alone: an exact radix
//    select on the remaining key bits of the candidates, and on the positions
//    of the tied ones (ties go to the lowest positions).
//  * A row whose threshold bin holds more candidates than the buffer takes a
//    slower exact path: one cluster-wide digit pass per remaining digit over
//    the slice, then an ordered emission (warp and block scans) in which ties
//    go to the lowest positions.
//  * sorted_index: the leader sorts the row's selected positions at the end.
#pragma once

#include "ptx.cuh"

namespace dstopk {

struct TopkParams {
  const void* scores;
  const int32_t* valid_len;
  int32_t* out_idx;
  void* out_val;
  int* status;
  int batch, n, k;
  int slice;         // elements per CTA, a multiple of 8
  int return_value;
  int sorted;        // write the selection in ascending position order
};

constexpr int kD0 = 12;               // width of the first digit
constexpr int kHistBins = 1 << kD0;   // 4096
constexpr int kCandCap = 2048;        // candidates the leader can hold
constexpr int kStashCap = 1024;       // keys a CTA can stash during pass 0

// float32 rows: 32-bit keys; digits 12 (pass 0), then 11 and 9.
struct F32Keys {
  using Raw = uint32_t;
  static constexpr int kBits = 32, kBytes = 4, kVec = 4;
  static constexpr int kNumLater = 2;  // digits after the first
  static constexpr uint32_t kNegInf = 0xFF800000u;
  __device__ __forceinline__ static int later_shift(int p) { return p == 0 ? 9 : 0; }
  __device__ __forceinline__ static int later_width(int p) { return p == 0 ? 11 : 9; }
  // larger key <=> larger value; -0 folds onto +0; every NaN maps to the top key.
  __device__ __forceinline__ static uint32_t key(uint32_t b) {
    if ((b & 0x7FFFFFFFu) > 0x7F800000u) return 0xFFFFFFFFu;
    if (b == 0x80000000u) b = 0u;
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
  }
  __device__ __forceinline__ static uint32_t slot(const uint4& v, int j) {
    return j == 0 ? v.x : (j == 1 ? v.y : (j == 2 ? v.z : v.w));
  }
  // The smallest value whose key is >= t, as a float: key(x) >= t holds
  // exactly when !(x < bound(t)) for every x that is not a NaN, and a NaN x
  // passes too (it has the top key).  For t above key(+inf), and t below
  // key(-inf), bound(t) is a NaN and every x passes: a superset, never a miss.
  __device__ __forceinline__ static float bound(uint32_t t) {
    return __uint_as_float((t & 0x80000000u) ? (t & 0x7FFFFFFFu) : ~t);
  }
  // !(element j of v < tf): one float compare instead of a key conversion
  __device__ __forceinline__ static bool ge(const uint4& v, int j, float tf) {
    return !(__uint_as_float(slot(v, j)) < tf);
  }
};

// bfloat16 rows: 16-bit keys; digits 12 (pass 0), then 4.
struct BF16Keys {
  using Raw = uint16_t;
  static constexpr int kBits = 16, kBytes = 2, kVec = 8;
  static constexpr int kNumLater = 1;
  static constexpr uint32_t kNegInf = 0xFF80u;
  __device__ __forceinline__ static int later_shift(int) { return 0; }
  __device__ __forceinline__ static int later_width(int) { return 4; }
  __device__ __forceinline__ static uint32_t key(uint32_t b) {
    b &= 0xFFFFu;
    if ((b & 0x7FFFu) > 0x7F80u) return 0xFFFFu;
    if (b == 0x8000u) b = 0u;
    return (b & 0x8000u) ? (~b & 0xFFFFu) : (b | 0x8000u);
  }
  __device__ __forceinline__ static uint32_t slot(const uint4& v, int j) {
    const uint32_t w = (j >> 1) == 0 ? v.x : ((j >> 1) == 1 ? v.y : ((j >> 1) == 2 ? v.z : v.w));
    return (j & 1) ? (w >> 16) : (w & 0xFFFFu);
  }
  // as F32Keys::bound, for 16-bit keys (a bfloat16 is the top half of a float)
  __device__ __forceinline__ static float bound(uint32_t t) {
    return __uint_as_float(((t & 0x8000u) ? (t & 0x7FFFu) : (~t & 0xFFFFu)) << 16);
  }
  __device__ __forceinline__ static bool ge(const uint4& v, int j, float tf) {
    const uint32_t w = (j >> 1) == 0 ? v.x : ((j >> 1) == 1 ? v.y : ((j >> 1) == 2 ? v.z : v.w));
    return !(__uint_as_float((j & 1) ? (w & 0xFFFF0000u) : (w << 16)) < tf);
  }
};

struct TopkCtrl {
  uint32_t res[4];     // leader -> every CTA: digit bin of the k-th key, keys still to take, keys in the bin
  uint32_t glob_out;   // leader: output slots handed out to the CTAs for final keys
  uint32_t glob_cand;  // leader: candidate slots handed out
  uint32_t loc_out;    // this CTA: final keys written
  uint32_t loc_cand;   // this CTA: candidates sent
  uint32_t bcast[4];   // broadcast scratch inside the CTA
  uint32_t base, take;
  uint32_t stash_cnt;  // this CTA: keys stashed in pass 0
  uint32_t tie_cnt;    // leader: ties listed
};

// shared memory: histogram | leader's reduction histogram, later its candidate
// buffer | stash | control block | scan scratch | per-CTA counts
constexpr int kSmemHist = 0;
constexpr int kSmemRegion = kSmemHist + kHistBins * 4;      // 16 KiB
constexpr int kSmemCandRaw = kSmemRegion;                   // u32[kCandCap]
constexpr int kSmemCandIdx = kSmemRegion + kCandCap * 4;    // u32[kCandCap]
constexpr int kSmemStashRaw = kSmemRegion + 2 * kCandCap * 4;  // u32[kStashCap]
constexpr int kSmemStashIdx = kSmemStashRaw + kStashCap * 4;   // u32[kStashCap]
constexpr int kSmemCtrl = kSmemStashIdx + kStashCap * 4;
constexpr int kSmemWtot = kSmemCtrl + 128;
constexpr int kSmemCnt = kSmemWtot + 32 * 4;                // every CTA: (gt, eq) of each CTA, 2 x u32[16]
constexpr int kTopkSmemBytes = kSmemCnt + 2 * 16 * 4;
static_assert(sizeof(TopkCtrl) <= 128, "ctrl block");
static_assert(kHistBins <= 2 * kCandCap, "the reduction histogram must fit the candidate region");
static_assert(2048 <= kCandCap, "the sort buffer (k <= 2048) reuses the candidate positions");

// Warp-aggregated histogram increment for a run of `cnt` equal digits: when
// every active lane of the warp carries the same digit, one atomic adds the
// warp's total (sorted or constant rows would otherwise put 32 lanes on one
// shared-memory word).
__device__ __forceinline__ void hist_add_run(uint32_t* h, uint32_t bin, uint32_t cnt) {
  const uint32_t mask = __activemask();
  const int lead = __ffs(mask) - 1;
  const uint32_t first = __shfl_sync(mask, bin, lead);
  if (__all_sync(mask, bin == first)) {
    const uint32_t tot = __reduce_add_sync(mask, cnt);
    if ((int)(threadIdx.x & 31) == lead) atomicAdd(h + bin, tot);
  } else {
    atomicAdd(h + bin, cnt);
  }
}

template <int NT>
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t* wtot, uint32_t& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t t = __shfl_up_sync(0xFFFFFFFFu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) wtot[warp] = incl;
  __syncthreads();
  uint32_t base = 0, tot = 0;
#pragma unroll
  for (int w = 0; w < NT / 32; ++w) {
    const uint32_t t = wtot[w];
    base += (w < warp) ? t : 0u;
    tot += t;
  }
  __syncthreads();
  total = tot;
  return base + incl - v;
}

template <int NT>
__device__ __forceinline__ uint32_t block_sum(uint32_t v, uint32_t* wtot) {
  uint32_t total;
  block_excl_scan<NT>(v, wtot, total);
  return total;
}

// Inside one CTA: in a histogram of nb bins find b with
// #(bins > b) < krem <= #(bins >= b); `above` / `inbin` return the counts
// above and inside it.  Every thread gets the result.  The caller must pass a
// __syncthreads() before `wtot` / `bcast` are written again.
template <int NT>
__device__ __forceinline__ uint32_t block_find_bin(const uint32_t* h, int nb, int krem, uint32_t* wtot,
                                                   uint32_t* bcast, uint32_t& above, uint32_t& inbin) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int bpt = (nb + NT - 1) / NT;
  const int r0 = threadIdx.x * bpt;  // this thread's bins, from the top: nb-1-r0, nb-2-r0, ...
  uint32_t s = 0;
  for (int r = r0; r < min(nb, r0 + bpt); ++r) s += h[nb - 1 - r];
  uint32_t incl = s;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t t = __shfl_up_sync(0xFFFFFFFFu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) wtot[warp] = incl;
  if (threadIdx.x == 0) {
    bcast[0] = 0u;
    bcast[1] = 0u;
    bcast[2] = 0u;
  }
  __syncthreads();
  uint32_t excl = incl - s;
#pragma unroll
  for (int w = 0; w < NT / 32; ++w) excl += (w < warp) ? wtot[w] : 0u;
  if (excl < (uint32_t)krem && (uint32_t)krem <= excl + s) {
    uint32_t acc = excl;
    for (int r = r0; r < min(nb, r0 + bpt); ++r) {
      const uint32_t c = h[nb - 1 - r];
      if (acc + c >= (uint32_t)krem) {
        bcast[0] = (uint32_t)(nb - 1 - r);
        bcast[1] = acc;
        bcast[2] = c;
        break;
      }
      acc += c;
    }
  }
  __syncthreads();
  above = bcast[1];
  inbin = bcast[2];
  return min(bcast[0], (uint32_t)(nb - 1));
}

// Streams the CTA's slice [i0, i0 + m) of a row.  fv(e, word) is called for
// every 16-byte word that lies inside the slice (e = row index of its first
// element), with UNROLL independent 128-bit loads per thread in flight;
// fe(e, raw) for each element of the (at most two) words that the slice
// covers only in part.
template <class K, int NT, int UNROLL, class FV, class FE>
__device__ __forceinline__ void stream_slice(const typename K::Raw* grow, int i0, int m, FV&& fv, FE&& fe) {
  if (m <= 0) return;
  const uintptr_t base = reinterpret_cast<uintptr_t>(grow);
  const uintptr_t a0 = base + (uintptr_t)i0 * K::kBytes;
  const uintptr_t a1 = a0 + (uintptr_t)m * K::kBytes;
  const uintptr_t f0 = (a0 + 15u) & ~uintptr_t(15);  // first full word
  const uintptr_t f1 = a1 & ~uintptr_t(15);          // end of the full words
  const int nfull = f1 > f0 ? (int)((f1 - f0) >> 4) : 0;
  const uint4* wp = reinterpret_cast<const uint4*>(f0);
  const int e_f0 = (int)((f0 - base) / K::kBytes);
  int w = threadIdx.x;
  for (; w + (UNROLL - 1) * NT < nfull; w += UNROLL * NT) {
    uint4 r[UNROLL];
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) r[u] = __ldg(wp + w + u * NT);
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) fv(e_f0 + (w + u * NT) * K::kVec, r[u]);
  }
  for (; w < nfull; w += NT) fv(e_f0 + w * K::kVec, __ldg(wp + w));
  // elements outside the full words: fewer than 2 * kVec
  const int head = nfull > 0 ? (int)((f0 - a0) / K::kBytes) : m;
  const int tail_start = nfull > 0 ? (int)((f1 - base) / K::kBytes) : i0 + m;
  const int tail = i0 + m - tail_start;
  const int t = threadIdx.x;
  if (t < head) fe(i0 + t, (uint32_t)grow[i0 + t]);
  if (nfull > 0 && t >= 32 && t - 32 < tail) fe(tail_start + t - 32, (uint32_t)grow[tail_start + t - 32]);
}

__device__ __forceinline__ void dsmem_st_u32(uint32_t addr, uint32_t v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

// The leader publishes (b, krem, count) into the control block of every CTA of
// the cluster with remote stores; after the next cluster barrier each CTA reads
// its own copy (no remote load on the critical path).
__device__ __forceinline__ void leader_publish(TopkCtrl* ctrl, uint32_t csize, uint32_t b, uint32_t krem,
                                               uint32_t cnt) {
  if (threadIdx.x < csize) {
    const uint32_t a = dsmem_map(smem_u32(&ctrl->res[0]), threadIdx.x);
    dsmem_st_u32(a, b);
    dsmem_st_u32(a + 4, krem);
    dsmem_st_u32(a + 8, cnt);
  }
}

__device__ __forceinline__ uint32_t dsmem_atom_add_u32(uint32_t addr, uint32_t v) {
  uint32_t old;
  asm volatile("atom.relaxed.cluster.shared::cluster.add.u32 %0, [%1], %2;" : "=r"(old) : "r"(addr), "r"(v) : "memory");
  return old;
}

template <class K, int NT>
__global__ void __launch_bounds__(NT, 1024 / NT) topk_cluster_kernel(const TopkParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  uint32_t* hist = reinterpret_cast<uint32_t*>(smem + kSmemHist);
  uint32_t* hred = reinterpret_cast<uint32_t*>(smem + kSmemRegion);
  uint32_t* cand_raw = reinterpret_cast<uint32_t*>(smem + kSmemCandRaw);
  uint32_t* cand_idx = reinterpret_cast<uint32_t*>(smem + kSmemCandIdx);
  TopkCtrl* ctrl = reinterpret_cast<TopkCtrl*>(smem + kSmemCtrl);
  uint32_t* wtot = reinterpret_cast<uint32_t*>(smem + kSmemWtot);
  uint32_t* cnt_gt = reinterpret_cast<uint32_t*>(smem + kSmemCnt);
  uint32_t* cnt_eq = cnt_gt + 16;
  uint32_t* stash_raw = reinterpret_cast<uint32_t*>(smem + kSmemStashRaw);
  uint32_t* stash_idx = reinterpret_cast<uint32_t*>(smem + kSmemStashIdx);
  using Raw = typename K::Raw;
  constexpr int kShift0 = K::kBits - kD0;

  const int tid = threadIdx.x;
  const uint32_t crank = cluster_ctarank();
  const uint32_t csize = cluster_nctarank();
  const int row = blockIdx.x / csize;
  pdl_wait();
  pdl_launch_dependents();

  int L = p.n;
  if (p.valid_len) {
    const int v = p.valid_len[row];
    if (tid == 0 && crank == 0) debug_range(v >= 0 && v <= p.n, p.status);
    L = v < 0 ? 0 : (v > p.n ? p.n : v);
  }
  const int kk = min(p.k, L);
  int32_t* out_idx = p.out_idx + (size_t)row * p.k;
  Raw* out_val = p.return_value ? reinterpret_cast<Raw*>(p.out_val) + (size_t)row * p.k : nullptr;

  // padding slots kk..k-1 (written by the leader CTA)
  if (crank == 0) {
    for (int j = kk + tid; j < p.k; j += NT) {
      out_idx[j] = -1;
      if (out_val) out_val[j] = (Raw)K::kNegInf;
    }
  }
  if (kk == 0) return;  // uniform across the cluster: nothing to select in this row

  const int i0 = (int)crank * p.slice;
  const int m = max(0, min(p.slice, L - i0));  // eligible scores in this slice
  const Raw* grow = reinterpret_cast<const Raw*>(p.scores) + (size_t)row * p.n;

  for (int i = tid; i < kHistBins; i += NT) hist[i] = 0u;
  if (crank == 0)
    for (int i = tid; i < kHistBins; i += NT) hred[i] = 0u;
  if (tid == 0) {
    ctrl->glob_out = 0u;
    ctrl->glob_cand = 0u;
    ctrl->loc_out = 0u;
    ctrl->loc_cand = 0u;
    ctrl->stash_cnt = 0u;
  }
  __syncthreads();
  cluster_arrive();  // every CTA's reduction histogram and counters are zeroed before anyone uses them

  // ---- pass 0: stream the slice; histogram of the top 12 key bits.  The
  // first loads of every thread form a sample: from its histogram the CTA
  // picks a digit b_est comfortably below its share of the row's threshold
  // and from then on stashes every key with digit >= b_est, so that pass 1
  // can skip the re-read of the slice.
  constexpr int U = 4;
  const uintptr_t rbase = reinterpret_cast<uintptr_t>(grow);
  const uintptr_t a0 = rbase + (uintptr_t)i0 * K::kBytes;
  const uintptr_t a1 = a0 + (uintptr_t)max(m, 0) * K::kBytes;
  const uintptr_t f0 = (a0 + 15u) & ~uintptr_t(15);
  const uintptr_t f1 = a1 & ~uintptr_t(15);
  const int nfull = (m > 0 && f1 > f0) ? (int)((f1 - f0) >> 4) : 0;
  const uint4* wp = reinterpret_cast<const uint4*>(f0);
  const int e_f0 = (int)((f0 - rbase) / K::kBytes);
  // the (fewer than 2 * kVec) elements outside the full words
  const int head = m <= 0 ? 0 : (nfull > 0 ? (int)((f0 - a0) / K::kBytes) : m);
  const int tail_start = nfull > 0 ? (int)((f1 - rbase) / K::kBytes) : i0 + m;
  const int tail = m <= 0 ? 0 : i0 + m - tail_start;
  int pe = -1;
  uint32_t praw = 0;
  if (tid < head) pe = i0 + tid;
  else if (nfull > 0 && tid >= 32 && tid - 32 < tail) pe = tail_start + tid - 32;
  if (pe >= 0) praw = (uint32_t)grow[pe];

  // digits of a 16-byte word; one histogram update per word (a warp-wide
  // atomic when all its digits agree across the warp: sorted or constant rows)
  auto digits = [&](const uint4& v, uint32_t (&d)[K::kVec]) {
#pragma unroll
    for (int j = 0; j < K::kVec; ++j) d[j] = K::key(K::slot(v, j)) >> kShift0;
  };
  auto hist_digits = [&](const uint32_t (&d)[K::kVec]) {
    bool same = true;
#pragma unroll
    for (int j = 1; j < K::kVec; ++j) same &= d[j] == d[0];
    if (same) {
      hist_add_run(hist, d[0], K::kVec);
    } else {
#pragma unroll
      for (int j = 0; j < K::kVec; ++j) atomicAdd(hist + d[j], 1u);
    }
  };
  uint4 sw[U];
#pragma unroll
  for (int u = 0; u < U; ++u)
    if (tid + u * NT < nfull) sw[u] = __ldg(wp + tid + u * NT);
#pragma unroll
  for (int u = 0; u < U; ++u) {
    if (tid + u * NT < nfull) {
      uint32_t d[K::kVec];
      digits(sw[u], d);
      hist_digits(d);
    }
  }
  if (pe >= 0) atomicAdd(hist + (K::key(praw) >> kShift0), 1u);
  // register mode: the whole slice is in this thread's first loads (sw, praw)
  const bool in_regs = nfull <= U * NT;
  uint32_t b_est = 0;
  if (!in_regs) {
    __syncthreads();
    {
      const int ns = U * NT * K::kVec + head + tail;
      const int target = min(ns, 2 * (int)((long)kk * ns / max(L, 1)) + 16);
      uint32_t above, inbin;
      b_est = block_find_bin<NT>(hist, kHistBins, target, wtot, ctrl->bcast, above, inbin);
    }
    auto stash_one = [&](int e, uint32_t raw) {
      const uint32_t pos = atomicAdd(&ctrl->stash_cnt, 1u);
      if (pos < (uint32_t)kStashCap) {
        stash_raw[pos] = raw;
        stash_idx[pos] = (uint32_t)e;
      }
    };
    auto stash_digits = [&](int e0, const uint4& v, const uint32_t (&d)[K::kVec]) {
      bool hit = false;
#pragma unroll
      for (int j = 0; j < K::kVec; ++j) hit |= d[j] >= b_est;
      if (hit) {
#pragma unroll
        for (int j = 0; j < K::kVec; ++j)
          if (d[j] >= b_est) stash_one(e0 + j, K::slot(v, j));
      }
    };
#pragma unroll
    for (int u = 0; u < U; ++u) {
      uint32_t d[K::kVec];
      digits(sw[u], d);  // all U sample words exist: nfull > U * NT
      stash_digits(e_f0 + (tid + u * NT) * K::kVec, sw[u], d);
    }
    if (pe >= 0 && (K::key(praw) >> kShift0) >= b_est) stash_one(pe, praw);
    int w = tid + U * NT;
    for (; w + (U - 1) * NT < nfull; w += U * NT) {
      uint4 r[U];
#pragma unroll
      for (int u = 0; u < U; ++u) r[u] = __ldg(wp + w + u * NT);
#pragma unroll
      for (int u = 0; u < U; ++u) {
        uint32_t d[K::kVec];
        digits(r[u], d);
        hist_digits(d);
        stash_digits(e_f0 + (w + u * NT) * K::kVec, r[u], d);
      }
    }
    for (; w < nfull; w += NT) {
      const uint4 r = __ldg(wp + w);
      uint32_t d[K::kVec];
      digits(r, d);
      hist_digits(d);
      stash_digits(e_f0 + w * K::kVec, r, d);
    }
  }
  __syncthreads();
  cluster_wait();

  const uint32_t leader_hred = dsmem_map(smem_u32(hred), 0);
  const uint32_t leader_ctrl = dsmem_map(smem_u32(ctrl), 0);
  for (int b = tid; b < kHistBins; b += NT) {
    const uint32_t c = hist[b];
    if (c) dsmem_red_add_u32(leader_hred + 4u * b, c);
  }
  cluster_sync();
  if (crank == 0) {
    uint32_t above, inbin;
    const uint32_t b = block_find_bin<NT>(hred, kHistBins, kk, wtot, ctrl->bcast, above, inbin);
    leader_publish(ctrl, csize, b, (uint32_t)(kk - (int)above), inbin);
  }
  cluster_sync();
  const uint32_t b0 = min(ctrl->res[0], (uint32_t)(kHistBins - 1));
  int krem = (int)ctrl->res[1];
  const uint32_t bcount = ctrl->res[2];
  const bool all_taken = bcount == (uint32_t)krem;  // the whole bin is selected

  if (all_taken || bcount <= (uint32_t)kCandCap) {
    // ---- fast path.  Final keys: digits >= fin_lo; candidates: digit b0
    // (unless the whole bin is taken).  This CTA's counts of both come from its
    // pass-0 histogram; one remote atomic each reserves its ranges.
    const uint32_t fin_lo = all_taken ? b0 : b0 + 1;
    uint32_t nfin = 0;
    for (int b = tid; b < kHistBins; b += NT) nfin += ((uint32_t)b >= fin_lo) ? hist[b] : 0u;
    nfin = block_sum<NT>(nfin, wtot);
    if (tid == 0) {
      ctrl->bcast[0] = dsmem_atom_add_u32(leader_ctrl + offsetof(TopkCtrl, glob_out), nfin);
      ctrl->bcast[1] = all_taken ? 0u : dsmem_atom_add_u32(leader_ctrl + offsetof(TopkCtrl, glob_cand), hist[b0]);
    }
    __syncthreads();
    const uint32_t fin_base = ctrl->bcast[0], cand_base = ctrl->bcast[1];
    const uint32_t lcand_raw = dsmem_map(smem_u32(cand_raw), 0);
    const uint32_t lcand_idx = dsmem_map(smem_u32(cand_idx), 0);
    // pass 1: re-read the slice (L2); a word holding a final key or a
    // candidate reserves its slots with one shared-memory atomic per kind
    auto emit = [&](int e0, const uint32_t* raw, int cnt) {
      uint32_t fin = 0, cand = 0;
      for (int j = 0; j < cnt; ++j) {
        const uint32_t d = K::key(raw[j]) >> kShift0;
        fin |= (uint32_t)(d >= fin_lo) << j;
        cand |= (uint32_t)(!all_taken && d == b0) << j;
      }
      if (fin) {
        uint32_t slot = fin_base + atomicAdd(&ctrl->loc_out, (uint32_t)__popc(fin));
        for (int j = 0; j < cnt; ++j) {
          if ((fin >> j) & 1u) {
            if (slot < (uint32_t)kk) {
              out_idx[slot] = e0 + j;
              if (out_val) out_val[slot] = (Raw)raw[j];
            }
            ++slot;
          }
        }
      }
      if (cand) {
        uint32_t cs = cand_base + atomicAdd(&ctrl->loc_cand, (uint32_t)__popc(cand));
        for (int j = 0; j < cnt; ++j) {
          if ((cand >> j) & 1u) {
            if (cs < (uint32_t)kCandCap) {
              dsmem_st_u32(lcand_raw + 4u * cs, raw[j]);
              dsmem_st_u32(lcand_idx + 4u * cs, (uint32_t)(e0 + j));
            }
            ++cs;
          }
        }
      }
    };
    if (in_regs) {
      // the slice is still in registers
#pragma unroll
      for (int u = 0; u < U; ++u) {
        if (tid + u * NT < nfull) {
          uint32_t raw[K::kVec];
          bool hit = false;
#pragma unroll
          for (int j = 0; j < K::kVec; ++j) {
            raw[j] = K::slot(sw[u], j);
            hit |= (K::key(raw[j]) >> kShift0) >= b0;
          }
          if (hit) emit(e_f0 + (tid + u * NT) * K::kVec, raw, K::kVec);
        }
      }
      if (pe >= 0) emit(pe, &praw, 1);
    } else if (ctrl->stash_cnt <= (uint32_t)kStashCap && b_est <= b0) {
      // the stash holds every key of this slice with digit >= b0
      const int ns = (int)ctrl->stash_cnt;
      for (int i = tid; i < ns; i += NT) {
        const uint32_t raw = stash_raw[i];
        emit((int)stash_idx[i], &raw, 1);
      }
    } else {
      stream_slice<K, NT, 4>(
          grow, i0, m,
          [&](int e0, const uint4& v) {
            uint32_t raw[K::kVec];
            bool hit = false;
#pragma unroll
            for (int j = 0; j < K::kVec; ++j) {
              raw[j] = K::slot(v, j);
              hit |= (K::key(raw[j]) >> kShift0) >= b0;
            }
            if (hit) emit(e0, raw, K::kVec);
          },
          [&](int e, uint32_t raw) { emit(e, &raw, 1); });
    }
    cluster_sync();  // every final key is written and every candidate has arrived
    if (crank != 0) return;
    if (!all_taken) {
      // ---- the leader alone: exact select among the candidates
      const int nc = min((int)bcount, kCandCap);
      uint32_t prefix = b0;
      int shift = kShift0;
      for (int pass = 0; pass < K::kNumLater; ++pass) {
        const int sh = K::later_shift(pass);
        const int wd = K::later_width(pass);
        const int nb = 1 << wd;
        for (int i = tid; i < nb; i += NT) hist[i] = 0u;
        __syncthreads();
        for (int i = tid; i < nc; i += NT) {
          const uint32_t kv = K::key(cand_raw[i]);
          if ((kv >> shift) == prefix) atomicAdd(hist + ((kv >> sh) & (uint32_t)(nb - 1)), 1u);
        }
        __syncthreads();
        uint32_t above, inbin;
        const uint32_t b = block_find_bin<NT>(hist, nb, krem, wtot, ctrl->bcast, above, inbin);
        krem -= (int)above;
        prefix = (prefix << wd) | b;
        shift = sh;
        if (inbin == (uint32_t)krem) break;  // the whole sub-bin is selected
      }
      // keys above the threshold are taken, and `krem` of the ties at it, the
      // lowest positions first: a radix select on the complemented positions
      // of the ties finds the position cut
      uint32_t ntie = 0;
      for (int i = tid; i < nc; i += NT) ntie += (K::key(cand_raw[i]) >> shift) == prefix;
      ntie = block_sum<NT>(ntie, wtot);
      auto put_sel = [&](int e, uint32_t raw) {
        const uint32_t slot = atomicAdd(&ctrl->glob_out, 1u);  // after the final keys
        if (slot < (uint32_t)kk) {
          out_idx[slot] = e;
          if (out_val) out_val[slot] = (Raw)raw;
        }
      };
      if ((uint32_t)krem >= ntie || ntie > (uint32_t)kStashCap) {
        uint32_t cut = 0xFFFFFFFFu;  // ties with position <= cut are taken
        if ((uint32_t)krem < ntie) {
          // many ties: radix select on the complemented positions
          uint32_t pfx = 0;
          int want = krem;
          for (int pass = 0; pass < 3; ++pass) {
            const int sh = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
            const int wd = pass == 2 ? 10 : 11;
            const int psh = pass == 0 ? 32 : (pass == 1 ? 21 : 10);
            const int nb = 1 << wd;
            for (int i = tid; i < nb; i += NT) hist[i] = 0u;
            __syncthreads();
            for (int i = tid; i < nc; i += NT) {
              if ((K::key(cand_raw[i]) >> shift) != prefix) continue;
              const uint32_t ck = ~cand_idx[i];
              if (pass == 0 || (ck >> psh) == pfx) atomicAdd(hist + ((ck >> sh) & (uint32_t)(nb - 1)), 1u);
            }
            __syncthreads();
            uint32_t above, inbin;
            const uint32_t b = block_find_bin<NT>(hist, nb, want, wtot, ctrl->bcast, above, inbin);
            want -= (int)above;
            pfx = (pass == 0 ? 0u : (pfx << wd)) | b;
          }
          cut = ~pfx;  // positions are distinct: exactly krem ties have position <= cut
        }
        for (int i = tid; i < nc; i += NT) {
          const uint32_t raw = cand_raw[i];
          const uint32_t top = K::key(raw) >> shift;
          const uint32_t e = cand_idx[i];
          if (top > prefix || (top == prefix && e <= cut)) put_sel((int)e, raw);
        }
      } else {
        // few ties: list them, rank each by counting lower positions
        if (tid == 0) ctrl->tie_cnt = 0u;
        __syncthreads();
        for (int i = tid; i < nc; i += NT) {
          const uint32_t raw = cand_raw[i];
          const uint32_t top = K::key(raw) >> shift;
          if (top > prefix) {
            put_sel((int)cand_idx[i], raw);
          } else if (top == prefix) {
            const uint32_t t = atomicAdd(&ctrl->tie_cnt, 1u);
            stash_idx[t] = cand_idx[i];
            stash_raw[t] = raw;
          }
        }
        __syncthreads();
        const int nt = (int)ntie;
        for (int i = tid; i < nt; i += NT) {
          const uint32_t me = stash_idx[i];
          int rank = 0;
          for (int j = 0; j < nt; ++j) rank += stash_idx[j] < me;
          if (rank < krem) put_sel((int)me, stash_raw[i]);
        }
      }
    }
    if (p.sorted) {
      // ---- ascending positions: bitonic sort of the row's selection
      __syncthreads();
      int np = 1;
      while (np < kk) np <<= 1;
      uint32_t* sidx = cand_idx;  // np <= 2048 entries; the candidates are done with
      for (int i = tid; i < np; i += NT) sidx[i] = i < kk ? (uint32_t)out_idx[i] : 0xFFFFFFFFu;
      __syncthreads();
      for (int len = 2; len <= np; len <<= 1) {
        for (int st = len >> 1; st > 0; st >>= 1) {
          for (int i = tid; i < np; i += NT) {
            const int j = i ^ st;
            if (j > i) {
              const uint32_t a = sidx[i], b = sidx[j];
              if ((a > b) == ((i & len) == 0)) {
                sidx[i] = b;
                sidx[j] = a;
              }
            }
          }
          __syncthreads();
        }
      }
      for (int i = tid; i < kk; i += NT) {
        out_idx[i] = (int)sidx[i];
        if (out_val) out_val[i] = grow[sidx[i]];
      }
    }
    return;
  }

  // ---- exact path for a crowded threshold bin: one cluster-wide pass per
  // remaining digit over the slice (from L2), then an ordered emission, which
  // also writes ascending positions.
  uint32_t prefix = b0;
  int lvl_shift = kShift0;
  uint32_t gt_local, eq_local;
  {
    uint32_t a = 0;
    for (int b = tid; b < kHistBins; b += NT) a += (b > (int)b0) ? hist[b] : 0u;
    gt_local = block_sum<NT>(a, wtot);
    eq_local = hist[b0];
  }
  for (int pass = 0; pass < K::kNumLater; ++pass) {
    const int sh = K::later_shift(pass);
    const int wd = K::later_width(pass);
    const int nb = 1 << wd;
    const int psh = lvl_shift;
    __syncthreads();
    for (int i = tid; i < kHistBins; i += NT) hist[i] = 0u;
    if (crank == 0)
      for (int i = tid; i < kHistBins; i += NT) hred[i] = 0u;
    cluster_sync();  // the leader's reduction histogram is cleared before any push
    auto add = [&](uint32_t raw) {
      const uint32_t kv = K::key(raw);
      if ((kv >> psh) == prefix) atomicAdd(hist + ((kv >> sh) & (uint32_t)(nb - 1)), 1u);
    };
    stream_slice<K, NT, 4>(
        grow, i0, m,
        [&](int, const uint4& v) {
#pragma unroll
          for (int j = 0; j < K::kVec; ++j) add(K::slot(v, j));
        },
        [&](int, uint32_t raw) { add(raw); });
    __syncthreads();
    for (int b = tid; b < nb; b += NT) {
      const uint32_t c = hist[b];
      if (c) dsmem_red_add_u32(leader_hred + 4u * b, c);
    }
    cluster_sync();
    if (crank == 0) {
      uint32_t above, inbin;
      const uint32_t b = block_find_bin<NT>(hred, nb, krem, wtot, ctrl->bcast, above, inbin);
      leader_publish(ctrl, csize, b, (uint32_t)(krem - (int)above), inbin);
    }
    cluster_sync();
    const uint32_t bs = min(ctrl->res[0], (uint32_t)(nb - 1));
    krem = (int)ctrl->res[1];
    const uint32_t bc = ctrl->res[2];
    uint32_t a = 0;
    for (int b = tid; b < nb; b += NT) a += (b > (int)bs) ? hist[b] : 0u;
    gt_local += block_sum<NT>(a, wtot);
    eq_local = hist[bs];
    prefix = (prefix << wd) | bs;
    lvl_shift = sh;
    if (bc == (uint32_t)krem) break;  // uniform
  }
  // exchange (gt, eq): every CTA stores its pair into every CTA's arrays
  if (tid < (int)csize) {
    dsmem_st_u32(dsmem_map(smem_u32(cnt_gt + crank), tid), gt_local);
    dsmem_st_u32(dsmem_map(smem_u32(cnt_eq + crank), tid), eq_local);
  }
  cluster_sync();
  if (tid == 0) {
    uint32_t base = 0, eq_before = 0;
    for (uint32_t r = 0; r < crank; ++r) {
      const uint32_t g = cnt_gt[r], e = cnt_eq[r];
      const int tk = max(0, min((int)e, krem - (int)eq_before));
      base += g + (uint32_t)tk;
      eq_before += e;
    }
    ctrl->base = base;
    ctrl->take = (uint32_t)max(0, min((int)eq_local, krem - (int)eq_before));
  }
  __syncthreads();
  const uint32_t base = ctrl->base, take = ctrl->take;
  const uint32_t mine = gt_local + take;
  if (mine > 0) {
    uint32_t gt_run = 0, tie_run = 0;
    for (int c0 = 0; c0 < m; c0 += NT) {
      const int e = i0 + c0 + tid;
      const bool in = c0 + tid < m;
      uint32_t raw = 0, top = 0;
      if (in) {
        raw = (uint32_t)grow[e];
        top = K::key(raw) >> lvl_shift;
      }
      const bool isg = in && top > prefix;
      const bool ise = in && top == prefix;
      uint32_t total;
      const uint32_t excl = block_excl_scan<NT>((uint32_t)isg | ((uint32_t)ise << 16), wtot, total);
      const uint32_t gb = gt_run + (excl & 0xFFFFu);
      const uint32_t tb = tie_run + (excl >> 16);
      if (isg || (ise && tb < take)) {
        const uint32_t pos = base + gb + min(tb, take);
        if (pos < (uint32_t)kk) {
          out_idx[pos] = e;
          if (out_val) out_val[pos] = (Raw)raw;
        }
      }
      gt_run += total & 0xFFFFu;
      tie_run += total >> 16;
      if (gt_run + min(tie_run, take) >= mine) break;  // uniform
    }
  }
}

}  // namespace dstopk
