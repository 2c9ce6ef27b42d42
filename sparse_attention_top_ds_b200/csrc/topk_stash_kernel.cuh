// topk_stash_kernel.cuh -- row-wise top-k in one pass over the scores.
//
// What it computes: for each row, the k largest of the first L = valid_len
// scores, ties to the lower position (DeepSelect hub page, use-case
// paragraphs: top-k of a bfloat16 indexer score row, and of a float32 logit
// row over a ~129K vocabulary; options sorted_index and return_value).
//
// How (B200 design, not the pages' design):
//  * A row is handled by one CTA, or by a cluster of C = 2 or 4 CTAs that
//    split it into contiguous slices when there are few rows.  Each CTA draws
//    a strided sample of its slice and takes from it a key threshold t that,
//    with a wide statistical margin, leaves at least min(k, slice) keys of the
//    slice at or above it and not many more.  It then streams the slice once
//    from HBM through a cp.async ring in shared memory and stashes every score
//    whose key is >= t, with its position.
//  * The k largest of a slice always contain that slice's share of the row's
//    k largest, so a CTA only checks its own count: the stash must hold at
//    least min(k, slice) keys and fit.  In a cluster every CTA then copies its
//    stash into the leader CTA (distributed shared memory): a pair's partner
//    into a receive area of the leader's own as soon as it has streamed,
//    behind one cluster barrier; four CTAs into the leader's ring, behind two.
//  * The row's k-th key is at or above tmax, the largest of the CTAs'
//    thresholds.  The leader counts the merged stash's keys >= tmax in 4096
//    bins of their offset above tmax (2^12 float32 keys, or single bfloat16
//    keys; the last bin takes everything above), finds the bin of the k-th
//    key, and resolves only that bin: when it holds at most 32 entries, the
//    emission visit lists them and one warp sorts them; otherwise a radix pass
//    over a list of the bin's keys (none for bfloat16), then positions for
//    ties.  When the k-th key lies in the last bin (or a CTA's stash was
//    redone, see below), the leader instead selects from the whole stash, one
//    radix pass per digit below the common prefix of its smallest and largest
//    key.  Every selected entry is written out with one warp-level atomic per
//    visit, and sorted_index sorts the selection by position first.
//  * A CTA whose stash came out short or too long (an unlucky sample, many
//    equal keys) re-reads its slice from L2 and finds its exact k-th (key,
//    position) with radix passes over the slice, then stashes exactly that
//    many.
//  * Rows whose scorer counted them (float32 rows of ds_indexer_topk with an
//    exact histogram of their keys' top 12 bits) skip the sample: the
//    threshold is the lower edge of the bin that holds the row's k-th key, so
//    the union of the stashes is complete by construction and only the
//    stash's capacity is checked.
#pragma once

#include "ptx.cuh"
#include "topk_kernel.cuh"

namespace dstopk {

constexpr int kTsThreads = 1024;
constexpr int kTsStages = 3;            // cp.async ring stages
constexpr int kTsStageWords = 3072;     // 16-byte words per stage: a 144 KiB ring
constexpr int kTsSample = 4096;         // sampled scores per CTA
constexpr int kTsPosBits = 24;          // positions are below 2^24
constexpr int kTsCap = 4096;            // stash entries per CTA (k <= 2048)
constexpr int kTsMaxCluster = 4;

// Phase stamps of the DS_DEBUG build: thread 0 of CTA b records %globaltimer
// at the end of each phase in ts_stamps[b][i] (read out by
// ds_debug_stash_stamps); the release build compiles them away.
constexpr int kTsStampCtas = 1024, kTsStampSlots = 10;
#ifdef DS_DEBUG
__device__ unsigned long long ts_stamps[kTsStampCtas][kTsStampSlots];
#define TS_STAMP(i)                                                                     \
  do {                                                                                  \
    if (threadIdx.x == 0 && blockIdx.x < (unsigned)kTsStampCtas) ts_stamps[blockIdx.x][i] = globaltimer_ns(); \
  } while (0)
#else
#define TS_STAMP(i) \
  do {              \
  } while (0)
#endif

struct TsParams {
  const void* scores;
  uint32_t* ghist;   // float32 rows: [batch, 4096] exact key histograms, or null (cleared here after use)
  const int32_t* valid_len;
  int32_t* out_idx;
  void* out_val;
  int batch, n, k;
  int slice;         // elements per CTA, a multiple of 8
  int return_value;
  int sorted;
  int* status;       // device status word (DS_DEBUG range checks)
};

struct TsCtrl {
  uint32_t cnt;             // this CTA: keys stashed (may run past the cap)
  uint32_t out;             // leader: selected entries written
  uint32_t bcast[4];
  uint32_t ok[16];          // every CTA: each CTA's verdict
  uint32_t tab[16];         // leader: each CTA's stash count
  uint32_t wtot[32];        // scan scratch: warp totals
  uint32_t wex[33];         // scan scratch: their exclusive prefixes, then the total
  uint32_t part[32][kTsMaxCluster];  // per-warp partial counts
  uint32_t above_of[kTsMaxCluster];
  uint32_t tval[16];        // every CTA: each CTA's stash threshold
  uint32_t cutk, cutp;      // leader: the cut inside the k-th key's bin
};

// Shared memory, in order: histogram u32[4096] (the stash's offsets above the
// threshold during the stream, then the radix passes' histogram, then the
// sorted selection: positions u32[2048], raw scores u32[2048]) | control | this CTA's
// stash (raw u32[cap], position u32[cap]) | cp.async ring of kTsStages stages.
// The last ring stage holds the sample's histogram until the ring reaches it.
// In a cluster the leader receives the stash of CTA c >= 1 in its ring (free
// by then) at (c - 1) stash sizes.
__host__ __device__ constexpr int ts_off_ctrl(int) { return 4096 * 4; }
__host__ __device__ constexpr int ts_off_stash(int C) { return ts_off_ctrl(C) + 1024; }
__host__ __device__ constexpr int ts_off_ring(int C) { return ts_off_stash(C) + kTsCap * 8; }
__host__ __device__ constexpr int ts_ring_bytes() { return kTsStages * kTsStageWords * 16; }
// A pair (C = 2) receives the partner's stash in an area of its own after the
// ring, so the partner can send it as soon as it has streamed.
__host__ __device__ constexpr int ts_smem_bytes(int C) {
  return ts_off_ring(C) + ts_ring_bytes() + (C == 2 ? kTsCap * 8 : 0);
}
static_assert(sizeof(TsCtrl) <= 1024, "control block");
static_assert(ts_off_ctrl(1) % 16 == 0 && ts_off_stash(1) % 16 == 0 && ts_off_ring(1) % 16 == 0,
              "the control block, the stash and the ring start on 16-byte boundaries");
static_assert(ts_smem_bytes(kTsMaxCluster) <= 227 * 1024 && ts_smem_bytes(2) <= 227 * 1024, "shared memory");
static_assert((kTsMaxCluster - 1) * kTsCap * 8 <= ts_ring_bytes(), "received stashes fit the ring");

// Exclusive block-wide scan of one value per thread (every thread calls it):
// a shuffle scan in each warp, then warp 0 scans the warp totals.
template <int NT>
__device__ __forceinline__ uint32_t ts_block_scan(uint32_t v, TsCtrl* ctrl, uint32_t& total) {
  static_assert(NT % 32 == 0 && NT / 32 <= 32, "one warp scans the warp totals");
  constexpr int NW = NT / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t t = __shfl_up_sync(0xFFFFFFFFu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) ctrl->wtot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const uint32_t x = lane < NW ? ctrl->wtot[lane] : 0u;
    uint32_t y = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t t = __shfl_up_sync(0xFFFFFFFFu, y, o);
      if (lane >= o) y += t;
    }
    if (lane < NW) ctrl->wex[lane] = y - x;
    if (lane == 31) ctrl->wex[32] = y;
  }
  __syncthreads();
  total = ctrl->wex[32];
  return ctrl->wex[warp] + incl - v;
}

// In a histogram of nb bins find b with #(bins > b) < krem <= #(bins >= b);
// `above` / `inbin` return the counts above and inside it.  Every thread calls
// it and gets the result; a __syncthreads() must separate two calls.  Each
// thread owns ceil(nb / NT) consecutive bins counted from the top.
template <int NT>
__device__ __forceinline__ uint32_t ts_find_bin(const uint32_t* h, int nb, uint32_t krem, TsCtrl* ctrl,
                                                uint32_t& above, uint32_t& inbin) {
  const int bpt = (nb + NT - 1) / NT;
  const int r0 = (int)threadIdx.x * bpt;  // first rank (0 = the top bin)
  const int r1 = min(nb, r0 + bpt);
  uint32_t s = 0u;
  if ((bpt & 3) == 0 && r1 - r0 == bpt) {
    // bins nb-r1 .. nb-1-r0 are 16-byte aligned groups of four
    for (int r = r0; r < r1; r += 4) {
      const uint4 v = *reinterpret_cast<const uint4*>(h + nb - 4 - r);
      s += v.x + v.y + v.z + v.w;
    }
  } else {
    for (int r = r0; r < r1; ++r) s += h[nb - 1 - r];
  }
  // two barriers: the warp totals out; every warp scans all of them itself
  static_assert(NT % 32 == 0 && NT / 32 <= 32, "one warp's lanes cover the warp totals");
  constexpr int NW = NT / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t incl = s;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t t = __shfl_up_sync(0xFFFFFFFFu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) ctrl->wtot[warp] = incl;
  __syncthreads();
  const uint32_t wt = lane < NW ? ctrl->wtot[lane] : 0u;
  uint32_t wi = wt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t t = __shfl_up_sync(0xFFFFFFFFu, wi, o);
    if (lane >= o) wi += t;
  }
  const uint32_t wex = __shfl_sync(0xFFFFFFFFu, wi - wt, warp);
  const uint32_t total = __shfl_sync(0xFFFFFFFFu, wi, 31);
  const uint32_t excl = wex + incl - s;
  if (threadIdx.x == 0 && (krem == 0u || krem > total)) {  // no such bin
    ctrl->bcast[0] = 0u;
    ctrl->bcast[1] = 0u;
    ctrl->bcast[2] = 0u;
  }
  if (excl < krem && krem <= excl + s) {
    uint32_t acc = excl;
    for (int r = r0; r < r1; ++r) {
      const uint32_t c = h[nb - 1 - r];
      if (acc + c >= krem) {
        ctrl->bcast[0] = (uint32_t)(nb - 1 - r);
        ctrl->bcast[1] = acc;
        ctrl->bcast[2] = c;
        break;
      }
      acc += c;
    }
  }
  __syncthreads();
  above = ctrl->bcast[1];
  inbin = ctrl->bcast[2];
  return min(ctrl->bcast[0], (uint32_t)(nb - 1));
}

// Where an exact selection of the kth largest (key, then lower position)
// cuts: an element is taken when the top bits of its key (key >> kshift)
// exceed kprefix, or equal it and its position is <= pcut.
struct TsCut {
  uint32_t kprefix;
  int kshift;
  uint32_t pcut;
};

__device__ __forceinline__ uint32_t ts_top(uint32_t key, int shift) { return shift >= 32 ? 0u : key >> shift; }

__device__ __forceinline__ bool ts_taken(const TsCut& c, uint32_t key, uint32_t pos) {
  const uint32_t top = ts_top(key, c.kshift);
  return top > c.kprefix || (top == c.kprefix && pos <= c.pcut);
}

// Exact radix select of the kth largest (key, lower position) among the
// elements that visit(f) hands to f(key, position) (at least kth of them,
// kth >= 1; positions below 2^24 and distinct).  Every visited key has top
// bits ts_top(key, shift0) == prefix0 (shift0 = K::kBits: nothing known), so
// the passes take 12-bit key digits from bit shift0 down; only if ties at the
// kth key remain, two 12-bit passes on the complemented positions of the tied
// elements.  Every thread of the block calls it.
template <class K, int NT, class Visit>
__device__ __forceinline__ TsCut ts_select(Visit&& visit, int kth, uint32_t* hist, TsCtrl* ctrl,
                                           uint32_t prefix0 = 0u, int shift0 = K::kBits) {
  uint32_t prefix = prefix0;
  int shift = shift0;
  int krem = kth;
  while (shift > 0) {
    const int wd = shift < 12 ? shift : 12;
    const int sh = shift - wd;
    const uint32_t mask = (1u << wd) - 1u;
    for (int i = threadIdx.x; i <= (int)mask; i += NT) hist[i] = 0u;
    __syncthreads();
    const uint32_t pf = prefix;
    const int sf = shift;
    visit([&](uint32_t key, uint32_t) {
      if (ts_top(key, sf) == pf) atomicAdd(hist + ((key >> sh) & mask), 1u);
    });
    __syncthreads();
    uint32_t above, inbin;
    const uint32_t b = ts_find_bin<NT>(hist, (int)mask + 1, (uint32_t)krem, ctrl, above, inbin);
    krem -= (int)above;
    prefix = (prefix << wd) | b;
    shift = sh;
    if (inbin == (uint32_t)krem) return TsCut{prefix, shift, 0xFFFFFFFFu};  // the whole bin is taken
  }
  // prefix is the kth key; krem of its ties are taken, the lowest positions first
  const uint32_t tkey = prefix;
  uint32_t pp = 0;
  int ps = kTsPosBits;
  for (int pass = 0; pass < 2; ++pass) {
    const int sh = ps - 12;
    for (int i = threadIdx.x; i < 4096; i += NT) hist[i] = 0u;
    __syncthreads();
    const uint32_t pf = pp;
    const int sf = ps;
    visit([&](uint32_t key, uint32_t pos) {
      const uint32_t cp = ((1u << kTsPosBits) - 1u) - pos;
      if (key == tkey && (cp >> sf) == pf) atomicAdd(hist + ((cp >> sh) & 4095u), 1u);
    });
    __syncthreads();
    uint32_t above, inbin;
    const uint32_t b = ts_find_bin<NT>(hist, 4096, (uint32_t)krem, ctrl, above, inbin);
    krem -= (int)above;
    pp = (pp << 12) | b;
    ps = sh;
    if (inbin == (uint32_t)krem) break;
  }
  // taken ties: complemented position >= pp << ps
  return TsCut{tkey, 0, ((1u << kTsPosBits) - 1u) - (pp << ps)};
}

// Block-wide minimum and maximum of one value per thread (every thread calls
// it and gets both).
template <int NT>
__device__ __forceinline__ void ts_block_minmax(uint32_t lo, uint32_t hi, TsCtrl* ctrl, uint32_t& gmin,
                                                uint32_t& gmax) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    lo = min(lo, __shfl_xor_sync(0xFFFFFFFFu, lo, o));
    hi = max(hi, __shfl_xor_sync(0xFFFFFFFFu, hi, o));
  }
  if (lane == 0) {
    ctrl->wtot[warp] = lo;
    ctrl->wex[warp] = hi;
  }
  __syncthreads();
  if (warp == 0) {
    uint32_t a = lane < NT / 32 ? ctrl->wtot[lane] : 0xFFFFFFFFu;
    uint32_t b = lane < NT / 32 ? ctrl->wex[lane] : 0u;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      a = min(a, __shfl_xor_sync(0xFFFFFFFFu, a, o));
      b = max(b, __shfl_xor_sync(0xFFFFFFFFu, b, o));
    }
    if (lane == 0) {
      ctrl->bcast[0] = a;
      ctrl->bcast[1] = b;
    }
  }
  __syncthreads();
  gmin = ctrl->bcast[0];
  gmax = ctrl->bcast[1];
}

// Hands out n consecutive slots of *counter to each lane of a warp (all 32
// lanes call it); returns this lane's first slot.
__device__ __forceinline__ uint32_t ts_warp_alloc(uint32_t n, uint32_t* counter) {
  const int lane = threadIdx.x & 31;
  uint32_t incl = n;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t t = __shfl_up_sync(0xFFFFFFFFu, incl, o);
    if (lane >= o) incl += t;
  }
  const uint32_t total = __shfl_sync(0xFFFFFFFFu, incl, 31);
  uint32_t base = 0;
  if (total != 0u) {
    if (lane == 0) base = atomicAdd(counter, total);
    base = __shfl_sync(0xFFFFFFFFu, base, 0);
  }
  return base + incl - n;
}



// Block-wide sums of C <= kTsMaxCluster values per thread (every thread calls
// it); the sums land in out[0 .. C).
template <int NT>
__device__ __forceinline__ void ts_block_sums(const uint32_t (&v)[kTsMaxCluster], int C, TsCtrl* ctrl,
                                              uint32_t* out) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int c = 0; c < kTsMaxCluster; ++c) {
    uint32_t x = v[c];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xFFFFFFFFu, x, o);
    if (lane == 0) ctrl->part[warp][c] = x;
  }
  __syncthreads();
  if (warp == 0) {
#pragma unroll
    for (int c = 0; c < kTsMaxCluster; ++c) {
      uint32_t x = lane < NT / 32 ? ctrl->part[lane][c] : 0u;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xFFFFFFFFu, x, o);
      if (lane == 0 && c < C) out[c] = x;
    }
  }
  __syncthreads();
}

template <class K, int NT>
__global__ void __launch_bounds__(NT, 1) topk_stash_kernel(const TsParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  using Raw = typename K::Raw;
  constexpr int kShift0 = K::kBits - 12;
  constexpr int stage_words = kTsStageWords;
  constexpr int V = stage_words / NT;  // words per thread per stage
  static_assert(V * NT == stage_words && V * K::kVec <= 32, "ring stage: one hit bit per score in a word");

  const int tid = threadIdx.x;
  const uint32_t crank = cluster_ctarank();
  const uint32_t csize = cluster_nctarank();
  const int C = (int)csize;
  uint32_t* hist = reinterpret_cast<uint32_t*>(smem);  // radix histogram
  TsCtrl* ctrl = reinterpret_cast<TsCtrl*>(smem + ts_off_ctrl(C));
  uint32_t* st_raw = reinterpret_cast<uint32_t*>(smem + ts_off_stash(C));
  uint32_t* st_pos = st_raw + kTsCap;
  uint8_t* ring = smem + ts_off_ring(C);
  uint32_t* shist = reinterpret_cast<uint32_t*>(ring + (size_t)(kTsStages - 1) * stage_words * 16);

  TS_STAMP(0);  // start
  const int row = (int)(blockIdx.x / csize);
  // (arrive now, wait before the first access to another CTA's shared
  // memory: by then every CTA of the cluster is running)
  if (C > 1) cluster_arrive_relaxed();
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
  if (crank == 0) {
    for (int j = kk + tid; j < p.k; j += NT) {
      out_idx[j] = -1;
      if (out_val) out_val[j] = (Raw)K::kNegInf;
    }
  }
  if (kk == 0) return;  // uniform across the cluster

  const int i0 = (int)crank * p.slice;
  const int m = max(0, min(p.slice, L - i0));  // eligible scores of this slice
  const int need = min(kk, m);                 // the stash must hold at least this many
  const Raw* grow = reinterpret_cast<const Raw*>(p.scores) + (size_t)row * p.n;

  // the slice as full 16-byte words plus fewer than 2 * kVec loose elements
  const uintptr_t rbase = reinterpret_cast<uintptr_t>(grow);
  const uintptr_t a0 = rbase + (uintptr_t)i0 * K::kBytes;
  const uintptr_t a1 = a0 + (uintptr_t)m * K::kBytes;
  const uintptr_t f0 = (a0 + 15u) & ~uintptr_t(15);
  const uintptr_t f1 = a1 & ~uintptr_t(15);
  const int nfull = (m > 0 && f1 > f0) ? (int)((f1 - f0) >> 4) : 0;
  const uint4* wp = reinterpret_cast<const uint4*>(f0);
  const int e_f0 = (int)((f0 - rbase) / K::kBytes);
  const int head = m <= 0 ? 0 : (nfull > 0 ? (int)((f0 - a0) / K::kBytes) : m);
  const int tail_start = nfull > 0 ? (int)((f1 - rbase) / K::kBytes) : i0 + m;
  const int tail = m <= 0 ? 0 : i0 + m - tail_start;
  int pe = -1;  // this thread's loose element, if any
  if (tid < head) pe = i0 + tid;
  else if (nfull > 0 && tid >= 32 && tid - 32 < tail) pe = tail_start + tid - 32;

  if (tid == 0) {
    ctrl->cnt = 0u;
    ctrl->out = 0u;
    ctrl->bcast[3] = 0u;
  }
  // the leader's histogram of the stash's offsets above the threshold
  // (zeroed before the first barrier below)
  constexpr int kRel = K::kBits == 32 ? 12 : 0;
  for (int i = tid; i < 4096; i += NT) hist[i] = 0u;

  TS_STAMP(1);  // prologue
  // ---- a strided sample of the full words (64 evenly spaced runs of run_w
  // words) when the slice does not fit the stash whole
  constexpr int SW = kTsSample / K::kVec;
  constexpr int SPT = (SW + NT - 1) / NT;
  constexpr int kRuns = 64;
  const bool counted = K::kBits == 32 && p.ghist != nullptr;  // the threshold comes from the row's histogram
  const bool sampled = !counted && m > kTsCap;
  const int run_w = sampled ? min(nfull, SW) / kRuns : 0;  // >= 7: a sampled slice has > 4096 scores
  const int sw = kRuns * run_w;                            // sampled words, <= nfull
  uint4 s[SPT];
#pragma unroll
  for (int j = 0; j < SPT; ++j) {
    const int idx = tid + j * NT;
    if (idx < sw) {
      const int ru = idx / run_w, o = idx - ru * run_w;
      s[j] = __ldg(wp + (int)(((long long)ru * (nfull - run_w)) / (kRuns - 1)) + o);
    }
  }
  uint32_t praw = 0;
  if (pe >= 0) praw = (uint32_t)grow[pe];

  // ---- the cp.async ring: a thread copies V words per stage and later
  // processes exactly those words, so the ring needs no block barrier.  (A
  // ring of bulk copies, one thread issuing each stage, streamed slower: a
  // copy-only read of these rows takes 8.4 us with 16-byte loads from every
  // thread and 9.7 us through a bulk-copy ring.)
  const int nst = (nfull + stage_words - 1) / stage_words;
  auto issue = [&](int st) {
    if (st < nst) {
      const int slot = st % kTsStages;
#pragma unroll
      for (int v = 0; v < V; ++v) {
        const int w = st * stage_words + v * NT + tid;
        if (w < nfull) {
          const uint32_t dst = smem_u32(ring + ((size_t)slot * stage_words + v * NT + tid) * 16);
          asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(wp + w) : "memory");
        }
      }
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };

  // ---- threshold: the sample's key of rank rk, which leaves an expected
  // need + 4 standard deviations + 8 keys of the slice above it.  For float32
  // keys the lower edge of its 12-bit bin is close enough (a second digit
  // pass costs more than the few extra keys stashed); for bfloat16 keys, with
  // only 4 bits below the first digit, the second digit keeps the stash small.
  uint32_t t = 0u;
  if (counted) {
    // the bin of the row's kk-th key from the scorer's counts
    const uint4* gh = reinterpret_cast<const uint4*>(p.ghist + (size_t)row * 4096);
    for (int i = tid; i < 1024; i += NT) reinterpret_cast<uint4*>(shist)[i] = __ldcg(gh + i);
    for (int st = 0; st < kTsStages - 1; ++st) issue(st);
    __syncthreads();
    uint32_t above, inbin;
    const uint32_t b0 = ts_find_bin<NT>(shist, 4096, (uint32_t)kk, ctrl, above, inbin);
    t = b0 << kShift0;
  } else if (sampled) {
    // the stream's first stages load while the sample is counted (the
    // histogram lives in the ring's last stage, loaded later)
    for (int st = 0; st < kTsStages - 1; ++st) issue(st);
    for (int i = tid; i < 4096; i += NT) shist[i] = 0u;
    __syncthreads();
#pragma unroll
    for (int j = 0; j < SPT; ++j) {
      if (tid + j * NT < sw) {
#pragma unroll
        for (int e = 0; e < K::kVec; ++e) atomicAdd(shist + (K::key(K::slot(s[j], e)) >> kShift0), 1u);
      }
    }
    __syncthreads();
    TS_STAMP(2);  // sample counted
    const int ns = sw * K::kVec;
    const float lam = (float)need * (float)ns / (float)m;
    const int rk = min(ns, (int)ceilf(lam + 4.0f * sqrtf(lam) + 8.0f));
    uint32_t above, inbin;
    const uint32_t b1 = ts_find_bin<NT>(shist, 4096, (uint32_t)rk, ctrl, above, inbin);
    if constexpr (K::kBits == 32) {
      t = b1 << kShift0;
    } else {
    constexpr int W2 = kShift0 >= 11 ? 11 : kShift0;
    constexpr int SH2 = kShift0 - W2;
    for (int i = tid; i < (1 << W2); i += NT) shist[i] = 0u;
    __syncthreads();
#pragma unroll
    for (int j = 0; j < SPT; ++j) {
      if (tid + j * NT < sw) {
#pragma unroll
        for (int e = 0; e < K::kVec; ++e) {
          const uint32_t kv = K::key(K::slot(s[j], e));
          if ((kv >> kShift0) == b1) atomicAdd(shist + ((kv >> SH2) & ((1u << W2) - 1u)), 1u);
        }
      }
    }
    __syncthreads();
    uint32_t a2, i2;
    const uint32_t b2 = ts_find_bin<NT>(shist, 1 << W2, (uint32_t)(rk - (int)above), ctrl, a2, i2);
    t = ((b1 << W2) | b2) << SH2;
    }
  } else {
    for (int st = 0; st < kTsStages - 1; ++st) issue(st);
    __syncthreads();  // the zeroed histogram and counters
  }

  // ---- one pass: every key >= t is stashed with its position; a warp takes
  // its stash slots with one atomic per stage.  The test is a float compare
  // against bound(t) (exact, or a superset that the stash's checks catch)
  // into a 32-bit hit mask; only the set bits are then visited.
  TS_STAMP(3);  // threshold
  const float tf = K::bound(t);
  for (int st = 0; st < nst; ++st) {
    issue(st + kTsStages - 1);
    asm volatile("cp.async.wait_group %0;" ::"n"(kTsStages - 1) : "memory");
    const int slot = st % kTsStages;
    uint4 x[V];
    uint32_t hits = 0u;  // one bit per score of this thread's words
#pragma unroll
    for (int v = 0; v < V; ++v) {
      const int w = st * stage_words + v * NT + tid;
      x[v] = make_uint4(0u, 0u, 0u, 0u);
      if (w < nfull) {
        x[v] = *reinterpret_cast<const uint4*>(ring + ((size_t)slot * stage_words + v * NT + tid) * 16);
#pragma unroll
        for (int j = 0; j < K::kVec; ++j) hits |= (uint32_t)K::ge(x[v], j, tf) << (v * K::kVec + j);
      }
    }
    uint32_t pos = ts_warp_alloc((uint32_t)__popc(hits), &ctrl->cnt);
    // only the hits are visited (a warp runs as many rounds as its busiest lane)
    while (hits) {
      const int j = __ffs(hits) - 1;
      hits &= hits - 1u;
      const int v = j / K::kVec, e = j % K::kVec;
      // the hit's 32-bit word (4 per 16-byte word), then its half for bfloat16
      constexpr int kPerWord = K::kVec / 4;
      const int wj = j / kPerWord;
      uint32_t word = 0u;
#pragma unroll
      for (int q = 0; q < V * 4; ++q) {
        const uint4& xv = x[q / 4];
        const uint32_t c = (q & 3) == 0 ? xv.x : ((q & 3) == 1 ? xv.y : ((q & 3) == 2 ? xv.z : xv.w));
        word = q == wj ? c : word;
      }
      const uint32_t raw = kPerWord == 1 ? word : ((j & 1) ? (word >> 16) : (word & 0xFFFFu));
      if (pos < (uint32_t)kTsCap) {
        st_raw[pos] = raw;
        st_pos[pos] = (uint32_t)(e_f0 + (st * stage_words + v * NT + tid) * K::kVec + e);
      }
      ++pos;
    }
  }
  asm volatile("cp.async.wait_group 0;" ::: "memory");
  if (pe >= 0) {
    const uint32_t key = K::key(praw);
    if (key >= t) {
      const uint32_t slot = atomicAdd(&ctrl->cnt, 1u);
      if (slot < (uint32_t)kTsCap) {
        st_raw[slot] = praw;
        st_pos[slot] = (uint32_t)pe;
      }
    }
  }
  __syncthreads();

  TS_STAMP(4);  // streamed
  // ---- in a cluster, every stash goes to the leader: a pair's partner into
  // the leader's receive area, as soon as it has streamed; with four CTAs,
  // stash c into the leader's ring (free once every CTA has streamed) at
  // (c - 1) stash sizes
  uint32_t* recv = reinterpret_cast<uint32_t*>(ring + ts_ring_bytes());
  auto region = [&](int c) -> uint32_t* {
    if (c == 0) return st_raw;
    return C == 2 ? recv : reinterpret_cast<uint32_t*>(ring + (size_t)(c - 1) * kTsCap * 8);
  };
  auto ship = [&](uint32_t n) {
    const uint32_t nv = (n + 3u) >> 2;
    const uint32_t dst = dsmem_map(smem_u32(region((int)crank)), 0);
    for (uint32_t v = tid; v < 2u * nv; v += NT) {
      const bool israw = v < nv;
      const uint32_t o = 16u * (israw ? v : v - nv);
      const uint4 x = *reinterpret_cast<const uint4*>(reinterpret_cast<const uint8_t*>(israw ? st_raw : st_pos) + o);
      asm volatile("st.shared::cluster.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(dst + (israw ? 0u : 4u * kTsCap) + o),
                   "r"(x.x), "r"(x.y), "r"(x.z), "r"(x.w)
                   : "memory");
    }
    if (tid == 0) dsmem_st_u32(dsmem_map(smem_u32(&ctrl->tab[crank]), 0), n);
  };

  uint32_t cnt = ctrl->cnt;
  const bool ok = (counted || cnt >= (uint32_t)need) && cnt <= (uint32_t)kTsCap;
  bool all_ok = ok;
  // tmax, the largest of the CTAs' thresholds: with every stash complete, the
  // row's k-th key is >= the threshold of each slice that holds k keys (and
  // slices that hold fewer have t = 0), so every key at or above the k-th is
  // >= tmax and in a stash
  uint32_t tmax = t;
  if (C > 1) {
    cluster_wait();  // (the arrival at the start) every CTA of the cluster is running
    if (C == 2) {
      // one cluster barrier: the partner's stash, thresholds and verdicts in
      // (writing the stash remotely during the stream instead slowed the
      // stream more than it saved here)
      if (ok && crank != 0) ship(cnt);
      if (tid < C) {
        dsmem_st_u32(dsmem_map(smem_u32(&ctrl->tval[crank]), (uint32_t)tid), t);
        dsmem_st_u32(dsmem_map(smem_u32(&ctrl->ok[crank]), (uint32_t)tid), ok ? 1u : 0u);
      }
      cluster_sync();
    } else {
      if (tid < C) dsmem_st_u32(dsmem_map(smem_u32(&ctrl->tval[crank]), (uint32_t)tid), t);
      cluster_sync();  // every CTA has streamed: the leader's ring is free
      if (ok && crank != 0) ship(cnt);
      if (tid < C) dsmem_st_u32(dsmem_map(smem_u32(&ctrl->ok[crank]), (uint32_t)tid), ok ? 1u : 0u);
      cluster_sync();
    }
    for (int c = 0; c < C; ++c) {
      all_ok &= ctrl->ok[c] != 0u;
      tmax = max(tmax, ctrl->tval[c]);
    }
  }
  if (tid == 0 && crank == 0) ctrl->tab[0] = cnt;
  // every CTA of the row has read the row's counts: the leader clears them
  // for the next call
  if (counted && crank == 0) {
    uint4* gh = reinterpret_cast<uint4*>(p.ghist + (size_t)row * 4096);
    for (int i = tid; i < 1024; i += NT) gh[i] = make_uint4(0u, 0u, 0u, 0u);
  }

  if (!all_ok) {
    // ---- exact fallback (uniform decision; only CTAs with a bad stash work):
    // radix passes over the slice (re-read from L2) find its need-th largest
    // (key, lower position); then exactly its need largest are stashed
    if (!ok) {
      auto visit_slice = [&](auto&& f) {
        stream_slice<K, NT, 4>(
            grow, i0, m,
            [&](int e0, const uint4& v) {
#pragma unroll
              for (int j = 0; j < K::kVec; ++j) f(K::key(K::slot(v, j)), (uint32_t)(e0 + j));
            },
            [&](int e, uint32_t raw) { f(K::key(raw), (uint32_t)e); });
      };
      const TsCut cut = ts_select<K, NT>(visit_slice, need, hist, ctrl);
      if (tid == 0) ctrl->cnt = 0u;
      __syncthreads();
      auto take = [&](uint32_t raw, int e) {
        const uint32_t key = K::key(raw);
        if (ts_taken(cut, key, (uint32_t)e)) {
          const uint32_t slot = atomicAdd(&ctrl->cnt, 1u);
          if (slot < (uint32_t)kTsCap) {
            st_raw[slot] = raw;
            st_pos[slot] = (uint32_t)e;
          }
        }
      };
      stream_slice<K, NT, 4>(
          grow, i0, m,
          [&](int e0, const uint4& v) {
#pragma unroll
            for (int j = 0; j < K::kVec; ++j) take(K::slot(v, j), e0 + j);
          },
          [&](int e, uint32_t raw) { take(raw, e); });
      __syncthreads();
      cnt = ctrl->cnt;  // == need
      if (crank != 0) ship(cnt);
      else if (tid == 0) ctrl->tab[0] = cnt;
    }
    if (C > 1) cluster_sync();
    else __syncthreads();
  }
  TS_STAMP(5);  // merged (every CTA)
  if (crank != 0) return;

  // ---- the leader: the kk largest of the (merged) stash
  __syncthreads();
  auto visit_stash = [&](auto&& f) {
    for (int c = 0; c < C; ++c) {
      const int nc = min((int)ctrl->tab[c], kTsCap);
      const uint32_t* rr = region(c);
      const uint32_t* rp = rr + kTsCap;
      int i = tid;
      for (; i + NT < nc; i += 2 * NT) {
        const uint32_t a0 = rr[i], a1 = rr[i + NT], q0 = rp[i], q1 = rp[i + NT];
        f(K::key(a0), q0);
        f(K::key(a1), q1);
      }
      if (i < nc) f(K::key(rr[i]), rp[i]);
    }
  };
  // The stash's keys >= tmax, counted in 4096 bins of their offset above
  // tmax (2^12 float32 keys or one bfloat16 key per bin, the last bin taking
  // everything above), place the k-th key: only its bin fb is resolved
  // (mode 1: all of the bin is taken; mode 2: a cut inside it, from a warp
  // sort of the bin's entries when they are few).
  int mode = 0;
  uint32_t fb = 0u, above_f = 0u;
  int krem_f = 0;
  TsCut cut = TsCut{0u, 0, 0u};
  if (all_ok) {
    visit_stash([&](uint32_t key, uint32_t) {
      if (key >= tmax) atomicAdd(hist + min(4095u, (key - tmax) >> kRel), 1u);
    });
    __syncthreads();
    TS_STAMP(6);  // leader: stash counted
    uint32_t above, inbin;
    const uint32_t b = ts_find_bin<NT>(hist, 4096, (uint32_t)kk, ctrl, above, inbin);
    TS_STAMP(7);  // leader: bin of the k-th key
    if (b < 4095u && above < (uint32_t)kk && above + inbin >= (uint32_t)kk) {
      fb = b;
      const int krem = kk - (int)above;
      above_f = above;
      krem_f = krem;
      if (inbin == (uint32_t)krem) {
        mode = 1;
      } else if (inbin <= 32u) {
        mode = 3;  // resolved during the emission (below)
      } else {
        mode = 2;
        // the bin's entries, listed in the ring's last stage (clear of the
        // received stashes): inbin of them
        constexpr int kListCap = 2048;
        uint32_t* lk = shist;
        uint32_t* lp = shist + kListCap;
        visit_stash([&](uint32_t key, uint32_t pos) {
          if (key >= tmax && min(4095u, (key - tmax) >> kRel) == b) {
            const uint32_t s = atomicAdd(&ctrl->bcast[3], 1u);
            if (s < (uint32_t)kListCap) {
              lk[s] = key;
              lp[s] = pos;
            }
          }
        });
        __syncthreads();
        if (inbin <= 32u) {
          if (tid < 32) {
            // bitonic sort of the (at most 32) entries, greatest first: larger
            // key, then lower position; lane krem - 1 holds the cut
            uint32_t key = tid < (int)inbin ? lk[tid] : 0u;
            uint32_t pos = tid < (int)inbin ? lp[tid] : 0xFFFFFFFFu;
#pragma unroll
            for (int w = 2; w <= 32; w <<= 1) {
#pragma unroll
              for (int j = w >> 1; j > 0; j >>= 1) {
                const uint32_t ok2 = __shfl_xor_sync(0xFFFFFFFFu, key, j);
                const uint32_t op2 = __shfl_xor_sync(0xFFFFFFFFu, pos, j);
                const bool other_greater = ok2 > key || (ok2 == key && op2 < pos);
                const bool keep_greater = ((tid & j) == 0) == ((tid & w) == 0);
                if (other_greater == keep_greater) {
                  key = ok2;
                  pos = op2;
                }
              }
            }
            if (tid == krem - 1) {
              ctrl->cutk = key;
              ctrl->cutp = pos;
            }
          }
          __syncthreads();
          cut = TsCut{ctrl->cutk, 0, ctrl->cutp};
        } else if (inbin <= (uint32_t)kListCap) {
          const int nl = (int)inbin;
          auto visit_list = [&](auto&& f) {
            for (int i = tid; i < nl; i += NT) f(lk[i], lp[i]);
          };
          cut = ts_select<K, NT>(visit_list, krem, hist, ctrl, (tmax >> kRel) + b, kRel);
        } else {
          cut = ts_select<K, NT>(visit_stash, krem, hist, ctrl, (tmax >> kRel) + b, kRel);
        }
      }
    }
  }
  TS_STAMP(8);  // leader: the bin resolved (mode 1 or 2)
  if (mode == 0) {
    // the stash's keys share their top bits between its smallest and largest
    // key: the radix digits start below that common prefix, so the first pass
    // spreads the stash over many bins
    __syncthreads();
    uint32_t lo = 0xFFFFFFFFu, hi = 0u;
    visit_stash([&](uint32_t key, uint32_t) {
      lo = min(lo, key);
      hi = max(hi, key);
    });
    uint32_t gmin, gmax;
    ts_block_minmax<NT>(lo, hi, ctrl, gmin, gmax);
    const int common = gmin == gmax ? K::kBits : __clz(gmin ^ gmax) - (32 - K::kBits);
    const int shift0 = K::kBits - common;
    cut = ts_select<K, NT>(visit_stash, kk, hist, ctrl, ts_top(gmax, shift0), shift0);
  }
  auto taken = [&](uint32_t key, uint32_t pos) -> bool {
    if (mode == 0) return ts_taken(cut, key, pos);
    if (key < tmax) return false;
    const uint32_t rel = min(4095u, (key - tmax) >> kRel);
    return rel > fb || (rel == fb && (mode == 1 || ts_taken(cut, key, pos)));
  };
  // every selected entry (exactly kk): one warp-level slot allocation per
  // visit (a ballot and one atomic); with sorted_index gathered in shared
  // memory first.  (Slots from a counting visit and a prefix over the warps,
  // without atomics, came out slower: the visit costs more than the atomics.)
  uint32_t* sel_pos = hist;
  uint32_t* sel_raw = hist + 2048;
  const bool sorted = p.sorted != 0;
  const int lane = tid & 31;
  const uint32_t lt = (1u << lane) - 1u;
  auto emit = [&](uint32_t slot, uint32_t pos, uint32_t raw) {
    if (sorted) {
      sel_pos[slot] = pos;
      sel_raw[slot] = raw;
    } else {
      out_idx[slot] = (int32_t)pos;
      if (out_val) out_val[slot] = (Raw)raw;
    }
  };
  if (mode == 3) {
    // One visit: the keys above the bin go out (slots 0 .. above - 1) and the
    // bin's entries (at most 32) are listed; then one warp sorts them
    // (bitonic, larger key then lower position first) and writes the first
    // krem of them at slots above .. kk - 1.
    uint32_t* lk = shist;
    uint32_t* lp = shist + 32;
    uint32_t* lr = shist + 64;
    for (int c = 0; c < C; ++c) {
      const int nc = min((int)ctrl->tab[c], kTsCap);
      const uint32_t* rr = region(c);
      const uint32_t* rp = rr + kTsCap;
      for (int base = 0; base < nc; base += NT) {
        const int i = base + tid;
        uint32_t raw = 0u, pos = 0u, key = 0u;
        bool up = false, inb = false;
        if (i < nc) {
          raw = rr[i];
          pos = rp[i];
          key = K::key(raw);
          if (key >= tmax) {
            const uint32_t rel = min(4095u, (key - tmax) >> kRel);
            up = rel > fb;
            inb = rel == fb;
          }
        }
        const uint32_t m = __ballot_sync(0xFFFFFFFFu, up);
        uint32_t wb = 0u;
        if (m != 0u) {
          if (lane == 0) wb = atomicAdd(&ctrl->out, (uint32_t)__popc(m));
          wb = __shfl_sync(0xFFFFFFFFu, wb, 0);
        }
        const uint32_t slot = wb + (uint32_t)__popc(m & lt);
        if (up && slot < above_f) emit(slot, pos, raw);
        if (inb) {
          const uint32_t s = atomicAdd(&ctrl->bcast[3], 1u);
          if (s < 32u) {
            lk[s] = key;
            lp[s] = pos;
            lr[s] = raw;
          }
        }
      }
    }
    __syncthreads();
    if (tid < 32) {
      const int n = (int)min(ctrl->bcast[3], 32u);
      uint32_t key = tid < n ? lk[tid] : 0u;
      uint32_t pos = tid < n ? lp[tid] : 0xFFFFFFFFu;
      uint32_t raw = tid < n ? lr[tid] : 0u;
#pragma unroll
      for (int w = 2; w <= 32; w <<= 1) {
#pragma unroll
        for (int j = w >> 1; j > 0; j >>= 1) {
          const uint32_t ok2 = __shfl_xor_sync(0xFFFFFFFFu, key, j);
          const uint32_t op2 = __shfl_xor_sync(0xFFFFFFFFu, pos, j);
          const uint32_t or2 = __shfl_xor_sync(0xFFFFFFFFu, raw, j);
          const bool other_greater = ok2 > key || (ok2 == key && op2 < pos);
          const bool keep_greater = ((tid & j) == 0) == ((tid & w) == 0);
          if (other_greater == keep_greater) {
            key = ok2;
            pos = op2;
            raw = or2;
          }
        }
      }
      if (tid < krem_f) emit(above_f + (uint32_t)tid, pos, raw);
    }
  } else {
  for (int c = 0; c < C; ++c) {
    const int nc = min((int)ctrl->tab[c], kTsCap);
    const uint32_t* rr = region(c);
    const uint32_t* rp = rr + kTsCap;
    for (int base = 0; base < nc; base += NT) {
      const int i = base + tid;
      uint32_t raw = 0u, pos = 0u;
      bool take = false;
      if (i < nc) {
        raw = rr[i];
        pos = rp[i];
        take = taken(K::key(raw), pos);
      }
      const uint32_t m = __ballot_sync(0xFFFFFFFFu, take);
      uint32_t wb = 0u;
      if (m != 0u) {
        if (lane == 0) wb = atomicAdd(&ctrl->out, (uint32_t)__popc(m));
        wb = __shfl_sync(0xFFFFFFFFu, wb, 0);
      }
      const uint32_t slot = wb + (uint32_t)__popc(m & lt);
      if (take && slot < (uint32_t)kk) emit(slot, pos, raw);
    }
  }
  }
  TS_STAMP(9);  // leader: thread 0's part of the emission written
  if (!sorted) return;
  __syncthreads();
  // ascending positions: bitonic sort of (position, score) pairs
  int np = 1;
  while (np < kk) np <<= 1;
  for (int i = kk + tid; i < np; i += NT) sel_pos[i] = 0xFFFFFFFFu;
  __syncthreads();
  for (int len = 2; len <= np; len <<= 1) {
    for (int st = len >> 1; st > 0; st >>= 1) {
      for (int i = tid; i < np; i += NT) {
        const int j = i ^ st;
        if (j > i) {
          const uint32_t a = sel_pos[i], b = sel_pos[j];
          if ((a > b) == ((i & len) == 0)) {
            sel_pos[i] = b;
            sel_pos[j] = a;
            const uint32_t x = sel_raw[i];
            sel_raw[i] = sel_raw[j];
            sel_raw[j] = x;
          }
        }
      }
      __syncthreads();
    }
  }
  for (int j = tid; j < kk; j += NT) {
    out_idx[j] = (int32_t)sel_pos[j];
    if (out_val) out_val[j] = (Raw)sel_raw[j];
  }
}

}  // namespace dstopk
