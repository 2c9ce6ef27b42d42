// select_phase.cuh -- the selection that follows the indexer score in
// ds_indexer_topk when a row's scores come from several CTAs (few rows, as in
// decode).
//
// What it computes (NKI pull request "Add DeepSeek-V4 CSA attention kernels",
// "How the algorithm works", steps table row 3, and "The top-k on the GPSIMD
// engine": the index scores feed the top-k as they are produced, with a
// final top-k over the chunks): the k largest of a row's float32 scores at
// positions s < valid_len, ties to the lower position.
//
// How (B200 design):
//  * While the scorer's epilogue produces a row's scores it counts them in an
//    exact histogram of the top 12 bits of their order-preserving keys, and
//    every scorer CTA adds its counts into the row's global histogram.  The
//    selection starts from that histogram: the bin b0 holding the k-th largest
//    key comes from one block-wide scan, with no sampling and no pass over the
//    scores spent on it.
//  * A cluster of CTAs per row then streams the row once, each CTA a slice:
//    keys above b0 go straight to the output (slots from the leader CTA's
//    counter, one remote atomic per warp), keys inside b0 (the candidates) to
//    the leader's shared memory.  The leader resolves the candidates with an
//    exact radix select on their remaining 20 key bits (10-bit digits), and
//    for keys equal to the k-th on their positions.  A threshold bin too
//    crowded for the leader (many equal scores) is resolved the same way from
//    the scores themselves.
//  * The code runs once per CTA and is bound by the latency of its dependent
//    steps: helpers are inlined, loops over rows are not unrolled (per-row
//    state in shared memory), and global loads go out in batches, the next
//    batch in flight while one is processed.
#pragma once

#include "topk_stash_kernel.cuh"

namespace dstopk {

constexpr int kSelBins = 4096;  // first digit: the top 12 key bits
constexpr int kSelShift = 20;   // key >> kSelShift is the first digit
constexpr int kSelDigit = 10;   // later key digits (the candidates' 20 low bits in two passes)
constexpr int kSelPosDigit = 8; // position digits (24 bits in three passes)

// Control block of a selection over up to NR rows at once (NTH threads).
template <int NR, int NTH>
struct MrCtrl {
  uint32_t wtot[NR][32];   // scan scratch: warp totals
  uint32_t wex[NR][33];    // their exclusive prefixes
  uint32_t res[NR][4];     // per row: bin, count above it, count inside it
  uint32_t out[NR];        // per row: selection slots handed out
  uint32_t cnt[NR];        // per row: candidates listed
  uint32_t part[NR][NTH];  // per row and thread: its bins' count
  uint32_t incl[NR][NTH];  // per row and thread: inclusive warp prefix
};

// For nr <= NR histograms of nb bins (bin b of row r read as get(r, b)), find
// per row the bin b with #(keys in bins > b) < target(r) <= #(keys in bins >= b);
// the results land in c->res[r] = {bin, above, inbin} ({0, 0, 0} when target
// is 0).  Every thread calls it; two block barriers serve all rows.
template <int NTH, int NR, class Get, class Target>
__device__ __forceinline__ void mr_find_bin(Get&& get, int nb, int nr, Target&& target, MrCtrl<NR, NTH>* c) {
  static_assert(NTH % 32 == 0 && NTH / 32 <= 32 && NR <= NTH / 32, "one warp's lanes cover a row's warp totals");
  constexpr int NW = NTH / 32;
  const int tid = (int)threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int bpt = (nb + NTH - 1) / NTH;
  const int r0 = tid * bpt;  // first rank owned (0 = the top bin)
  const int r1 = min(nb, r0 + bpt);
  if (tid < nr) {
    c->res[tid][0] = 0u;
    c->res[tid][1] = 0u;
    c->res[tid][2] = 0u;
  }
#pragma unroll 1
  for (int r = 0; r < nr; ++r) {
    uint32_t a = 0u;
    for (int i = r0; i < r1; ++i) a += get(r, nb - 1 - i);
    uint32_t in = a;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t t = __shfl_up_sync(0xFFFFFFFFu, in, o);
      if (lane >= o) in += t;
    }
    c->part[r][tid] = a;
    c->incl[r][tid] = in;
    if (lane == 31) c->wtot[r][warp] = in;
  }
  __syncthreads();
  // two barriers in all: every warp scans a row's warp totals itself
#pragma unroll 1
  for (int r = 0; r < nr; ++r) {
    const uint32_t x = lane < NW ? c->wtot[r][lane] : 0u;
    uint32_t y = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t t = __shfl_up_sync(0xFFFFFFFFu, y, o);
      if (lane >= o) y += t;
    }
    const uint32_t wex = __shfl_sync(0xFFFFFFFFu, y - x, warp);
    const uint32_t tg = target(r), a = c->part[r][tid];
    const uint32_t excl = wex + c->incl[r][tid] - a;
    if (excl < tg && tg <= excl + a) {
      uint32_t acc = excl;
      for (int i = r0; i < r1; ++i) {
        const uint32_t n = get(r, nb - 1 - i);
        if (acc + n >= tg) {
          c->res[r][0] = (uint32_t)(nb - 1 - i);
          c->res[r][1] = acc;
          c->res[r][2] = n;
          break;
        }
        acc += n;
      }
    }
  }
  __syncthreads();
}

// Where a selection cuts inside one row's threshold bin: a key is taken when
// its top bits (key >> kshift) exceed kprefix, or equal it with the position
// at or below pcut.
struct SelCut {
  uint32_t kprefix;
  int kshift;
  uint32_t pcut;
};

__device__ __forceinline__ bool sel_taken(const SelCut& c, uint32_t key, uint32_t pos) {
  const uint32_t top = c.kshift >= 32 ? 0u : key >> c.kshift;
  return top > c.kprefix || (top == c.kprefix && pos <= c.pcut);
}

// Per-row state of a selection, in shared memory.
struct RowSel {
  uint32_t kk;      // selection size: min(k, valid length)
  uint32_t b0;      // threshold bin (top 12 key bits of the kk-th largest key)
  uint32_t krem;    // keys still to take inside the current digit bin
  uint32_t ncand;   // candidates listed
  uint32_t gather;  // the candidates are resolved from the list
  uint32_t live;    // the candidate resolution is still running
  uint32_t all;     // every key of bin b0 is taken
  uint32_t L;       // valid positions
  SelCut cut;       // the cut inside b0 once resolved
  uint32_t pp;      // position-pass prefix
};

// Exact selection among each live row's candidates (cand(r, i) -> key, pos;
// all with top key bits rs[r].b0): the rs[r].krem largest by (key, lower
// position), recorded in rs[r].cut.  Digit passes of 10 key bits, then (for
// rows still tied at one key) 8-bit passes on the complemented positions; each
// pass serves every row.  `hist` holds nr x 1024 counters.  Every thread calls it.
template <int NTH, int NR, class Cand>
__device__ __forceinline__ void mr_resolve(Cand&& cand, int nr, RowSel* rs, uint32_t* hist, MrCtrl<NR, NTH>* c) {
  constexpr int HB = 1 << kSelDigit;
  constexpr int PB = 1 << kSelPosDigit;
  const int tid = (int)threadIdx.x;
  // key digits: bits [19:10], then [9:0]; then position digits
  constexpr int kKeyPasses = kSelShift / kSelDigit, kPosPasses = kTsPosBits / kSelPosDigit;
#pragma unroll 1
  for (int pass = 0; pass < kKeyPasses + kPosPasses; ++pass) {
    const bool keys = pass < kKeyPasses;
    bool any = false;
    for (int r = 0; r < nr; ++r) any |= rs[r].live != 0u;
    if (!any) break;  // uniform
    const int nb = keys ? HB : PB;
    for (int i = tid; i < nr * nb; i += NTH) hist[i] = 0u;
    __syncthreads();
#pragma unroll 1
    for (int r = 0; r < nr; ++r) {
      if (!rs[r].live) continue;
      const SelCut cu = rs[r].cut;  // keys: prefix at shift; positions: prefix at shift 0, pp so far
      const int ps = kTsPosBits - (pass - kKeyPasses) * kSelPosDigit;  // position bits above the digit
      const uint32_t pp = rs[r].pp;
      const int n = (int)rs[r].ncand;
      for (int i = tid; i < n; i += NTH) {
        uint32_t key, pos;
        cand(r, i, key, pos);
        if (keys) {
          if ((key >> cu.kshift) == cu.kprefix)
            atomicAdd(hist + r * nb + ((key >> (cu.kshift - kSelDigit)) & (HB - 1)), 1u);
        } else {
          const uint32_t cp = ((1u << kTsPosBits) - 1u) - pos;
          if (key == cu.kprefix && (ps >= 32 ? 0u : cp >> ps) == pp)
            atomicAdd(hist + r * nb + ((cp >> (ps - kSelPosDigit)) & (PB - 1)), 1u);
        }
      }
    }
    __syncthreads();
    mr_find_bin<NTH, NR>([&](int r, int x) { return hist[r * nb + x]; }, nb, nr,
                         [&](int r) { return rs[r].live ? rs[r].krem : 0u; }, c);
    if (tid < nr && rs[tid].live) {
      RowSel& q = rs[tid];
      q.krem -= c->res[tid][1];
      if (keys) {
        q.cut.kprefix = (q.cut.kprefix << kSelDigit) | c->res[tid][0];
        q.cut.kshift -= kSelDigit;
      } else {
        const int ps = kTsPosBits - (pass - kKeyPasses + 1) * kSelPosDigit;
        q.pp = (q.pp << kSelPosDigit) | c->res[tid][0];
        // taken ties: complemented position >= pp << ps
        q.cut.pcut = ((1u << kTsPosBits) - 1u) - (q.pp << ps);
      }
      if (c->res[tid][2] == q.krem) q.live = 0u;  // the whole sub-bin is taken
    }
    __syncthreads();
  }
}

// Bitonic sort of nr rows of (position, value) pairs by position ascending
// (row r: n(r) <= 2048 pairs at pos + r * 2048, val + r * 2048).  Every
// thread calls it.
template <int NTH, class N>
__device__ __forceinline__ void mr_sort_pairs(uint32_t* pos, uint32_t* val, int nr, N&& n) {
  int np = 1;
  for (int r = 0; r < nr; ++r)
    while (np < (int)n(r)) np <<= 1;
  for (int i = (int)threadIdx.x; i < nr * np; i += NTH) {
    const int r = i / np, j = i % np;
    if (j >= (int)n(r)) pos[r * 2048 + j] = 0xFFFFFFFFu;
  }
  __syncthreads();
  for (int len = 2; len <= np; len <<= 1) {
    for (int st = len >> 1; st > 0; st >>= 1) {
      for (int i = (int)threadIdx.x; i < nr * np; i += NTH) {
        const int r = i / np, a = i % np, b = a ^ st;
        if (b > a) {
          uint32_t* p = pos + r * 2048;
          const uint32_t x = p[a], y = p[b];
          if ((x > y) == ((a & len) == 0)) {
            p[a] = y;
            p[b] = x;
            uint32_t* v = val + r * 2048;
            const uint32_t t = v[a];
            v[a] = v[b];
            v[b] = t;
          }
        }
      }
      __syncthreads();
    }
  }
}

// ------------------------------------------------------------------ split rows

constexpr int kHsThreads = 256;
constexpr int kHsCap = 2048;  // candidates the leader can hold (in the histogram's place)

struct HsParams {
  const float* scores;      // [B, S]: row t at scores + t * S, valid at s < valid_len[t]
  uint32_t* ghist;          // [B, 4096] key histograms; cleared here for the next launch
  const int32_t* valid_len; // [B] or null
  int32_t* out_idx;         // [B, k]
  float* out_score;         // [B, k] or null
  int B, S, k;
  int slice;                // positions per CTA, a multiple of 4
  int sorted;
  int* status;              // device status word (DS_DEBUG range checks)
};

// Shared memory of topk_hist_select_kernel (about 23 KiB, so that several CTAs
// share an SM): the row's histogram, whose space then holds the leader's
// candidates (raw[cap], pos[cap]), a 1024-bin pass histogram, and the control
// blocks.
struct HsSmem {
  static constexpr int kOffHist = 0;                        // u32[4096], later the candidates
  static constexpr int kOffCand = kOffHist;
  static constexpr int kOffPass = kOffHist + kSelBins * 4;  // u32[1024]
  static constexpr int kOffCtrl = kOffPass + (1 << kSelDigit) * 4;  // MrCtrl, TsCtrl, RowSel
  // each control block on a 16-byte boundary (TsCtrl holds 8-byte mbarriers)
  static constexpr int kOffTs = kOffCtrl + (int)((sizeof(MrCtrl<1, kHsThreads>) + 15) / 16 * 16);
  static constexpr int kOffRow = kOffTs + (int)((sizeof(TsCtrl) + 15) / 16 * 16);
  static constexpr int kBytes = (kOffRow + (int)sizeof(RowSel) + 127) / 128 * 128;
};
static_assert(HsSmem::kOffTs % 16 == 0 && HsSmem::kOffRow % 16 == 0, "control blocks aligned");
static_assert(kHsCap * 8 <= kSelBins * 4, "the candidates fit the histogram's space");

__device__ __forceinline__ uint32_t dsmem_atom_add(uint32_t addr, uint32_t v) {
  uint32_t old;
  asm volatile("atom.relaxed.cluster.shared::cluster.add.u32 %0, [%1], %2;" : "=r"(old) : "r"(addr), "r"(v) : "memory");
  return old;
}

__device__ __forceinline__ void dsmem_st(uint32_t addr, uint32_t v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

// One cluster of C CTAs per row (C = the launch's cluster size): the row's
// threshold bin from its global histogram, then one pass over the row split
// into C slices (keys above the bin go straight out, keys inside it to the
// leader), then the leader resolves the candidates.
__global__ void __launch_bounds__(kHsThreads) topk_hist_select_kernel(const HsParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  uint32_t* hist = reinterpret_cast<uint32_t*>(smem + HsSmem::kOffHist);
  uint32_t* pass_hist = reinterpret_cast<uint32_t*>(smem + HsSmem::kOffPass);
  MrCtrl<1, kHsThreads>* c = reinterpret_cast<MrCtrl<1, kHsThreads>*>(smem + HsSmem::kOffCtrl);
  TsCtrl* tc = reinterpret_cast<TsCtrl*>(smem + HsSmem::kOffTs);
  RowSel* rs = reinterpret_cast<RowSel*>(smem + HsSmem::kOffRow);
  uint32_t* cand_raw = reinterpret_cast<uint32_t*>(smem + HsSmem::kOffCand);
  uint32_t* cand_pos = cand_raw + kHsCap;
  const int tid = (int)threadIdx.x, lane = tid & 31;
  const uint32_t crank = cluster_ctarank(), csize = cluster_nctarank();
  const int row = (int)(blockIdx.x / csize);
  pdl_wait();
  pdl_launch_dependents();
  int L = p.S;
  if (p.valid_len) {
    const int v = p.valid_len[row];
    if (tid == 0 && crank == 0) debug_range(v >= 0 && v <= p.S, p.status);
    L = v < 0 ? 0 : (v > p.S ? p.S : v);
  }
  const int kk = min(p.k, L);
  int32_t* out_idx = p.out_idx + (size_t)row * p.k;
  float* out_score = p.out_score ? p.out_score + (size_t)row * p.k : nullptr;
  if (crank == 0)
    for (int j = kk + tid; j < p.k; j += kHsThreads) {
      out_idx[j] = -1;
      if (out_score) out_score[j] = -INFINITY;
    }
  if (kk == 0) return;  // uniform over the cluster; the row's histogram is all zero

  const uint32_t* srow = reinterpret_cast<const uint32_t*>(p.scores + (size_t)row * p.S);
  uint32_t* gh = p.ghist + (size_t)row * kSelBins;
  // this CTA's slice, loaded while the histogram comes in
  const int i0 = (int)crank * p.slice;
  const int m = max(0, min(p.slice, L - i0));
  constexpr int V = 8;  // scores per thread per round
  uint32_t rv[V], nx[V];
#pragma unroll
  for (int u = 0; u < V; ++u) {
    const int i = u * kHsThreads + tid;
    rv[u] = i < m ? __ldcg(srow + i0 + i) : 0u;
  }
  for (int i = tid; i < kSelBins / 4; i += kHsThreads)
    reinterpret_cast<uint4*>(hist)[i] = __ldcg(reinterpret_cast<const uint4*>(gh) + i);
  if (tid == 0) {
    c->out[0] = 0u;
    c->cnt[0] = 0u;
  }
  __syncthreads();
  mr_find_bin<kHsThreads, 1>([&](int, int b) { return hist[b]; }, kSelBins, 1, [&](int) { return (uint32_t)kk; },
                             c);
  const uint32_t b0 = c->res[0][0];
  const uint32_t krem = (uint32_t)kk - c->res[0][1];
  const bool all = c->res[0][2] == krem;
  const bool gather = !all && c->res[0][2] <= (uint32_t)kHsCap;
  const uint32_t fin_lo = all ? b0 : b0 + 1u;
  cluster_sync();  // every CTA has its copy of the histogram and the leader's counters are zero
  // the histogram goes back to zero for the next launch, each CTA a share
  for (int i = (int)crank * kHsThreads + tid; i < kSelBins / 4; i += (int)csize * kHsThreads)
    reinterpret_cast<uint4*>(gh)[i] = make_uint4(0u, 0u, 0u, 0u);

  // ---- the slice: selected keys straight out, candidates to the leader
  const uint32_t l_out = dsmem_map(smem_u32(&c->out[0]), 0);
  const uint32_t l_cnt = dsmem_map(smem_u32(&c->cnt[0]), 0);
  const uint32_t l_craw = dsmem_map(smem_u32(cand_raw), 0);
  const uint32_t l_cpos = dsmem_map(smem_u32(cand_pos), 0);
  const int rounds = (m + V * kHsThreads - 1) / (V * kHsThreads);
#pragma unroll 1
  for (int it = 0; it < rounds; ++it) {
    if (it + 1 < rounds) {  // the next round's loads in flight while this one is classified
#pragma unroll
      for (int u = 0; u < V; ++u) {
        const int i = ((it + 1) * V + u) * kHsThreads + tid;
        nx[u] = i < m ? __ldcg(srow + i0 + i) : 0u;
      }
    }
    uint32_t fm = 0u, cm = 0u;
#pragma unroll
    for (int u = 0; u < V; ++u) {
      const bool in = (it * V + u) * kHsThreads + tid < m;
      const uint32_t d = F32Keys::key(rv[u]) >> kSelShift;
      fm |= (uint32_t)(in && d >= fin_lo) << u;
      cm |= (uint32_t)(in && gather && d == b0) << u;
    }
    // warp-wide slot allocation in the leader (one remote atomic per warp and kind)
    const uint32_t nf = (uint32_t)__popc(fm), nc = (uint32_t)__popc(cm);
    uint32_t fi = nf, ci = nc;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t a = __shfl_up_sync(0xFFFFFFFFu, fi, o), b = __shfl_up_sync(0xFFFFFFFFu, ci, o);
      if (lane >= o) {
        fi += a;
        ci += b;
      }
    }
    const uint32_t ftot = __shfl_sync(0xFFFFFFFFu, fi, 31), ctot = __shfl_sync(0xFFFFFFFFu, ci, 31);
    uint32_t fb = 0u, cb = 0u;
    if (lane == 0) {
      if (ftot) fb = dsmem_atom_add(l_out, ftot);
      if (ctot) cb = dsmem_atom_add(l_cnt, ctot);
    }
    uint32_t fo = __shfl_sync(0xFFFFFFFFu, fb, 0) + fi - nf;
    uint32_t co = __shfl_sync(0xFFFFFFFFu, cb, 0) + ci - nc;
    while (fm | cm) {
      const int u = __ffs(fm | cm) - 1;
      const uint32_t bit = 1u << u;
      const uint32_t pos = (uint32_t)(i0 + (it * V + u) * kHsThreads + tid);
      uint32_t raw = 0u;
#pragma unroll
      for (int x = 0; x < V; ++x) raw = x == u ? rv[x] : raw;
      if (fm & bit) {
        if (fo < (uint32_t)kk) {
          out_idx[fo] = (int32_t)pos;
          if (out_score) out_score[fo] = __uint_as_float(raw);
        }
        ++fo;
      } else {
        if (co < (uint32_t)kHsCap) {
          dsmem_st(l_craw + 4u * co, raw);
          dsmem_st(l_cpos + 4u * co, pos);
        }
        ++co;
      }
      fm &= ~bit;
      cm &= ~bit;
    }
#pragma unroll
    for (int u = 0; u < V; ++u) rv[u] = nx[u];
  }
  cluster_sync();  // every selected key is out and every candidate is in the leader
  if (crank != 0) return;

  // ---- the leader: the krem largest candidates
  if (!all) {
    if (gather) {
      if (tid == 0) {
        RowSel& q = rs[0];
        q.kk = (uint32_t)kk;
        q.b0 = b0;
        q.krem = krem;
        q.ncand = min(c->cnt[0], (uint32_t)kHsCap);
        q.live = 1u;
        q.cut = SelCut{b0, kSelShift, 0xFFFFFFFFu};
        q.pp = 0u;
      }
      __syncthreads();
      mr_resolve<kHsThreads, 1>(
          [&](int, int i, uint32_t& key, uint32_t& pos) {
            key = F32Keys::key(cand_raw[i]);
            pos = cand_pos[i];
          },
          1, rs, pass_hist, c);
      const SelCut cu = rs[0].cut;
      for (int i = tid; i < (int)rs[0].ncand; i += kHsThreads) {
        const uint32_t raw = cand_raw[i], pos = cand_pos[i];
        if (sel_taken(cu, F32Keys::key(raw), pos)) {
          const uint32_t s = atomicAdd(&c->out[0], 1u);
          if (s < (uint32_t)kk) {
            out_idx[s] = (int32_t)pos;
            if (out_score) out_score[s] = __uint_as_float(raw);
          }
        }
      }
    } else {
      // more keys in the threshold bin than the leader can hold: straight
      // from the row
      auto visit = [&](auto&& f) {
        for (int i = tid; i < L; i += kHsThreads) f(F32Keys::key(__ldcg(srow + i)), (uint32_t)i);
      };
      const TsCut tcut = ts_select<F32Keys, kHsThreads>(visit, (int)krem, cand_raw, tc, b0, kSelShift);
      for (int i = tid; i < L; i += kHsThreads) {
        const uint32_t raw = __ldcg(srow + i), key = F32Keys::key(raw);
        if ((key >> kSelShift) == b0 && ts_taken(tcut, key, (uint32_t)i)) {
          const uint32_t s = atomicAdd(&c->out[0], 1u);
          if (s < (uint32_t)kk) {
            out_idx[s] = i;
            if (out_score) out_score[s] = __uint_as_float(raw);
          }
        }
      }
    }
  }
  if (!p.sorted) return;
  // ---- ascending positions: the selection read back (the other CTAs' part
  // is visible after the cluster barrier) and sorted; scores gathered again
  __syncthreads();
  uint32_t* sp = cand_pos;  // 2048 positions and their scores (the candidates are done with)
  uint32_t* sv = cand_raw;
  for (int j = tid; j < kk; j += kHsThreads) {
    const uint32_t pos = (uint32_t)__ldcg(out_idx + j);
    const bool in = pos < (uint32_t)L;  // always, unless the row's histogram disagreed with its scores
    sp[j] = in ? pos : 0xFFFFFFFFu;
    sv[j] = in ? __ldcg(srow + pos) : 0u;
  }
  __syncthreads();
  mr_sort_pairs<kHsThreads>(sp, sv, 1, [&](int) { return (uint32_t)kk; });
  for (int j = tid; j < kk; j += kHsThreads) {
    out_idx[j] = sp[j] == 0xFFFFFFFFu ? -1 : (int32_t)sp[j];
    if (out_score) out_score[j] = __uint_as_float(sv[j]);
  }
}

}  // namespace dstopk
