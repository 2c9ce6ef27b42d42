// topk_kernel.cuh -- row-wise top-k with one thread-block cluster per row.
//
// What it computes: for each row, the k largest of the first L = valid_len
// scores, ties to the lower position (DeepSelect hub page, use-case
// paragraphs: top-k of a bfloat16 indexer score row, and of a float32 logit
// row over a ~129K vocabulary; options sorted_index and return_value).
//
// How (B200 design, not the pages' design):
//  * A row is split into C contiguous slices, one per CTA of a cluster of C
//    CTAs.  Each CTA pulls its slice into shared memory with bulk TMA copies
//    (the row is read from HBM exactly once) and turns every score into an
//    order-preserving unsigned key in place, building the histogram of the
//    first radix digit (11 bits) as the chunks land.
//  * The histograms are added into the leader CTA through distributed shared
//    memory; the leader finds the digit bin holding the k-th key and every CTA
//    reads it back.  One more pass over the slice moves the keys above that bin
//    to a selection list and the keys inside it to a small candidate list; the
//    remaining digits (float32: 11 + 10 bits, bfloat16: 5 bits) are resolved on
//    the candidate lists only.  A CTA whose share of the bin overflows its list
//    scans its whole slice instead (same result, slower).
//  * Output slots: keys above the threshold, then ties, the ties going to the
//    lowest positions of the row (CTA order = position order).  With
//    sorted_index the selection is written by an ordered pass over the slice
//    (warp scans + a block scan per chunk) and so comes out in ascending
//    position order.  Values are re-read bit-exactly from global memory.
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
  int slice;  // elements per CTA, a multiple of 8
  int return_value;
  int sorted;  // write the selection in ascending position order
};

// float32 rows: 32-bit keys, digits of 11, 11 and 10 bits.
struct F32Keys {
  using Raw = uint32_t;
  static constexpr int kBytes = 4, kVec = 4, kPasses = 3;
  static constexpr uint32_t kNegInf = 0xFF800000u;
  __device__ __forceinline__ static int shift(int p) { return p == 0 ? 21 : (p == 1 ? 10 : 0); }
  __device__ __forceinline__ static int width(int p) { return p == 2 ? 10 : 11; }
  // larger key <=> larger value; -0 folds onto +0; every NaN maps to the top key.
  __device__ __forceinline__ static uint32_t key(uint32_t b) {
    if ((b & 0x7FFFFFFFu) > 0x7F800000u) return 0xFFFFFFFFu;
    if (b == 0x80000000u) b = 0u;
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
  }
  __device__ __forceinline__ static uint32_t slot(const uint4& v, int j) {
    return j == 0 ? v.x : (j == 1 ? v.y : (j == 2 ? v.z : v.w));
  }
  __device__ __forceinline__ static uint4 keys4(uint4 v) {
    return make_uint4(key(v.x), key(v.y), key(v.z), key(v.w));
  }
};

// bfloat16 rows: 16-bit keys, digits of 11 and 5 bits.
struct BF16Keys {
  using Raw = uint16_t;
  static constexpr int kBytes = 2, kVec = 8, kPasses = 2;
  static constexpr uint32_t kNegInf = 0xFF80u;
  __device__ __forceinline__ static int shift(int p) { return p == 0 ? 5 : 0; }
  __device__ __forceinline__ static int width(int p) { return p == 0 ? 11 : 5; }
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
  __device__ __forceinline__ static uint32_t key2(uint32_t w) { return key(w & 0xFFFFu) | (key(w >> 16) << 16); }
  __device__ __forceinline__ static uint4 keys4(uint4 v) {
    return make_uint4(key2(v.x), key2(v.y), key2(v.z), key2(v.w));
  }
};

constexpr int kHistBins = 2048;        // largest digit: 11 bits
constexpr int kChunkBytes = 16384;     // one TMA copy / mbarrier per 16 KiB
constexpr int kMaxChunks = 16;
constexpr int kMaxSliceBytes = 184320; // 180 KiB of scores per CTA
constexpr int kSelCap = 2048;          // keys above the first-digit bin (< k <= 2048)
constexpr int kCandCap = 1024;         // keys inside the first-digit bin, per CTA

struct TopkCtrl {
  uint32_t bstar;     // leader -> all: digit of the k-th key in this pass
  int32_t krem;       // leader -> all: keys still to take inside that digit
  uint32_t bcount;    // leader -> all: keys of the whole cluster inside that digit
  uint32_t pad0;
  uint32_t gt;        // this CTA: keys above the threshold
  uint32_t eq;        // this CTA: keys equal to the threshold
  uint32_t base;      // this CTA: first output slot
  uint32_t take;      // this CTA: ties it selects
  uint32_t bcast[4];  // broadcast scratch inside the CTA
  uint32_t sel_cnt;   // entries in the selection list
  uint32_t cand_cnt;  // entries in the candidate list
  uint32_t tie_cnt;   // entries in the tie list
  uint32_t out_cnt;   // output slots handed out (list mode)
};

constexpr int kSmemHist = 0;
constexpr int kSmemHred = kSmemHist + kHistBins * 4;
constexpr int kSmemCtrl = kSmemHred + kHistBins * 4;
constexpr int kSmemWtot = kSmemCtrl + 128;
constexpr int kSmemMbar = kSmemWtot + 32 * 4;
constexpr int kSmemSel = kSmemMbar + kMaxChunks * 8;
constexpr int kSmemCandKey = kSmemSel + kSelCap * 4;
constexpr int kSmemCandIdx = kSmemCandKey + kCandCap * 4;
constexpr int kSmemTie = kSmemCandIdx + kCandCap * 4;
constexpr int kSmemData = ((kSmemTie + kCandCap * 4) + 127) / 128 * 128;
static_assert(sizeof(TopkCtrl) <= 128, "ctrl block");

__host__ __device__ constexpr int topk_smem_bytes(int slice_bytes) { return kSmemData + slice_bytes + 32; }

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

template <class K, int NT>
__global__ void __launch_bounds__(NT, 1) topk_cluster_kernel(const TopkParams p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  uint32_t* hist = reinterpret_cast<uint32_t*>(smem + kSmemHist);
  uint32_t* hred = reinterpret_cast<uint32_t*>(smem + kSmemHred);
  TopkCtrl* ctrl = reinterpret_cast<TopkCtrl*>(smem + kSmemCtrl);
  uint32_t* wtot = reinterpret_cast<uint32_t*>(smem + kSmemWtot);
  const uint32_t mbar0 = smem_u32(smem + kSmemMbar);
  const uint32_t data = smem_u32(smem + kSmemData);

  const int tid = threadIdx.x;
  const uint32_t crank = cluster_ctarank();
  const uint32_t csize = cluster_nctarank();
  const int row = blockIdx.x / csize;

  int L = p.n;
  if (p.valid_len) {
    const int v = p.valid_len[row];
    L = v < 0 ? 0 : (v > p.n ? p.n : v);
  }
  const int kk = min(p.k, L);
  int32_t* out_idx = p.out_idx + (size_t)row * p.k;
  typename K::Raw* out_val = p.return_value ? reinterpret_cast<typename K::Raw*>(p.out_val) + (size_t)row * p.k
                                            : nullptr;

  // padding slots kk..k-1 (written by the leader CTA)
  if (crank == 0) {
    for (int j = kk + tid; j < p.k; j += NT) {
      out_idx[j] = -1;
      if (out_val) out_val[j] = (typename K::Raw)K::kNegInf;
    }
  }
  if (kk == 0) return;  // uniform across the cluster: nothing to select in this row

  const int i0 = (int)crank * p.slice;
  const int m = max(0, min(p.slice, L - i0));  // eligible scores in this slice
  const typename K::Raw* grow = reinterpret_cast<const typename K::Raw*>(p.scores) + (size_t)row * p.n;
  const char* gslice = reinterpret_cast<const char*>(grow + i0);
  const uint32_t off = (uint32_t)(reinterpret_cast<uintptr_t>(gslice) & 15u);
  const uint32_t nbytes = off + (uint32_t)m * K::kBytes;
  const int nwords = m ? (int)((nbytes + 15u) >> 4) : 0;
  const int wf0 = off ? 1 : 0;               // first word fully inside the slice
  const int wf1 = m ? (int)(nbytes >> 4) : 0; // one past the last full word
  const int nfull = wf1 > wf0 ? wf1 - wf0 : 0;
  const uint32_t full_bytes = (uint32_t)nfull * 16u;
  const int nchunks = (int)((full_bytes + kChunkBytes - 1) / kChunkBytes);

  // ---- set-up: histograms, mbarriers, partially covered words
  for (int i = tid; i < kHistBins; i += NT) {
    hist[i] = 0u;
    hred[i] = 0u;
  }
  if (tid == 0) {
    for (int j = 0; j < nchunks; ++j) mbar_init(mbar0 + 8 * j, 1);
    fence_mbar_init();
    ctrl->sel_cnt = 0u;
    ctrl->cand_cnt = 0u;
    ctrl->tie_cnt = 0u;
    ctrl->out_cnt = 0u;
  }
  // The (at most two) words that the slice covers only in part are loaded
  // element by element; their other slots are never read as keys.
  int pw0 = -1, pw1 = -1;
  if (nwords > 0) {
    if (!(0 >= wf0 && 0 < wf1)) pw0 = 0;
    if (nwords - 1 > 0 && !(nwords - 1 >= wf0 && nwords - 1 < wf1)) pw1 = nwords - 1;
  }
  if (tid < 2 * K::kVec) {
    const int w = (tid < K::kVec) ? pw0 : pw1, j = tid % K::kVec;
    if (w >= 0) {
      const int b = 16 * w + j * K::kBytes - (int)off;
      if (b >= 0 && b / K::kBytes < m) {
        const uint32_t kv = K::key((uint32_t)grow[i0 + b / K::kBytes]);
        if (K::kBytes == 4)
          *reinterpret_cast<uint32_t*>(smem + kSmemData + 16 * w + j * 4) = kv;
        else
          *reinterpret_cast<uint16_t*>(smem + kSmemData + 16 * w + j * 2) = (uint16_t)kv;
      }
    }
  }
  __syncthreads();
  cluster_arrive();  // every CTA's reduction histogram is zeroed before anyone pushes

  if (tid == 0 && nchunks > 0) {
    const uint64_t pol = policy_evict_first();
    const char* src = gslice - off + 16 * wf0;
    for (int j = 0; j < nchunks; ++j) {
      const uint32_t bytes = min((uint32_t)kChunkBytes, full_bytes - (uint32_t)j * kChunkBytes);
      mbar_arrive_expect_tx(mbar0 + 8 * j, bytes);
      bulk_g2s_hint(data + 16 * wf0 + j * kChunkBytes, src + (size_t)j * kChunkBytes, bytes, mbar0 + 8 * j, pol);
    }
  }

  auto word_valid = [&](int w, int j) -> bool {
    const int b = 16 * w + j * K::kBytes - (int)off;
    return b >= 0 && b < m * K::kBytes;
  };

  // ---- pass 0: digit histogram while the slice lands; keys written in place
  {
    const int s0 = K::shift(0);
    if (tid < 2) {
      const int w = tid == 0 ? pw0 : pw1;
      if (w >= 0) {
        const uint4 v = lds128(data + 16 * w);
#pragma unroll
        for (int j = 0; j < K::kVec; ++j)
          if (word_valid(w, j)) atomicAdd(hist + (K::slot(v, j) >> s0), 1u);
      }
    }
    for (int c = 0; c < nchunks; ++c) {
      mbar_wait_bounded(mbar0 + 8 * c, 0, p.status);
      const int w_lo = wf0 + c * (kChunkBytes / 16);
      const int w_hi = min(wf1, w_lo + kChunkBytes / 16);
      for (int w = w_lo + tid; w < w_hi; w += NT) {
        const uint4 kv = K::keys4(lds128(data + 16 * w));
        sts128(data + 16 * w, kv);
        const uint32_t b0 = K::slot(kv, 0) >> s0;
        bool same = true;
#pragma unroll
        for (int j = 1; j < K::kVec; ++j) same &= (K::slot(kv, j) >> s0) == b0;
        if (same) {
          hist_add_run(hist, b0, K::kVec);
        } else {
#pragma unroll
          for (int j = 0; j < K::kVec; ++j) atomicAdd(hist + (K::slot(kv, j) >> s0), 1u);
        }
      }
    }
  }
  __syncthreads();
  cluster_wait();

  // ---- radix passes
  uint32_t* sel_idx = reinterpret_cast<uint32_t*>(smem + kSmemSel);
  uint32_t* cand_key = reinterpret_cast<uint32_t*>(smem + kSmemCandKey);
  uint32_t* cand_idx = reinterpret_cast<uint32_t*>(smem + kSmemCandIdx);
  uint32_t* tie_idx = reinterpret_cast<uint32_t*>(smem + kSmemTie);
  const uint32_t leader_hred = dsmem_map(smem_u32(hred), 0);
  const uint32_t leader_ctrl = dsmem_map(smem_u32(ctrl), 0);
  int krem = kk;
  uint32_t prefix = 0;
  int lvl_shift = 0;
  uint32_t gt_local = 0, eq_local = 0;
  bool use_list = false;  // per CTA: later digits resolved on the candidate list

  auto elem_of = [&](int w, int j) -> int { return (16 * w + j * K::kBytes - (int)off) / K::kBytes; };

  for (int pass = 0; pass < K::kPasses; ++pass) {
    const int sh = K::shift(pass);
    const int nb = 1 << K::width(pass);
    if (pass > 0) {
      const int psh = K::shift(pass - 1);
      if (use_list) {
        const int nc = min((int)ctrl->cand_cnt, kCandCap);
        for (int i = tid; i < nc; i += NT) {
          const uint32_t kv = cand_key[i];
          if ((kv >> psh) == prefix) atomicAdd(hist + ((kv >> sh) & (uint32_t)(nb - 1)), 1u);
        }
      } else {
        for (int w = tid; w < nwords; w += NT) {
          const uint4 v = lds128(data + 16 * w);
          const bool full = (w >= wf0 && w < wf1);
          uint32_t b0 = 0xFFFFFFFFu;
          bool same = full;
#pragma unroll
          for (int j = 0; j < K::kVec; ++j) {
            const uint32_t kv = K::slot(v, j);
            const bool hit = (full || word_valid(w, j)) && (kv >> psh) == prefix;
            const uint32_t b = hit ? ((kv >> sh) & (uint32_t)(nb - 1)) : 0xFFFFFFFEu;
            if (j == 0) b0 = b;
            same &= (b == b0) && hit;
          }
          if (same) {
            hist_add_run(hist, b0, K::kVec);
          } else {
#pragma unroll
            for (int j = 0; j < K::kVec; ++j) {
              const uint32_t kv = K::slot(v, j);
              if ((full || word_valid(w, j)) && (kv >> psh) == prefix)
                atomicAdd(hist + ((kv >> sh) & (uint32_t)(nb - 1)), 1u);
            }
          }
        }
      }
      __syncthreads();
    }
    // push the local histogram into the leader
    for (int b = tid; b < nb; b += NT) {
      const uint32_t c = hist[b];
      if (c) dsmem_red_add_u32(leader_hred + 4u * b, c);
    }
    cluster_sync();
    if (crank == 0) {
      if (tid == 0) {
        ctrl->bstar = 0u;
        ctrl->krem = krem;
        ctrl->bcount = 0u;
      }
      // find the digit b* with  #(digits > b*) < krem <= #(digits >= b*)
      const int bpt = (nb + NT - 1) / NT;
      const int r0 = tid * bpt;
      uint32_t s = 0;
      for (int r = r0; r < min(nb, r0 + bpt); ++r) s += hred[nb - 1 - r];
      uint32_t total;
      const uint32_t excl = block_excl_scan<NT>(s, wtot, total);
      if (excl < (uint32_t)krem && (uint32_t)krem <= excl + s) {
        uint32_t acc = excl;
        for (int r = r0; r < min(nb, r0 + bpt); ++r) {
          const uint32_t c = hred[nb - 1 - r];
          if (acc + c >= (uint32_t)krem) {
            ctrl->bstar = (uint32_t)(nb - 1 - r);
            ctrl->krem = krem - (int)acc;
            ctrl->bcount = c;
            break;
          }
          acc += c;
        }
      }
      __syncthreads();
      for (int b = tid; b < nb; b += NT) hred[b] = 0u;
    }
    cluster_sync();
    if (tid == 0) {
      ctrl->bcast[0] = dsmem_ld_u32(leader_ctrl + offsetof(TopkCtrl, bstar));
      ctrl->bcast[1] = dsmem_ld_u32(leader_ctrl + offsetof(TopkCtrl, krem));
      ctrl->bcast[2] = dsmem_ld_u32(leader_ctrl + offsetof(TopkCtrl, bcount));
    }
    __syncthreads();
    const uint32_t bstar = min(ctrl->bcast[0], (uint32_t)(nb - 1));
    krem = (int)ctrl->bcast[1];
    const uint32_t bcount = ctrl->bcast[2];
    uint32_t above = 0;
    for (int b = tid; b < nb; b += NT) above += (b > (int)bstar) ? hist[b] : 0u;
    above = block_sum<NT>(above, wtot);
    gt_local += above;
    eq_local = hist[bstar];
    prefix = (prefix << K::width(pass)) | bstar;
    lvl_shift = sh;
    __syncthreads();
    for (int b = tid; b < nb; b += NT) hist[b] = 0u;
    if (pass == 0) {
      // keys above the bin go to the selection list, keys inside it to the
      // candidate list (when this CTA's share fits)
      use_list = eq_local <= (uint32_t)kCandCap;
      if (use_list) {
        for (int w = tid; w < nwords; w += NT) {
          const uint4 v = lds128(data + 16 * w);
          const bool full = (w >= wf0 && w < wf1);
#pragma unroll
          for (int j = 0; j < K::kVec; ++j) {
            const uint32_t kv = K::slot(v, j);
            const uint32_t d = kv >> sh;
            if (d >= prefix && (full || word_valid(w, j))) {
              if (d > prefix) {
                const uint32_t pos = atomicAdd(&ctrl->sel_cnt, 1u);
                if (pos < (uint32_t)kSelCap) sel_idx[pos] = (uint32_t)elem_of(w, j);
              } else {
                const uint32_t pos = atomicAdd(&ctrl->cand_cnt, 1u);
                if (pos < (uint32_t)kCandCap) {
                  cand_key[pos] = kv;
                  cand_idx[pos] = (uint32_t)elem_of(w, j);
                }
              }
            }
          }
        }
      }
    }
    __syncthreads();
    if (bcount == (uint32_t)krem) break;  // the whole digit bin is selected: threshold found
  }

  // ---- exchange (gt, eq) across the cluster; derive output base and tie share
  if (tid == 0) {
    ctrl->gt = gt_local;
    ctrl->eq = eq_local;
  }
  cluster_sync();
  if (tid == 0) {
    uint32_t base = 0, eq_before = 0;
    for (uint32_t r = 0; r < crank; ++r) {
      const uint32_t a = dsmem_map(smem_u32(ctrl), r);
      const uint32_t g = dsmem_ld_u32(a + offsetof(TopkCtrl, gt));
      const uint32_t e = dsmem_ld_u32(a + offsetof(TopkCtrl, eq));
      const int tk = max(0, min((int)e, krem - (int)eq_before));
      base += g + (uint32_t)tk;
      eq_before += e;
    }
    ctrl->base = base;
    ctrl->take = (uint32_t)max(0, min((int)eq_local, krem - (int)eq_before));
  }
  __syncthreads();
  cluster_arrive();  // this CTA no longer reads other CTAs' shared memory

  const uint32_t base = ctrl->base, take = ctrl->take;
  const uint32_t mine = gt_local + take;
  auto put = [&](uint32_t pos, int e_idx) {
    if (pos < (uint32_t)kk) {  // always true when the counts are consistent
      out_idx[pos] = i0 + e_idx;
      if (out_val) out_val[pos] = grow[i0 + e_idx];
    }
  };

  if (mine > 0 && (p.sorted || !use_list)) {
    // ---- ordered emission over the whole slice (ascending positions)
    uint32_t gt_run = 0, tie_run = 0;
    for (int w0 = 0; w0 < nwords; w0 += NT) {
      const int w = w0 + tid;
      uint4 v = make_uint4(0, 0, 0, 0);
      const bool inw = w < nwords;
      if (inw) v = lds128(data + 16 * w);
      const bool full = inw && (w >= wf0 && w < wf1);
      uint32_t g = 0, e = 0, gm = 0, em = 0;
#pragma unroll
      for (int j = 0; j < K::kVec; ++j) {
        const bool ok = inw && (full || word_valid(w, j));
        const uint32_t top = K::slot(v, j) >> lvl_shift;
        const bool isg = ok && top > prefix;
        const bool ise = ok && top == prefix;
        g += isg;
        e += ise;
        gm |= (uint32_t)isg << j;
        em |= (uint32_t)ise << j;
      }
      uint32_t total;
      const uint32_t excl = block_excl_scan<NT>(g | (e << 16), wtot, total);
      if (total != 0) {
        uint32_t gb = gt_run + (excl & 0xFFFFu);
        uint32_t tb = tie_run + (excl >> 16);
#pragma unroll
        for (int j = 0; j < K::kVec; ++j) {
          const bool isg = (gm >> j) & 1u, ise = (em >> j) & 1u;
          if (isg || (ise && tb < take)) put(base + gb + min(tb, take), elem_of(w, j));
          gb += isg;
          tb += ise;
        }
      }
      gt_run += total & 0xFFFFu;
      tie_run += total >> 16;
      if (gt_run + min(tie_run, take) >= mine) break;  // uniform: every selected key is written
    }
  } else if (mine > 0) {
    // ---- list emission: selection list, then candidates above / at the threshold
    const int ns = min((int)ctrl->sel_cnt, kSelCap);
    for (int i = tid; i < ns; i += NT) put(base + atomicAdd(&ctrl->out_cnt, 1u), (int)sel_idx[i]);
    const int nc = min((int)ctrl->cand_cnt, kCandCap);
    for (int i = tid; i < nc; i += NT) {
      const uint32_t top = cand_key[i] >> lvl_shift;
      if (top > prefix) {
        put(base + atomicAdd(&ctrl->out_cnt, 1u), (int)cand_idx[i]);
      } else if (top == prefix && take > 0) {
        const uint32_t t = atomicAdd(&ctrl->tie_cnt, 1u);
        tie_idx[t] = cand_idx[i];
      }
    }
    __syncthreads();
    const int nt = (int)ctrl->tie_cnt;
    if (take >= (uint32_t)nt) {
      for (int i = tid; i < nt; i += NT) put(base + gt_local + (uint32_t)i, (int)tie_idx[i]);
    } else {
      // the `take` lowest positions among this CTA's ties
      for (int i = tid; i < nt; i += NT) {
        const uint32_t me = tie_idx[i];
        uint32_t rank = 0;
        for (int j = 0; j < nt; ++j) rank += tie_idx[j] < me;
        if (rank < take) put(base + gt_local + rank, (int)me);
      }
    }
  }
  cluster_wait();  // keep this CTA's shared memory alive until the cluster is done reading it
}

}  // namespace dstopk
