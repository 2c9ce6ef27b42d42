// rowcluster_kernel.cuh -- fused lightning-indexer score + top-k, one thread-block
// cluster per query row.
//
// What it computes (NKI pull request "Add DeepSeek-V4 CSA attention kernels",
// "How the algorithm works", steps table rows 2 and 3, and "The top-k on the
// GPSIMD engine": the score of every compressed position and its top-k in one
// launch, the score row never written out):
//     score[t, s] = sum_h w[t, h] * max(0, q[t, h, :] . k[s, :]),  s < valid_len[t]
// then the k highest scores of the row, ties to the lower position.
//
// How (B200 design):
//  * The CS CTAs of a cluster split the row's positions, PPC each.  A CTA
//    scores its 128-position key tiles on the tensor cores: D[s, h] =
//    K[s, :] . Q[t, h, :] with M = 128 positions, N = 64 heads, K = 128 channels,
//    the key tiles streamed by TMA through a 4-deep ring, the accumulator in one
//    of four TMEM buffers; two groups of four epilogue warps take alternate
//    tiles, apply ReLU, the per-head weight and the head sum, keep the scores in
//    shared memory and count their leading 12-bit radix digits in a local
//    histogram.  Tiles at or past valid_len are neither loaded nor scored.
//  * After one cluster barrier every CTA copies its scores into the leader CTA
//    through distributed shared memory (the leader's key ring is free by then)
//    and adds its non-zero histogram bins into the leader's histogram.  After a
//    second barrier the leader alone selects: the threshold bin from the merged
//    histogram, one pass over the row that emits every key above the bin and
//    lists the positions inside it, then a radix select over the listed
//    positions on (lower 20 key bits, complemented position), whose values are
//    all distinct, so the k-th one is unique and ties fall to the lower position.
#pragma once

#include <cuda.h>

#include "ptx.cuh"
#include "tcgen05.cuh"
#include "topk_kernel.cuh"

namespace dstopk {

constexpr int kRcThreads = 320;   // TMA warp, MMA warp, 2 x 4 epilogue warps
constexpr int kRcStages = 4;      // key-tile ring
constexpr int kRcBufs = 4;        // TMEM accumulators of 64 columns
constexpr int kRcMaxS = 32768;    // positions a row may have (leader buffer; 15-bit positions)
constexpr int kRcMaxPPC = 4096;   // positions per CTA
constexpr int kRcHeads = 64;      // the MMA's N; heads past H are zero-filled and weighted 0

struct RowClusterParams {
  const float* w;            // [B, H]
  const int32_t* valid_len;  // [B] or null
  int32_t* out_idx;          // [B, k]
  float* out_score;          // [B, k] or null
  int* status;
  int B, H, S, k;
  int ppc;                   // positions per CTA, a multiple of 128
};

struct RcSmem {
  static constexpr int kKHalf = 128 * 128;                       // 128 positions x 64 channels, bf16
  static constexpr int kStage = 2 * kKHalf;
  static constexpr int kOffRegion = 0;                           // key ring, then the leader's score row
  static constexpr int kOffQ = kOffRegion + kRcStages * kStage;  // 64 heads x 128 channels
  static constexpr int kOffSc = kOffQ + 2 * kRcHeads * 128;      // local scores, kRcMaxPPC floats
  static constexpr int kOffList = kOffQ;                         // leader: listed positions (u16) over q + scores
  static constexpr int kListCap = (kOffSc + kRcMaxPPC * 4 - kOffQ) / 2;
  static constexpr int kOffHist = kOffSc + kRcMaxPPC * 4;        // 4096 bins
  static constexpr int kOffW = kOffHist + 4096 * 4;              // 64 weights
  static constexpr int kOffCtl = kOffW + kRcHeads * 4;           // control words
  static constexpr int kOffBar = kOffCtl + 256;                  // 17 mbarriers
  static constexpr int kBytes = kOffBar + 256 + 1024;            // + alignment slack
  static_assert(kRcStages * kStage >= kRcMaxS * 4, "the leader's score row reuses the key ring");
};

// Hands out `n` consecutive slots of `*counter` to every lane of a warp (all 32
// lanes call it); returns this lane's first slot.
__device__ __forceinline__ uint32_t rc_warp_alloc(uint32_t n, uint32_t* counter) {
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

// Selection key of a position inside the threshold bin: the 20 key bits below
// the leading digit, then the complemented position (larger = lower position).
__device__ __forceinline__ uint64_t rc_composite(uint32_t key, int pos) {
  return ((uint64_t)(key & 0xFFFFFu) << 15) | (uint64_t)(uint32_t)(kRcMaxS - 1 - pos);
}

__global__ void __launch_bounds__(kRcThreads, 1)
    indexer_topk_rowcluster_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                                   const RowClusterParams p) {
  using SM = RcSmem;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  float* sc = reinterpret_cast<float*>(smem + SM::kOffSc);
  float* w_s = reinterpret_cast<float*>(smem + SM::kOffW);
  uint32_t* hist = reinterpret_cast<uint32_t*>(smem + SM::kOffHist);
  uint32_t* ctl = reinterpret_cast<uint32_t*>(smem + SM::kOffCtl);  // [0..1] counters, [12] TMEM base
  uint32_t* wtot = ctl + 16;                                          // scan scratch, one word per warp
  uint32_t* bcast = ctl + 48;
  const uint32_t bar = sbase + SM::kOffBar;
  auto BAR = [&](int i) -> uint32_t { return bar + 8u * (uint32_t)i; };
  // mbarriers: q, key full[4], key empty[4], accumulator full[4], accumulator empty[4]
  constexpr int kBQ = 0, kBKF = 1, kBKE = 5, kBAF = 9, kBAE = 13;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t crank = cluster_ctarank();
  const uint32_t csize = cluster_nctarank();
  const int row = (int)(blockIdx.x / csize);
  int L = p.S;
  if (p.valid_len) {
    L = p.valid_len[row];
    L = L < 0 ? 0 : (L > p.S ? p.S : L);
  }
  const int pos_lo = (int)crank * p.ppc;
  const int nact = max(0, min(p.ppc / 128, (L - pos_lo + 127) / 128));  // tiles holding a scored position

  if (tid == 0) {
    for (int i = 0; i < 17; ++i) mbar_init(BAR(i), i >= kBAE ? 4u : 1u);
    fence_mbar_init();
    if (nact > 0) {
      mbar_arrive_expect_tx(BAR(kBQ), 2 * kRcHeads * 128);
      tma_load_3d(sbase + SM::kOffQ, &tm_q, 0, 0, row, BAR(kBQ));
      tma_load_3d(sbase + SM::kOffQ + kRcHeads * 128, &tm_q, 64, 0, row, BAR(kBQ));
      for (int i = 0; i < min(nact, kRcStages); ++i) {
        const int pos0 = pos_lo + i * 128;
        mbar_arrive_expect_tx(BAR(kBKF + i), SM::kStage);
        tma_load_2d(sbase + SM::kOffRegion + i * SM::kStage, &tm_k, 0, pos0, BAR(kBKF + i));
        tma_load_2d(sbase + SM::kOffRegion + i * SM::kStage + SM::kKHalf, &tm_k, 64, pos0, BAR(kBKF + i));
      }
    }
  }
  for (int i = tid; i < 4096; i += kRcThreads) hist[i] = 0u;
  uint32_t* tmem_slot = ctl + 12;
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), kRcBufs * 64);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  // ------------------------------------------------------------ scores
  if (warp == 0) {
    if (lane == 0) {
      for (int i = kRcStages; i < nact; ++i) {
        const int s = i % kRcStages, r = i / kRcStages;
        if (!mbar_wait_bounded(BAR(kBKE + s), (uint32_t)((r & 1) ^ 1), p.status)) break;
        const int pos0 = pos_lo + i * 128;
        mbar_arrive_expect_tx(BAR(kBKF + s), SM::kStage);
        tma_load_2d(sbase + SM::kOffRegion + s * SM::kStage, &tm_k, 0, pos0, BAR(kBKF + s));
        tma_load_2d(sbase + SM::kOffRegion + s * SM::kStage + SM::kKHalf, &tm_k, 64, pos0, BAR(kBKF + s));
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && nact > 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, kRcHeads);
      bool ok = mbar_wait_bounded(BAR(kBQ), 0u, p.status);
      for (int i = 0; i < nact && ok; ++i) {
        const int s = i % kRcStages, r = i / kRcStages;
        const int b = i % kRcBufs, u = i / kRcBufs;
        if (!mbar_wait_bounded(BAR(kBAE + b), (uint32_t)((u & 1) ^ 1), p.status)) break;
        if (!mbar_wait_bounded(BAR(kBKF + s), (uint32_t)(r & 1), p.status)) break;
        tc_fence_after();
        const uint32_t a_base = sbase + SM::kOffRegion + s * SM::kStage;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t koff = (uint32_t)(kk & 3) * 32u;
          const uint64_t adesc = sw128_kmajor_desc(a_base + (uint32_t)(kk >> 2) * SM::kKHalf + koff);
          const uint64_t bdesc =
              sw128_kmajor_desc(sbase + SM::kOffQ + (uint32_t)(kk >> 2) * (kRcHeads * 128) + koff);
          mma_bf16_ss(tmem_base + (uint32_t)(b * 64), adesc, bdesc, idesc, kk > 0 ? 1u : 0u);
        }
        mma_commit(BAR(kBKE + s));
        mma_commit(BAR(kBAF + b));
      }
    }
  } else {
    const int gr = (warp - 2) >> 2;  // this group takes tiles gr, gr + 2, ...
    const int qd = warp & 3;         // TMEM lane quarter a warp may read
    const uint32_t lane_addr = (uint32_t)(qd * 32) << 16;
    for (int i = tid - 64; i < kRcHeads; i += kRcThreads - 64)
      w_s[i] = (i < p.H) ? p.w[(size_t)row * p.H + i] : 0.0f;
    named_bar_sync(1, kRcThreads - 64);
    for (int i = gr; i < nact; i += 2) {
      const int b = i % kRcBufs, u = i / kRcBufs;
      if (!mbar_wait_bounded(BAR(kBAF + b), (uint32_t)(u & 1), p.status)) break;
      tc_fence_after();
      uint32_t r[64];
#pragma unroll
      for (int c = 0; c < 64; c += 16)
        tmem_ld16(tmem_base + lane_addr + (uint32_t)(b * 64 + c), *reinterpret_cast<uint32_t(*)[16]>(r + c));
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(kBAE + b));
      float acc = 0.0f;
#pragma unroll
      for (int x = 0; x < 64; ++x) acc = fmaf(w_s[x], fmaxf(__uint_as_float(r[x]), 0.0f), acc);
      const int loc = i * 128 + qd * 32 + lane;
      sc[loc] = acc;
      if (pos_lo + loc < L) atomicAdd(hist + (F32Keys::key(__float_as_uint(acc)) >> 20), 1u);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, kRcBufs * 64);

  // ------------------------------------------------------------ scores and histogram -> leader
  cluster_sync();  // every CTA is done with its key ring; the leader's ring becomes the score row
  {
    const int nscored = max(0, min(p.ppc, L - pos_lo));
    const uint32_t dst = dsmem_map(sbase + SM::kOffRegion + (uint32_t)pos_lo * 4u, 0);
    const int nv = (nscored + 3) / 4;
    for (int v = tid; v < nv; v += kRcThreads) {
      const uint4 x = reinterpret_cast<const uint4*>(sc)[v];
      asm volatile("st.shared::cluster.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(dst + 16u * (uint32_t)v), "r"(x.x),
                   "r"(x.y), "r"(x.z), "r"(x.w)
                   : "memory");
    }
    if (crank != 0 && nscored > 0) {
      const uint32_t hdst = dsmem_map(sbase + SM::kOffHist, 0);
      for (int i = tid; i < 4096; i += kRcThreads) {
        const uint32_t c = hist[i];
        if (c) dsmem_red_add_u32(hdst + 4u * (uint32_t)i, c);
      }
    }
  }
  cluster_sync();
  if (crank != 0) return;

  // ------------------------------------------------------------ the leader selects
  const float* R = reinterpret_cast<const float*>(smem + SM::kOffRegion);
  uint16_t* list = reinterpret_cast<uint16_t*>(smem + SM::kOffList);
  int32_t* oidx = p.out_idx + (size_t)row * p.k;
  float* osc = p.out_score ? p.out_score + (size_t)row * p.k : nullptr;
  const int kk = min(p.k, L);
  for (int j = kk + tid; j < p.k; j += kRcThreads) {
    oidx[j] = -1;
    if (osc) osc[j] = -INFINITY;
  }
  if (kk == 0) return;
  if (tid == 0) {
    ctl[0] = 0u;  // output slots handed out
    ctl[1] = 0u;  // positions listed
  }
  uint32_t above, inbin;
  const uint32_t b0 = block_find_bin<kRcThreads>(hist, 4096, kk, wtot, bcast, above, inbin);
  uint32_t krem = (uint32_t)kk - above;
  const bool use_list = inbin <= (uint32_t)SM::kListCap;
  // one pass over the row: keys above the threshold bin are selected, positions inside it listed
  {
    const int nv = (L + 3) >> 2;
    for (int base = 0; base < nv; base += kRcThreads) {
      const int v = base + tid;
      float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
      if (v < nv) x = reinterpret_cast<const float4*>(R)[v];
      const float xs[4] = {x.x, x.y, x.z, x.w};
      uint32_t sel = 0u, cand = 0u;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        if (4 * v + e < L) {
          const uint32_t d = F32Keys::key(__float_as_uint(xs[e])) >> 20;
          sel |= (uint32_t)(d > b0) << e;
          cand |= (uint32_t)(d == b0) << e;
        }
      }
      uint32_t slot = rc_warp_alloc((uint32_t)__popc(sel), &ctl[0]);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        if ((sel >> e) & 1u) {
          if (slot < (uint32_t)kk) {
            oidx[slot] = 4 * v + e;
            if (osc) osc[slot] = xs[e];
          }
          ++slot;
        }
      }
      if (use_list) {
        uint32_t ls = rc_warp_alloc((uint32_t)__popc(cand), &ctl[1]);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          if ((cand >> e) & 1u) {
            if (ls < (uint32_t)SM::kListCap) list[ls] = (uint16_t)(4 * v + e);
            ++ls;
          }
        }
      }
    }
  }
  __syncthreads();
  // radix select on the composite keys of the threshold bin: digits of 12, 12 and 11 bits
  const int nsrc = use_list ? (int)inbin : L;
  auto src_pos = [&](int j) -> int { return use_list ? (int)list[j] : j; };
  uint64_t prefix = 0;
  int shift = 35;
  for (int pass = 0; pass < 3 && inbin != krem; ++pass) {
    const int sh = pass == 0 ? 23 : (pass == 1 ? 11 : 0);
    const int wd = pass == 2 ? 11 : 12;
    const int nb = 1 << wd;
    for (int i = tid; i < nb; i += kRcThreads) hist[i] = 0u;
    __syncthreads();
    for (int j = tid; j < nsrc; j += kRcThreads) {
      const int pos = src_pos(j);
      const uint32_t key = F32Keys::key(__float_as_uint(R[pos]));
      if ((key >> 20) != b0) continue;
      const uint64_t c = rc_composite(key, pos);
      if ((c >> shift) == prefix) atomicAdd(hist + (uint32_t)((c >> sh) & (uint64_t)(nb - 1)), 1u);
    }
    __syncthreads();
    uint32_t ab, ib;
    const uint32_t b = block_find_bin<kRcThreads>(hist, nb, (int)krem, wtot, bcast, ab, ib);
    krem -= ab;
    inbin = ib;
    prefix = (prefix << wd) | b;
    shift = sh;
  }
  // the rest of the selection: every listed position at or above the threshold
  for (int base = 0; base < nsrc; base += kRcThreads) {
    const int j = base + tid;
    bool take = false;
    int pos = 0;
    float val = 0.f;
    if (j < nsrc) {
      pos = src_pos(j);
      val = R[pos];
      const uint32_t key = F32Keys::key(__float_as_uint(val));
      take = (key >> 20) == b0 && (rc_composite(key, pos) >> shift) >= prefix;
    }
    const uint32_t slot = rc_warp_alloc(take ? 1u : 0u, &ctl[0]);
    if (take && slot < (uint32_t)kk) {
      oidx[slot] = pos;
      if (osc) osc[slot] = val;
    }
  }
}

}  // namespace dstopk
