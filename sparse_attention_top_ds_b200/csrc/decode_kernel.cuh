// decode_kernel.cuh -- fused lightning-indexer score + top-k for a decode step.
//
// What it computes (NKI pull request "Add DeepSeek-V4 CSA attention kernels",
// "How the algorithm works", steps table rows 2 and 3, and "The top-k on the
// GPSIMD engine": scoring fused with the selection so that the score row does
// not go back in full):
//     score[t, s] = sum_h w[t, h] * max(0, q[t, h, :] . k[s, :])
// for up to 8 query rows against one bf16 key cache, then the k highest scores
// of each row (ties to the lower position), in ONE cooperative launch.
//
// How (B200 design):
//  1. Each CTA scores its run of 128-position key tiles for all rows on the
//     tensor cores (tcgen05, accumulator in TMEM, split into two 256-column
//     halves of 4 rows each so the epilogue of one half overlaps the MMAs of
//     the other; a half whose rows are all past the tile's positions is
//     skipped).  The scores stay in shared memory.
//  2. Per row, a 4096-bin histogram of the top 12 bits of the order-preserving
//     float key, plus a 256-bin coarse copy, is added into a small global
//     table (only non-empty bins; 8 replicas spread the atomics).  One
//     grid-wide barrier.
//  3. Every CTA finds each row's threshold bin with two short reads (coarse,
//     then the 16 fine bins under it); keys above it are written out at once,
//     keys inside it are appended to a per-row candidate list.
//  4. The last CTA to finish a row (an atomic ticket, no waiting) resolves that
//     row's candidates exactly: radix select on the remaining key bits, ties
//     to the lowest positions.
// Only the candidates (a few per cent of a row) ever leave the chip.
#pragma once

#include <cuda.h>

#include "ptx.cuh"
#include "tcgen05.cuh"
#include "topk_kernel.cuh"

namespace dstopk {

constexpr int kDecRows = 8;        // query rows of one call (at most)
constexpr int kDecHeads = 64;      // padded heads
constexpr int kDecStages = 2;      // key-tile ring
constexpr int kDecMaxTiles = 4;    // 128-position tiles per CTA
constexpr int kDecThreads = 320;   // TMA warp, MMA warp, 8 epilogue warps

struct DecodeParams {
  const float* w;           // [B, H]
  const int32_t* valid_len; // [B] or null
  int32_t* out_idx;         // [B, k]
  float* out_score;         // [B, k] or null
  int* status;
  int B, H, S, k;
  int tiles_per_cta;
  uint32_t* ctl;            // control table, see DecodeCtl
  uint32_t* cand;           // [B][S][2] candidates: raw score bits, position
};

// Layout of the control table (u32 offsets): two copies, then a parity word
// and an exit counter.  A call uses the copy the parity word names and clears
// the other one for the next call; the last CTA to leave flips the parity, so
// consecutive calls (eager or replayed from a CUDA graph) alternate on their
// own.  The table is zeroed once when it is allocated.
constexpr int kDecRep = 8;  // replicas of the global histograms (CTA c adds into replica c % kDecRep)

struct DecodeCtl {
  static constexpr int kFine = 0;                                   // [kDecRep][8][4096]
  static constexpr int kCoarse = kFine + kDecRep * kDecRows * 4096; // [kDecRep][8][256]
  static constexpr int kCtr = kCoarse + kDecRep * kDecRows * 256;   // [8][4]: out, cand, ticket, -
  static constexpr int kBar = kCtr + kDecRows * 4;                  // grid barrier
  static constexpr int kSize = kBar + 4;                            // per copy
  static constexpr int kParity = 2 * kSize;                         // which copy is in use
  static constexpr int kExit = kParity + 1;                         // CTAs that have finished
  static constexpr int kTotal = kExit + 3;
};

struct DecodeSmem {
  static constexpr int kQHalf = 512 * 128;                           // rows x 64 channels x 2 B
  static constexpr int kOffQ = 0;                                     // 128 KiB (later: histograms)
  static constexpr int kOffK = kOffQ + 2 * kQHalf;                    // 64 KiB (later: coarse / candidates)
  static constexpr int kKHalf = 128 * 128;
  static constexpr int kStage = 2 * kKHalf;
  static constexpr int kOffW = kOffK + kDecStages * kStage;           // 2 KiB
  static constexpr int kOffSc = kOffW + kDecRows * kDecHeads * 4;     // scores [8][kDecMaxTiles*128]
  static constexpr int kOffCtrl = kOffSc + kDecRows * kDecMaxTiles * 128 * 4;
  static constexpr int kOffBar = kOffCtrl + 1024;
  static constexpr int kBytes = kOffBar + 128 + 1024;                 // + alignment slack
  static_assert(kDecRows * 4096 * 4 <= 2 * kQHalf, "histograms reuse the query region");
};

struct DecodeRowCtl {
  uint32_t b0, krem, bcount, kk;
  uint32_t def_base, cand_base, loc_def, loc_cand;
  uint32_t dmin, dmax, final_row, pad;  // dmin: whole bin taken; pad: the row's valid length
};

__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ uint32_t f32_key(uint32_t b) {
  if ((b & 0x7FFFFFFFu) > 0x7F800000u) return 0xFFFFFFFFu;
  if (b == 0x80000000u) b = 0u;
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

__global__ void __launch_bounds__(kDecThreads, 1)
    indexer_topk_decode_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                               const DecodeParams p) {
  using SM = DecodeSmem;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  float* w_s = reinterpret_cast<float*>(smem + SM::kOffW);
  float* sc = reinterpret_cast<float*>(smem + SM::kOffSc);
  DecodeRowCtl* rc = reinterpret_cast<DecodeRowCtl*>(smem + SM::kOffCtrl);
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + SM::kOffCtrl + 8 * sizeof(DecodeRowCtl));
  uint32_t* wtot = misc + 16;  // 32 words of scan scratch
  uint32_t* bcast = misc + 48;
  const uint32_t bar = sbase + SM::kOffBar;
  auto BAR = [&](int i) -> uint32_t { return bar + 8u * (uint32_t)i; };
  // barriers: q[2], kfull[2], kempty[2], afull[2], aempty[2]
  constexpr int kBQ = 0, kBKF = 2, kBKE = 4, kBAF = 6, kBAE = 8;
  uint32_t* tmem_slot = misc + 60;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = gridDim.x;
  const int TPC = p.tiles_per_cta;
  const int ntiles = (p.S + 127) / 128;
  const int tile_lo = blockIdx.x * TPC;
  const int tile_hi = min(ntiles, tile_lo + TPC);
  const uint32_t parity = __ldcg(p.ctl + DecodeCtl::kParity) & 1u;
  uint32_t* ctl = p.ctl + parity * DecodeCtl::kSize;
  uint32_t* ctl_next = p.ctl + (parity ^ 1u) * DecodeCtl::kSize;

  // loads start at once: the queries and the first ring of key tiles of this
  // CTA, before anything else waits on memory (tiles past every valid length
  // are loaded too, and simply not used)
  const int nload = min(max(tile_hi - tile_lo, 0), kDecStages);
  if (tid == 0) {
    for (int i = 0; i < 10; ++i) mbar_init(BAR(i), (i == kBAE || i == kBAE + 1) ? 4 : 1);
    fence_mbar_init();
    if (nload > 0) {
      for (int g = 0; g < 2; ++g) {  // queries of rows 4g..4g+3, both channel halves
        mbar_arrive_expect_tx(BAR(kBQ + g), 2 * 256 * 128);
        tma_load_3d(sbase + SM::kOffQ + g * 256 * 128, &tm_q, 0, 0, 4 * g, BAR(kBQ + g));
        tma_load_3d(sbase + SM::kOffQ + SM::kQHalf + g * 256 * 128, &tm_q, 64, 0, 4 * g, BAR(kBQ + g));
      }
      for (int i = 0; i < nload; ++i) {
        const int pos0 = (tile_lo + i) * 128;
        mbar_arrive_expect_tx(BAR(kBKF + i), SM::kStage);
        tma_load_2d(sbase + SM::kOffK + i * SM::kStage, &tm_k, 0, pos0, BAR(kBKF + i));
        tma_load_2d(sbase + SM::kOffK + i * SM::kStage + SM::kKHalf, &tm_k, 64, pos0, BAR(kBKF + i));
      }
    }
  }
  // valid lengths; the largest per half of the rows decides which tiles / halves run
  int vlh[2] = {0, 0};
  for (int t = 0; t < kDecRows; ++t) {
    int v = 0;
    if (t < p.B) {
      v = p.valid_len ? p.valid_len[t] : p.S;
      v = v < 0 ? 0 : (v > p.S ? p.S : v);
    }
    vlh[t >> 2] = max(vlh[t >> 2], v);
  }
  const int act_hi = min(tile_hi, (max(vlh[0], vlh[1]) + 127) / 128);
  const int nact = max(0, act_hi - tile_lo);
  auto half_active = [&](int g, int i) { return (tile_lo + i) * 128 < vlh[g]; };
  // clear the other copy of the control table for the next call
  for (int i = blockIdx.x * kDecThreads + tid; i < DecodeCtl::kSize; i += G * kDecThreads) ctl_next[i] = 0u;
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  // ------------------------------------------------------------ 1. scores
  if (warp == 0) {
    if (lane == 0) {
      for (int i = kDecStages; i < nact; ++i) {
        const int s = i % kDecStages, r = i / kDecStages;
        if (!mbar_wait_bounded(BAR(kBKE + s), (r & 1) ^ 1, p.status)) break;
        const int pos0 = (tile_lo + i) * 128;
        mbar_arrive_expect_tx(BAR(kBKF + s), SM::kStage);
        tma_load_2d(sbase + SM::kOffK + s * SM::kStage, &tm_k, 0, pos0, BAR(kBKF + s));
        tma_load_2d(sbase + SM::kOffK + s * SM::kStage + SM::kKHalf, &tm_k, 64, pos0, BAR(kBKF + s));
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && nact > 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, 256);
      bool ok = true;
      bool qready[2] = {false, false};
      for (int i = 0; i < nact && ok; ++i) {
        const int s = i % kDecStages, r = i / kDecStages;
        if (!mbar_wait_bounded(BAR(kBKF + s), r & 1, p.status)) break;
        const uint32_t a_base = sbase + SM::kOffK + s * SM::kStage;
        for (int g = 0; g < 2; ++g) {
          if (!half_active(g, i)) continue;
          if (!qready[g]) {
            if (!mbar_wait_bounded(BAR(kBQ + g), 0, p.status)) {
              ok = false;
              break;
            }
            qready[g] = true;
          }
          if (!mbar_wait_bounded(BAR(kBAE + g), (i & 1) ^ 1, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t koff = (uint32_t)(kk & 3) * 32u;
            const uint64_t adesc = sw128_kmajor_desc(a_base + (uint32_t)(kk >> 2) * SM::kKHalf + koff);
            const uint32_t b_addr = sbase + SM::kOffQ + (uint32_t)(kk >> 2) * SM::kQHalf + (uint32_t)g * 256u * 128u + koff;
            mma_bf16_ss(tmem_base + (uint32_t)(g * 256), adesc, sw128_kmajor_desc(b_addr), idesc, kk > 0 ? 1u : 0u);
          }
          mma_commit(BAR(kBAF + g));
        }
        mma_commit(BAR(kBKE + s));
      }
      for (int g = 0; g < 2; ++g)
        if (!qready[g]) mbar_wait_bounded(BAR(kBQ + g), 0, p.status);
    }
    // loads issued but never consumed (tiles past every valid length) are
    // waited for, so no copy is in flight when the region is reused
    if (lane == 0 && nload > 0) {
      if (nact == 0)
        for (int g = 0; g < 2; ++g) mbar_wait_bounded(BAR(kBQ + g), 0, p.status);
      for (int i = nact; i < nload; ++i) mbar_wait_bounded(BAR(kBKF + i), 0, p.status);
    }
  } else {
    // per-head weights (zero for padded heads and absent rows), loaded by the
    // epilogue warps only
    for (int i = tid - 64; i < kDecRows * kDecHeads; i += kDecThreads - 64) {
      const int t = i / kDecHeads, h = i % kDecHeads;
      w_s[i] = (t < p.B && h < p.H) ? p.w[(size_t)t * p.H + h] : 0.0f;
    }
    named_bar_sync(1, kDecThreads - 64);
    const int g = (warp - 2) >> 2;  // rows 4g .. 4g+3
    const int qd = warp & 3;
    const int lrow = qd * 32 + lane;
    const uint32_t lane_addr = (uint32_t)(qd * 32) << 16;
    int vl[4];
    for (int j = 0; j < 4; ++j) {
      const int t = 4 * g + j;
      int v = 0;
      if (t < p.B) {
        v = p.valid_len ? p.valid_len[t] : p.S;
        v = v < 0 ? 0 : (v > p.S ? p.S : v);
      }
      vl[j] = v;
    }
    for (int i = 0; i < TPC; ++i) {
      const int pos = (tile_lo + i) * 128 + lrow;
      const bool ran = i < nact && half_active(g, i);
      if (ran) {
        if (!mbar_wait_bounded(BAR(kBAF + g), i & 1, p.status)) break;
        tc_fence_after();
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float acc = -INFINITY;
        if (ran) {
          const uint32_t col = tmem_base + lane_addr + (uint32_t)(g * 256 + j * 64);
          uint32_t r[64];
#pragma unroll
          for (int c = 0; c < 64; c += 16) tmem_ld16(col + (uint32_t)c, *reinterpret_cast<uint32_t(*)[16]>(r + c));
          tmem_wait_ld();
          acc = 0.0f;
#pragma unroll
          for (int x = 0; x < 64; ++x) acc = fmaf(w_s[(4 * g + j) * 64 + x], fmaxf(__uint_as_float(r[x]), 0.0f), acc);
        }
        sc[(4 * g + j) * (kDecMaxTiles * 128) + i * 128 + lrow] = (pos < vl[j]) ? acc : -INFINITY;
      }
      if (ran) {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(BAR(kBAE + g));
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, 512);

  // ------------------------------------------------------------ 2. histograms
  uint32_t* hist = reinterpret_cast<uint32_t*>(smem + SM::kOffQ);       // [8][4096]
  for (int i = tid; i < kDecRows * 4096 / 4; i += kDecThreads)
    reinterpret_cast<uint4*>(hist)[i] = make_uint4(0u, 0u, 0u, 0u);
  if (tid < kDecRows) {
    int L = 0;
    if (tid < p.B) {
      L = p.valid_len ? p.valid_len[tid] : p.S;
      L = L < 0 ? 0 : (L > p.S ? p.S : L);
    }
    rc[tid].kk = (uint32_t)L;  // holds L until the threshold step
    rc[tid].loc_def = 0u;
    rc[tid].loc_cand = 0u;
    rc[tid].final_row = 0u;
  }
  __syncthreads();
  const int npos = TPC * 128;
  const int pos0 = tile_lo * 128;
  for (int e = tid; e < p.B * npos; e += kDecThreads) {
    const int t = e / npos, lp = e - t * npos;
    if (pos0 + lp >= (int)rc[t].kk) continue;  // kk holds the row's valid length here
    atomicAdd(hist + t * 4096 + (f32_key(__float_as_uint(sc[t * (kDecMaxTiles * 128) + lp])) >> 20), 1u);
  }
  __syncthreads();
  // push the non-empty bins into this CTA's replica of the global table
  {
    uint32_t* gf = ctl + DecodeCtl::kFine + (blockIdx.x % kDecRep) * (kDecRows * 4096);
    uint32_t* gc = ctl + DecodeCtl::kCoarse + (blockIdx.x % kDecRep) * (kDecRows * 256);
    for (int pr = tid; pr < p.B * 256; pr += kDecThreads) {
      const uint32_t* hb = hist + pr * 16;  // row pr / 256, coarse bin pr % 256
      const uint4 a0 = reinterpret_cast<const uint4*>(hb)[0], a1 = reinterpret_cast<const uint4*>(hb)[1];
      const uint4 a2 = reinterpret_cast<const uint4*>(hb)[2], a3 = reinterpret_cast<const uint4*>(hb)[3];
      const uint32_t v[16] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w,
                              a2.x, a2.y, a2.z, a2.w, a3.x, a3.y, a3.z, a3.w};
      uint32_t c = 0;
#pragma unroll
      for (int j = 0; j < 16; ++j) c += v[j];
      if (c == 0u) continue;
      atomicAdd(gc + pr, c);
#pragma unroll
      for (int j = 0; j < 16; ++j)
        if (v[j]) atomicAdd(gf + pr * 16 + j, v[j]);
    }
  }
  // ------------------------------------------------------------ grid barrier
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    atomicAdd(ctl + DecodeCtl::kBar, 1u);
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t it = 0;; ++it) {
      if (ld_acquire_gpu(ctl + DecodeCtl::kBar) >= (uint32_t)G) break;
      if ((it & 63u) == 0 && globaltimer_ns() - t0 > kWaitLimitNs) {
        record_status(p.status, kErrTimeout);
        break;
      }
    }
    __threadfence();
  }
  __syncthreads();

  // ------------------------------------------------------------ 3. threshold bins, emission
  if (warp < p.B) {
    const int t = warp;
    const int L = (int)rc[t].kk;
    const uint32_t kk = (uint32_t)min(p.k, L);
    __syncwarp();
    uint32_t b0 = 0, above = 0, bcount = 0;
    if (kk > 0) {
      // coarse bins, highest first: lane l holds bins 255-8l .. 248-8l
      const uint32_t* cg = ctl + DecodeCtl::kCoarse + t * 256;
      uint32_t c[8], s = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) c[j] = 0u;
#pragma unroll
      for (int r = 0; r < kDecRep; ++r)
#pragma unroll
        for (int j = 0; j < 8; ++j) c[j] += __ldcg(cg + r * (kDecRows * 256) + 255 - 8 * lane - j);
#pragma unroll
      for (int j = 0; j < 8; ++j) s += c[j];
      uint32_t incl = s;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t x = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= o) incl += x;
      }
      const uint32_t excl = incl - s;
      const bool mine = excl < kk && kk <= incl;
      const uint32_t who = __ballot_sync(0xFFFFFFFFu, mine);
      uint32_t cb = 0, acc = 0;
      if (mine) {
        acc = excl;
        for (int j = 0; j < 8; ++j) {
          if (acc + c[j] >= kk) {
            cb = 255u - 8u * lane - j;
            break;
          }
          acc += c[j];
        }
      }
      const int src = who ? __ffs(who) - 1 : 0;
      cb = __shfl_sync(0xFFFFFFFFu, cb, src);
      acc = __shfl_sync(0xFFFFFFFFu, acc, src);
      // the 16 fine bins under cb, highest first
      uint32_t f = 0u;
      if (lane < 16)
#pragma unroll
        for (int r = 0; r < kDecRep; ++r)
          f += __ldcg(ctl + DecodeCtl::kFine + r * (kDecRows * 4096) + t * 4096 + cb * 16 + 15 - lane);
      uint32_t fi = f;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t x = __shfl_up_sync(0xFFFFFFFFu, fi, o);
        if (lane >= o) fi += x;
      }
      const bool m2 = lane < 16 && acc + fi - f < kk && kk <= acc + fi;
      const uint32_t w2 = __ballot_sync(0xFFFFFFFFu, m2);
      const int s2 = w2 ? __ffs(w2) - 1 : 0;
      b0 = cb * 16 + 15 - (uint32_t)s2;
      above = acc + __shfl_sync(0xFFFFFFFFu, fi - f, s2);
      bcount = __shfl_sync(0xFFFFFFFFu, f, s2);
    }
    if (lane == 0) {
      rc[t].pad = (uint32_t)L;
      rc[t].kk = kk;
      rc[t].b0 = b0;
      rc[t].krem = kk - above;
      rc[t].bcount = bcount;
      // this CTA's share: final keys (digits above b0, or the whole bin when it
      // is all taken) and candidates (inside b0)
      rc[t].dmin = (uint32_t)(bcount == kk - above);  // whole bin taken
    }
    // this CTA's share: final keys (digits above b0, or the whole bin when it
    // is all taken) and candidates (inside b0), summed by the warp
    const bool all = __shfl_sync(0xFFFFFFFFu, bcount == kk - above, 0);
    uint32_t nd = 0;
    if (kk > 0)
      for (uint32_t b = b0 + (all ? 0u : 1u) + lane; b < 4096u; b += 32u) nd += hist[t * 4096 + b];
    nd = __reduce_add_sync(0xFFFFFFFFu, nd);
    if (lane == 0) {
      const uint32_t nc = (kk > 0 && !all) ? hist[t * 4096 + b0] : 0u;
      // one 64-bit atomic reserves both ranges: final keys (low word) and
      // candidates (high word)
      unsigned long long old = 0;
      if (nd | nc)
        old = atomicAdd(reinterpret_cast<unsigned long long*>(ctl + DecodeCtl::kCtr + t * 4),
                        ((unsigned long long)nc << 32) | nd);
      rc[t].def_base = (uint32_t)old;
      rc[t].cand_base = (uint32_t)(old >> 32);
    }
  }
  __syncthreads();
  for (int e = tid; e < p.B * npos; e += kDecThreads) {
    const int t = e / npos, lp = e % npos;
    const uint32_t kk = rc[t].kk;
    if (kk == 0) continue;
    const int pos = pos0 + lp;
    if (pos >= (int)rc[t].pad) continue;  // pad holds L
    const uint32_t raw = __float_as_uint(sc[t * (kDecMaxTiles * 128) + lp]);
    const uint32_t d = f32_key(raw) >> 20;
    const uint32_t b0 = rc[t].b0;
    const bool all = rc[t].bcount == rc[t].krem;
    if (d > b0 || (all && d == b0)) {
      const uint32_t slot = rc[t].def_base + atomicAdd(&rc[t].loc_def, 1u);
      if (slot < kk) {
        p.out_idx[(size_t)t * p.k + slot] = pos;
        if (p.out_score) p.out_score[(size_t)t * p.k + slot] = __uint_as_float(raw);
      }
    } else if (d == b0) {
      const uint32_t cs = rc[t].cand_base + atomicAdd(&rc[t].loc_cand, 1u);
      if (cs < (uint32_t)p.S) {
        uint32_t* cp = p.cand + ((size_t)t * p.S + cs) * 2;
        cp[0] = raw;
        cp[1] = (uint32_t)pos;
      }
    }
  }
  // ------------------------------------------------------------ 4. finish each row in its own CTA
  // Row t is finished by CTA (t * G) / B once every CTA has counted itself in
  // on the row's ticket (a bounded wait; all CTAs are co-resident).
  __syncthreads();
  if (tid < p.B) {
    __threadfence();
    atomicAdd(ctl + DecodeCtl::kCtr + tid * 4 + 2, 1u);
  }
  for (int t = 0; t < p.B; ++t) {
    if ((int)blockIdx.x != (t * G) / p.B) continue;
    const uint32_t kk = rc[t].kk;
    int32_t* oidx = p.out_idx + (size_t)t * p.k;
    float* osc = p.out_score ? p.out_score + (size_t)t * p.k : nullptr;
    for (int j = (int)kk + tid; j < p.k; j += kDecThreads) {
      oidx[j] = -1;
      if (osc) osc[j] = -INFINITY;
    }
    if (kk == 0 || rc[t].bcount == rc[t].krem) continue;
    if (tid == 0) {
      const uint64_t w0 = globaltimer_ns();
      for (uint32_t it = 0;; ++it) {
        if (ld_acquire_gpu(ctl + DecodeCtl::kCtr + t * 4 + 2) >= (uint32_t)G) break;
        if ((it & 63u) == 0 && globaltimer_ns() - w0 > kWaitLimitNs) {
          record_status(p.status, kErrTimeout);
          break;
        }
      }
      __threadfence();
      misc[12] = __ldcg(ctl + DecodeCtl::kCtr + t * 4 + 0);  // final keys of the row: output slots taken
    }
    __syncthreads();
    // candidates of the row (raw score bits, position), staged in shared
    // memory when they fit (the key-tile region, free by now)
    const int nc = (int)min(rc[t].bcount, (uint32_t)p.S);
    const uint32_t* gcand = p.cand + (size_t)t * p.S * 2;
    constexpr int kStageCand = (kDecStages * SM::kStage) / 8;
    uint32_t* scand = reinterpret_cast<uint32_t*>(smem + SM::kOffK);
    const bool staged = nc <= kStageCand;
    if (staged) {
      // 16-byte loads, four in flight per thread
      const int nv = (2 * nc + 3) / 4;
      const uint4* g4 = reinterpret_cast<const uint4*>(gcand);
      uint4* s4 = reinterpret_cast<uint4*>(scand);
      for (int i = tid; i < nv; i += 4 * kDecThreads) {
        uint4 r[4];
#pragma unroll
        for (int u = 0; u < 4; ++u)
          if (i + u * kDecThreads < nv) r[u] = __ldcg(g4 + i + u * kDecThreads);
#pragma unroll
        for (int u = 0; u < 4; ++u)
          if (i + u * kDecThreads < nv) s4[i + u * kDecThreads] = r[u];
      }
    }
    const uint32_t* cand = staged ? scand : gcand;
    __syncthreads();
    uint32_t* h = hist;  // reuse: this CTA's histograms are no longer needed
    int krem = (int)rc[t].krem;
    uint32_t prefix = rc[t].b0;
    int shift = 20;
    for (int pass = 0; pass < 2; ++pass) {
      const int sh = pass == 0 ? 9 : 0;
      const int wd = pass == 0 ? 11 : 9;
      const int nb = 1 << wd;
      for (int i = tid; i < nb; i += kDecThreads) h[i] = 0u;
      __syncthreads();
      for (int i = tid; i < nc; i += kDecThreads) {
        const uint32_t kv = f32_key(cand[2 * i]);
        if ((kv >> shift) == prefix) atomicAdd(h + ((kv >> sh) & (uint32_t)(nb - 1)), 1u);
      }
      __syncthreads();
      uint32_t ab, inbin;
      const uint32_t b = block_find_bin<kDecThreads>(h, nb, krem, wtot, bcast, ab, inbin);
      krem -= (int)ab;
      prefix = (prefix << wd) | b;
      shift = sh;
      if (inbin == (uint32_t)krem) break;
    }
    // ties at the threshold: the lowest positions, by a radix select on the
    // complemented positions
    uint32_t ntie = 0;
    for (int i = tid; i < nc; i += kDecThreads) ntie += (f32_key(cand[2 * i]) >> shift) == prefix;
    ntie = block_sum<kDecThreads>(ntie, wtot);
    uint32_t cut = 0xFFFFFFFFu;
    if ((uint32_t)krem < ntie) {
      uint32_t pfx = 0;
      int want = krem;
      for (int pass = 0; pass < 3; ++pass) {
        const int sh = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
        const int wd = pass == 2 ? 10 : 11;
        const int psh = pass == 0 ? 32 : (pass == 1 ? 21 : 10);
        const int nb = 1 << wd;
        for (int i = tid; i < nb; i += kDecThreads) h[i] = 0u;
        __syncthreads();
        for (int i = tid; i < nc; i += kDecThreads) {
          if ((f32_key(cand[2 * i]) >> shift) != prefix) continue;
          const uint32_t ck = ~cand[2 * i + 1];
          if (pass == 0 || (ck >> psh) == pfx) atomicAdd(h + ((ck >> sh) & (uint32_t)(nb - 1)), 1u);
        }
        __syncthreads();
        uint32_t ab, inbin;
        const uint32_t b = block_find_bin<kDecThreads>(h, nb, want, wtot, bcast, ab, inbin);
        want -= (int)ab;
        pfx = (pass == 0 ? 0u : (pfx << wd)) | b;
      }
      cut = ~pfx;
    }
    for (int i = tid; i < nc; i += kDecThreads) {
      const uint32_t raw = cand[2 * i];
      const uint32_t top = f32_key(raw) >> shift;
      const uint32_t pos = cand[2 * i + 1];
      if (top > prefix || (top == prefix && pos <= cut)) {
        const uint32_t slot = atomicAdd(&misc[12], 1u);
        if (slot < kk) {
          oidx[slot] = (int)pos;
          if (osc) osc[slot] = __uint_as_float(raw);
        }
      }
    }
    __syncthreads();
  }
  // the last CTA to leave hands the other copy of the table to the next call
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    if (atomicInc(p.ctl + DecodeCtl::kExit, (uint32_t)G - 1u) == (uint32_t)G - 1u)
      atomicExch(p.ctl + DecodeCtl::kParity, parity ^ 1u);
  }
}

}  // namespace dstopk
