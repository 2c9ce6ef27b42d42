// indexer_kernel.cuh -- the lightning-indexer score on the tcgen05 tensor cores.
//
// What it computes (NKI pull request "Add DeepSeek-V4 CSA attention kernels",
// "How the algorithm works", steps table row 2):
//     score[t, s] = sum_h w[t, h] * max(0, q[t, h, :] . k[s, :]),   d = 128,
// for s < valid_len[t]; -inf at the other positions.
//
// How (B200 design):
//  * A CTA owns a group of NT query rows and a run of 128-position tiles of
//    the key cache.  The contraction D[s, (t,h)] = K[s, :] . Q[(t,h), :] is a
//    dense GEMM with M = 128 positions, N = NT x HP (rows x padded heads),
//    K = 128 channels: the key tile is operand A, the group's queries are
//    operand B, both bf16 and K-major in 128-byte-swizzled shared memory
//    written by TMA; the float32 accumulator lives in TMEM.
//  * Warp roles: warp 0 issues TMA loads (queries once, key tiles through a
//    ring of STAGES buffers), warp 1 owns TMEM and issues the MMAs from one
//    thread, warps 2..9 are the epilogue.  With N <= 256 the accumulator is
//    double-buffered in TMEM so the epilogue of one tile overlaps the MMAs of
//    the next.
//  * Epilogue: after tcgen05.ld each thread holds one position's per-head
//    products for its rows, so ReLU, the per-head weight (broadcast from
//    shared memory) and the head sum are a register loop with no shuffles.
//  * Positions at or past the group's largest valid_len are neither loaded
//    nor multiplied.
//  * The key tensor map is 4-D (64 channels, positions, 2 channel halves,
//    caches): one TMA copy brings a whole 128-position tile (32 KiB), its two
//    64-channel halves one after the other as the MMA reads them.  There is one
//    cache for every row, or one per row (then a group is one row and reads
//    cache t).
//
// With the selection (SEL = true; NKI pull request, "The top-k on the GPSIMD
// engine": the index scores feed the top-k as they are produced):
//  * The epilogue also counts every valid score of its rows in a shared-memory
//    histogram of the top 12 bits of its order-preserving key (16-bit counters,
//    two per word), and at the end adds the CTA's counts into the rows' global
//    histograms; only valid positions are stored.
//  * topk_hist_select_kernel (select_phase.cuh) then starts from the exact
//    threshold bin those histograms give: one pass over each row, no sampling
//    and no histogram pass of its own.
#pragma once

#include <cuda.h>

#include "ptx.cuh"
#include "tcgen05.cuh"
#include "select_phase.cuh"

namespace dstopk {

struct ScoreParams {
  const float* w;           // [B, H]
  const int32_t* valid_len; // [B] or null
  float* out;               // [B, S]: every score (SEL: valid positions only, read back by the selection)
  int* status;
  int B, H, S;
  int tiles_per_cta;        // 128-position tiles per CTA
  int ctas_per_group;       // CTAs sharing one group of NT rows
  int key_per_row;          // 1: row t reads key cache t (then NT == 1); 0: one cache for every row
  uint32_t* ghist;          // SEL: [B, 4096] key histograms, zero before the launch
  uint64_t wait_ns;         // limit of every bounded wait (0: the library default)
  int fault;                // testing the failure detection: 1 = CTA 0's first epilogue warp skips its
                            // first release of the accumulator, so that a wait runs out (0 otherwise)
};

template <int NT, int HP, int STAGES, bool SEL = false>
struct ScoreCfg {
  static constexpr int kN = NT * HP;                 // accumulator columns per tile
  static constexpr int kNmma = kN < 256 ? kN : 256;  // N of one MMA instruction
  static constexpr int kNumMma = kN / kNmma;
  static constexpr int kNbuf = 2;                    // TMEM accumulators: whole tiles alternate between them
  static constexpr int kEpiPerSlot = 8;              // epilogue warps releasing one accumulator
  static constexpr int kCols = kN * kNbuf;
  static constexpr int kTmemCols = kCols <= 32 ? 32 : (kCols <= 64 ? 64 : (kCols <= 128 ? 128 : (kCols <= 256 ? 256 : 512)));
  static constexpr int kQHalf = kN * 128;            // bytes: kN rows x 64 channels x 2 B
  static constexpr int kKHalf = 128 * 128;           // bytes: 128 positions x 64 channels x 2 B
  static constexpr int kStage = 2 * kKHalf;
  static constexpr int kEpiWarps = 8;
  static constexpr int kThreads = (2 + kEpiWarps) * 32;
  // shared-memory layout (offsets from a 1024-byte aligned base)
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + 2 * kQHalf;
  static constexpr int kOffW = kOffK + STAGES * kStage;
  static constexpr int kOffHist = kOffW + NT * HP * 4;          // SEL: u16 key histograms, 2 per word
  static constexpr int kHistBytes = SEL ? NT * (kSelBins / 2) * 4 : 0;
  static constexpr int kOffBar = kOffHist + kHistBytes;
  // (tiles whose key loads the MMA warp has waited for: the drain at the end)
  // barriers: qfull, kfull[STAGES], kempty[STAGES], afull[2], aempty[2], tmem slot
  static constexpr int kBarQ = 0;
  static constexpr int kBarKFull = 1;
  static constexpr int kBarKEmpty = 1 + STAGES;
  static constexpr int kBarAFull = 1 + 2 * STAGES;
  static constexpr int kBarAEmpty = 3 + 2 * STAGES;
  static constexpr int kNumBars = 5 + 2 * STAGES;
  static constexpr int kOffTmemSlot = kOffBar + kNumBars * 8;
  static constexpr int kOffConsumed = kOffTmemSlot + 8;
  static constexpr int kSmemBytes = kOffTmemSlot + 16 + 1024;  // + alignment slack
  static_assert(kN % 16 == 0 && kN <= 256 && kN % kNmma == 0, "bad tile");
  static_assert(HP % 16 == 0 && HP <= 64, "bad head padding");
  static_assert(kSmemBytes <= 227 * 1024, "shared memory");
  // SEL: 16-bit histogram counters hold the positions one CTA scores per row
  static constexpr int kMaxTilesPerCta = 65535 / 128;
};

// valid positions of row t, clamped to [0, S]
__device__ __forceinline__ int row_valid_len(const ScoreParams& p, int t) {
  int v = p.valid_len ? p.valid_len[t] : p.S;
  return v < 0 ? 0 : (v > p.S ? p.S : v);
}

template <int NT, int HP, int STAGES, bool SEL = false>
__global__ void __launch_bounds__(ScoreCfg<NT, HP, STAGES, SEL>::kThreads, 1)
    indexer_score_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                         const ScoreParams p) {
  using C = ScoreCfg<NT, HP, STAGES, SEL>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  float* w_s = reinterpret_cast<float*>(smem + C::kOffW);
  const uint32_t bar = sbase + C::kOffBar;
  auto BAR = [&](int i) -> uint32_t { return bar + 8u * (uint32_t)i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffTmemSlot);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int group = blockIdx.x / p.ctas_per_group;
  const int part = blockIdx.x % p.ctas_per_group;
  const int t0 = group * NT;
  const int ntiles = (p.S + 127) / 128;
  const int tile_lo = part * p.tiles_per_cta;
  const int tile_hi = min(ntiles, tile_lo + p.tiles_per_cta);

  pdl_wait();
  // largest valid length in the group: tiles at or past it are not computed
  int maxvl = 0;
  for (int t = 0; t < NT; ++t) {
    if (t0 + t < p.B) {
      int v = p.valid_len ? p.valid_len[t0 + t] : p.S;
      if (threadIdx.x == 0 && blockIdx.x % p.ctas_per_group == 0) debug_range(v >= 0 && v <= p.S, p.status);
      v = v < 0 ? 0 : (v > p.S ? p.S : v);
      maxvl = max(maxvl, v);
    }
  }
  const int act_hi = min(tile_hi, (maxvl + 127) / 128);
  const int kcache = p.key_per_row ? t0 : 0;  // the key cache of this group (its one row, with per-row caches)
  const int nact = max(0, act_hi - tile_lo);  // tiles that need the tensor cores

  if (threadIdx.x == 0) {
    mbar_init(BAR(C::kBarQ), 1);
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(BAR(C::kBarKFull + s), 1);
      mbar_init(BAR(C::kBarKEmpty + s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(BAR(C::kBarAFull + b), 1);
      mbar_init(BAR(C::kBarAEmpty + b), C::kEpiPerSlot);
    }
    fence_mbar_init();
    // start the loads at once: the queries and the first ring of key tiles
    if (nact > 0) {
      mbar_arrive_expect_tx(BAR(C::kBarQ), 2 * C::kQHalf);
      tma_load_3d(sbase + C::kOffQ, &tm_q, 0, 0, t0, BAR(C::kBarQ));
      tma_load_3d(sbase + C::kOffQ + C::kQHalf, &tm_q, 64, 0, t0, BAR(C::kBarQ));
      for (int i = 0; i < min(nact, STAGES); ++i) {
        const int pos0 = (tile_lo + i) * 128;
        mbar_arrive_expect_tx(BAR(C::kBarKFull + i), C::kStage);
        tma_load_4d(sbase + C::kOffK + i * C::kStage, &tm_k, 0, pos0, 0, kcache, BAR(C::kBarKFull + i));
      }
    }
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), C::kTmemCols);
    tmem_relinquish();
  }
  // per-head weights of the group (zero for padded heads and absent rows)
  for (int i = threadIdx.x; i < NT * HP; i += C::kThreads) {
    const int t = i / HP, h = i % HP;
    w_s[i] = (t0 + t < p.B && h < p.H) ? p.w[(size_t)(t0 + t) * p.H + h] : 0.0f;
  }
  uint32_t* hist16 = reinterpret_cast<uint32_t*>(smem + C::kOffHist);  // SEL: [NT][2048] words
  if constexpr (SEL) {
    for (int i = threadIdx.x; i < NT * (kSelBins / 2); i += C::kThreads) hist16[i] = 0u;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  uint32_t* consumed = reinterpret_cast<uint32_t*>(smem + C::kOffConsumed);  // [0] tiles, [1] queries
  const uint64_t wait_ns = p.wait_ns;
  int issued = min(nact, STAGES);  // thread 0: key tiles whose loads are issued
  if (warp == 0) {
    // ---------------- TMA producer
    if (lane == 0 && nact > 0) {
      for (int i = STAGES; i < nact; ++i) {
        const int s = i % STAGES, r = i / STAGES;
        if (!mbar_wait_bounded(BAR(C::kBarKEmpty + s), (r & 1) ^ 1, p.status, wait_ns)) break;
        const int pos0 = (tile_lo + i) * 128;
        mbar_arrive_expect_tx(BAR(C::kBarKFull + s), C::kStage);
        tma_load_4d(sbase + C::kOffK + s * C::kStage, &tm_k, 0, pos0, 0, kcache, BAR(C::kBarKFull + s));
        issued = i + 1;
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer
    if (lane == 0 && nact > 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, C::kNmma);
      bool ok = mbar_wait_bounded(BAR(C::kBarQ), 0, p.status, wait_ns);
      consumed[1] = ok ? 1u : 0u;
      consumed[0] = 0u;
      for (int i = 0; i < nact && ok; ++i) {
        const int s = i % STAGES, r = i / STAGES;
        if (!mbar_wait_bounded(BAR(C::kBarKFull + s), r & 1, p.status, wait_ns)) break;
        consumed[0] = (uint32_t)(i + 1);
        const uint32_t a_base = sbase + C::kOffK + s * C::kStage;
        // the whole tile in accumulator buffer i % 2
        const int slot = i % C::kNbuf;
        const int use = i / C::kNbuf;
        if (!mbar_wait_bounded(BAR(C::kBarAEmpty + slot), (use & 1) ^ 1, p.status, wait_ns)) break;
        tc_fence_after();
        const uint32_t d_base = tmem_base + (uint32_t)(slot * C::kN);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t koff = (uint32_t)(kk & 3) * 32u;  // 16 channels = 32 bytes inside the swizzled row
          const uint64_t adesc = sw128_kmajor_desc(a_base + (uint32_t)(kk >> 2) * C::kKHalf + koff);
#pragma unroll
          for (int j = 0; j < C::kNumMma; ++j) {
            const uint32_t b_addr = sbase + C::kOffQ + (uint32_t)(kk >> 2) * C::kQHalf +
                                    (uint32_t)(j * C::kNmma) * 128u + koff;
            mma_bf16_ss(d_base + (uint32_t)(j * C::kNmma), adesc, sw128_kmajor_desc(b_addr), idesc,
                        kk > 0 ? 1u : 0u);
          }
        }
        mma_commit(BAR(C::kBarAFull + slot));
        mma_commit(BAR(C::kBarKEmpty + s));
      }
    }
  } else {
    // ---------------- epilogue: 8 warps; TMEM lane quarter = warp % 4
    const int e = warp - 2;
    const int qd = warp & 3;
    const int hf = e >> 2;  // which half of the group's rows
    const int row = qd * 32 + lane;
    const uint32_t lane_addr = (uint32_t)(qd * 32) << 16;
    constexpr int TPH = (NT + 1) / 2;  // rows per epilogue half
    int vl[TPH];
#pragma unroll
    for (int j = 0; j < TPH; ++j) {
      const int tl = hf * TPH + j;
      const int t = t0 + tl;
      int v = 0;
      if (tl < NT && t < p.B) {
        v = p.valid_len ? p.valid_len[t] : p.S;
        v = v < 0 ? 0 : (v > p.S ? p.S : v);
      }
      vl[j] = v;
    }
    int done = nact;  // tiles scored: fewer once a wait has run out
    for (int i = 0; i < nact; ++i) {
      const int b = i % C::kNbuf;  // TMEM buffer of this tile
      const int slot = b;
      const int u = i / C::kNbuf;
      if (!mbar_wait_bounded(BAR(C::kBarAFull + slot), u & 1, p.status, wait_ns)) {  // status records it
        done = i;
        break;
      }
      tc_fence_after();
      const int s = (tile_lo + i) * 128 + row;
#pragma unroll
      for (int j = 0; j < TPH; ++j) {
        const int tl = hf * TPH + j;  // row inside the group
        if (tl >= NT) break;
        const uint32_t col = tmem_base + lane_addr + (uint32_t)(b * C::kN + tl * HP);
        uint32_t r[HP];
#pragma unroll
        for (int c = 0; c < HP; c += 16) tmem_ld16(col + (uint32_t)c, *reinterpret_cast<uint32_t(*)[16]>(r + c));
        tmem_wait_ld();
        float acc = 0.0f;
#pragma unroll
        for (int x = 0; x < HP; ++x) acc = fmaf(w_s[tl * HP + x], fmaxf(__uint_as_float(r[x]), 0.0f), acc);
        const int t = t0 + tl;
        if constexpr (SEL) {
          // valid positions: counted, and stored for the selection
          if (t < p.B && s < vl[j]) {
            const uint32_t bin = F32Keys::key(__float_as_uint(acc)) >> kSelShift;
            atomicAdd(hist16 + tl * (kSelBins / 2) + (bin >> 1), 1u << ((bin & 1u) << 4));
            p.out[(size_t)t * p.S + s] = acc;
          }
        } else {
          if (t < p.B && s < p.S) p.out[(size_t)t * p.S + s] = (s < vl[j]) ? acc : -INFINITY;
        }
      }
      tc_fence_before();
      __syncwarp();
      // (testing the failure detection: CTA 0's first epilogue warp may skip
      // its first release, so that the MMA warp's wait for this buffer runs out)
      const bool skip = p.fault == 1 && blockIdx.x == 0 && e == 0 && i == 0;
      if (lane == 0 && !skip) mbar_arrive(BAR(C::kBarAEmpty + slot));
    }
    // after a wait that ran out, the valid positions left still get a score:
    // -inf (counted too), so that the rows and their histograms stay in step
    if constexpr (SEL) {
      const uint32_t bin_ninf = F32Keys::key(__float_as_uint(-INFINITY)) >> kSelShift;
      for (int i = done; i < nact; ++i) {
        const int s = (tile_lo + i) * 128 + row;
#pragma unroll
        for (int j = 0; j < TPH; ++j) {
          const int tl = hf * TPH + j;
          const int t = t0 + tl;
          if (tl < NT && t < p.B && s < vl[j]) {
            atomicAdd(hist16 + tl * (kSelBins / 2) + (bin_ninf >> 1), 1u << ((bin_ninf & 1u) << 4));
            p.out[(size_t)t * p.S + s] = -INFINITY;
          }
        }
      }
    }
    // tiles past the group's valid lengths (and, after a wait that ran out,
    // the tiles left): no products, -inf (the selection never reads them)
    for (int tile = tile_lo + done; !SEL && tile < tile_hi; ++tile) {
      const int s = tile * 128 + row;
#pragma unroll
      for (int j = 0; j < TPH; ++j) {
        const int tl = hf * TPH + j;
        const int t = t0 + tl;
        if (tl < NT && t < p.B && s < p.S) p.out[(size_t)t * p.S + s] = -INFINITY;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // after a wait that ran out, key tiles (or the queries) may still be on
  // their way into shared memory: wait for them (bounded) before the CTA ends
  if (threadIdx.x == 0 && nact > 0) {
    if (consumed[1] == 0u) mbar_wait_bounded(BAR(C::kBarQ), 0, p.status, wait_ns);
    for (int j = (int)consumed[0]; j < issued; ++j)
      mbar_wait_bounded(BAR(C::kBarKFull + j % STAGES), (uint32_t)((j / STAGES) & 1), p.status, wait_ns);
  }
  if (warp == 1) tmem_dealloc(tmem_base, C::kTmemCols);
  if constexpr (SEL) {
    // every score is counted: add this CTA's counts into the rows' global
    // histograms (the selection kernel reads them once this grid has finished)
    for (int tl = 0; tl < NT && t0 + tl < p.B; ++tl) {
      uint32_t* gh = p.ghist + (size_t)(t0 + tl) * kSelBins;
      for (int i = threadIdx.x; i < kSelBins / 2; i += C::kThreads) {
        const uint32_t v = hist16[tl * (kSelBins / 2) + i];
        if (v & 0xFFFFu) atomicAdd(gh + 2 * i, v & 0xFFFFu);
        if (v >> 16) atomicAdd(gh + 2 * i + 1, v >> 16);
      }
    }
  }
  // the next kernel (the selection over these rows) may launch only now:
  // launched earlier its CTAs would crowd onto the few SMs this grid leaves free
  pdl_launch_dependents();
}

}  // namespace dstopk
