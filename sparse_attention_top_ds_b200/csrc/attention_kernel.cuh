// attention_kernel.cuh -- multi-query decode attention over the selected
// compressed rows plus a sliding window, on the tcgen05 tensor cores.
//
// What it computes (NKI pull request "Add DeepSeek-V4 CSA attention kernels",
// "How the algorithm works" and steps table row 4 "Concatenate and attend";
// K and V are one embedding, "The top-k on the GPSIMD engine"): for batch row
// b and query head h, over the attended rows r (the selected cache rows, then
// the window rows),
//     out[b,h,:] = sum_r e^{z_r} row_r / (sum_r e^{z_r} + e^{sink_h}),
//     z_r = scale * (q[b,h,:] . row_r),   lse[b,h] = log of the denominator.
//
// How (B200 design).  Every batch row has 128 heads that share the same rows,
// so both products are dense: S = Q . R^T (M = heads, N = rows, K = d) and
// O = P . R (M = heads, N = d, K = rows).  Splitting the rows over CTAs would
// leave a float32 partial O of heads x d per CTA -- for d = 512 four times
// the bytes of the rows themselves -- so the two products are split
// differently, in two launches joined by programmatic dependent launch:
//  * score kernel: a CTA owns a batch row, a tile of 128 heads and a chunk of
//    64 attended slots.  The queries arrive by TMA (128-byte swizzle), the 64
//    rows are gathered with cp.async straight into the same layout, S goes to
//    TMEM, and four softmax warps (a TMEM lane per head) turn it into the
//    chunk's weights 2^(z - max_chunk) in bf16.  The weight tile (16 KiB,
//    already in the MMA operand layout) goes back to global memory with one
//    bulk copy, with the chunk's (max, sum) per head.
//  * weighted-sum kernel: a CTA owns a batch row, a tile of 128 heads and a
//    64-column slice of d.  It reads the (max, sum) of every chunk of the row,
//    so it knows the row's softmax maximum and normaliser, then streams the
//    chunks through a ring: the weight tile by bulk copy, the 64-column slice
//    of the chunk's rows by cp.async (the rows are in L2 from the score
//    kernel).  Each weight row is rescaled in place by 2^(max_chunk - max)/sum
//    and O_slice += P . R_slice runs on the tensor cores, the row slice being
//    the MN-major B operand.  The accumulator is the final output: it is
//    rounded to bf16 and written, with lse, and no combine pass is needed.
#pragma once

#include <cuda.h>

#include "ptx.cuh"
#include "tcgen05.cuh"

namespace dstopk {

constexpr int kAttnRows = 64;       // attended slots per chunk (N of S = Q . R^T)
constexpr int kAttnHeads = 128;     // query heads per CTA (M of both products)
constexpr int kAttnThreads = 256;   // score kernel: 8 warps
constexpr int kAttnMaxD = 512;
constexpr int kAttnTile = kAttnHeads * kAttnRows * 2;  // bytes of one chunk's bf16 weight tile
constexpr int kPvSlice = 64;        // weighted-sum kernel: output columns per CTA

struct AttnParams {
  const uint16_t* kv;      // bf16 compressed caches
  long long kv_bstride;    // elements from one batch row's cache to the next
  const uint16_t* win;     // bf16 [B, W, D] or null
  const int32_t* idx;      // [B, k] or null
  const int32_t* win_len;  // [B] or null
  const float* sink;       // [H] or null
  uint8_t* ptile;          // [B][HT][NS] weight tiles of kAttnTile bytes
  uint8_t* vtile;          // [B][D/64][NS] row tiles: the chunk's 64 rows, one 64-column block, 8 KiB
  float2* ml;              // [B][HT][NS][128]: (chunk max in log2 units, sum of the chunk's weights)
  uint16_t* out;           // bf16 [B, H, D]
  float* lse;              // [B, H] or null
  int* status;
  uint64_t wait_ns;        // limit of every bounded wait (0: the library default)
  int T, k, W, B, H, D, HT, NS;
  float scale_log2;        // scale * log2(e)
};

// Where slot j of batch row b reads its row from; null if the slot is skipped.
__device__ __forceinline__ const uint16_t* attn_row_src(const AttnParams& p, int b, int j) {
  if (j < p.k) {
    const int r = p.idx[(size_t)b * p.k + j];
    debug_range(r >= -1 && r < p.T, p.status);
    if (r >= 0 && r < p.T) return p.kv + (long long)b * p.kv_bstride + (long long)r * p.D;
  } else if (j < p.k + p.W) {
    int wl = p.win_len ? p.win_len[b] : p.W;
    debug_range(wl >= 0 && wl <= p.W, p.status);
    wl = wl < 0 ? 0 : (wl > p.W ? p.W : wl);
    const int i = j - p.k;
    if (i < wl) return p.win + ((long long)b * p.W + i) * p.D;
  }
  return nullptr;
}

// Pack two floats into bf16x2, round to nearest even: `lo` in the low half.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t u;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(u) : "f"(hi), "f"(lo));
  return u;
}

// ------------------------------------------------------------------ score kernel

constexpr int kRowTile = kAttnRows * 128;  // bytes of one chunk's rows in one 64-column block

// Shared-memory layout for head_dim D (byte offsets from a 1024-aligned base):
// queries D/64 blocks of 128 rows x 128 B | rows D/64 blocks of 64 x 128 B |
// row flags (64 B) | mbarriers: queries, S | TMEM slot.
struct AttnSmem {
  __host__ __device__ static constexpr int q_off() { return 0; }
  __host__ __device__ static constexpr int kv_off(int D) { return (D / 64) * 16384; }
  __host__ __device__ static constexpr int flag_off(int D) { return kv_off(D) + (D / 64) * kRowTile; }
  __host__ __device__ static constexpr int bar_off(int D) { return flag_off(D) + kAttnRows; }
  __host__ __device__ static constexpr int slot_off(int D) { return bar_off(D) + 16; }
  __host__ __device__ static constexpr int bytes(int D) { return slot_off(D) + 16 + 1024; }  // + alignment slack
};

// tm_q views the queries [rows][D] as (64 channels, rows, D/64 blocks), so one
// box of (64, 128, D/64) lands in shared memory block by block, each block
// 128 rows x 128 B in the 128-byte-swizzled layout.
__global__ void __launch_bounds__(kAttnThreads, 1)
    sparse_attn_score_kernel(const __grid_constant__ CUtensorMap tm_q, const AttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const int D = p.D, DB = D >> 6;
  const uint32_t q_s = sbase + AttnSmem::q_off();
  const uint32_t kv_s = sbase + AttnSmem::kv_off(D);
  uint8_t* flags = smem + AttnSmem::flag_off(D);
  const uint32_t bar_q = sbase + AttnSmem::bar_off(D);
  const uint32_t bar_s = bar_q + 8;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + AttnSmem::slot_off(D));

  const int split = blockIdx.x, ht = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  constexpr uint32_t kCols = 64;

  if (tid == 0) {
    mbar_init(bar_q, 1);
    mbar_init(bar_s, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), kCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // the slots (and the queries) may be written by the kernel just before this one
  pdl_wait();
  // let the weighted-sum kernel launch now: its CTAs take SMs as these exit,
  // and wait (griddepcontrol.wait) for this whole grid before reading
  pdl_launch_dependents();
  if (tid == 0) {
    mbar_arrive_expect_tx(bar_q, (uint32_t)DB * 16384u);
    tma_load_3d(q_s, &tm_q, 0, b * p.H + ht * kAttnHeads, 0, bar_q);
  }
  // gather: thread t moves 16-byte piece c8 = t % 8 of rows t / 8 and t / 8 + 32
  // of every 64-column block, all loads in flight at once, into the swizzled
  // layout (piece c8 of row r goes to position c8 ^ (r & 7) of the row's 128
  // bytes); skipped rows become zeros.  The first head tile also stores each
  // block's row tile for the weighted-sum kernel.
  {
    const int r0 = tid >> 3, r1 = r0 + 32, c8 = tid & 7;
    const uint16_t* s0 = attn_row_src(p, b, split * kAttnRows + r0);
    const uint16_t* s1 = attn_row_src(p, b, split * kAttnRows + r1);
    if (c8 == 0) {
      flags[r0] = s0 != nullptr;
      flags[r1] = s1 != nullptr;
    }
    uint4 v0[kAttnMaxD / 64], v1[kAttnMaxD / 64];
#pragma unroll
    for (int db = 0; db < kAttnMaxD / 64; ++db) {
      if (db < DB) {
        v0[db] = s0 ? __ldcg(reinterpret_cast<const uint4*>(s0 + db * 64 + c8 * 8)) : make_uint4(0, 0, 0, 0);
        v1[db] = s1 ? __ldcg(reinterpret_cast<const uint4*>(s1 + db * 64 + c8 * 8)) : make_uint4(0, 0, 0, 0);
      }
    }
    const uint32_t o0 = (uint32_t)r0 * 128u + ((uint32_t)(c8 ^ (r0 & 7)) << 4);
    const uint32_t o1 = (uint32_t)r1 * 128u + ((uint32_t)(c8 ^ (r1 & 7)) << 4);
    uint8_t* vt = (ht == 0) ? p.vtile + ((size_t)b * DB * p.NS + split) * kRowTile : nullptr;
#pragma unroll
    for (int db = 0; db < kAttnMaxD / 64; ++db) {
      if (db < DB) {
        sts128(kv_s + (uint32_t)db * kRowTile + o0, v0[db]);
        sts128(kv_s + (uint32_t)db * kRowTile + o1, v1[db]);
        if (vt) {
          uint8_t* t = vt + (size_t)db * p.NS * kRowTile;
          *reinterpret_cast<uint4*>(t + o0) = v0[db];
          *reinterpret_cast<uint4*>(t + o1) = v1[db];
        }
      }
    }
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();

  // ---- S = Q . R^T into TMEM columns [0, 64)
  if (tid == 0) {
    const bool ok = mbar_wait_bounded(bar_q, 0, p.status, p.wait_ns);
    tc_fence_after();
    if (ok) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, kAttnRows);
      // the start address is the descriptor's low field (in 16-byte units), so
      // moving through the tiles is an add on the first descriptor
      const uint64_t a0 = sw128_kmajor_desc(q_s), b0 = sw128_kmajor_desc(kv_s);
      for (int db = 0; db < DB; ++db) {
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_bf16_ss(tmem, a0 + (uint64_t)((db * 16384 + kk * 32) >> 4), b0 + (uint64_t)((db * kRowTile + kk * 32) >> 4),
                      idesc, (db | kk) != 0 ? 1u : 0u);
      }
    }
    mma_commit(bar_s);  // arrives even when nothing was issued, so that no one waits for ever
  }

  // ---- the chunk's weights: all 8 warps, TMEM lane = head (lane quarter =
  // warp % 4), warps 0..3 taking rows 0..31 of the chunk and warps 4..7 rows
  // 32..63; the two halves of a head swap their maxima and sums through shared
  // memory.  Each thread writes its half of the head's 128-byte row of the
  // tile straight to global memory, in the swizzled order the weighted-sum
  // kernel's MMAs read.
  const size_t chunk = ((size_t)b * p.HT + ht) * p.NS + split;
  {
    const int half = warp >> 2;
    const int h = (warp & 3) * 32 + lane;
    float* xch = reinterpret_cast<float*>(smem + AttnSmem::kv_off(D));  // the row tiles are no longer read
    mbar_wait_bounded(bar_s, 0, p.status, p.wait_ns);
    __syncwarp();
    tc_fence_after();
    const uint32_t taddr = tmem + ((uint32_t)((warp & 3) * 32) << 16) + (uint32_t)(half * 32);
    uint32_t r[32];
    tmem_ld16(taddr, *reinterpret_cast<uint32_t(*)[16]>(r));
    tmem_ld16(taddr + 16u, *reinterpret_cast<uint32_t(*)[16]>(r + 16));
    const uint4 fa = *reinterpret_cast<const uint4*>(flags + half * 32);
    const uint4 fb = *reinterpret_cast<const uint4*>(flags + half * 32 + 16);
    const uint32_t fw[8] = {fa.x, fa.y, fa.z, fa.w, fb.x, fb.y, fb.z, fb.w};
    tmem_wait_ld();
    float z[32];
    float m = -INFINITY;
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const bool v = ((fw[j >> 2] >> ((j & 3) * 8)) & 0xffu) != 0;
      z[j] = v ? __uint_as_float(r[j]) * p.scale_log2 : -INFINITY;
      m = fmaxf(m, z[j]);
    }
    xch[half * kAttnHeads + h] = m;
    named_bar_sync(1, kAttnThreads);
    m = fmaxf(m, xch[(1 - half) * kAttnHeads + h]);
    const float mu = m == -INFINITY ? 0.0f : m;  // exp2(-inf - mu) = 0 for every skipped row
    float l = 0.0f;
    uint4* trow = reinterpret_cast<uint4*>(p.ptile + chunk * (size_t)kAttnTile + (size_t)h * 128u);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      uint32_t pk[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int j = c * 8 + i * 2;
        const uint32_t u = pack_bf16x2(exp2f(z[j] - mu), exp2f(z[j + 1] - mu));
        l += __uint_as_float(u << 16) + __uint_as_float(u & 0xffff0000u);
        pk[i] = u;
      }
      trow[(half * 4 + c) ^ (h & 7)] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
    }
    xch[2 * kAttnHeads + half * kAttnHeads + h] = l;
    named_bar_sync(1, kAttnThreads);
    if (half == 0) p.ml[chunk * kAttnHeads + h] = make_float2(m, l + xch[3 * kAttnHeads + h]);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kCols);
  }
}

// ------------------------------------------------------------------ weighted-sum kernel

// Warp roles: lane 0 of warp 0 loads; warps 1..8 rescale the weight rows (two
// threads per head, half a row each) and later read the accumulator; warp 9
// owns TMEM and issues the MMAs from one thread.  A ring stage holds K
// consecutive chunks: their weight tiles (K x 16 KiB) and their row tiles for
// this CTA's 64 columns (K x 8 KiB), each a contiguous run in global memory
// fetched by one bulk copy (large copies keep the copy engine near its peak).
// Stages pass full -> ready -> empty through mbarriers, so no CTA-wide
// barrier sits in the loop.
//
// With G = 2 the chunks of a batch row are split between the two CTAs of a
// cluster.  Both know the row's softmax maximum and normaliser, so their two
// accumulators are partial sums of the same normalised output: each CTA sends
// the partner the 32 columns the partner finalises, by st.async into the
// partner's shared memory completing on the partner's mbarrier, and each
// writes 32 columns.
constexpr int kPvWarps = 10;
constexpr int kPvRescale = 256;  // rescaling threads (warps 1..8)
// K chunks per ring stage, S ring stages
template <int K, int S>
struct PvSmem {
  static constexpr int kStage = K * (kAttnTile + kRowTile);
  // ring | partner's columns (128 heads x 32 floats) | (max, sum) of every chunk
  // of the row | mbarriers full[S], ready[S], empty[S], ml, done, recv | TMEM slot
  __host__ __device__ static constexpr int recv_off() { return S * kStage; }
  __host__ __device__ static constexpr int ml_off() { return recv_off() + kAttnHeads * 32 * 4; }
  __host__ __device__ static constexpr int bar_off(int NS) { return ml_off() + NS * kAttnHeads * 8; }
  __host__ __device__ static constexpr int slot_off(int NS) { return bar_off(NS) + (3 * S + 3) * 8; }
  __host__ __device__ static constexpr int bytes(int NS) { return slot_off(NS) + 16 + 1024; }
};

// Columns [LO, LO + 32) of one head's accumulator, held as r[0..31]:
// optionally add the partner's share from `recv` (the head's 128 bytes, whose
// 16-byte piece i sits at position i ^ sw), round to bf16 and store.
template <bool ADD>
__device__ __forceinline__ void pv_emit(const uint32_t (&r)[32], const float* recv, int sw, uint16_t* dst) {
  uint4* d4 = reinterpret_cast<uint4*>(dst);
  const float4* r4 = reinterpret_cast<const float4*>(recv);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    float a[8] = {0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f};
    if (ADD) {
      const float4 x = r4[(2 * q) ^ sw], y = r4[(2 * q + 1) ^ sw];
      a[0] = x.x, a[1] = x.y, a[2] = x.z, a[3] = x.w, a[4] = y.x, a[5] = y.y, a[6] = y.z, a[7] = y.w;
    }
    float v[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) v[e] = __uint_as_float(r[8 * q + e]) + a[e];
    d4[q] = make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                       pack_bf16x2(v[6], v[7]));
  }
}

template <int K, int S>
__global__ void __launch_bounds__(kPvWarps * 32, 1) sparse_attn_pv_kernel(const AttnParams p) {
  using L_ = PvSmem<K, S>;
  constexpr int kPvStages = S;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const int NS = p.NS;
  const int G = gridDim.y, g = blockIdx.y;  // chunk group = rank in the cluster
  const int NSg = (NS + G - 1) / G;
  const int c0 = g * NSg, nmine = max(0, min(NS, c0 + NSg) - c0);
  const int nstage = (nmine + K - 1) / K;   // ring uses of this CTA
  const float2* ml_s = reinterpret_cast<const float2*>(smem + L_::ml_off());
  float* recv = reinterpret_cast<float*>(smem + L_::recv_off());
  const uint32_t full0 = sbase + L_::bar_off(NS);
  const uint32_t ready0 = full0 + 8u * kPvStages, empty0 = ready0 + 8u * kPvStages;
  const uint32_t bar_ml = empty0 + 8u * kPvStages, bar_done = bar_ml + 8u, bar_recv = bar_done + 8u;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L_::slot_off(NS));
  const int slice = blockIdx.x, ht = blockIdx.z % p.HT, b = blockIdx.z / p.HT;
  const int DB = p.D >> 6;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  constexpr uint32_t kCols = kPvSlice;
  constexpr float kLog2e = 1.4426950408889634f;
  constexpr float kLn2 = 0.6931471805599453f;

  if (tid == 0) {
    for (int s = 0; s < kPvStages; ++s) {
      mbar_init(full0 + 8u * s, 1);             // the producer's expect_tx
      mbar_init(ready0 + 8u * s, kPvRescale);   // the rescaling threads
      mbar_init(empty0 + 8u * s, 1);            // the MMAs' commit
    }
    mbar_init(bar_ml, 1);
    mbar_init(bar_done, 1);
    mbar_init(bar_recv, 1);
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(smem_u32(tmem_slot), kCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (G == 2) cluster_sync();  // the partner's mbarriers exist before anything targets them
  const uint32_t tmem = *tmem_slot;
  pdl_wait();  // the tiles and statistics come from the score kernel

  const size_t row0 = ((size_t)b * p.HT + ht) * NS;          // this row's first weight tile
  const size_t vrow0 = ((size_t)b * DB + slice) * NS;         // this row's first row tile of this slice
  float M = -INFINITY, L = 0.0f;  // head h's softmax maximum and normaliser (warps 1..8)
  // warps 1..8 own half a head row per thread; a warp may only read its TMEM
  // lane quarter (warp % 4), so warp w takes heads 32 (w % 4) .. + 31, and
  // warps 1..4 the first half of each row, warps 5..8 the second
  const int h = ((warp & 3) << 5) | lane;
  const int half = (warp - 1) >> 2;
  if (warp == 0) {
    // ---------------- producer
    if (lane == 0) {
      if (NS > 0) {
        const uint32_t bytes = (uint32_t)NS * kAttnHeads * 8u;
        mbar_arrive_expect_tx(bar_ml, bytes);
        bulk_g2s(sbase + L_::ml_off(), p.ml + row0 * kAttnHeads, bytes, bar_ml);
      }
      for (int j = 0; j < nstage; ++j) {
        const int s = j % kPvStages;
        const int c = c0 + j * K, n = min(K, c0 + nmine - c);
        if (j >= kPvStages)
          mbar_wait_bounded(empty0 + 8u * s, (uint32_t)((j / kPvStages - 1) & 1), p.status, p.wait_ns);
        const uint32_t st = sbase + (uint32_t)s * L_::kStage;
        mbar_arrive_expect_tx(full0 + 8u * s, (uint32_t)n * (kAttnTile + kRowTile));
        bulk_g2s(st, p.ptile + (row0 + c) * (size_t)kAttnTile, (uint32_t)n * kAttnTile, full0 + 8u * s);
        bulk_g2s(st + (uint32_t)K * kAttnTile, p.vtile + (vrow0 + c) * (size_t)kRowTile, (uint32_t)n * kRowTile,
                 full0 + 8u * s);
      }
    }
  } else if (warp <= 8) {
    // ---------------- rescaling: head h's weights of every chunk, to the row's
    // maximum and normaliser.  Every 16-byte piece of a row takes the same
    // factor, so the thread visits its pieces in the order q ^ (h % 8): eight
    // consecutive heads then touch eight different bank groups.
    const int hg = ht * kAttnHeads + h;
    const float sink_l2 = (p.sink && hg < p.H) ? p.sink[hg] * kLog2e : -INFINITY;
    M = sink_l2;
    if (NS > 0) mbar_wait_bounded(bar_ml, 0, p.status, p.wait_ns);
    for (int c = 0; c < NS; ++c) {
      const float2 v = ml_s[c * kAttnHeads + h];
      if (v.y > 0.0f) M = fmaxf(M, v.x);
    }
    if (M > -INFINITY && sink_l2 > -INFINITY) L = exp2f(sink_l2 - M);
    for (int c = 0; c < NS; ++c) {
      const float2 v = ml_s[c * kAttnHeads + h];
      if (v.y > 0.0f) L = fmaf(v.y, exp2f(v.x - M), L);
    }
    const float invL = L > 0.0f ? 1.0f / L : 0.0f;
    for (int j = 0; j < nstage; ++j) {
      const int s = j % kPvStages;
      const int c = c0 + j * K, n = min(K, c0 + nmine - c);
      mbar_wait_bounded(full0 + 8u * s, (uint32_t)((j / kPvStages) & 1), p.status, p.wait_ns);
      for (int t = 0; t < n; ++t) {
        const float2 v = ml_s[(c + t) * kAttnHeads + h];
        const float f = v.y > 0.0f ? exp2f(v.x - M) * invL : 0.0f;
        const uint32_t prow = sbase + (uint32_t)s * L_::kStage + (uint32_t)t * kAttnTile + (uint32_t)h * 128u;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint32_t a = prow + ((uint32_t)((half * 4 + q) ^ (h & 7)) << 4);
          uint4 x = lds128(a);
          uint32_t* w = reinterpret_cast<uint32_t*>(&x);
#pragma unroll
          for (int e = 0; e < 4; ++e)
            w[e] = pack_bf16x2(__uint_as_float(w[e] << 16) * f, __uint_as_float(w[e] & 0xffff0000u) * f);
          sts128(a, x);
        }
      }
      fence_proxy_async_smem();
      mbar_arrive(ready0 + 8u * s);
    }
  } else if (lane == 0) {
    // ---------------- MMA issuer: O_slice += P'_chunk . R_slice
    constexpr uint32_t idesc = idesc_bf16_f32(128, kPvSlice) | (1u << 16);  // B is MN-major
    for (int j = 0; j < nstage; ++j) {
      const int s = j % kPvStages;
      const int n = min(K, c0 + nmine - (c0 + j * K));
      mbar_wait_bounded(ready0 + 8u * s, (uint32_t)((j / kPvStages) & 1), p.status, p.wait_ns);
      fence_proxy_async_smem();
      tc_fence_after();
      const uint32_t st = sbase + (uint32_t)s * L_::kStage;
      const uint64_t a0 = sw128_kmajor_desc(st), b0 = sw128_mnmajor_desc(st + (uint32_t)K * kAttnTile, 8192u, 1024u);
      for (int t = 0; t < n; ++t) {
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_bf16_ss(tmem, a0 + (uint64_t)((t * kAttnTile + kk * 32) >> 4), b0 + (uint64_t)((t * kRowTile + kk * 2048) >> 4),
                      idesc, (j | t | kk) != 0 ? 1u : 0u);
      }
      mma_commit(empty0 + 8u * s);
    }
    mma_commit(bar_done);  // after every MMA above (or at once if there were none)
  }

  // ---- epilogue: warps 1..8, thread (h, half) holds columns [32 half, 32 half + 32)
  if (warp >= 1 && warp <= 8) {
    uint32_t r[32];
    if (nmine > 0) {
      mbar_wait_bounded(bar_done, 0, p.status, p.wait_ns);
      __syncwarp();
      tc_fence_after();
      const uint32_t taddr = tmem + ((uint32_t)((warp & 3) * 32) << 16) + (uint32_t)(half * 32);
      tmem_ld16(taddr, *reinterpret_cast<uint32_t(*)[16]>(r));
      tmem_ld16(taddr + 16u, *reinterpret_cast<uint32_t(*)[16]>(r + 16));
      tmem_wait_ld();
    } else {
#pragma unroll
      for (int i = 0; i < 32; ++i) r[i] = 0u;
    }
    const int hg = ht * kAttnHeads + h;
    uint16_t* orow = p.out + ((size_t)b * p.H + hg) * p.D + (size_t)slice * kPvSlice + half * 32;
    if (G == 2) {
      if (half != g) {
        // these 32 columns are finalised by the partner (CTA `half` of the pair);
        // piece q goes to position q ^ (h % 8) of the head's 128 bytes, so that
        // eight consecutive heads write (and later read) eight bank groups
        const uint32_t dst = dsmem_map(smem_u32(recv + h * 32), (uint32_t)half);
        const uint32_t rbar = dsmem_map(bar_recv, (uint32_t)half);
#pragma unroll
        for (int q = 0; q < 8; ++q)
          asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.b32 [%0], {%1, %2, %3, %4}, [%5];" ::
                           "r"(dst + 16u * (uint32_t)(q ^ (h & 7))), "r"(r[4 * q]), "r"(r[4 * q + 1]), "r"(r[4 * q + 2]),
                       "r"(r[4 * q + 3]),
                       "r"(rbar)
                       : "memory");
      } else {
        if (h == 0) mbar_arrive_expect_tx(bar_recv, kAttnHeads * 32 * 4);  // 128 heads x 32 columns from the partner
        mbar_wait_bounded(bar_recv, 0, p.status, p.wait_ns);
        if (hg < p.H) pv_emit<true>(r, recv + h * 32, h & 7, orow);
      }
    } else if (hg < p.H) {
      pv_emit<false>(r, recv, 0, orow);
    }
    if (half == 0 && hg < p.H && slice == 0 && g == 0 && p.lse)
      p.lse[(size_t)b * p.H + hg] = L > 0.0f ? (M + log2f(L)) * kLn2 : -INFINITY;
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, kCols);
  }
  pdl_launch_dependents();
}

}  // namespace dstopk
