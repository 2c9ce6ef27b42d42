// qproj_kernel.cuh -- the indexer query projection as a GEMV on the CUDA cores.
//
// What it computes (NKI pull request "Add DeepSeek-V4 CSA attention kernels",
// "How the algorithm works", steps table row 2: the indexer query is projected
// into 128 channels per head; the launch list runs that projection as a GEMV
// ahead of the scoring launch):
//     q[t, n] = sum_i x[t, i] * Wq[n, i]     n < heads * 128, rounded to bf16
//     w[t, h] = sum_i x[t, i] * Ww[h, i]     h < heads, float32
// with float32 accumulation of the exact bf16 products.
//
// How (B200 design).  For a decode step (a handful of tokens) every weight is
// used by at most 8 tokens: the op streams the weight matrix from HBM once and
// is bound by HBM, so it runs on the CUDA cores, not the tensor cores.
//  * A warp owns 4 output rows (weight rows); its 32 lanes split the input
//    width in 16-byte pieces (8 channels), lane l taking pieces l, l + 32, ...
//    A lane has every weight piece of a 6-piece block in flight at once
//    (4 rows x 6 x 16 B), so an SM has ~100 KB of weight loads outstanding.
//  * The group's 8 token rows sit in shared memory; a lane reads the 8 token
//    pieces at its position once per block and uses them for all 4 rows.
//  * The products go through Blackwell's packed fma.rn.f32x2: one instruction
//    accumulates two consecutive channels of the same (row, token) into a
//    pair of partial sums.
//  * The 32 lanes' partial sums are reduced through a per-warp transpose in
//    shared memory: lane l ends with the sum of (row l / 8, token l % 8).
//  * More than 8 tokens run as groups of 8 (grid y); each group streams the
//    weights again, from L2 after the first.
#pragma once

#include <cuda_runtime.h>

#include "ptx.cuh"

namespace dstopk {

constexpr int kQpThreads = 256;  // 8 warps
constexpr int kQpRows = 4;       // weight rows per warp task
constexpr int kQpTok = 8;        // tokens per group
constexpr int kQpBlock = 6;      // 16-byte pieces per lane per block of the input width
constexpr int kQpMaxIn = 8192;   // largest input width (shared memory holds 8 token rows)

struct QpParams {
  const uint16_t* x;   // bf16 [T, d_in]
  const uint16_t* wq;  // bf16 [heads * 128, d_in]
  const uint16_t* ww;  // bf16 [heads, d_in] or null
  uint16_t* q;         // bf16 [T, heads * 128]
  float* w;            // f32 [T, heads] or null
  int T, d_in, nq, nrows;  // nq = heads * 128; nrows = nq (+ heads with ww)
  int heads;
};

// d = a * b + d on two float32 lanes at once.
__device__ __forceinline__ void ffma2(float2& d, float2 a, float2 b) {
  uint64_t dd = (uint64_t)__float_as_uint(d.x) | ((uint64_t)__float_as_uint(d.y) << 32);
  const uint64_t aa = (uint64_t)__float_as_uint(a.x) | ((uint64_t)__float_as_uint(a.y) << 32);
  const uint64_t bb = (uint64_t)__float_as_uint(b.x) | ((uint64_t)__float_as_uint(b.y) << 32);
  asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(dd) : "l"(aa), "l"(bb));
  d.x = __uint_as_float((uint32_t)dd);
  d.y = __uint_as_float((uint32_t)(dd >> 32));
}

// The two bf16 of a packed pair, widened exactly to float32.
__device__ __forceinline__ float2 bf16x2_f32(uint32_t u) {
  return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xffff0000u));
}

__device__ __forceinline__ uint32_t qp_round_bf16(float v) {
  uint32_t u;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(u) : "f"(0.0f), "f"(v));
  return u & 0xffffu;
}

__global__ void __launch_bounds__(kQpThreads) indexer_qproj_kernel(const QpParams p) {
  extern __shared__ __align__(16) uint8_t qp_smem[];
  uint16_t* xs = reinterpret_cast<uint16_t*>(qp_smem);                       // [8][d_in]
  float* red = reinterpret_cast<float*>(qp_smem + (size_t)kQpTok * p.d_in * 2);  // [8 warps][32][33]
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int t0 = blockIdx.y * kQpTok;
  const int ntok = min(kQpTok, p.T - t0);
  const int npieces = p.d_in >> 3;  // 16-byte pieces per row

  pdl_wait();  // x may come from the kernel just before this one
  // the group's token rows (zeros past the last token)
  {
    const uint4* src = reinterpret_cast<const uint4*>(p.x + (size_t)t0 * p.d_in);
    uint4* dst = reinterpret_cast<uint4*>(xs);
    for (int i = tid; i < kQpTok * npieces; i += kQpThreads)
      dst[i] = (i / npieces < ntok) ? __ldg(src + i) : make_uint4(0, 0, 0, 0);
  }
  __syncthreads();

  float* wred = red + warp * 32 * 33;
  const int ntasks = (p.nrows + kQpRows - 1) / kQpRows;
  for (int task = blockIdx.x * 8 + warp; task < ntasks; task += gridDim.x * 8) {
    const int r0 = task * kQpRows;
    const uint4* wrow[kQpRows];
#pragma unroll
    for (int r = 0; r < kQpRows; ++r) {
      const int n = min(r0 + r, p.nrows - 1);  // rows past the end repeat the last one (not stored)
      wrow[r] = reinterpret_cast<const uint4*>(n < p.nq ? p.wq + (size_t)n * p.d_in : p.ww + (size_t)(n - p.nq) * p.d_in);
    }
    float2 acc[kQpRows][kQpTok];
#pragma unroll
    for (int r = 0; r < kQpRows; ++r)
#pragma unroll
      for (int t = 0; t < kQpTok; ++t) acc[r][t] = make_float2(0.0f, 0.0f);

    for (int base = lane; base < npieces; base += 32 * kQpBlock) {
      uint4 wv[kQpBlock][kQpRows];
#pragma unroll
      for (int j = 0; j < kQpBlock; ++j) {
        const int c = base + 32 * j;
#pragma unroll
        for (int r = 0; r < kQpRows; ++r)
          wv[j][r] = c < npieces ? __ldcg(wrow[r] + c) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int j = 0; j < kQpBlock; ++j) {
        const int c = base + 32 * j;
        if (c >= npieces) break;
#pragma unroll
        for (int t = 0; t < kQpTok; ++t) {
          const uint4 xv = reinterpret_cast<const uint4*>(xs + (size_t)t * p.d_in)[c];
          const float2 x0 = bf16x2_f32(xv.x), x1 = bf16x2_f32(xv.y), x2 = bf16x2_f32(xv.z), x3 = bf16x2_f32(xv.w);
#pragma unroll
          for (int r = 0; r < kQpRows; ++r) {
            ffma2(acc[r][t], bf16x2_f32(wv[j][r].x), x0);
            ffma2(acc[r][t], bf16x2_f32(wv[j][r].y), x1);
            ffma2(acc[r][t], bf16x2_f32(wv[j][r].z), x2);
            ffma2(acc[r][t], bf16x2_f32(wv[j][r].w), x3);
          }
        }
      }
    }
    // reduce over the 32 lanes: lane l ends with (row l / 8, token l % 8)
#pragma unroll
    for (int r = 0; r < kQpRows; ++r)
#pragma unroll
      for (int t = 0; t < kQpTok; ++t) wred[lane * 33 + r * kQpTok + t] = acc[r][t].x + acc[r][t].y;
    __syncwarp();
    float sum = 0.0f;
#pragma unroll 8
    for (int l = 0; l < 32; ++l) sum += wred[l * 33 + lane];
    __syncwarp();
    const int n = r0 + (lane >> 3), t = lane & 7;
    if (n < p.nrows && t < ntok) {
      if (n < p.nq) p.q[(size_t)(t0 + t) * p.nq + n] = (uint16_t)qp_round_bf16(sum);
      else p.w[(size_t)(t0 + t) * p.heads + (n - p.nq)] = sum;
    }
  }
  pdl_launch_dependents();
}

}  // namespace dstopk

#include "tcgen05.cuh"

namespace dstopk {

// ------------------------------------------------------------------ tensor-core projection
//
// For input widths that are a multiple of 64 the products run on the tcgen05
// tensor cores, fed by TMA: D[row, token] = W[row, :] . x[token, :] with
// M = 128 weight rows per CTA, N = 16 tokens (one token group) and K = the
// input width.  The weights stream from HBM in 3-D TMA boxes of up to
// 4 x 64 channels x 128 rows (64 KiB: large copies keep the copy engine near
// its peak), every box of a CTA in flight at once through a 3-stage ring; the
// 16 token rows come with each box.  One MMA does 128 x 16 x 16 products, so
// the CUDA cores only issue copies and MMAs.  (Measured on this GPU: the same
// kernel fed by ld.global.v4 from 512 threads, the whole 192 KiB block in
// flight, took 14 us per launch against 10-11 us with TMA.)  A cluster pair
// splits the input width (G = 2) when one CTA per row block would leave most
// SMs idle; each CTA then finalises 64 of the 128 rows, receiving the
// partner's partial sums by st.async.  The per-head weight rows (Ww) form one
// more row block.
constexpr int kQtStages = 3;
constexpr int kQtTok = 16;                         // tokens per group (MMA N)
constexpr int kQtWBox = 4 * 128 * 128;             // bytes of a 4-block weight box (64 KiB)
constexpr int kQtXBox = 4 * kQtTok * 128;          // bytes of a 4-block token box (8 KiB)
constexpr int kQtStage = kQtWBox + kQtXBox;
struct QtSmem {
  static constexpr int kRecv = kQtStages * kQtStage;         // partner's rows: 64 x 16 floats
  static constexpr int kBar = kRecv + 64 * kQtTok * 4;       // full[3], empty[3], done, recv
  static constexpr int kSlot = kBar + (2 * kQtStages + 2) * 8;
  static constexpr int kBytes = kSlot + 16 + 1024;
};

struct QtParams {
  uint16_t* q;     // bf16 [T, nq]
  float* w;        // f32 [T, heads] or null
  int* status;
  uint64_t wait_ns;        // limit of every bounded wait (0: the library default)
  int T, nq, heads, nblk;  // nblk = input width / 64
  int bpb;                 // 64-channel blocks per box (1 or 4)
  int nqb;                 // row blocks of Wq (nq / 128)
};

__global__ void __launch_bounds__(128, 1)
    indexer_qproj_tc_kernel(const __grid_constant__ CUtensorMap tm_wq, const __grid_constant__ CUtensorMap tm_ww,
                            const __grid_constant__ CUtensorMap tm_x, const QtParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  float* recv = reinterpret_cast<float*>(smem + QtSmem::kRecv);
  const uint32_t full0 = sbase + QtSmem::kBar, empty0 = full0 + 8u * kQtStages;
  const uint32_t bar_done = empty0 + 8u * kQtStages, bar_recv = bar_done + 8u;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + QtSmem::kSlot);
  const int rb = blockIdx.x, G = gridDim.y, g = blockIdx.y, tg = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool is_w = rb >= p.nqb;                    // the per-head weight rows
  const CUtensorMap* tw = is_w ? &tm_ww : &tm_wq;
  const int row0 = is_w ? 0 : rb * 128;
  // this CTA's 64-channel blocks [b0, b0 + per), in boxes of bpb blocks
  const int per = p.nblk / G, b0 = g * per, nbox = per / p.bpb;
  const uint32_t box_bytes = (uint32_t)p.bpb * (128 * 128 + kQtTok * 128);

  if (tid == 0) {
    for (int s = 0; s < kQtStages; ++s) {
      mbar_init(full0 + 8u * s, 1);
      mbar_init(empty0 + 8u * s, 1);
    }
    mbar_init(bar_done, 1);
    mbar_init(bar_recv, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), 32);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (G == 2) cluster_sync();  // the partner's mbarriers exist before anything targets them
  const uint32_t tmem = *tmem_slot;
  pdl_wait();  // the token rows may come from the kernel just before this one

  if (tid == 0) {
    auto load = [&](int i) {
      const int s = i % kQtStages;
      const uint32_t st = sbase + (uint32_t)s * kQtStage;
      const int blk = b0 + i * p.bpb;
      mbar_arrive_expect_tx(full0 + 8u * s, box_bytes);
      tma_load_3d(st, tw, 0, row0, blk, full0 + 8u * s);
      tma_load_3d(st + kQtWBox, &tm_x, 0, tg * kQtTok, blk, full0 + 8u * s);
    };
    tma_prefetch_desc(tw);
    tma_prefetch_desc(&tm_x);
    for (int i = 0; i < min(nbox, kQtStages); ++i) load(i);
    constexpr uint32_t idesc = idesc_bf16_f32(128, kQtTok);
    bool ok = true;
    for (int i = 0; i < nbox && ok; ++i) {
      const int s = i % kQtStages;
      ok = mbar_wait_bounded(full0 + 8u * s, (uint32_t)((i / kQtStages) & 1), p.status, p.wait_ns);
      tc_fence_after();
      const uint32_t st = sbase + (uint32_t)s * kQtStage;
      const uint64_t a0 = sw128_kmajor_desc(st), x0 = sw128_kmajor_desc(st + kQtWBox);
      for (int bk = 0; bk < p.bpb; ++bk) {
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_bf16_ss(tmem, a0 + (uint64_t)((bk * 128 * 128 + kk * 32) >> 4),
                      x0 + (uint64_t)((bk * kQtTok * 128 + kk * 32) >> 4), idesc, (i | bk | kk) != 0 ? 1u : 0u);
      }
      mma_commit(empty0 + 8u * s);
      if (ok && i + kQtStages < nbox) {
        ok = mbar_wait_bounded(empty0 + 8u * s, (uint32_t)((i / kQtStages) & 1), p.status, p.wait_ns);
        if (ok) load(i + kQtStages);  // refill only a stage its MMAs have finished with
      }
    }
    mma_commit(bar_done);
  }

  // ---- epilogue: thread = weight row (TMEM lane), 16 token columns
  mbar_wait_bounded(bar_done, 0, p.status, p.wait_ns);
  __syncwarp();
  tc_fence_after();
  uint32_t r[16];
  tmem_ld16(tmem + ((uint32_t)(warp * 32) << 16), r);
  tmem_wait_ld();
  const int row = warp * 32 + lane;
  bool mine = true;
  if (G == 2) {
    const int owner = row >> 6;  // CTA g finalises rows 64 g .. 64 g + 63
    mine = owner == g;
    if (!mine) {
      const uint32_t dst = dsmem_map(smem_u32(recv + (row & 63) * kQtTok), (uint32_t)owner);
      const uint32_t rbar = dsmem_map(bar_recv, (uint32_t)owner);
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4)
        asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.b32 [%0], {%1, %2, %3, %4}, [%5];" ::
                         "r"(dst + 16u * q4), "r"(r[4 * q4]), "r"(r[4 * q4 + 1]), "r"(r[4 * q4 + 2]), "r"(r[4 * q4 + 3]),
                     "r"(rbar)
                     : "memory");
    } else {
      if ((row & 63) == 0) mbar_arrive_expect_tx(bar_recv, 64 * kQtTok * 4);
      mbar_wait_bounded(bar_recv, 0, p.status, p.wait_ns);
#pragma unroll
      for (int t = 0; t < kQtTok; ++t)
        r[t] = __float_as_uint(__uint_as_float(r[t]) + recv[(row & 63) * kQtTok + t]);
    }
  }
  if (mine) {
    const int t0 = tg * kQtTok;
#pragma unroll
    for (int t = 0; t < kQtTok; ++t) {
      if (t0 + t >= p.T) break;
      const float v = __uint_as_float(r[t]);
      if (!is_w) p.q[(size_t)(t0 + t) * p.nq + row0 + row] = (uint16_t)qp_round_bf16(v);
      else if (row < p.heads) p.w[(size_t)(t0 + t) * p.heads + row] = v;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 32);
  }
  pdl_launch_dependents();
}

}  // namespace dstopk
