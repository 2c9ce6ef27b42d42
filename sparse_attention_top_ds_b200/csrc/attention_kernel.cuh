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
// How (B200 design): split-KV, one launch for the partial attentions and one
// that combines them.
//  * A CTA owns one batch row, a tile of 128 query heads (the M of every MMA)
//    and a run of 64 attended slots.  The queries arrive by TMA in the
//    128-byte-swizzled layout; the 64 rows are gathered with cp.async
//    straight into the same layout, each row read once from HBM.
//  * S = Q . R^T (M = 128 heads, N = 64 rows, K = d) accumulates in TMEM.
//    Four softmax warps (one TMEM lane per head) take the chunk's maximum,
//    write the weights 2^(z - max) as bf16 into shared memory and sum the
//    rounded weights.
//  * O = P . R (M = 128, N = d in pieces of at most 256, K = 64 rows) takes the
//    gathered tile again, now as the MN-major B operand: the bytes that served
//    as the keys serve unchanged as the values, so nothing is transposed or
//    read twice.  O overwrites S in TMEM (the softmax has read S by then).
//  * The epilogue stores O unnormalised with the chunk's (max, sum) in a
//    head-fastest layout, so that every warp store is 512 contiguous bytes.
//  * The combine kernel rescales the chunks by 2^(max_chunk - max_all), adds
//    the sink to the normaliser, and writes out (bf16) and lse.
#pragma once

#include <cuda.h>

#include "ptx.cuh"
#include "tcgen05.cuh"

namespace dstopk {

constexpr int kAttnRows = 64;       // attended slots per CTA (N of S = Q . R^T)
constexpr int kAttnHeads = 128;     // query heads per CTA (M of both products)
constexpr int kAttnThreads = 256;   // 8 warps
constexpr int kAttnMaxD = 512;

struct AttnParams {
  const uint16_t* kv;      // bf16 compressed caches
  long long kv_bstride;    // elements from one batch row's cache to the next
  const uint16_t* win;     // bf16 [B, W, D] or null
  const int32_t* idx;      // [B, k] or null
  const int32_t* win_len;  // [B] or null
  float* opart;            // [B][HT][NS][D/4][128] float4: unnormalised O per chunk
  float2* ml;              // [B][HT][NS][128]: (max of the chunk in log2 units, sum of weights)
  int* status;
  int T, k, W, B, H, D, HT, NS;
  float scale_log2;        // scale * log2(e)
};

// Shared-memory layout for head_dim D (byte offsets from a 1024-aligned base):
// queries D/64 blocks of 128 rows x 128 B | rows D/64 blocks of 64 x 128 B |
// weights 128 x 128 B | row sources (64 pointers) | valid mask | 3 mbarriers |
// TMEM slot.
struct AttnSmem {
  __host__ __device__ static constexpr int q_off() { return 0; }
  __host__ __device__ static constexpr int kv_off(int D) { return (D / 64) * 16384; }
  __host__ __device__ static constexpr int p_off(int D) { return kv_off(D) + (D / 64) * 8192; }
  __host__ __device__ static constexpr int src_off(int D) { return p_off(D) + 16384; }
  __host__ __device__ static constexpr int mask_off(int D) { return src_off(D) + kAttnRows * 8; }
  __host__ __device__ static constexpr int bar_off(int D) { return mask_off(D) + 16; }
  __host__ __device__ static constexpr int slot_off(int D) { return bar_off(D) + 32; }
  __host__ __device__ static constexpr int bytes(int D) { return slot_off(D) + 16 + 1024; }  // + alignment slack
};

__host__ __device__ constexpr uint32_t attn_tmem_cols(int D) {
  return D <= 64 ? 64u : (D <= 128 ? 128u : (D <= 256 ? 256u : 512u));
}

// Pack two floats into bf16x2, round to nearest even: `lo` in the low half.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t u;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(u) : "f"(hi), "f"(lo));
  return u;
}

__global__ void __launch_bounds__(kAttnThreads, 1)
    sparse_attn_partial_kernel(const __grid_constant__ CUtensorMap tm_q, const AttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const int D = p.D, DB = D >> 6;
  const uint32_t q_s = sbase + AttnSmem::q_off();
  const uint32_t kv_s = sbase + AttnSmem::kv_off(D);
  const uint32_t p_s = sbase + AttnSmem::p_off(D);
  const uint16_t** src = reinterpret_cast<const uint16_t**>(smem + AttnSmem::src_off(D));
  uint32_t* mask = reinterpret_cast<uint32_t*>(smem + AttnSmem::mask_off(D));
  const uint32_t bar_q = sbase + AttnSmem::bar_off(D);
  const uint32_t bar_s = bar_q + 8, bar_o = bar_q + 16;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + AttnSmem::slot_off(D));

  const int split = blockIdx.x, ht = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t ncols = attn_tmem_cols(D);

  if (tid == 0) {
    mbar_init(bar_q, 1);
    mbar_init(bar_s, 1);
    mbar_init(bar_o, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), ncols);
    tmem_relinquish();
  }
  // the slots (and the queries) may be written by the kernel just before this one
  pdl_wait();
  if (tid == 0) {
    tma_prefetch_desc(&tm_q);
    mbar_arrive_expect_tx(bar_q, (uint32_t)DB * 16384u);
    for (int db = 0; db < DB; ++db)
      tma_load_2d(q_s + (uint32_t)db * 16384u, &tm_q, db * 64, b * p.H + ht * kAttnHeads, bar_q);
  }
  // where each of the 64 slots reads its row from (null: skipped)
  if (tid < kAttnRows) {
    const int j = split * kAttnRows + tid;
    const uint16_t* s = nullptr;
    if (j < p.k) {
      const int r = p.idx[(size_t)b * p.k + j];
      if (r >= 0 && r < p.T) s = p.kv + (long long)b * p.kv_bstride + (long long)r * D;
    } else if (j < p.k + p.W) {
      int wl = p.win_len ? p.win_len[b] : p.W;
      wl = wl < 0 ? 0 : (wl > p.W ? p.W : wl);
      const int i = j - p.k;
      if (i < wl) s = p.win + ((long long)b * p.W + i) * D;
    }
    src[tid] = s;
    const uint32_t bal = __ballot_sync(0xffffffffu, s != nullptr);
    if (lane == 0) mask[warp] = bal;
  }
  __syncthreads();

  // gather: 16-byte pieces into the swizzled layout (piece c8 of row r goes to
  // position c8 ^ (r & 7) of the row's 128 bytes); skipped rows become zeros
  for (int c = tid; c < DB * 512; c += kAttnThreads) {
    const int db = c >> 9, rem = c & 511, r = rem >> 3, c8 = rem & 7;
    const uint16_t* s = src[r];
    const uint32_t dst = kv_s + (uint32_t)db * 8192u + (uint32_t)r * 128u + ((uint32_t)(c8 ^ (r & 7)) << 4);
    const void* g = s ? static_cast<const void*>(s + db * 64 + c8 * 8) : static_cast<const void*>(p.kv);
    const uint32_t nbytes = s ? 16u : 0u;
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(g), "r"(nbytes) : "memory");
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
  asm volatile("cp.async.wait_group 0;" ::: "memory");
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // ---- S = Q . R^T into TMEM columns [0, 64)
  if (tid == 0) {
    const bool ok = mbar_wait_bounded(bar_q, 0, p.status);
    tc_fence_after();
    if (ok) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, kAttnRows);
      for (int db = 0; db < DB; ++db) {
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t a = sw128_kmajor_desc(q_s + (uint32_t)db * 16384u + (uint32_t)kk * 32u);
          const uint64_t bd = sw128_kmajor_desc(kv_s + (uint32_t)db * 8192u + (uint32_t)kk * 32u);
          mma_bf16_ss(tmem, a, bd, idesc, (db | kk) != 0 ? 1u : 0u);
        }
      }
    }
    mma_commit(bar_s);  // arrives even when nothing was issued, so that no one waits for ever
  }

  // ---- softmax of the chunk: warps 0..3, TMEM lane = head
  float m_row = -INFINITY, l_row = 0.0f;
  if (warp < 4) {
    mbar_wait_bounded(bar_s, 0, p.status);
    __syncwarp();
    tc_fence_after();
    const uint32_t taddr = tmem + ((uint32_t)(warp * 32) << 16);
    uint32_t r[64];
#pragma unroll
    for (int c = 0; c < 4; ++c) tmem_ld16(taddr + (uint32_t)(c * 16), *reinterpret_cast<uint32_t(*)[16]>(r + c * 16));
    tmem_wait_ld();
    const uint32_t m0 = mask[0], m1 = mask[1];
    float z[64];
#pragma unroll
    for (int j = 0; j < 64; ++j) {
      const bool v = ((j < 32 ? m0 >> j : m1 >> (j - 32)) & 1u) != 0;
      z[j] = v ? __uint_as_float(r[j]) * p.scale_log2 : -INFINITY;
      m_row = fmaxf(m_row, z[j]);
    }
    const int h = warp * 32 + lane;
    const uint32_t prow = p_s + (uint32_t)h * 128u;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      uint32_t pk[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int j = c * 8 + i * 2;
        const float e0 = z[j] == -INFINITY ? 0.0f : exp2f(z[j] - m_row);
        const float e1 = z[j + 1] == -INFINITY ? 0.0f : exp2f(z[j + 1] - m_row);
        const uint32_t u = pack_bf16x2(e0, e1);
        l_row += __uint_as_float(u << 16) + __uint_as_float(u & 0xffff0000u);
        pk[i] = u;
      }
      sts128(prow + ((uint32_t)(c ^ (h & 7)) << 4), make_uint4(pk[0], pk[1], pk[2], pk[3]));
    }
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();

  // ---- O = P . R: the gathered tile again, as the MN-major B operand
  if (tid == 0) {
    tc_fence_after();
    for (int n0 = 0; n0 < D; n0 += 256) {
      const int N = D - n0 < 256 ? D - n0 : 256;
      const uint32_t idesc = idesc_bf16_f32(128, N) | (1u << 16);  // B is MN-major
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint64_t a = sw128_kmajor_desc(p_s + (uint32_t)kk * 32u);
        const uint64_t bd =
            sw128_mnmajor_desc(kv_s + (uint32_t)(n0 / 64) * 8192u + (uint32_t)kk * 2048u, 8192u, 1024u);
        mma_bf16_ss(tmem + (uint32_t)n0, a, bd, idesc, kk > 0 ? 1u : 0u);
      }
    }
    mma_commit(bar_o);
  }

  // ---- epilogue: 8 warps, TMEM lane quarter = warp % 4, column half = warp / 4
  mbar_wait_bounded(bar_o, 0, p.status);
  __syncwarp();
  tc_fence_after();
  {
    const int qd = warp & 3, half = warp >> 2;
    const int hrow = qd * 32 + lane;
    const uint32_t taddr = tmem + ((uint32_t)(qd * 32) << 16);
    const size_t chunk = ((size_t)b * p.HT + ht) * p.NS + split;
    float4* op = reinterpret_cast<float4*>(p.opart) + chunk * (size_t)(D / 4) * kAttnHeads + hrow;
    const int c_lo = half * (D / 2), c_hi = c_lo + D / 2;
    for (int c0 = c_lo; c0 < c_hi; c0 += 32) {
      uint32_t r[32];
      tmem_ld16(taddr + (uint32_t)c0, *reinterpret_cast<uint32_t(*)[16]>(r));
      tmem_ld16(taddr + (uint32_t)(c0 + 16), *reinterpret_cast<uint32_t(*)[16]>(r + 16));
      tmem_wait_ld();
#pragma unroll
      for (int i = 0; i < 8; ++i)
        op[(size_t)(c0 / 4 + i) * kAttnHeads] = make_float4(__uint_as_float(r[4 * i]), __uint_as_float(r[4 * i + 1]),
                                                            __uint_as_float(r[4 * i + 2]), __uint_as_float(r[4 * i + 3]));
    }
    if (warp < 4) p.ml[chunk * kAttnHeads + hrow] = make_float2(m_row, l_row);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, ncols);
  }
  pdl_launch_dependents();
}

// ------------------------------------------------------------------ combine

struct AttnCombineParams {
  const float* opart;
  const float2* ml;
  const float* sink;   // [H] or null
  uint16_t* out;       // bf16 [B, H, D]
  float* lse;          // [B, H] or null
  int B, H, D, HT, NS;
};

// Grid (D/64 column blocks, ceil(H/32) head groups, B); 4 warps.  Lane = head,
// warp w covers 16 columns, so every load of a chunk's O is 512 contiguous
// bytes.
__global__ void __launch_bounds__(128) sparse_attn_combine_kernel(const AttnCombineParams p) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cb = blockIdx.x, b = blockIdx.z;
  const int h = blockIdx.y * 32 + lane;
  pdl_wait();
  if (h >= p.H) return;
  constexpr float kLog2e = 1.4426950408889634f;
  constexpr float kLn2 = 0.6931471805599453f;
  const int ht = h / kAttnHeads, hl = h % kAttnHeads;
  const size_t base = ((size_t)b * p.HT + ht) * p.NS;
  const float2* ml = p.ml + base * kAttnHeads + hl;
  const float sink_l2 = p.sink ? p.sink[h] * kLog2e : -INFINITY;
  float M = sink_l2;
  for (int s = 0; s < p.NS; ++s) {
    const float2 v = ml[(size_t)s * kAttnHeads];
    if (v.y > 0.0f) M = fmaxf(M, v.x);
  }
  float L = p.sink ? exp2f(sink_l2 - M) : 0.0f;
  float acc[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) acc[i] = 0.0f;
  const int cc0 = cb * 16 + warp * 4;  // first float4 column of this warp
  const float4* op = reinterpret_cast<const float4*>(p.opart) + base * (size_t)(p.D / 4) * kAttnHeads + hl;
  for (int s = 0; s < p.NS; ++s) {
    const float2 v = ml[(size_t)s * kAttnHeads];
    if (v.y > 0.0f) {
      const float w = exp2f(v.x - M);
      L = fmaf(w, v.y, L);
      const float4* o = op + (size_t)s * (p.D / 4) * kAttnHeads;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float4 x = o[(size_t)(cc0 + i) * kAttnHeads];
        acc[4 * i] = fmaf(w, x.x, acc[4 * i]);
        acc[4 * i + 1] = fmaf(w, x.y, acc[4 * i + 1]);
        acc[4 * i + 2] = fmaf(w, x.z, acc[4 * i + 2]);
        acc[4 * i + 3] = fmaf(w, x.w, acc[4 * i + 3]);
      }
    }
  }
  const float inv = L > 0.0f ? 1.0f / L : 0.0f;
  uint32_t pk[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) pk[i] = pack_bf16x2(acc[2 * i] * inv, acc[2 * i + 1] * inv);
  uint4* dst = reinterpret_cast<uint4*>(p.out + ((size_t)b * p.H + h) * p.D + (size_t)cc0 * 4);
  dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
  dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
  if (cb == 0 && warp == 0 && p.lse) p.lse[(size_t)b * p.H + h] = L > 0.0f ? (M + log2f(L)) * kLn2 : -INFINITY;
}

}  // namespace dstopk
