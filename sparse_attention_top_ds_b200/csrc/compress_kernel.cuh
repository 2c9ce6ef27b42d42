// compress_kernel.cuh -- the compressor's 4:1 fold as a gated weighted sum.
//
// What it computes (NKI pull request "Add DeepSeek-V4 CSA attention kernels",
// "How the algorithm works", steps table row 1: the compressor folds 4 tokens
// into 1 with a gated weighted sum, once every 4 decode steps).  The pages do
// not give the gate; the reading implemented here (also the oracle's) is a
// per-token gate score s_i = g . x_i from one gate vector g, weights
// a = softmax(s_0..s_3), and the folded row sum_i a_i x_i.
//
// How: a decode step folds one group of 4 rows per batch row -- a few KiB --
// so the op is latency bound.  One warp per batch row: the lanes split the
// row width in 16-byte pieces, reduce the 4 gate scores with shuffles, take
// the softmax in registers and write the folded row, rounded to bf16, at the
// caller's stride (for instance straight into the compressed cache).
#pragma once

#include <cuda_runtime.h>

#include "ptx.cuh"

namespace dstopk {

constexpr int kCfWarps = 8;
constexpr int kCfMaxD = 4096;

struct CfParams {
  const uint16_t* rows;   // bf16: batch row b's 4 rows start at rows + b * rows_bstride, D apart
  const uint16_t* gate;   // bf16 [D]
  uint16_t* out;          // bf16: batch row b's folded row at out + b * out_bstride
  long long rows_bstride, out_bstride;
  int B, D;
};

__device__ __forceinline__ float2 cf_bf16x2(uint32_t u) {
  return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xffff0000u));
}

__device__ __forceinline__ uint32_t cf_pack(float lo, float hi) {
  uint32_t u;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(u) : "f"(hi), "f"(lo));
  return u;
}

__global__ void __launch_bounds__(kCfWarps * 32) compress_fold_kernel(const CfParams p) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.x * kCfWarps + warp;
  pdl_wait();  // the rows may be written by the kernel just before this one
  if (b < p.B) {
    const uint16_t* x = p.rows + (long long)b * p.rows_bstride;
    const int npieces = p.D >> 3;
    // pass 1: the 4 gate scores
    float s[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    for (int c = lane; c < npieces; c += 32) {
      const uint4 gv = __ldg(reinterpret_cast<const uint4*>(p.gate) + c);
      const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint4 xv = __ldg(reinterpret_cast<const uint4*>(x + (size_t)i * p.D) + c);
        const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 gg = cf_bf16x2(gw[e]), xx = cf_bf16x2(xw[e]);
          s[i] = fmaf(gg.x, xx.x, s[i]);
          s[i] = fmaf(gg.y, xx.y, s[i]);
        }
      }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) s[i] += __shfl_xor_sync(0xffffffffu, s[i], o);
    // the softmax over the 4 tokens
    const float m = fmaxf(fmaxf(s[0], s[1]), fmaxf(s[2], s[3]));
    float a[4], sum = 0.0f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      a[i] = expf(s[i] - m);
      sum += a[i];
    }
    const float inv = 1.0f / sum;
    // pass 2: the weighted sum, written at the caller's stride
    uint16_t* o = p.out + (long long)b * p.out_bstride;
    for (int c = lane; c < npieces; c += 32) {
      float acc[8] = {0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint4 xv = __ldg(reinterpret_cast<const uint4*>(x + (size_t)i * p.D) + c);
        const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
        const float wi = a[i] * inv;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 xx = cf_bf16x2(xw[e]);
          acc[2 * e] = fmaf(wi, xx.x, acc[2 * e]);
          acc[2 * e + 1] = fmaf(wi, xx.y, acc[2 * e + 1]);
        }
      }
      reinterpret_cast<uint4*>(o)[c] = make_uint4(cf_pack(acc[0], acc[1]), cf_pack(acc[2], acc[3]),
                                                  cf_pack(acc[4], acc[5]), cf_pack(acc[6], acc[7]));
    }
  }
  pdl_launch_dependents();
}

}  // namespace dstopk
