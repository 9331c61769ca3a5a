// Pooled operands of the rectification pass (Rectified SpaAttn, abstract:
// the omitted keys' attention is recovered from pooled query-key
// interactions).  An omitted key block j stands for s_j copies of its mean
// key and mean value, so the pass needs the block means of K and of V as
// bf16 rows (the tensor cores' operand type): one CTA per (key block,
// batch-head, K or V) sums the block's valid rows in fp32 with 16-byte
// coalesced loads and writes the mean, rounded once to bf16.  Rows past the
// last key block are written as zeros.
#pragma once

#include "common.cuh"

namespace vsa {

constexpr int kPoolBfThreads = 256;

template <int D>
__global__ void __launch_bounds__(kPoolBfThreads) pool_kv_bf16_kernel(const __nv_bfloat16 *__restrict__ k,
                                                                      const __nv_bfloat16 *__restrict__ v,
                                                                      int n_pad, int n_valid, int bk, int n_rows,
                                                                      __nv_bfloat16 *__restrict__ k_bar,
                                                                      __nv_bfloat16 *__restrict__ v_bar) {
  constexpr int C = D / 8;                 // 16-byte chunks per row
  constexpr int R = kPoolBfThreads / C;    // row groups
  __shared__ float part[R][D];
  const int j = blockIdx.x, bh = blockIdx.y;
  const bool is_v = blockIdx.z == 1;
  __nv_bfloat16 *dst = (is_v ? v_bar : k_bar) + ((size_t)bh * n_rows + j) * D;
  const int t = threadIdx.x, c = t % C, g = t / C;
  const int r0 = j * bk;
  const int cnt = max(0, min(bk, n_valid - r0));
  if (j * bk >= n_pad || cnt == 0) {
    for (int i = t; i < D / 2; i += kPoolBfThreads)
      reinterpret_cast<__nv_bfloat162 *>(dst)[i] = __floats2bfloat162_rn(0.f, 0.f);
    return;
  }
  const __nv_bfloat16 *src = (is_v ? v : k) + ((size_t)bh * n_pad + r0) * D;
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;
  for (int r = g; r < cnt; r += R) {
    const uint4 x = __ldg(reinterpret_cast<const uint4 *>(src + (size_t)r * D) + c);
    const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&x);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = __bfloat1622float2(h[e]);
      acc[2 * e] += f.x;
      acc[2 * e + 1] += f.y;
    }
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) part[g][c * 8 + e] = acc[e];
  __syncthreads();
  const float inv = 1.f / static_cast<float>(cnt);
  for (int col2 = t; col2 < D / 2; col2 += kPoolBfThreads) {
    float s0 = 0.f, s1 = 0.f;
#pragma unroll 4
    for (int gg = 0; gg < R; ++gg) {
      s0 += part[gg][2 * col2];
      s1 += part[gg][2 * col2 + 1];
    }
    reinterpret_cast<__nv_bfloat162 *>(dst)[col2] = __floats2bfloat162_rn(s0 * inv, s1 * inv);
  }
}

}  // namespace vsa
