// a1 Pooling: block means of Q and K over their valid rows.
//
// Rectified SpaAttn (abstract) scores blocks through pooled query-key
// interactions; HyperVAttention section 4.1 takes a centroid as the mean of
// its tokens.  One CTA reads one 128-row chunk of one (batch, head) of Q or K
// exactly once with 16-byte coalesced loads, sums 16-row groups in fp32 in
// shared memory and writes every requested granularity from those sums:
// Q at (bq, 64) rows, K at (bk, 16) rows.  HBM-bound: the only traffic is the
// read of Q and K plus the small fp32 outputs.
#pragma once

#include "common.cuh"

namespace vsa {

constexpr int kPoolRows = 128;
constexpr int kPoolThreads = 256;

struct PoolOut {
  float *coarse;  // [BH, n_pad / coarse_rows, d]
  int coarse_rows;
  float *fine;  // [BH, n_pad / fine_rows, d] or null
  int fine_rows;
};

template <int D>
__global__ void __launch_bounds__(kPoolThreads) pool_kernel(const __nv_bfloat16 *__restrict__ q,
                                                            const __nv_bfloat16 *__restrict__ k, int n_pad,
                                                            int n_valid, PoolOut out_q, PoolOut out_k) {
  constexpr int C = D / 8;                 // 16-byte chunks per row
  constexpr int R = kPoolThreads / C;      // row groups
  constexpr int RPG = kPoolRows / R;       // rows per thread
  constexpr int G16 = kPoolRows / 16;      // 16-row groups in the chunk
  __shared__ float part[R][D];             // per row-group sums
  __shared__ float g16[G16][D];            // 16-row sums

  const int chunk = blockIdx.x;
  const int bh = blockIdx.y;
  const bool is_k = blockIdx.z == 1;
  const __nv_bfloat16 *src = (is_k ? k : q) + ((size_t)bh * n_pad + (size_t)chunk * kPoolRows) * D;
  const PoolOut out = is_k ? out_k : out_q;
  const int row0 = chunk * kPoolRows;

  const int t = threadIdx.x;
  const int c = t % C;
  const int g = t / C;
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;
  uint4 v[RPG];
#pragma unroll
  for (int r = 0; r < RPG; ++r) {
    const int row = g * RPG + r;
    if (row0 + row < n_valid) {
      v[r] = __ldg(reinterpret_cast<const uint4 *>(src + (size_t)row * D) + c);
    } else {
      v[r] = make_uint4(0, 0, 0, 0);
    }
  }
#pragma unroll
  for (int r = 0; r < RPG; ++r) {
    const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&v[r]);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      float2 f = __bfloat1622float2(h[e]);
      acc[2 * e] += f.x;
      acc[2 * e + 1] += f.y;
    }
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) part[g][c * 8 + e] = acc[e];
  __syncthreads();

  // 16-row group sums: R row groups of RPG rows; 16 / RPG of them per group.
  constexpr int PER16 = 16 / RPG;
  for (int i = t; i < G16 * D; i += kPoolThreads) {
    const int gg = i / D, col = i % D;
    float s = 0.f;
#pragma unroll
    for (int j = 0; j < PER16; ++j) s += part[gg * PER16 + j][col];
    g16[gg][col] = s;
  }
  __syncthreads();

  // Write a granularity of `rows` rows (a multiple of 16, at most 128).
  auto emit = [&](float *dst, int rows) {
    const int per_chunk = kPoolRows / rows;
    const int per = rows / 16;
    for (int i = t; i < per_chunk * D; i += kPoolThreads) {
      const int o = i / D, col = i % D;
      float s = 0.f;
      for (int j = 0; j < per; ++j) s += g16[o * per + j][col];
      const int start = row0 + o * rows;
      int cnt = n_valid - start;
      cnt = cnt < 0 ? 0 : (cnt > rows ? rows : cnt);
      const size_t blk = (size_t)bh * (n_pad / rows) + (size_t)(row0 / rows) + o;
      dst[blk * D + col] = cnt > 0 ? s / (float)cnt : 0.f;
    }
  };
  emit(out.coarse, out.coarse_rows);
  if (out.fine) emit(out.fine, out.fine_rows);
}

}  // namespace vsa
