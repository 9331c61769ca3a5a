// Exact LSE merge of two attention results over disjoint key supports
// (HyMoR-Attn abstract: Macro and Micro outputs combined by exact LSE
// merging).  With L = ln(e^{L_a} + e^{L_b}):
//     O = e^{L_a - L} O_a + e^{L_b - L} O_b.
// Elementwise and HBM-bound: one warp per row, 16-byte loads and stores.
#pragma once

#include "common.cuh"

namespace vsa {

struct MergeWeights {
  float wa, wb, lse;
};

// Both LSE may be -inf (empty support); the merge of two empties is empty.
__device__ __forceinline__ MergeWeights lse_merge_weights(float la, float lb) {
  MergeWeights m;
  const float mx = fmaxf(la, lb);
  if (mx == -INFINITY) {
    m.wa = 0.f;
    m.wb = 0.f;
    m.lse = -INFINITY;
    return m;
  }
  const float ea = expf(la - mx), eb = expf(lb - mx);
  const float s = ea + eb;
  m.lse = mx + logf(s);
  m.wa = ea / s;
  m.wb = eb / s;
  return m;
}

template <int D>
__global__ void lse_merge_kernel(const float *__restrict__ oa, const float *__restrict__ la,
                                 const float *__restrict__ ob, const float *__restrict__ lb, size_t rows,
                                 void *o_out, int out_fp32, float *lse_out) {
  const size_t row = (size_t)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const MergeWeights w = lse_merge_weights(la[row], lb[row]);
  constexpr int V = D / 4;  // float4 per row
  for (int c = lane; c < V; c += 32) {
    const float4 a = reinterpret_cast<const float4 *>(oa + row * D)[c];
    const float4 b = reinterpret_cast<const float4 *>(ob + row * D)[c];
    float4 r;
    r.x = w.wa * a.x + w.wb * b.x;
    r.y = w.wa * a.y + w.wb * b.y;
    r.z = w.wa * a.z + w.wb * b.z;
    r.w = w.wa * a.w + w.wb * b.w;
    if (out_fp32) {
      reinterpret_cast<float4 *>(static_cast<float *>(o_out) + row * D)[c] = r;
    } else {
      uint2 p;
      p.x = pack_bf16x2(r.x, r.y);
      p.y = pack_bf16x2(r.z, r.w);
      reinterpret_cast<uint2 *>(static_cast<__nv_bfloat16 *>(o_out) + row * D)[c] = p;
    }
  }
  __syncwarp();
  if (lane == 0) lse_out[row] = w.lse;
}

}  // namespace vsa
