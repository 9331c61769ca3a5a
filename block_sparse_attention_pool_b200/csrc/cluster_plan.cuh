// Layout of the cluster-aligned blocks (HyperVAttention section 2 Eq. (1),
// (4); section 4.3: every group of query clusters is one block row, executed
// in whole CTA tiles, its key clusters packed one after the other).
//
// Query side: the groups follow each other in ascending leader order; a
// group's rows are its member clusters in ascending order, each cluster's
// tokens in the cluster permutation's order, and the group is padded with
// zero rows to a whole number of 128-row tiles.  The plan writes
//   qmap[r]      the token of row r of that layout (-1: padding row of a
//                group, -2: row of an unused tile past the last group),
//   qinv[token]  the row of each token (-1 for tokens at or past n_valid),
//   tile_list[T] the group (its leader) of tile T, -1 for unused tiles,
// and, on the key side (keys stay in the cluster permutation's order, one
// cluster after the other), kc_off[j] = the first row of key cluster j.
//
// gather_rows_kernel moves rows by such a map: dst[i] = src[map[i]], a fill
// word for map -1, untouched for map -2 (one warp per row).
#pragma once

#include "common.cuh"

namespace vsa {

constexpr int kPlanThreads = 1024;
constexpr int kPlanMaxClusters = 1024;

struct PlanArgs {
  const int32_t *group_of;  // [BH][nq]
  const int32_t *sizes_q;   // [BH][nq]
  const int32_t *perm_q;    // [BH][n_pad]
  const int32_t *sizes_k;   // [BH][nk]
  int nq, nk, n_valid, n_pad, n_rows;
  int32_t *qmap;       // [BH][n_rows]
  int32_t *qinv;       // [BH][n_pad]
  int32_t *tile_list;  // [BH][n_rows / 128]
  int32_t *kc_off;     // [BH][nk]
  int *status;         // the launch's status word
};

// Exclusive prefix sum over the 1024 threads of the block; *total gets the sum.
__device__ __forceinline__ int block_exclusive_scan(int v, int *s_tmp, int *total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int ex = warp_exclusive_scan(v, lane);
  if (lane == 31) s_tmp[warp] = ex + v;
  __syncthreads();
  if (warp == 0) {
    const int x = s_tmp[lane];
    const int e = warp_exclusive_scan(x, lane);
    s_tmp[lane] = e;
    if (lane == 31) s_tmp[32] = e + x;
  }
  __syncthreads();
  const int r = s_tmp[warp] + ex;
  if (total) *total = s_tmp[32];
  __syncthreads();
  return r;
}

__global__ void __launch_bounds__(kPlanThreads) cluster_plan_kernel(const PlanArgs a) {
  __shared__ int s_size[kPlanMaxClusters];
  __shared__ int s_grp[kPlanMaxClusters];
  __shared__ int s_gsz[kPlanMaxClusters];
  __shared__ int s_goff[kPlanMaxClusters];
  __shared__ int s_row0[kPlanMaxClusters];
  __shared__ int s_qoff[kPlanMaxClusters];
  __shared__ int s_tmp[33];
  const int bh = blockIdx.x, t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const size_t hq = (size_t)bh * a.nq;

  int sz = 0, grp = t;
  if (t < a.nq) {
    sz = max(0, __ldg(a.sizes_q + hq + t));
    grp = __ldg(a.group_of + hq + t);
    // a group is named by its leader, which leads itself
    if (grp < 0 || grp >= a.nq || __ldg(a.group_of + hq + grp) != grp) {
      latch_status(a.status, VSA_ERR_BAD_INDEX);
      grp = t;
    }
  }
  s_size[t] = sz;
  s_grp[t] = grp;
  s_gsz[t] = 0;
  int n_q_tokens = 0;
  const int qoff = block_exclusive_scan(sz, s_tmp, &n_q_tokens);
  s_qoff[t] = qoff;
  if (t < a.nq) atomicAdd(&s_gsz[grp], sz);
  __syncthreads();
  const bool leader = t < a.nq && s_grp[t] == t;
  const int padded = leader ? ((s_gsz[t] + 127) / 128) * 128 : 0;
  int total = 0;
  const int goff = block_exclusive_scan(padded, s_tmp, &total);
  s_goff[t] = goff;
  __syncthreads();
  if (total > a.n_rows || n_q_tokens > a.n_pad) {
    if (t == 0) latch_status(a.status, VSA_ERR_CAPACITY);
    return;
  }
  if (t < a.nq) {
    int within = 0;
    for (int i = 0; i < t; ++i) within += s_grp[i] == grp ? s_size[i] : 0;
    s_row0[t] = s_goff[grp] + within;
  }
  // defaults: unused tiles and rows, padding rows, tokens without a row
  const int n_tiles = a.n_rows / 128;
  for (int T = t; T < n_tiles; T += kPlanThreads) a.tile_list[(size_t)bh * n_tiles + T] = -1;
  for (int r = t; r < a.n_rows; r += kPlanThreads) a.qmap[(size_t)bh * a.n_rows + r] = r < total ? -1 : -2;
  for (int i = t; i < a.n_pad; i += kPlanThreads) a.qinv[(size_t)bh * a.n_pad + i] = -1;
  __syncthreads();
  if (leader)
    for (int T = goff / 128; T < (goff + padded) / 128; ++T) a.tile_list[(size_t)bh * n_tiles + T] = t;
  for (int i = warp; i < a.nq; i += kPlanThreads / 32) {
    const int n = s_size[i], src0 = s_qoff[i], dst0 = s_row0[i];
    for (int e = lane; e < n; e += 32) {
      const int tok = __ldg(a.perm_q + (size_t)bh * a.n_pad + src0 + e);
      if (tok < 0 || tok >= a.n_valid) {
        latch_status(a.status, VSA_ERR_BAD_INDEX);
        continue;
      }
      a.qmap[(size_t)bh * a.n_rows + dst0 + e] = tok;
      a.qinv[(size_t)bh * a.n_pad + tok] = dst0 + e;
    }
  }
  // key clusters: first row of each in the permuted key sequence
  const int skv = t < a.nk ? max(0, __ldg(a.sizes_k + (size_t)bh * a.nk + t)) : 0;
  const int koff = block_exclusive_scan(skv, s_tmp, nullptr);
  if (t < a.nk) a.kc_off[(size_t)bh * a.nk + t] = koff;
}

__global__ void gather_rows_kernel(const uint32_t *__restrict__ src, const int32_t *__restrict__ map, int n_src,
                                   int n_dst, long long n_rows, int row_words, uint32_t fill,
                                   uint32_t *__restrict__ dst, int *status) {
  const long long row = (long long)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  if (row >= n_rows) return;
  const int lane = threadIdx.x & 31;
  const long long bh = row / n_dst;
  const int m = __ldg(map + row);
  if (m == -2) return;
  uint32_t *d = dst + row * row_words;
  if (m < -2 || m >= n_src) {
    if (lane == 0) latch_status(status, VSA_ERR_BAD_INDEX);
    return;
  }
  if (m == -1) {
    for (int w = lane; w < row_words; w += 32) d[w] = fill;
    return;
  }
  const uint32_t *s = src + (bh * n_src + m) * row_words;
  if ((row_words & 3) == 0) {
    const uint4 *s4 = reinterpret_cast<const uint4 *>(s);
    uint4 *d4 = reinterpret_cast<uint4 *>(d);
    for (int w = lane; w < row_words / 4; w += 32) d4[w] = __ldg(s4 + w);
  } else {
    for (int w = lane; w < row_words; w += 32) d[w] = __ldg(s + w);
  }
}

}  // namespace vsa
