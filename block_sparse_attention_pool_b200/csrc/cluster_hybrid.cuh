// Hybrid clustering across denoising steps (HyperVAttention section 4.2,
// Eq. (6)).  An anchor step runs the full 3D local-window clustering; its last
// assignment round also writes every token's Lowe ratio rho = d1 / d2, and the
// ceil(frac * N) tokens of largest rho (the ones most likely to change
// cluster) are cached.  An intermediate step revisits only those tokens: each
// is reassigned, with its current embedding, to the nearest centroid of the
// whole set; the clusters that gained or lost a token get the mean of their
// members' current embeddings, and sizes and permutation follow.
//
// Kernels (one (batch, head) per blockIdx.y unless stated):
//   subset_select_kernel  one CTA per head: the rank-n key of rho by a bitwise
//                         search (the largest key T with #(rho >= T) >= n),
//                         then an ordered compaction of the tokens above T
//                         and the first tokens equal to T (ties to the lower
//                         index), ascending
//   reassign_kernel       128 cached tokens per CTA against every centroid,
//                         staged 128 at a time, as an fp32 register-tiled
//                         product in shared memory (distance |mu|^2 - 2 x.mu,
//                         ties to the lower cell); marks the clusters a token
//                         left and joined
//   count_sort kernels    sizes and the permutation of any assignment: per
//                         1024-token chunk a histogram (count), one exclusive
//                         scan per head over (cluster, chunk) (scan), and a
//                         stable scatter in which one warp walks its chunk in
//                         token order, ranking equal clusters with a match
//                         mask (scatter)
//   refresh_kernel        one CTA per marked cluster: the mean of its members
//                         in permutation order (an emptied cluster keeps its
//                         centroid)
#pragma once

#include "common.cuh"

namespace vsa {

constexpr int kHybThreads = 1024;
constexpr int kSortChunk = 1024;
constexpr int kReTok = 128;  // cached tokens per reassignment CTA
constexpr int kReCen = 128;  // centroids per staged chunk

// ---- subset selection -------------------------------------------------------

__device__ __forceinline__ int hyb_block_sum(int v, int *s_tmp) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  v = warp_sum_int(v);
  if (lane == 0) s_tmp[warp] = v;
  __syncthreads();
  int t = 0;
  for (int w = 0; w < kHybThreads / 32; ++w) t += s_tmp[w];
  __syncthreads();
  return t;
}

__device__ __forceinline__ int hyb_block_excl(int v, int *s_tmp, int *total) {
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
  *total = s_tmp[32];
  __syncthreads();
  return r;
}

// rho >= 0: its float bits order like its value.
__global__ void __launch_bounds__(kHybThreads) subset_select_kernel(const float *__restrict__ ratio, int n_valid,
                                                                    int n_sub, int32_t *__restrict__ subset) {
  __shared__ int s_tmp[33];
  const int bh = blockIdx.x, t = threadIdx.x;
  const uint32_t *key = reinterpret_cast<const uint32_t *>(ratio) + (size_t)bh * n_valid;
  // each thread owns the contiguous tokens [lo, hi)
  const int per = (n_valid + kHybThreads - 1) / kHybThreads;
  const int lo = min(n_valid, t * per), hi = min(n_valid, lo + per);
  uint32_t T = 0u;
  for (int bit = 31; bit >= 0; --bit) {
    const uint32_t cand = T | (1u << bit);
    int c = 0;
    for (int i = lo; i < hi; ++i) c += __ldg(key + i) >= cand ? 1 : 0;
    if (hyb_block_sum(c, s_tmp) >= n_sub) T = cand;
  }
  int gt = 0, eq = 0;
  for (int i = lo; i < hi; ++i) {
    const uint32_t k = __ldg(key + i);
    gt += k > T ? 1 : 0;
    eq += k == T ? 1 : 0;
  }
  int n_gt = 0, n_eq = 0;
  hyb_block_excl(gt, s_tmp, &n_gt);
  const int eq_before = hyb_block_excl(eq, s_tmp, &n_eq);
  const int need = n_sub - n_gt;  // tokens equal to T that are taken, lowest index first
  const int take_eq = max(0, min(eq, need - eq_before));
  int total = 0;
  int pos = hyb_block_excl(gt + take_eq, s_tmp, &total);
  int eq_seen = 0;
  int32_t *dst = subset + (size_t)bh * n_sub;
  for (int i = lo; i < hi; ++i) {
    const uint32_t k = __ldg(key + i);
    bool take = k > T;
    if (k == T) take = eq_seen++ < take_eq;
    if (take && pos < n_sub) dst[pos++] = i;
  }
}

// ---- global reassignment of the cached tokens --------------------------------

template <int D>
struct ReLayout {
  static constexpr int kLd = D + 4;
  static constexpr int kOffX = 0;
  static constexpr int kOffC = kOffX + kReTok * kLd * 4;
  static constexpr int kBytes = kOffC + kReCen * kLd * 4;
};

template <int D>
__global__ void __launch_bounds__(256) reassign_kernel(const __nv_bfloat16 *__restrict__ x, int n_pad, int n_valid,
                                                       int n_cells, const float *__restrict__ mu,
                                                       const int32_t *__restrict__ subset, int n_sub,
                                                       int32_t *__restrict__ assign, int32_t *__restrict__ changed) {
  using L = ReLayout<D>;
  constexpr int kLd = L::kLd;
  constexpr int NB = kReCen / 16;
  extern __shared__ __align__(16) uint8_t re_smem_raw[];
  float(*sX)[kLd] = reinterpret_cast<float(*)[kLd]>(re_smem_raw + L::kOffX);
  float(*sC)[kLd] = reinterpret_cast<float(*)[kLd]>(re_smem_raw + L::kOffC);
  __shared__ int s_tok[kReTok];
  const int bh = blockIdx.y, tid = threadIdx.x;
  const int i0 = blockIdx.x * kReTok;
  if (tid < kReTok) {
    int tok = -1;
    if (i0 + tid < n_sub) {
      tok = __ldg(subset + (size_t)bh * n_sub + i0 + tid);
      if (tok < 0 || tok >= n_valid) {
        latch_status(VSA_ERR_BAD_INDEX);
        tok = -1;
      }
    }
    s_tok[tid] = tok;
  }
  __syncthreads();
  const __nv_bfloat16 *xb = x + (size_t)bh * n_pad * D;
  for (int e = tid; e < kReTok * (D / 8); e += 256) {
    const int i = e / (D / 8), k8 = e % (D / 8);
    const int tok = s_tok[i];
    float4 lo = make_float4(0.f, 0.f, 0.f, 0.f), hi = lo;
    if (tok >= 0) {
      const uint4 raw = __ldg(reinterpret_cast<const uint4 *>(xb + (size_t)tok * D) + k8);
      const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&raw.x));
      const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&raw.y));
      const float2 c = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&raw.z));
      const float2 d = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&raw.w));
      lo = make_float4(a.x, a.y, b.x, b.y);
      hi = make_float4(c.x, c.y, d.x, d.y);
    }
    *reinterpret_cast<float4 *>(&sX[i][8 * k8]) = lo;
    *reinterpret_cast<float4 *>(&sX[i][8 * k8 + 4]) = hi;
  }
  const int ty = tid >> 4, tx = tid & 15;
  float best[8];
  int bcell[8];
#pragma unroll
  for (int a = 0; a < 8; ++a) {
    best[a] = INFINITY;
    bcell[a] = 0x7fffffff;
  }
  const float *mub = mu + (size_t)bh * n_cells * D;
  for (int c0 = 0; c0 < n_cells; c0 += kReCen) {
    __syncthreads();  // the previous chunk's centroids are consumed
    for (int e = tid; e < kReCen * (D / 4); e += 256) {
      const int j = e / (D / 4), k4 = e % (D / 4);
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (c0 + j < n_cells) v = __ldg(reinterpret_cast<const float4 *>(mub + (size_t)(c0 + j) * D) + k4);
      *reinterpret_cast<float4 *>(&sC[j][4 * k4]) = v;
    }
    __syncthreads();
    float acc[8][NB], cn[NB];
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      cn[b] = 0.f;
#pragma unroll
      for (int a = 0; a < 8; ++a) acc[a][b] = 0.f;
    }
#pragma unroll 2
    for (int k = 0; k < D; k += 4) {
      float4 cv[NB];
#pragma unroll
      for (int b = 0; b < NB; ++b) {
        cv[b] = *reinterpret_cast<const float4 *>(&sC[tx + 16 * b][k]);
        cn[b] = fmaf(cv[b].x, cv[b].x, cn[b]);
        cn[b] = fmaf(cv[b].y, cv[b].y, cn[b]);
        cn[b] = fmaf(cv[b].z, cv[b].z, cn[b]);
        cn[b] = fmaf(cv[b].w, cv[b].w, cn[b]);
      }
#pragma unroll
      for (int a = 0; a < 8; ++a) {
        const float4 xv = *reinterpret_cast<const float4 *>(&sX[ty + 16 * a][k]);
#pragma unroll
        for (int b = 0; b < NB; ++b) {
          acc[a][b] = fmaf(xv.x, cv[b].x, acc[a][b]);
          acc[a][b] = fmaf(xv.y, cv[b].y, acc[a][b]);
          acc[a][b] = fmaf(xv.z, cv[b].z, acc[a][b]);
          acc[a][b] = fmaf(xv.w, cv[b].w, acc[a][b]);
        }
      }
    }
#pragma unroll
    for (int a = 0; a < 8; ++a)
#pragma unroll
      for (int b = 0; b < NB; ++b) {
        const int cell = c0 + tx + 16 * b;
        if (cell < n_cells) {
          const float dist = fmaf(-2.f, acc[a][b], cn[b]);
          if (dist < best[a] || (dist == best[a] && cell < bcell[a])) {
            best[a] = dist;
            bcell[a] = cell;
          }
        }
      }
  }
  int32_t *ab = assign + (size_t)bh * n_valid;
  int32_t *ch = changed + (size_t)bh * n_cells;
#pragma unroll
  for (int a = 0; a < 8; ++a) {
    float d = best[a];
    int c = bcell[a];
#pragma unroll
    for (int o = 1; o < 16; o <<= 1) {
      const float od = __shfl_xor_sync(0xffffffffu, d, o);
      const int oc = __shfl_xor_sync(0xffffffffu, c, o);
      if (od < d || (od == d && oc < c)) {
        d = od;
        c = oc;
      }
    }
    const int i = ty + 16 * a;
    const int tok = s_tok[i];
    if (tx == 0 && tok >= 0 && c < n_cells) {
      const int old = ab[tok];
      if (old != c) {
        ab[tok] = c;
        if (old >= 0 && old < n_cells) ch[old] = 1;
        ch[c] = 1;
      }
    }
  }
}

// ---- sizes and stable permutation of an assignment ---------------------------

// cnt[bh][u][chunk]: tokens of chunk with cluster u
__global__ void __launch_bounds__(256) sort_count_kernel(const int32_t *__restrict__ assign, int n_valid,
                                                         int n_cells, int n_chunks, int32_t *__restrict__ cnt) {
  extern __shared__ int hist[];
  const int chunk = blockIdx.x, bh = blockIdx.y;
  for (int u = threadIdx.x; u < n_cells; u += 256) hist[u] = 0;
  __syncthreads();
  const int32_t *ab = assign + (size_t)bh * n_valid;
  for (int i = chunk * kSortChunk + threadIdx.x; i < min(n_valid, (chunk + 1) * kSortChunk); i += 256) {
    const int u = __ldg(ab + i);
    if (u >= 0 && u < n_cells) atomicAdd(&hist[u], 1);
    else latch_status(VSA_ERR_BAD_INDEX);
  }
  __syncthreads();
  for (int u = threadIdx.x; u < n_cells; u += 256) cnt[((size_t)bh * n_cells + u) * n_chunks + chunk] = hist[u];
}

// In place: cnt -> exclusive prefix in (cluster, chunk) order; sizes[u] = the cluster's total.
__global__ void __launch_bounds__(kHybThreads) sort_scan_kernel(int32_t *__restrict__ cnt, int n_cells, int n_chunks,
                                                               int32_t *__restrict__ sizes) {
  __shared__ int s_tmp[33];
  const int bh = blockIdx.x, t = threadIdx.x;
  int32_t *c = cnt + (size_t)bh * n_cells * n_chunks;
  const int n = n_cells * n_chunks;
  const int per = (n + kHybThreads - 1) / kHybThreads;
  const int lo = min(n, t * per), hi = min(n, lo + per);
  int s = 0;
  for (int i = lo; i < hi; ++i) s += c[i];
  int total = 0;
  int run = hyb_block_excl(s, s_tmp, &total);
  for (int i = lo; i < hi; ++i) {
    const int v = c[i];
    c[i] = run;
    run += v;
  }
  __syncthreads();
  // cluster u spans [c[u * n_chunks], next cluster's start)
  for (int u = t; u < n_cells; u += kHybThreads) {
    const int start = c[u * n_chunks];
    const int end = u + 1 < n_cells ? c[(u + 1) * n_chunks] : total;
    sizes[(size_t)bh * n_cells + u] = end - start;
  }
}

// One warp per chunk, in token order: a token's rank among the chunk's tokens of
// its cluster is the count of earlier ones (running counters) plus its earlier
// peers in the same 32-token step.
__global__ void __launch_bounds__(32) sort_scatter_kernel(const int32_t *__restrict__ assign, int n_valid, int n_pad,
                                                          int n_cells, int n_chunks, const int32_t *__restrict__ off,
                                                          int32_t *__restrict__ perm) {
  extern __shared__ int seen[];
  const int chunk = blockIdx.x, bh = blockIdx.y, lane = threadIdx.x;
  for (int u = lane; u < n_cells; u += 32) seen[u] = 0;
  __syncwarp();
  const int32_t *ab = assign + (size_t)bh * n_valid;
  const int32_t *ob = off + (size_t)bh * n_cells * n_chunks;
  int32_t *pb = perm + (size_t)bh * n_pad;
  const int end = min(n_valid, (chunk + 1) * kSortChunk);
  for (int base = chunk * kSortChunk; base < end; base += 32) {
    const int i = base + lane;
    const bool in = i < end;
    int u = in ? __ldg(ab + i) : -1;
    if (u >= n_cells) u = -1;  // latched by the count kernel
    const uint32_t peers = __match_any_sync(0xffffffffu, u);
    const int before = __popc(peers & ((1u << lane) - 1u));
    const int r = u >= 0 ? seen[u] + before : 0;
    __syncwarp();
    if (u >= 0) {
      pb[ob[(size_t)u * n_chunks + chunk] + r] = i;
      if (before == 0) seen[u] += __popc(peers);
    }
    __syncwarp();
  }
  if (chunk == 0)
    for (int i = n_valid + lane; i < n_pad; i += 32) pb[i] = i;  // padding rows stay
}

// ---- centroids of the clusters that changed ----------------------------------

template <int D>
__global__ void __launch_bounds__(128) refresh_kernel(const __nv_bfloat16 *__restrict__ x, int n_pad, int n_cells,
                                                      int n_chunks, const int32_t *__restrict__ changed,
                                                      const int32_t *__restrict__ off, const int32_t *__restrict__ sizes,
                                                      const int32_t *__restrict__ perm, float *__restrict__ mu) {
  const int u = blockIdx.x, bh = blockIdx.y;
  if (!changed[(size_t)bh * n_cells + u]) return;
  const int m = sizes[(size_t)bh * n_cells + u];
  if (m == 0) return;  // an emptied cluster keeps its centroid
  const int start = off[((size_t)bh * n_cells + u) * n_chunks];
  const int32_t *pb = perm + (size_t)bh * n_pad + start;
  const __nv_bfloat16 *xb = x + (size_t)bh * n_pad * D;
  const float inv = 1.f / (float)m;
  for (int k = threadIdx.x; k < D; k += 128) {
    float s = 0.f;
    for (int r = 0; r < m; ++r) s += __bfloat162float(xb[(size_t)__ldg(pb + r) * D + k]);
    mu[((size_t)bh * n_cells + u) * D + k] = s * inv;
  }
}

}  // namespace vsa
