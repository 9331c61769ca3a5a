// 3D local-window clustering and the cluster permutation.
//
// HyperVAttention §4.1 Eq. (5): the T x H x W token lattice is cut into
// regular cells of (k_t, k_h, k_w) tokens with one centroid per cell,
// initialised from the token at the centre of the cell; every token is
// assigned to the nearest centroid (squared Euclidean distance) among the
// cells of a (w_t, w_h, w_w) window around its own cell, and a centroid is
// then the mean of its tokens.  §2 Eq. (1): Q, K, V are reordered so that the
// tokens of a cluster are contiguous; Eq. (4): the output is put back in
// token order.
//
// Kernels (one (batch, head) per blockIdx.y):
//   cluster_init_kernel    centroid u = the centre token of cell u
//   cluster_assign_kernel  one CTA per cell: the cell's tokens (<= 128) x the
//                          window's centroids (<= 128, in chunks of 32) as an
//                          fp32 register-tiled GEMM on shared memory;
//                          distance = |mu|^2 - 2 x.mu (|x|^2 is common to all
//                          candidates of a token); argmin with ties to the
//                          lower cell
//   cluster_update_kernel  one CTA per cluster: the tokens that can hold it
//                          are those whose window contains it, i.e. one box
//                          of the lattice; the CTA collects its members from
//                          that box in token order (ballot compaction) and
//                          sums them in that order, so centroids, sizes and
//                          the permutation are deterministic
//   cluster_perm_kernel    one CTA per cluster: its offset (sum of the sizes
//                          of lower clusters) and its members, in token order
//   permute_rows_kernel    one warp per row: gather (dst[i] = src[perm[i]])
//                          or scatter (dst[perm[i]] = src[i])
// A cell at the far edge of an axis holds the remaining tokens; the window of
// w cells spans offsets -((w-1)/2) .. w/2; an empty cluster keeps its
// centroid; padding rows (at or past T*H*W) keep their place in the
// permutation.
#pragma once

#include "common.cuh"

namespace vsa {

constexpr int kClusterThreads = 256;
constexpr int kClusterMaxTokens = 128;  // tokens per cell
constexpr int kClusterMaxWindow = 128;  // cells per window
constexpr int kClusterChunk = 32;       // window centroids per shared-memory chunk

struct ClusterGeom {
  int T, H, W;        // token lattice
  int kt, kh, kw;     // cell extents (tokens)
  int CT, CH, CW;     // cells per axis
  int wt, wh, ww;     // window (cells)
  int n_cells;
  int n_valid, n_pad;
};

__device__ __forceinline__ int win_lo(int w) { return -((w - 1) / 2); }
__device__ __forceinline__ int win_hi(int w) { return w / 2; }

// Token box [t0,t1) x [h0,h1) x [w0,w1) of the cells [c0, c1) along each axis.
struct TokBox {
  int t0, t1, h0, h1, w0, w1;
  __device__ int size() const { return (t1 - t0) * (h1 - h0) * (w1 - w0); }
  // the i-th token of the box in (t, h, w) order, as a flat lattice index
  __device__ int token(int i, const ClusterGeom &g) const {
    const int ew = w1 - w0, eh = h1 - h0;
    const int bw = i % ew, bh = (i / ew) % eh, bt = i / (ew * eh);
    return ((t0 + bt) * g.H + (h0 + bh)) * g.W + (w0 + bw);
  }
};

__device__ __forceinline__ TokBox cell_box(int ct0, int ct1, int ch0, int ch1, int cw0, int cw1,
                                           const ClusterGeom &g) {
  TokBox b;
  b.t0 = ct0 * g.kt;
  b.t1 = min(ct1 * g.kt, g.T);
  b.h0 = ch0 * g.kh;
  b.h1 = min(ch1 * g.kh, g.H);
  b.w0 = cw0 * g.kw;
  b.w1 = min(cw1 * g.kw, g.W);
  return b;
}

template <int D>
__global__ void cluster_init_kernel(const __nv_bfloat16 *__restrict__ x, ClusterGeom g, float *__restrict__ mu) {
  const int u = blockIdx.x, bh = blockIdx.y;
  const int cw = u % g.CW, ch = (u / g.CW) % g.CH, ct = u / (g.CW * g.CH);
  const TokBox b = cell_box(ct, ct + 1, ch, ch + 1, cw, cw + 1, g);
  const int t = b.t0 + (b.t1 - b.t0 - 1) / 2, h = b.h0 + (b.h1 - b.h0 - 1) / 2, w = b.w0 + (b.w1 - b.w0 - 1) / 2;
  const size_t row = (size_t)bh * g.n_pad + (size_t)((t * g.H + h) * g.W + w);
  float *dst = mu + ((size_t)bh * g.n_cells + u) * D;
  for (int k = threadIdx.x; k < D; k += blockDim.x) dst[k] = __bfloat162float(x[row * D + k]);
}

template <int D>
struct AssignSmem {
  static constexpr int kLd = D + 4;
  float X[kClusterMaxTokens][kLd];
  float C[kClusterChunk][kLd];
  float cnorm[kClusterChunk];
  int win[kClusterMaxWindow];
  int n_win;
};

template <int D>
__global__ void __launch_bounds__(kClusterThreads) cluster_assign_kernel(const __nv_bfloat16 *__restrict__ x,
                                                                         ClusterGeom g, const float *__restrict__ mu,
                                                                         int32_t *__restrict__ assign) {
  extern __shared__ __align__(16) uint8_t cluster_smem_raw[];
  AssignSmem<D> &sm = *reinterpret_cast<AssignSmem<D> *>(cluster_smem_raw);
  const int u0 = blockIdx.x, bh = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int cw = u0 % g.CW, ch = (u0 / g.CW) % g.CH, ct = u0 / (g.CW * g.CH);
  const TokBox box = cell_box(ct, ct + 1, ch, ch + 1, cw, cw + 1, g);
  const int n_tok = box.size();

  // window cells, ascending flat index (t-major loops)
  if (tid == 0) {
    int n = 0;
    for (int dt = win_lo(g.wt); dt <= win_hi(g.wt); ++dt)
      for (int dh = win_lo(g.wh); dh <= win_hi(g.wh); ++dh)
        for (int dw = win_lo(g.ww); dw <= win_hi(g.ww); ++dw) {
          const int t = ct + dt, h = ch + dh, w = cw + dw;
          if (t >= 0 && t < g.CT && h >= 0 && h < g.CH && w >= 0 && w < g.CW && n < kClusterMaxWindow)
            sm.win[n++] = (t * g.CH + h) * g.CW + w;
        }
    sm.n_win = n;
  }
  // the cell's tokens as fp32 rows (zero rows past n_tok)
  const __nv_bfloat16 *xb = x + (size_t)bh * g.n_pad * D;
  for (int e = tid; e < kClusterMaxTokens * (D / 2); e += kClusterThreads) {
    const int i = e / (D / 2), k2 = e % (D / 2);
    float2 v = make_float2(0.f, 0.f);
    if (i < n_tok) {
      const __nv_bfloat162 p = reinterpret_cast<const __nv_bfloat162 *>(xb + (size_t)box.token(i, g) * D)[k2];
      v = __bfloat1622float2(p);
    }
    sm.X[i][2 * k2] = v.x;
    sm.X[i][2 * k2 + 1] = v.y;
  }
  __syncthreads();
  const int n_win = sm.n_win;
  const float *mub = mu + (size_t)bh * g.n_cells * D;

  const int ty = tid >> 4, tx = tid & 15;
  float best_d[8];
  int best_c[8];
#pragma unroll
  for (int a = 0; a < 8; ++a) {
    best_d[a] = INFINITY;
    best_c[a] = 0x7fffffff;
  }
  for (int c0 = 0; c0 < n_win; c0 += kClusterChunk) {
    __syncthreads();  // the previous chunk's centroids are consumed
    for (int e = tid; e < kClusterChunk * (D / 4); e += kClusterThreads) {
      const int j = e / (D / 4), k4 = e % (D / 4);
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (c0 + j < n_win) v = reinterpret_cast<const float4 *>(mub + (size_t)sm.win[c0 + j] * D)[k4];
      *reinterpret_cast<float4 *>(&sm.C[j][4 * k4]) = v;
    }
    __syncthreads();
    // |mu|^2 of the chunk: warp w reduces rows 4w .. 4w+3 in a fixed order
    for (int j = warp * 4; j < warp * 4 + 4; ++j) {
      float s = 0.f;
      for (int k = lane; k < D; k += 32) s = fmaf(sm.C[j][k], sm.C[j][k], s);
      s = warp_sum(s);
      if (lane == 0) sm.cnorm[j] = s;
    }
    float acc[8][2];
#pragma unroll
    for (int a = 0; a < 8; ++a) acc[a][0] = acc[a][1] = 0.f;
#pragma unroll 4
    for (int k = 0; k < D; k += 4) {
      const float4 b0 = *reinterpret_cast<const float4 *>(&sm.C[tx][k]);
      const float4 b1 = *reinterpret_cast<const float4 *>(&sm.C[tx + 16][k]);
#pragma unroll
      for (int a = 0; a < 8; ++a) {
        const float4 xv = *reinterpret_cast<const float4 *>(&sm.X[ty + 16 * a][k]);
        acc[a][0] = fmaf(xv.x, b0.x, acc[a][0]);
        acc[a][0] = fmaf(xv.y, b0.y, acc[a][0]);
        acc[a][0] = fmaf(xv.z, b0.z, acc[a][0]);
        acc[a][0] = fmaf(xv.w, b0.w, acc[a][0]);
        acc[a][1] = fmaf(xv.x, b1.x, acc[a][1]);
        acc[a][1] = fmaf(xv.y, b1.y, acc[a][1]);
        acc[a][1] = fmaf(xv.z, b1.z, acc[a][1]);
        acc[a][1] = fmaf(xv.w, b1.w, acc[a][1]);
      }
    }
    __syncthreads();  // cnorm written by other warps
#pragma unroll
    for (int bb = 0; bb < 2; ++bb) {
      const int j = tx + 16 * bb;
      if (c0 + j < n_win) {
        const int cell = sm.win[c0 + j];
        const float cn = sm.cnorm[j];
#pragma unroll
        for (int a = 0; a < 8; ++a) {
          const float dist = fmaf(-2.f, acc[a][bb], cn);
          if (dist < best_d[a] || (dist == best_d[a] && cell < best_c[a])) {
            best_d[a] = dist;
            best_c[a] = cell;
          }
        }
      }
    }
  }
  // argmin across the 16 threads (tx) that share a token
  int32_t *ab = assign + (size_t)bh * g.n_valid;
#pragma unroll
  for (int a = 0; a < 8; ++a) {
    float d = best_d[a];
    int c = best_c[a];
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
    if (tx == 0 && i < n_tok) ab[box.token(i, g)] = c;
  }
}

// The members of cluster u in token order, collected into list[] (capacity
// = the size of the reverse-window box); returns their count.  Every thread
// of the CTA calls it.
__device__ __forceinline__ int cluster_members(int u, int bh, const ClusterGeom &g, const int32_t *__restrict__ assign,
                                               int32_t *list, int *warp_cnt) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int cw = u % g.CW, ch = (u / g.CW) % g.CH, ct = u / (g.CW * g.CH);
  // cells whose window holds u: offsets -hi .. -lo around u
  const TokBox box = cell_box(max(0, ct - win_hi(g.wt)), min(g.CT, ct - win_lo(g.wt) + 1),
                              max(0, ch - win_hi(g.wh)), min(g.CH, ch - win_lo(g.wh) + 1),
                              max(0, cw - win_hi(g.ww)), min(g.CW, cw - win_lo(g.ww) + 1), g);
  const int n_box = box.size();
  const int32_t *ab = assign + (size_t)bh * g.n_valid;
  int total = 0;
  for (int base = 0; base < n_box; base += kClusterThreads) {
    const int i = base + tid;
    int tok = -1;
    bool mine = false;
    if (i < n_box) {
      tok = box.token(i, g);
      mine = __ldg(ab + tok) == u;
    }
    const uint32_t bal = __ballot_sync(0xffffffffu, mine);
    if (lane == 0) warp_cnt[warp] = __popc(bal);
    __syncthreads();
    int before = 0, chunk = 0;
    for (int w = 0; w < kClusterThreads / 32; ++w) {
      const int c = warp_cnt[w];
      before += w < warp ? c : 0;
      chunk += c;
    }
    if (mine) list[total + before + __popc(bal & ((1u << lane) - 1u))] = tok;
    total += chunk;
    __syncthreads();  // warp_cnt is rewritten by the next round
  }
  return total;
}

template <int D>
__global__ void __launch_bounds__(kClusterThreads) cluster_update_kernel(const __nv_bfloat16 *__restrict__ x,
                                                                         ClusterGeom g, const int32_t *__restrict__ assign,
                                                                         float *__restrict__ mu, int32_t *__restrict__ sizes) {
  extern __shared__ __align__(16) uint8_t cluster_smem_raw[];
  int *warp_cnt = reinterpret_cast<int *>(cluster_smem_raw);
  int32_t *list = reinterpret_cast<int32_t *>(cluster_smem_raw) + 32;
  const int u = blockIdx.x, bh = blockIdx.y;
  const int m = cluster_members(u, bh, g, assign, list, warp_cnt);
  __syncthreads();
  if (threadIdx.x == 0) sizes[(size_t)bh * g.n_cells + u] = m;
  if (m == 0) return;  // an empty cluster keeps its centroid
  const __nv_bfloat16 *xb = x + (size_t)bh * g.n_pad * D;
  const float inv = 1.f / (float)m;
  for (int k = threadIdx.x; k < D; k += blockDim.x) {
    float s = 0.f;
#pragma unroll 8
    for (int r = 0; r < m; ++r) s += __bfloat162float(xb[(size_t)list[r] * D + k]);
    mu[((size_t)bh * g.n_cells + u) * D + k] = s * inv;
  }
}

__global__ void __launch_bounds__(kClusterThreads) cluster_perm_kernel(ClusterGeom g, const int32_t *__restrict__ assign,
                                                                       const int32_t *__restrict__ sizes,
                                                                       int32_t *__restrict__ perm) {
  extern __shared__ __align__(16) uint8_t cluster_smem_raw[];
  int *warp_cnt = reinterpret_cast<int *>(cluster_smem_raw);
  int32_t *list = reinterpret_cast<int32_t *>(cluster_smem_raw) + 32;
  __shared__ int s_off[kClusterThreads / 32];
  const int u = blockIdx.x, bh = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // offset of cluster u: the sizes of clusters 0 .. u-1
  int part = 0;
  const int32_t *sb = sizes + (size_t)bh * g.n_cells;
  for (int v = tid; v < u; v += kClusterThreads) part += sb[v];
  part = warp_sum_int(part);
  if (lane == 0) s_off[warp] = part;
  __syncthreads();
  int off = 0;
  for (int w = 0; w < kClusterThreads / 32; ++w) off += s_off[w];
  const int m = cluster_members(u, bh, g, assign, list, warp_cnt);
  __syncthreads();
  int32_t *pb = perm + (size_t)bh * g.n_pad;
  for (int r = tid; r < m; r += kClusterThreads) pb[off + r] = list[r];
  if (u == 0)
    for (int i = g.n_valid + tid; i < g.n_pad; i += kClusterThreads) pb[i] = i;  // padding rows stay
}

// One warp per row of row_words 32-bit words: gather dst[i] = src[perm[i]],
// or (inverse) scatter dst[perm[i]] = src[i].
__global__ void permute_rows_kernel(const uint32_t *__restrict__ src, const int32_t *__restrict__ perm, int n_pad,
                                    long long n_rows, int row_words, int inverse, uint32_t *__restrict__ dst) {
  const long long row = (long long)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  if (row >= n_rows) return;
  const int lane = threadIdx.x & 31;
  const long long bh = row / n_pad;
  const int p = __ldg(perm + row);
  if (p < 0 || p >= n_pad) {  // a caller-given permutation entry out of range: nothing is copied
    if (lane == 0) latch_status(VSA_ERR_BAD_INDEX);
    return;
  }
  const long long from = inverse ? row : bh * n_pad + p;
  const long long to = inverse ? bh * n_pad + p : row;
  const uint32_t *s = src + from * row_words;
  uint32_t *d = dst + to * row_words;
  if ((row_words & 3) == 0) {
    const uint4 *s4 = reinterpret_cast<const uint4 *>(s);
    uint4 *d4 = reinterpret_cast<uint4 *>(d);
    for (int w = lane; w < row_words / 4; w += 32) d4[w] = __ldg(s4 + w);
  } else {
    for (int w = lane; w < row_words; w += 32) d[w] = __ldg(s + w);
  }
}

}  // namespace vsa
