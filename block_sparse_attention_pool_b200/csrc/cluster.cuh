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
//                          window's centroids (<= 128, staged once) as an
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

// Shared memory of the assignment kernel: the cell's tokens and the window's
// centroids as fp32 rows (row stride D + 4 floats, 16-byte aligned) and the
// window's cell indices.  The centroid block is sized
// by the window (n_win rows, rounded up to 16).
template <int D>
struct AssignLayout {
  static constexpr int kLd = D + 4;
  static constexpr int kOffX = 0;
  static constexpr int kOffC = kOffX + kClusterMaxTokens * kLd * 4;
  static __host__ __device__ int off_win(int win_rows) { return kOffC + win_rows * kLd * 4; }
  static __host__ __device__ int bytes(int win_rows) { return off_win(win_rows) + kClusterMaxWindow * 4 + 16; }
};

// One CTA per cell.  Thread (ty, tx) scores tokens ty + 16 a (a < 8) against
// centroids tx + 16 b (b < NB): each 4-wide step of d loads 8 + NB float4 and
// issues 32 NB FMAs.  NB = ceil(window cells / 16) is a template parameter.
// RATIO: also write each token's Lowe ratio rho = d1 / d2 (HyperVAttention
// Eq. (6): Euclidean distances to the nearest and the second-nearest centroid
// of the window; 0 for a window of one centroid, 1 when both are 0).
template <int D, int NB, bool RATIO = false>
__global__ void __launch_bounds__(kClusterThreads) cluster_assign_kernel(const __nv_bfloat16 *__restrict__ x,
                                                                         ClusterGeom g, const float *__restrict__ mu,
                                                                         int32_t *__restrict__ assign,
                                                                         float *__restrict__ ratio) {
  using L = AssignLayout<D>;
  constexpr int kLd = L::kLd;
  constexpr int kRows = 16 * NB;
  extern __shared__ __align__(16) uint8_t cluster_smem_raw[];
  float(*sX)[kLd] = reinterpret_cast<float(*)[kLd]>(cluster_smem_raw + L::kOffX);
  float(*sC)[kLd] = reinterpret_cast<float(*)[kLd]>(cluster_smem_raw + L::kOffC);
  int *win = reinterpret_cast<int *>(cluster_smem_raw + L::off_win(kRows));
  __shared__ int s_tok[kClusterMaxTokens];  // lattice index of the cell's i-th token
  __shared__ int s_wcnt[kClusterMaxWindow / 32];
  const int u0 = blockIdx.x, bh = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int cw = u0 % g.CW, ch = (u0 / g.CW) % g.CH, ct = u0 / (g.CW * g.CH);
  const TokBox box = cell_box(ct, ct + 1, ch, ch + 1, cw, cw + 1, g);
  const int n_tok = box.size();

  // token table; window cells in (t, h, w) loop order = ascending flat index,
  // compacted by ballot over the first four warps
  int wcell = -1;
  if (tid < kClusterMaxTokens) s_tok[tid] = tid < n_tok ? box.token(tid, g) : -1;
  if (tid < kClusterMaxWindow) {
    if (tid < g.wt * g.wh * g.ww) {
      const int dw = tid % g.ww, dh = (tid / g.ww) % g.wh, dt = tid / (g.ww * g.wh);
      const int t = ct + win_lo(g.wt) + dt, h = ch + win_lo(g.wh) + dh, w = cw + win_lo(g.ww) + dw;
      if (t >= 0 && t < g.CT && h >= 0 && h < g.CH && w >= 0 && w < g.CW) wcell = (t * g.CH + h) * g.CW + w;
    }
    const uint32_t bal = __ballot_sync(0xffffffffu, wcell >= 0);
    if (lane == 0) s_wcnt[warp] = __popc(bal);
    __syncwarp();
    wcell = wcell >= 0 ? (wcell | (__popc(bal & ((1u << lane) - 1u)) << 24)) : -1;  // rank inside the warp
  }
  __syncthreads();
  int n_win = 0;
#pragma unroll
  for (int w = 0; w < kClusterMaxWindow / 32; ++w) n_win += s_wcnt[w];
  if (tid < kClusterMaxWindow && wcell >= 0) {
    int before = 0;
    for (int w = 0; w < warp; ++w) before += s_wcnt[w];
    const int pos = before + (wcell >> 24);
    if (pos < kRows) win[pos] = wcell & 0xffffff;
  }
  n_win = min(n_win, kRows);
  __syncthreads();

  // the cell's tokens (zero rows past n_tok) and the window's centroids (zero
  // rows past n_win), fp32
  const __nv_bfloat16 *xb = x + (size_t)bh * g.n_pad * D;
  for (int e = tid; e < kClusterMaxTokens * (D / 8); e += kClusterThreads) {
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
  const float *mub = mu + (size_t)bh * g.n_cells * D;
  for (int e = tid; e < kRows * (D / 4); e += kClusterThreads) {
    const int j = e / (D / 4), k4 = e % (D / 4);
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (j < n_win) v = __ldg(reinterpret_cast<const float4 *>(mub + (size_t)win[j] * D) + k4);
    *reinterpret_cast<float4 *>(&sC[j][4 * k4]) = v;
  }
  __syncthreads();

  // dot products and, alongside, |mu|^2 of this thread's centroids (every
  // thread that holds a centroid sums it in the same order)
  const int ty = tid >> 4, tx = tid & 15;
  float acc[8][NB], cn[NB], xn[8];
#pragma unroll
  for (int a = 0; a < 8; ++a) xn[a] = 0.f;
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
      if constexpr (RATIO) {
        xn[a] = fmaf(xv.x, xv.x, xn[a]);
        xn[a] = fmaf(xv.y, xv.y, xn[a]);
        xn[a] = fmaf(xv.z, xv.z, xn[a]);
        xn[a] = fmaf(xv.w, xv.w, xn[a]);
      }
#pragma unroll
      for (int b = 0; b < NB; ++b) {
        acc[a][b] = fmaf(xv.x, cv[b].x, acc[a][b]);
        acc[a][b] = fmaf(xv.y, cv[b].y, acc[a][b]);
        acc[a][b] = fmaf(xv.z, cv[b].z, acc[a][b]);
        acc[a][b] = fmaf(xv.w, cv[b].w, acc[a][b]);
      }
    }
  }
  int32_t *ab = assign + (size_t)bh * g.n_valid;
#pragma unroll
  for (int a = 0; a < 8; ++a) {
    float d = INFINITY, d2 = INFINITY;  // best and second-best |mu|^2 - 2 x.mu
    int c = 0x7fffffff;
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      const int j = tx + 16 * b;
      if (j < n_win) {
        const float dist = fmaf(-2.f, acc[a][b], cn[b]);
        const int cell = win[j];
        if (dist < d || (dist == d && cell < c)) {
          d2 = d;
          d = dist;
          c = cell;
        } else {
          d2 = fminf(d2, dist);
        }
      }
    }
    // argmin across the 16 threads (tx) that share a token; the second best is
    // the smaller of the losing best and the two second bests
#pragma unroll
    for (int o = 1; o < 16; o <<= 1) {
      const float od = __shfl_xor_sync(0xffffffffu, d, o);
      const int oc = __shfl_xor_sync(0xffffffffu, c, o);
      const float od2 = __shfl_xor_sync(0xffffffffu, d2, o);
      d2 = fminf(fminf(d2, od2), fmaxf(d, od));
      if (od < d || (od == d && oc < c)) {
        d = od;
        c = oc;
      }
    }
    const int i = ty + 16 * a;
    if (tx == 0 && i < n_tok) {
      ab[s_tok[i]] = c;
      if constexpr (RATIO) {
        const float e1 = fmaxf(0.f, xn[a] + d), e2 = d2 == INFINITY ? INFINITY : fmaxf(0.f, xn[a] + d2);
        const float rho = e2 == INFINITY ? 0.f : (e2 > 0.f ? sqrtf(e1) / sqrtf(e2) : 1.f);
        ratio[(size_t)bh * g.n_valid + s_tok[i]] = rho;
      }
    }
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
                                    long long n_rows, int row_words, int inverse, uint32_t *__restrict__ dst,
                                    int *status) {
  const long long row = (long long)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  if (row >= n_rows) return;
  const int lane = threadIdx.x & 31;
  const long long bh = row / n_pad;
  const int p = __ldg(perm + row);
  if (p < 0 || p >= n_pad) {  // a caller-given permutation entry out of range: nothing is copied
    if (lane == 0) latch_status(status, VSA_ERR_BAD_INDEX);
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
