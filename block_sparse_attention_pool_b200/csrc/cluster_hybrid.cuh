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
  // the counting passes read the keys interleaved (coalesced)
  uint32_t T = 0u;
  for (int bit = 31; bit >= 0; --bit) {
    const uint32_t cand = T | (1u << bit);
    int c = 0;
    for (int i = t; i < n_valid; i += kHybThreads) c += __ldg(key + i) >= cand ? 1 : 0;
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
                                                       int32_t *__restrict__ assign, int32_t *__restrict__ changed,
                                                       int *status) {
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
        latch_status(status, VSA_ERR_BAD_INDEX);
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
                                                         int n_cells, int n_chunks, int32_t *__restrict__ cnt,
                                                         int *status) {
  extern __shared__ int hist[];
  const int chunk = blockIdx.x, bh = blockIdx.y;
  for (int u = threadIdx.x; u < n_cells; u += 256) hist[u] = 0;
  __syncthreads();
  const int32_t *ab = assign + (size_t)bh * n_valid;
  for (int i = chunk * kSortChunk + threadIdx.x; i < min(n_valid, (chunk + 1) * kSortChunk); i += 256) {
    const int u = __ldg(ab + i);
    if (u >= 0 && u < n_cells) atomicAdd(&hist[u], 1);
    else latch_status(status, VSA_ERR_BAD_INDEX);
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

// ---- global reassignment on the tensor cores ---------------------------------
//
// The same product as reassign_kernel, 128 cached tokens x 128 centroids per
// step, on tcgen05: A = the tokens' bf16 rows (exact), B = each centroid
// split into two bf16 rows, mu = hi + lo with hi = bf16(mu) and
// lo = bf16(mu - hi), both multiplied into one fp32 TMEM accumulator (the
// split leaves an error below 2^-16 |mu|; the fp32 norms |mu|^2 come from the
// fp32 centroids).  The operand tiles are written by the threads into 128-byte
// swizzled shared memory, the B tiles of chunk c + 1 while the MMAs of chunk c
// run, and two TMEM accumulators let the argmin of chunk c - 1 (thread i =
// TMEM lane i = token i) overlap the MMAs of chunk c.

constexpr int kRtThreads = 128;

template <int D>
struct RtLayout {
  static constexpr int kChunk = 128 * 128;                    // 128 rows x 64 bf16
  static constexpr int kKc = D / 64;                          // 64-column chunks of d
  static constexpr int kOffA = 0;                             // [kKc] token tiles
  static constexpr int kOffB = kOffA + kKc * kChunk;          // [2 buffers][2 parts][kKc]
  static constexpr int kOffN = kOffB + 2 * 2 * kKc * kChunk;  // [2][128] |mu|^2
  static constexpr int kOffCtl = kOffN + 2 * 128 * 4;
  static constexpr int kBytes = kOffCtl + 64;
  static constexpr int kAlloc = kBytes + 1024;
};

struct RtCtl {
  uint64_t done[2];
  uint64_t fin;
  uint32_t tmem_base;
  AbortCtl abort;
};

// Row r of a 128-row K-major bf16 tile, 64 columns from v (32 packed pairs).
__device__ __forceinline__ void rt_store_row(uint8_t *tile, int r, const uint32_t (&v)[32]) {
  uint8_t *row = tile + (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll
  for (int q = 0; q < 8; ++q)
    *reinterpret_cast<uint4 *>(row + ((q ^ (r & 7)) << 4)) = make_uint4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
}

template <int D>
__global__ void __launch_bounds__(kRtThreads, 1)
    reassign_tc_kernel(const __nv_bfloat16 *__restrict__ x, int n_pad, int n_valid, int n_cells,
                       const float *__restrict__ mu, const int32_t *__restrict__ subset, int n_sub,
                       int32_t *__restrict__ assign, int32_t *__restrict__ changed, unsigned long long timeout_ns,
                       int *status) {
  using L = RtLayout<D>;
  extern __shared__ uint8_t rt_smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(rt_smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  float *s_norm = reinterpret_cast<float *>(smem + L::kOffN);
  RtCtl *ctl = reinterpret_cast<RtCtl *>(smem + L::kOffCtl);
  AbortCtl *abort = &ctl->abort;
  const int bh = blockIdx.y, t = threadIdx.x, warp = t >> 5;
  const int i = blockIdx.x * kReTok + t;
  int tok = -1;
  if (i < n_sub) {
    tok = __ldg(subset + (size_t)bh * n_sub + i);
    if (tok < 0 || tok >= n_valid) {
      latch_status(status, VSA_ERR_BAD_INDEX);
      tok = -1;
    }
  }
  // the token tile: thread t writes row t (zeros past the subset)
  {
    const uint4 *src = reinterpret_cast<const uint4 *>(x + ((size_t)bh * n_pad + (tok >= 0 ? tok : 0)) * D);
#pragma unroll
    for (int kc = 0; kc < L::kKc; ++kc) {
      uint32_t v[32];
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const uint4 w = tok >= 0 ? __ldg(src + kc * 8 + q) : make_uint4(0u, 0u, 0u, 0u);
        v[4 * q] = w.x;
        v[4 * q + 1] = w.y;
        v[4 * q + 2] = w.z;
        v[4 * q + 3] = w.w;
      }
      rt_store_row(smem + L::kOffA + kc * L::kChunk, t, v);
    }
  }
  if (t == 0) {
    mbar_init(&ctl->done[0], 1);
    mbar_init(&ctl->done[1], 1);
    mbar_init(&ctl->fin, 1);
    abort_init(&ctl->abort, status);
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(&ctl->tmem_base, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;
  const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
  constexpr uint32_t kId = idesc_bf16_f32(128, 128, false);
  const float *mub = mu + (size_t)bh * n_cells * D;
  const int n_chunks = (n_cells + 127) / 128;
  float best = INFINITY;
  int bcell = 0x7fffffff;
  bool ok = true;

  auto argmin_chunk = [&](int c) {
    const int buf = c & 1;
    const float *nrm = s_norm + buf * 128;
#pragma unroll 1
    for (int c0 = 0; c0 < 128; c0 += 32) {
      uint32_t d[32];
      tmem_ld32(tmem + lane_off + buf * 128u + c0, d);
      tmem_ld_wait();
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const int cell = c * 128 + c0 + j;
        const float dist = fmaf(-2.f, __uint_as_float(d[j]), nrm[c0 + j]);
        if (cell < n_cells && (dist < best || (dist == best && cell < bcell))) {
          best = dist;
          bcell = cell;
        }
      }
    }
  };

  for (int c = 0; c < n_chunks && ok; ++c) {
    const int buf = c & 1;
    if (c >= 2) {
      const bool w = mbar_wait(&ctl->done[buf], ((c - 2) >> 1) & 1, abort, timeout_ns);
      ok = __syncthreads_and(w ? 1 : 0) != 0;
      if (!ok) break;
    }
    // centroid c * 128 + t: split into bf16 hi / lo rows, and its fp32 norm
    {
      const int cell = c * 128 + t;
      const float4 *src = reinterpret_cast<const float4 *>(mub + (size_t)(cell < n_cells ? cell : 0) * D);
      float nrm = 0.f;
#pragma unroll
      for (int kc = 0; kc < L::kKc; ++kc) {
        uint32_t hi[32], lo[32];
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          const float4 f = cell < n_cells ? __ldg(src + kc * 16 + q) : make_float4(0.f, 0.f, 0.f, 0.f);
          nrm = fmaf(f.x, f.x, nrm);
          nrm = fmaf(f.y, f.y, nrm);
          nrm = fmaf(f.z, f.z, nrm);
          nrm = fmaf(f.w, f.w, nrm);
          const __nv_bfloat162 h0 = __floats2bfloat162_rn(f.x, f.y), h1 = __floats2bfloat162_rn(f.z, f.w);
          const float2 g0 = __bfloat1622float2(h0), g1 = __bfloat1622float2(h1);
          const __nv_bfloat162 l0 = __floats2bfloat162_rn(f.x - g0.x, f.y - g0.y);
          const __nv_bfloat162 l1 = __floats2bfloat162_rn(f.z - g1.x, f.w - g1.y);
          hi[2 * q] = *reinterpret_cast<const uint32_t *>(&h0);
          hi[2 * q + 1] = *reinterpret_cast<const uint32_t *>(&h1);
          lo[2 * q] = *reinterpret_cast<const uint32_t *>(&l0);
          lo[2 * q + 1] = *reinterpret_cast<const uint32_t *>(&l1);
        }
        rt_store_row(smem + L::kOffB + ((buf * 2 + 0) * L::kKc + kc) * L::kChunk, t, hi);
        rt_store_row(smem + L::kOffB + ((buf * 2 + 1) * L::kKc + kc) * L::kChunk, t, lo);
      }
      s_norm[buf * 128 + t] = nrm;
    }
    fence_proxy_async_smem();
    __syncthreads();
    if (t == 0) {
      tc_fence_after();
      bool first = true;
#pragma unroll
      for (int part = 0; part < 2; ++part)
#pragma unroll
        for (int kc = 0; kc < L::kKc; ++kc) {
          const uint64_t da = smem_desc_sw128(smem_addr(smem + L::kOffA + kc * L::kChunk), 16, 1024);
          const uint64_t db = smem_desc_sw128(smem_addr(smem + L::kOffB + ((buf * 2 + part) * L::kKc + kc) * L::kChunk),
                                              16, 1024);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            umma_bf16_ss(tmem + buf * 128u, da + 2 * kk, db + 2 * kk, kId, first ? 0u : 1u);
            first = false;
          }
        }
      umma_commit(&ctl->done[buf]);
    }
    if (c >= 1) {
      const bool w = mbar_wait(&ctl->done[(c - 1) & 1], ((c - 1) >> 1) & 1, abort, timeout_ns);
      ok = __syncthreads_and(w ? 1 : 0) != 0;
      if (!ok) break;
      tc_fence_after();
      argmin_chunk(c - 1);
    }
  }
  if (ok) {
    const int c = n_chunks - 1;
    const bool w = mbar_wait(&ctl->done[c & 1], (c >> 1) & 1, abort, timeout_ns);
    ok = __syncthreads_and(w ? 1 : 0) != 0;
    if (ok) {
      tc_fence_after();
      argmin_chunk(c);
    }
  }
  // every MMA of the CTA has completed before TMEM and shared memory are released
  if (t == 0) umma_commit(&ctl->fin);
  const bool fin = mbar_drain(&ctl->fin, 0, timeout_ns);
  if (!fin) raise_timeout(status);
  if (ok && tok >= 0 && bcell < n_cells) {
    int32_t *ab = assign + (size_t)bh * n_valid;
    const int old = ab[tok];
    if (old != bcell) {
      ab[tok] = bcell;
      int32_t *ch = changed + (size_t)bh * n_cells;
      if (old >= 0 && old < n_cells) ch[old] = 1;
      ch[bcell] = 1;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 256);
}

}  // namespace vsa
