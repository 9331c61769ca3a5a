// a2 + a3 Pooled scoring and block selection, and the explicit-mask path.
//
// HyperVAttention section 2 Eq. (2): S_ij = <mu_i, mu_j> / sqrt(d) and the
// size-weighted softmax P'_ij = s_j e^{S_ij} / sum_o s_o e^{S_io}; Eq. (3):
// row-wise Top-p, the smallest prefix of key blocks in descending P' whose
// mass reaches p; App. A.1 "Min-kc": a floor on the kept count; the LVSA
// abstract: rotating global anchor columns.
//
// One CTA owns 16 query-block rows of one (batch, head).  It stages the 16
// pooled query rows and 32-key chunks of the pooled keys in shared memory and
// computes the 16 x n_k logits with fp32 FFMA (no TF32, so the ranking
// matches an fp64 evaluation wherever two blocks differ by more than fp32
// rounding).  Each warp then ranks two rows: the n_k log-weights
// w = S + ln s_j, packed with the key index into 64-bit keys, are bitonic-
// sorted in registers (32 keys per lane at most, n_k <= 1024), the sorted
// weights are exponentiated and prefix-summed, and the kept prefix plus the
// anchors is written out as an ascending index list with ballot compaction.
// A fixed count (fixed_k > 0) needs the set of the k largest weights only: that
// instantiation keeps 32-bit keys, finds the k-th largest by a bitwise search
// and marks the set without sorting (same set as the sort, ties to the lower
// block index).
#pragma once

#include "common.cuh"

namespace vsa {

constexpr int kSelRows = 16;
constexpr int kSelThreads = 256;
constexpr int kSelChunk = 64;

struct SelectArgs {
  const float *q_pool;  // [BH, n_q, d]
  const float *k_pool;  // [BH, n_k, d]
  int n_q, n_k, bq, bk, n_valid;
  float scale;
  int k_min, fixed_k, n_anchor, anchor_rot;
  float cum_mass;
  int32_t *counts;  // [BH, n_q]
  int32_t *idx;     // [BH, n_q, n_k]
  uint8_t *mask;    // [BH, n_q, n_k] or null
  // cluster mode (HyperVAttention Eq. (2) on clusters): explicit sizes of the
  // query and key units [BH, n_q] / [BH, n_k] replace the block sizes implied
  // by n_valid; null in block mode
  const int32_t *q_sizes;
  const int32_t *k_sizes;
};

// Compare-exchange of the in-register pairs (i, i | J) of a bitonic substage.
template <int NR, int J>
__device__ __forceinline__ void bitonic_in_lane(uint64_t (&key)[NR], int lane, int kk) {
#pragma unroll
  for (int i = 0; i < NR; ++i) {
    if ((i & J) == 0) {
      const bool desc = ((lane * NR + i) & kk) == 0;
      const uint64_t a = key[i], b = key[i | J];
      const bool swap = desc ? (a < b) : (a > b);
      key[i] = swap ? b : a;
      key[i | J] = swap ? a : b;
    }
  }
}

template <int NR, int J>
__device__ __forceinline__ void bitonic_in_lane_dispatch(uint64_t (&key)[NR], int lane, int kk, int j) {
  if constexpr (J >= 1) {
    if (j == J) {
      bitonic_in_lane<NR, J>(key, lane, kk);
      return;
    }
    bitonic_in_lane_dispatch<NR, J / 2>(key, lane, kk, j);
  }
}

// Bitonic sort, descending, of NR * 32 64-bit keys held NR per lane; the key at
// sorted position e = lane * NR + i ends in register i of that lane.  The
// stage loops run at run time and only the per-register bodies are unrolled,
// which keeps the code small enough for the instruction cache.
template <int NR>
__device__ __forceinline__ void warp_bitonic_sort_desc(uint64_t (&key)[NR], int lane) {
  constexpr int N = NR * 32;
#pragma unroll 1
  for (int kk = 2; kk <= N; kk <<= 1) {
#pragma unroll 1
    for (int j = kk >> 1; j > 0; j >>= 1) {
      if (j >= NR) {
        // partner in lane ^ (j / NR), same register
        const int lx = j / NR;
        const bool lower = (lane & lx) == 0;
#pragma unroll
        for (int i = 0; i < NR; ++i) {
          const bool desc = ((lane * NR + i) & kk) == 0;
          const uint64_t other = __shfl_xor_sync(0xffffffffu, key[i], lx);
          const uint64_t mx = key[i] > other ? key[i] : other;
          const uint64_t mn = key[i] > other ? other : key[i];
          key[i] = (desc == lower) ? mx : mn;
        }
      } else {
        bitonic_in_lane_dispatch<NR, (NR > 1 ? NR / 2 : 0)>(key, lane, kk, j);
      }
    }
  }
}

// Fixed count: mark in the warp bitmap the m largest of the row's score keys
// (element j = 32 i + lane in register i; equal keys go to the lower j;
// 1 <= m <= number of real elements, padding keys are 0).  The set needs no
// order, so instead of a sort the m-th largest key H is found bit by bit
// (the largest H with #(key >= H) >= m), and of the keys equal to H the
// lowest-index ones fill the rank.  Word i of the bitmap is register i's ballot.
template <int NR>
__device__ __forceinline__ void mark_top_m(const uint32_t (&hk)[NR], int m, int lane, uint32_t *bits) {
  uint32_t H = 0u;
#pragma unroll 1
  for (int b = 31; b >= 0; --b) {
    const uint32_t cand = H | (1u << b);
    unsigned c = 0u;
#pragma unroll
    for (int i = 0; i < NR; ++i) c += hk[i] >= cand ? 1u : 0u;
    if (static_cast<int>(__reduce_add_sync(0xffffffffu, c)) >= m) H = cand;
  }
  unsigned above = 0u;
#pragma unroll
  for (int i = 0; i < NR; ++i) above += hk[i] > H ? 1u : 0u;
  const int need = m - static_cast<int>(__reduce_add_sync(0xffffffffu, above));
  const uint32_t lt = (1u << lane) - 1u;
  int before = 0;  // keys equal to H at lower element indices
#pragma unroll
  for (int i = 0; i < NR; ++i) {
    const uint32_t eq = __ballot_sync(0xffffffffu, hk[i] == H);
    const bool sel = hk[i] > H || (hk[i] == H && before + __popc(eq & lt) < need);
    const uint32_t word = __ballot_sync(0xffffffffu, sel);
    if (lane == (i & 31)) bits[i] = word;
    before += __popc(eq);
  }
}

// Emit the ascending index list of the set bits of a per-warp bitmap of n bits
// (word w covers indices [32w, 32w + 32)); returns the count.
__device__ __forceinline__ int emit_bitmap_list(const uint32_t *bits, int n, int lane, int32_t *dst,
                                                uint8_t *mask_row) {
  int total = 0;
  for (int w0 = 0; w0 * 32 < n; w0 += 32) {
    const int w = w0 + lane;
    const uint32_t word = (w * 32 < n) ? bits[w] : 0u;
    const int cnt = __popc(word);
    const int off = warp_exclusive_scan(cnt, lane);
    uint32_t rest = word;
    int o = total + off;
    while (rest) {
      const int b = __ffs(rest) - 1;
      rest &= rest - 1;
      dst[o++] = w * 32 + b;
    }
    if (mask_row && w * 32 < n) {
      const int lim = min(32, n - w * 32);
      for (int b = 0; b < lim; ++b) mask_row[w * 32 + b] = (word >> b) & 1u;
    }
    total += __shfl_sync(0xffffffffu, off + cnt, 31);
  }
  return total;
}

// Dynamic shared memory of select_blocks_kernel: the query rows and a key
// chunk (rows padded to d + 4 floats), the logits of the CTA's rows (nkp
// columns), one 32-word bitmap per warp.  The host sizes the launch with this.
__host__ __device__ constexpr size_t select_smem_bytes(int d, int nkp) {
  return (size_t)(kSelRows + kSelChunk) * (d + 4) * 4 + (size_t)kSelRows * nkp * 4 + 8 * 32 * 4;
}

template <int D, int NR, bool BY_RANK>
__global__ void __launch_bounds__(kSelThreads) select_blocks_kernel(SelectArgs a) {
  constexpr int DP = D + 4;  // padded row stride (floats)
  extern __shared__ __align__(16) float sel_smem[];
  float *qs = sel_smem;                       // [kSelRows][DP]
  float *ks = qs + kSelRows * DP;             // [kSelChunk][DP]
  const int nkp = NR * 32;
  float *S = ks + kSelChunk * DP;             // [kSelRows][nkp]
  uint32_t *bitmap = reinterpret_cast<uint32_t *>(S + kSelRows * nkp);  // [8 warps][32]

  const int bh = blockIdx.y;
  const int row0 = blockIdx.x * kSelRows;
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const float *qp = a.q_pool + (size_t)bh * a.n_q * D;
  const float *kp = a.k_pool + (size_t)bh * a.n_k * D;

  for (int i = t; i < kSelRows * (D / 4); i += kSelThreads) {
    const int r = i / (D / 4), c4 = i % (D / 4);
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (row0 + r < a.n_q) v = __ldg(reinterpret_cast<const float4 *>(qp + (size_t)(row0 + r) * D) + c4);
    *reinterpret_cast<float4 *>(qs + r * DP + c4 * 4) = v;
  }

  // ---- logits: warp w -> rows 2w, 2w+1; lane -> keys lane, lane + 32 of the chunk
  const int r0 = 2 * warp;
  for (int k0 = 0; k0 < a.n_k; k0 += kSelChunk) {
    __syncthreads();
    for (int i = t; i < kSelChunk * (D / 4); i += kSelThreads) {
      const int r = i / (D / 4), c4 = i % (D / 4);
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (k0 + r < a.n_k) v = __ldg(reinterpret_cast<const float4 *>(kp + (size_t)(k0 + r) * D) + c4);
      *reinterpret_cast<float4 *>(ks + r * DP + c4 * 4) = v;
    }
    __syncthreads();
    float s00 = 0.f, s01 = 0.f, s10 = 0.f, s11 = 0.f;
    const float *q0 = qs + r0 * DP, *q1 = qs + (r0 + 1) * DP;
    const float *ka = ks + lane * DP, *kb = ks + (lane + 32) * DP;
#pragma unroll 8
    for (int c = 0; c < D; c += 4) {
      const float4 x0 = *reinterpret_cast<const float4 *>(q0 + c);
      const float4 x1 = *reinterpret_cast<const float4 *>(q1 + c);
      const float4 ya = *reinterpret_cast<const float4 *>(ka + c);
      const float4 yb = *reinterpret_cast<const float4 *>(kb + c);
      s00 = fmaf(x0.x, ya.x, s00); s00 = fmaf(x0.y, ya.y, s00); s00 = fmaf(x0.z, ya.z, s00); s00 = fmaf(x0.w, ya.w, s00);
      s01 = fmaf(x0.x, yb.x, s01); s01 = fmaf(x0.y, yb.y, s01); s01 = fmaf(x0.z, yb.z, s01); s01 = fmaf(x0.w, yb.w, s01);
      s10 = fmaf(x1.x, ya.x, s10); s10 = fmaf(x1.y, ya.y, s10); s10 = fmaf(x1.z, ya.z, s10); s10 = fmaf(x1.w, ya.w, s10);
      s11 = fmaf(x1.x, yb.x, s11); s11 = fmaf(x1.y, yb.y, s11); s11 = fmaf(x1.z, yb.z, s11); s11 = fmaf(x1.w, yb.w, s11);
    }
    if (k0 + lane < nkp) {
      S[r0 * nkp + k0 + lane] = s00 * a.scale;
      S[(r0 + 1) * nkp + k0 + lane] = s10 * a.scale;
    }
    if (k0 + lane + 32 < nkp) {
      S[r0 * nkp + k0 + lane + 32] = s01 * a.scale;
      S[(r0 + 1) * nkp + k0 + lane + 32] = s11 * a.scale;
    }
  }
  __syncthreads();

  // ---- per-row ranking and selection, two rows per warp
  const float ln_bk = logf((float)a.bk);
  uint32_t *bits = bitmap + warp * 32;
  for (int rr = 0; rr < kSelRows / 8; ++rr) {
    const int r = warp * (kSelRows / 8) + rr;
    const int qi = row0 + r;
    if (qi >= a.n_q) break;
    const size_t orow = (size_t)bh * a.n_q + qi;
    int32_t *dst = a.idx + orow * a.n_k;
    uint8_t *mrow = a.mask ? a.mask + orow * a.n_k : nullptr;
    const bool q_has_rows = a.q_sizes ? __ldg(a.q_sizes + orow) > 0 : qi * a.bq < a.n_valid;

    if constexpr (BY_RANK) {
      // fixed count (fixed_k > 0): the k largest log-weights, no order needed
      uint32_t hk[NR];
#pragma unroll
      for (int i = 0; i < NR; ++i) {
        const int j = i * 32 + lane;
        uint32_t kv = 0u;
        if (j < a.n_k) {
          const int sj = a.k_sizes ? __ldg(a.k_sizes + (size_t)bh * a.n_k + j) : min(a.bk, max(0, a.n_valid - j * a.bk));
          const float w = sj > 0 ? S[r * nkp + j] + (sj == a.bk ? ln_bk : logf((float)sj)) : -INFINITY;
          kv = float_key(w);
        }
        hk[i] = kv;
      }
      bits[lane] = 0u;
      __syncwarp();
      if (q_has_rows) mark_top_m<NR>(hk, min(a.fixed_k, a.n_k), lane, bits);
      __syncwarp();
      if (q_has_rows && lane == 0 && a.n_anchor > 0) {
        const int step = a.n_k / a.n_anchor;
        for (int tt = 0; tt < a.n_anchor; ++tt) {
          const int j = (int)(((long long)a.anchor_rot + (long long)tt * step) % a.n_k);
          atomicOr(&bits[j >> 5], 1u << (j & 31));
        }
      }
    } else {
      // Load: element j = i*32 + lane goes to register i (any start placement
      // sorts to the same result).
      uint64_t key[NR];
  #pragma unroll
      for (int i = 0; i < NR; ++i) {
        const int j = i * 32 + lane;
        if (j < a.n_k) {
          const int sj = a.k_sizes ? __ldg(a.k_sizes + (size_t)bh * a.n_k + j) : min(a.bk, max(0, a.n_valid - j * a.bk));
          const float w = sj > 0 ? S[r * nkp + j] + (sj == a.bk ? ln_bk : logf((float)sj)) : -INFINITY;
          key[i] = ((uint64_t)float_key(w) << 32) | (uint64_t)(0xffffffffu - (uint32_t)j);
        } else {
          key[i] = 0ull;
        }
      }
      warp_bitonic_sort_desc<NR>(key, lane);

      int m = 0;
      if (q_has_rows) {
        if (a.fixed_k > 0) {
          m = min(a.fixed_k, a.n_k);
        } else {
          int m_p = 0;
          if (a.cum_mass > 0.f) {
            const float wmax = key_float((uint32_t)(__shfl_sync(0xffffffffu, key[0], 0) >> 32));
            float p[NR];
            float lsum = 0.f;
  #pragma unroll
            for (int i = 0; i < NR; ++i) {
              const bool real = key[i] != 0ull;
              const float w = key_float((uint32_t)(key[i] >> 32));
              p[i] = (real && w != -INFINITY) ? expf(w - wmax) : 0.f;
              lsum += p[i];
              p[i] = lsum;  // inclusive lane-local prefix
            }
            // exclusive prefix of lane totals
            float base = lsum;
  #pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
              const float y = __shfl_up_sync(0xffffffffu, base, o);
              if (lane >= o) base += y;
            }
            const float total = __shfl_sync(0xffffffffu, base, 31);
            base -= lsum;
            const float target = a.cum_mass * total;
            int first = 0x7fffffff;
  #pragma unroll
            for (int i = NR - 1; i >= 0; --i)
              if (base + p[i] >= target) first = lane * NR + i;
  #pragma unroll
            for (int o = 16; o > 0; o >>= 1) first = min(first, __shfl_xor_sync(0xffffffffu, first, o));
            m_p = first == 0x7fffffff ? a.n_k : first + 1;
          }
          m = min(a.n_k, max(a.k_min, m_p));
        }
      }

      // mark the kept prefix and the anchors
      bits[lane] = 0u;
      __syncwarp();
      if (q_has_rows) {
  #pragma unroll
        for (int i = 0; i < NR; ++i) {
          if (lane * NR + i < m) {
            const int j = (int)(0xffffffffu - (uint32_t)(key[i] & 0xffffffffull));
            atomicOr(&bits[j >> 5], 1u << (j & 31));
          }
        }
        if (lane == 0 && a.n_anchor > 0) {
          const int step = a.n_k / a.n_anchor;
          for (int tt = 0; tt < a.n_anchor; ++tt) {
            const int j = (int)(((long long)a.anchor_rot + (long long)tt * step) % a.n_k);
            atomicOr(&bits[j >> 5], 1u << (j & 31));
          }
        }
      }
    }
    __syncwarp();
    const int total = emit_bitmap_list(bits, a.n_k, lane, dst, mrow);
    if (lane == 0) a.counts[orow] = total;
    __syncwarp();
  }
}

// ---- rows of more than 1024 key units ----------------------------------------
// The same selection rule for rows too long for a warp's registers, one CTA
// per row.  The kept set is the top m of the log-weights (ties to the lower
// index) for m = fixed_k, or m = max(k_min, m_p) where m_p, the length of the
// shortest descending prefix whose mass reaches cum_mass, comes from the value
// H* of its last element: the largest H with mass(w >= H) >= cum_mass (the
// mass above a value only falls as the value rises), plus the few elements
// tied at H* that the prefix needs.  Both searches run bit by bit over the
// order-preserving 32-bit keys, so no sort is needed.
constexpr int kLongThreads = 256;
constexpr int kLongPerThread = 16;
constexpr int kSelLongMax = kLongThreads * kLongPerThread;  // 4096 key units

__device__ __forceinline__ unsigned block_sum_u32(unsigned v, unsigned *red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  v = __reduce_add_sync(0xffffffffu, v);
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  unsigned t = 0u;
#pragma unroll
  for (int w = 0; w < kLongThreads / 32; ++w) t += red[w];
  return t;
}

__device__ __forceinline__ float block_sum_f32(float v, float *red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float t = 0.f;
#pragma unroll
  for (int w = 0; w < kLongThreads / 32; ++w) t += red[w];
  return t;
}

template <int D>
__global__ void __launch_bounds__(kLongThreads) select_long_kernel(SelectArgs a) {
  __shared__ __align__(16) float qs[D];
  __shared__ uint32_t bits[kSelLongMax / 32];
  __shared__ float red_f[kLongThreads / 32];
  __shared__ unsigned red_u[kLongThreads / 32];
  __shared__ unsigned scan[kLongThreads / 32];
  const int qi = blockIdx.x, bh = blockIdx.y;
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const size_t orow = (size_t)bh * a.n_q + qi;
  const float *qp = a.q_pool + orow * D;
  const float *kp = a.k_pool + (size_t)bh * a.n_k * D;
  for (int c = t; c < D; c += kLongThreads) qs[c] = __ldg(qp + c);
  for (int w = t; w < kSelLongMax / 32; w += kLongThreads) bits[w] = 0u;
  __syncthreads();
  const bool q_has_rows = a.q_sizes ? __ldg(a.q_sizes + orow) > 0 : qi * a.bq < a.n_valid;
  const float ln_bk = logf((float)a.bk);

  // log-weights of this thread's units j = i * 256 + t, as order-preserving keys (0 = no unit)
  uint32_t hk[kLongPerThread];
  float wv[kLongPerThread];
  float wmax = -INFINITY;
#pragma unroll
  for (int i = 0; i < kLongPerThread; ++i) {
    const int j = i * kLongThreads + t;
    hk[i] = 0u;
    wv[i] = -INFINITY;
    if (j < a.n_k) {
      const float4 *k4 = reinterpret_cast<const float4 *>(kp + (size_t)j * D);
      float acc = 0.f;
#pragma unroll 8
      for (int c = 0; c < D / 4; ++c) {
        const float4 y = __ldg(k4 + c);
        acc = fmaf(qs[4 * c], y.x, acc);
        acc = fmaf(qs[4 * c + 1], y.y, acc);
        acc = fmaf(qs[4 * c + 2], y.z, acc);
        acc = fmaf(qs[4 * c + 3], y.w, acc);
      }
      const int sj = a.k_sizes ? __ldg(a.k_sizes + (size_t)bh * a.n_k + j) : min(a.bk, max(0, a.n_valid - j * a.bk));
      const float w = sj > 0 ? acc * a.scale + (sj == a.bk ? ln_bk : logf((float)sj)) : -INFINITY;
      hk[i] = float_key(w);
      wv[i] = w;
      wmax = fmaxf(wmax, w);
    }
  }

  int m = 0;
  if (q_has_rows) {
    if (a.fixed_k > 0) {
      m = min(a.fixed_k, a.n_k);
    } else {
      int m_p = 0;
      if (a.cum_mass > 0.f) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) wmax = fmaxf(wmax, __shfl_xor_sync(0xffffffffu, wmax, o));
        __syncthreads();
        if (lane == 0) red_f[warp] = wmax;
        __syncthreads();
        float gmax = -INFINITY;
#pragma unroll
        for (int w = 0; w < kLongThreads / 32; ++w) gmax = fmaxf(gmax, red_f[w]);
        float p[kLongPerThread];
        float lsum = 0.f;
#pragma unroll
        for (int i = 0; i < kLongPerThread; ++i) {
          p[i] = wv[i] != -INFINITY ? expf(wv[i] - gmax) : 0.f;
          lsum += p[i];
        }
        const float target = a.cum_mass * block_sum_f32(lsum, red_f);
        // H* = the largest key whose upper set holds the target mass
        uint32_t H = 0u;
#pragma unroll 1
        for (int b = 31; b >= 0; --b) {
          const uint32_t cand = H | (1u << b);
          float f = 0.f;
#pragma unroll
          for (int i = 0; i < kLongPerThread; ++i) f += hk[i] >= cand ? p[i] : 0.f;
          if (block_sum_f32(f, red_f) >= target) H = cand;
        }
        float above = 0.f, tie_p = 0.f;
        unsigned n_above = 0u, n_tie = 0u;
#pragma unroll
        for (int i = 0; i < kLongPerThread; ++i) {
          if (hk[i] > H) {
            above += p[i];
            ++n_above;
          } else if (hk[i] == H && hk[i] != 0u) {
            tie_p = p[i];
            ++n_tie;
          }
        }
        const float mass_above = block_sum_f32(above, red_f);
        const unsigned cnt_above = block_sum_u32(n_above, red_u);
        const unsigned cnt_tie = block_sum_u32(n_tie, red_u);
        const float ptie = block_sum_f32(n_tie ? tie_p : 0.f, red_f) / fmaxf(1.f, (float)block_sum_u32(n_tie ? 1u : 0u, red_u));
        int need = 1;
        if (cnt_tie > 1u && ptie > 0.f) need = (int)ceilf((target - mass_above) / ptie);
        need = max(1, min((int)cnt_tie, need));
        m_p = cnt_tie == 0u ? a.n_k : (int)cnt_above + need;
      }
      m = min(a.n_k, max(a.k_min, m_p));
    }
  }

  if (m > 0) {
    // the m largest keys, ties to the lower index: the m-th largest value H,
    // then the lowest-index keys equal to H for the rest of the rank
    uint32_t H = 0u;
#pragma unroll 1
    for (int b = 31; b >= 0; --b) {
      const uint32_t cand = H | (1u << b);
      unsigned c = 0u;
#pragma unroll
      for (int i = 0; i < kLongPerThread; ++i) c += hk[i] >= cand ? 1u : 0u;
      if ((int)block_sum_u32(c, red_u) >= m) H = cand;
    }
    unsigned above = 0u;
#pragma unroll
    for (int i = 0; i < kLongPerThread; ++i) above += hk[i] > H ? 1u : 0u;
    const int need = m - (int)block_sum_u32(above, red_u);
    int before = 0;  // keys equal to H at lower indices (index order: i-major, then thread)
    const uint32_t lt = (1u << lane) - 1u;
#pragma unroll 1
    for (int i = 0; i < kLongPerThread; ++i) {
      const bool eq = hk[i] == H;
      const uint32_t bal = __ballot_sync(0xffffffffu, eq);
      __syncthreads();
      if (lane == 0) scan[warp] = __popc(bal);
      __syncthreads();
      int wbase = 0, tot = 0;
      for (int w = 0; w < kLongThreads / 32; ++w) {
        if (w < warp) wbase += scan[w];
        tot += scan[w];
      }
      const int j = i * kLongThreads + t;
      const bool sel = hk[i] > H || (eq && before + wbase + __popc(bal & lt) < need);
      if (sel && j < a.n_k) atomicOr(&bits[j >> 5], 1u << (j & 31));
      before += tot;
    }
  }
  if (q_has_rows && t == 0 && a.n_anchor > 0) {
    const int step = a.n_k / a.n_anchor;
    for (int tt = 0; tt < a.n_anchor; ++tt) {
      const int j = (int)(((long long)a.anchor_rot + (long long)tt * step) % a.n_k);
      atomicOr(&bits[j >> 5], 1u << (j & 31));
    }
  }
  __syncthreads();
  if (warp == 0) {
    const int total = emit_bitmap_list(bits, a.n_k, lane, a.idx + orow * a.n_k, a.mask ? a.mask + orow * a.n_k : nullptr);
    if (lane == 0) a.counts[orow] = total;
  }
}

// Explicit uint8 block mask -> ascending lists: one warp per row.
// Rows longer than 1024 columns go in segments of 1024.
__global__ void mask_to_lists_kernel(const uint8_t *__restrict__ mask, int rows, int n_k,
                                     int32_t *__restrict__ counts, int32_t *__restrict__ idx) {
  __shared__ uint32_t bitmap[8][32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int row = blockIdx.x * 8 + warp;
  if (row >= rows) return;
  const uint8_t *m = mask + (size_t)row * n_k;
  uint32_t *bits = bitmap[warp];
  int total = 0;
  for (int seg = 0; seg < n_k; seg += 1024) {
    const int n = min(1024, n_k - seg);
    uint32_t word = 0u;
    for (int b = 0; b < 32; ++b) {
      const int j = lane * 32 + b;
      if (j < n && m[seg + j] != 0) word |= 1u << b;
    }
    bits[lane] = word;
    __syncwarp();
    int32_t *dst = idx + (size_t)row * n_k + total;
    const int c = emit_bitmap_list(bits, n, lane, dst, nullptr);
    __syncwarp();
    // emit_bitmap_list writes indices within the segment: shift them
    for (int e = lane; e < c; e += 32) dst[e] += seg;
    total += c;
    __syncwarp();
  }
  if (lane == 0) counts[row] = total;
}

}  // namespace vsa
