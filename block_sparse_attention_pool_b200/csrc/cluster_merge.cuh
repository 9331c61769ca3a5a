// Hardware-aware cluster merging (HyperVAttention section 4.3, Eq. (7)-(10),
// Algorithm 1 "Parallel Agglomerative Merging").
//
// A group S of query clusters costs C(S) = ceil(s_q(S) / tau_q) *
// ceil(w_k(S) / tau_k) tiles, s_q the summed query sizes and w_k the summed
// sizes of the union chi(S) of the key clusters its members selected (Eq. (8);
// counted in tiles, i.e. Eq. (8) divided by tau_q * tau_k, which orders every
// candidate the same way).  Each round splits the active groups by a given bit
// per group leader (the random bipartition, passed in), evaluates every
// cross pair (A, B), lets each A pick the B of smallest dC = C(A u B) - C(A) -
// C(B) (Eq. (10)), keeps for each B the A of smallest dC among those that
// picked it, and applies the pairs with dC < 0 at once.
//
// The pair evaluation is a dense contraction: w_k(A u B) = w_k(A) + w_k(B) -
// I(A, B) with I(A, B) = sum_j chi_j(A) chi_j(B) s^k_j, i.e. I = X_A diag(s)
// X_B^T over the 0/1 membership rows X.  It runs on the tensor cores: a CTA
// takes 128 A-groups x 128 B-groups, builds the fp16 operand tiles in shared
// memory straight from the groups' chi bitmasks (A: 0/1, B: chi_j * digit_j
// of the key sizes in base 2048, one pass per nonzero digit, at most three),
// accumulates each digit's product in its own fp32 TMEM accumulator (every
// partial sum is an integer below 2^24, so exact), and the epilogue (thread i
// owns TMEM lane i = A-group i) turns each column into dC and keeps its
// row's minimum; CTAs of the same A-rows combine through a 64-bit atomicMin
// on (dC, B index).
//
// Groups are identified by their lowest member (the leader).  A query cluster
// of size zero keeps nothing and can never lower a cost, so it never merges
// and is left out of the rounds.
#pragma once

#include <cuda_fp16.h>

#include "common.cuh"
#include "select.cuh"

namespace vsa {

constexpr int kMergeMaxClusters = 1024;  // query and key clusters per head
constexpr int kMergeWords = 32;          // chi bitmask words per group
constexpr int kMergeTile = 128;          // groups per CTA side
constexpr int kMergeThreads = 128;
constexpr int kMergeHeadThreads = 1024;
constexpr int kMergeChunkKeys = 64;                   // key clusters per operand chunk
constexpr int kMergeTileBytes = kMergeTile * 128;     // 128 rows x 64 fp16
constexpr long long kDcBias = 1ll << 52;              // dC field of the pair key: dC + 2^52 (clamped)
constexpr unsigned long long kNoPair = ~0ull;

struct MergeWs {
  int32_t *lead;              // [BH][nq] leader of each cluster's group
  int32_t *gsq;               // [BH][nq] query tokens of the group (at leaders)
  int32_t *gwk;               // [BH][nq] summed sizes of chi(group) (at leaders)
  uint32_t *chi;              // [BH][nq][32] chi(group) bitmask (at leaders)
  int32_t *list;              // [BH][2][nq] this round's A and B leaders, ascending
  int32_t *nlist;             // [BH][2]
  unsigned long long *best;   // [BH][nq] per A index: (dC + bias) << 10 | B index
  int32_t *passes;            // [BH] digits of the largest key size (1..3)
};

struct MergeArgs {
  const int32_t *sizes_q;  // [BH][nq]
  const int32_t *sizes_k;  // [BH][nk]
  const int32_t *counts;   // [BH][nq]
  const int32_t *idx;      // [BH][nq][nk]
  const uint8_t *sides;    // [BH][rounds][nq]
  int nq, nk, rounds;
  int tau_q, tau_k;
  float inv_tau_q, inv_tau_k;
  int32_t *group_of;       // [BH][nq]
  int32_t *g_counts;       // [BH][nq]
  int32_t *g_idx;          // [BH][nq][nk]
  MergeWs ws;
  unsigned long long timeout_ns;
  int *status;             // the launch's status word
};

// ceil(x / tau) for x >= 0: a float estimate corrected to the exact quotient.
__device__ __forceinline__ long long ceil_div_tiles(long long x, int tau, float inv_tau) {
  if (x <= 0) return 0;
  long long q = static_cast<long long>(static_cast<float>(x) * inv_tau);
  while (q > 0 && q * tau > x) --q;
  while ((q + 1) * tau <= x) ++q;
  return q + (q * tau < x ? 1 : 0);
}

__device__ __forceinline__ long long group_cost(long long sq, long long wk, const MergeArgs &a) {
  return ceil_div_tiles(sq, a.tau_q, a.inv_tau_q) * ceil_div_tiles(wk, a.tau_k, a.inv_tau_k);
}

// Block-wide (1024 threads, thread g = group g): this round's A and B lists.
__device__ void merge_build_lists(const MergeArgs &a, int bh, int r, int *s_tot) {
  const int g = threadIdx.x, lane = g & 31, warp = g >> 5;
  const size_t hb = (size_t)bh * a.nq;
  bool in_a = false, in_b = false;
  if (g < a.nq && a.ws.lead[hb + g] == g && a.ws.gsq[hb + g] > 0) {
    const bool side = a.sides[((size_t)bh * a.rounds + r) * a.nq + g] != 0;
    in_a = !side;
    in_b = side;
  }
  const uint32_t ba = __ballot_sync(0xffffffffu, in_a), bb = __ballot_sync(0xffffffffu, in_b);
  if (lane == 0) {
    s_tot[warp] = __popc(ba);
    s_tot[32 + warp] = __popc(bb);
  }
  __syncthreads();
  if (warp == 0) {
    const int x = s_tot[lane], y = s_tot[32 + lane];
    const int ex = warp_exclusive_scan(x, lane), ey = warp_exclusive_scan(y, lane);
    s_tot[lane] = ex;
    s_tot[32 + lane] = ey;
    if (lane == 31) {
      s_tot[64] = ex + x;
      s_tot[65] = ey + y;
    }
  }
  __syncthreads();
  const uint32_t lt = (1u << lane) - 1u;
  int32_t *la = a.ws.list + (size_t)bh * 2 * a.nq;
  if (in_a) {
    const int p = s_tot[warp] + __popc(ba & lt);
    la[p] = g;
    a.ws.best[hb + p] = kNoPair;
  }
  if (in_b) la[a.nq + s_tot[32 + warp] + __popc(bb & lt)] = g;
  if (g == 0) {
    a.ws.nlist[2 * bh] = s_tot[64];
    a.ws.nlist[2 * bh + 1] = s_tot[65];
  }
}

// Block-wide: the final groups -- group_of, and each leader's chi(S) as an
// ascending list (0 entries at non-leaders).
__device__ void merge_emit(const MergeArgs &a, int bh) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const size_t hb = (size_t)bh * a.nq;
  for (int i = warp; i < a.nq; i += kMergeHeadThreads / 32) {
    const int l = a.ws.lead[hb + i];
    int cnt = 0;
    if (l == i) cnt = emit_bitmap_list(a.ws.chi + (hb + i) * kMergeWords, a.nk, lane, a.g_idx + (hb + i) * a.nk, nullptr);
    if (lane == 0) {
      a.g_counts[hb + i] = cnt;
      a.group_of[hb + i] = l;
    }
  }
}

// One CTA per (batch, head): singleton groups from the kept lists.
__global__ void __launch_bounds__(kMergeHeadThreads) merge_init_kernel(const MergeArgs a) {
  __shared__ uint32_t wbits[kMergeHeadThreads / 32][kMergeWords];
  __shared__ int s_tot[66];
  __shared__ int s_max;
  const int bh = blockIdx.x, t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const size_t hb = (size_t)bh * a.nq;
  if (t == 0) s_max = 0;
  __syncthreads();
  bool bad_size = false;
  for (int j = t; j < a.nk; j += kMergeHeadThreads) {
    const int s = __ldg(a.sizes_k + (size_t)bh * a.nk + j);
    if (s < 0) bad_size = true;
    else atomicMax(&s_max, s);
  }
  for (int i = warp; i < a.nq; i += kMergeHeadThreads / 32) {
    const int c = __ldg(a.counts + hb + i);
    const int32_t *row = a.idx + (hb + i) * a.nk;
    bool bad = c < 0 || c > a.nk;
    wbits[warp][lane] = 0u;
    __syncwarp();
    int wk = 0;
    for (int e = lane; !bad && e < c; e += 32) {
      const int j = __ldg(row + e);
      if (j < 0 || j >= a.nk || (e > 0 && __ldg(row + e - 1) >= j)) {
        bad = true;
      } else {
        atomicOr(&wbits[warp][j >> 5], 1u << (j & 31));
        wk += max(0, __ldg(a.sizes_k + (size_t)bh * a.nk + j));
      }
    }
    bad = __any_sync(0xffffffffu, bad);
    wk = warp_sum_int(wk);
    __syncwarp();
    a.ws.chi[(hb + i) * kMergeWords + lane] = bad ? 0u : wbits[warp][lane];
    if (lane == 0) {
      const int s = __ldg(a.sizes_q + hb + i);
      if (bad || s < 0) latch_status(a.status, VSA_ERR_BAD_INDEX);
      a.ws.gsq[hb + i] = max(0, s);
      a.ws.gwk[hb + i] = bad ? 0 : wk;
      a.ws.lead[hb + i] = i;
    }
    __syncwarp();
  }
  if (bad_size) latch_status(a.status, VSA_ERR_BAD_INDEX);
  __syncthreads();
  if (t == 0) a.ws.passes[bh] = s_max >= (1 << 22) ? 3 : (s_max >= 2048 ? 2 : 1);
  if (a.rounds > 0) merge_build_lists(a, bh, 0, s_tot);
  else merge_emit(a, bh);
}

struct MergeCtl {
  uint64_t done[2];  // the MMAs reading operand buffer b have completed
  uint64_t fin;      // every MMA of the CTA has completed
  uint32_t tmem_base;
  AbortCtl abort;
};

struct MergeSmem {
  static constexpr int kOffA = 0;                                 // [2] A tiles
  static constexpr int kOffB = kOffA + 2 * kMergeTileBytes;       // [2][3] B tiles
  static constexpr int kOffH = kOffB + 6 * kMergeTileBytes;       // [3][512] fp16 digit pairs
  static constexpr int kOffCol = kOffH + 3 * 512 * 4;             // [128] s_q, [128] w_k, [128] cost (int64)
  static constexpr int kOffCtl = kOffCol + 128 * 16;
  static constexpr int kBytes = kOffCtl + 64;
  static constexpr int kAlloc = kBytes + 1024;
};

// fp16 of a digit in [0, 2048): exact.
__device__ __forceinline__ uint32_t half_bits(int v) {
  return static_cast<uint32_t>(__half_as_ushort(__int2half_rn(v)));
}

// Row r of a 128 x 64 fp16 K-major tile in the 128-byte swizzled layout the
// MMA descriptor expects: eight 16-byte chunks, chunk q stored at q ^ (r & 7).
__device__ __forceinline__ void store_row_sw128(uint8_t *tile, int r, const uint32_t (&v)[32]) {
  uint8_t *row = tile + (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll
  for (int q = 0; q < 8; ++q)
    *reinterpret_cast<uint4 *>(row + ((q ^ (r & 7)) << 4)) = make_uint4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
}

// Lane masks of two fp16 values from two bits.
__device__ __forceinline__ uint32_t pair_mask(uint32_t two_bits) {
  return ((0u - (two_bits & 1u)) & 0xffffu) | ((0u - ((two_bits >> 1) & 1u)) << 16);
}

// Instruction descriptor of kind::f16 with fp16 A/B, fp32 D, both K-major.
__host__ __device__ constexpr uint32_t idesc_f16_f32(int M, int N) {
  return (1u << 4) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// One CTA per (128 A-groups, 128 B-groups, batch-head) of round r.
__global__ void __launch_bounds__(kMergeThreads, 1) merge_pairs_kernel(const MergeArgs a) {
  const int tb = blockIdx.x, ta = blockIdx.y, bh = blockIdx.z;
  const int nA = a.ws.nlist[2 * bh], nB = a.ws.nlist[2 * bh + 1];
  if (ta * kMergeTile >= nA || tb * kMergeTile >= nB) return;
  extern __shared__ uint8_t merge_smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(merge_smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  using L = MergeSmem;
  uint32_t *hv2 = reinterpret_cast<uint32_t *>(smem + L::kOffH);
  int *col_sq = reinterpret_cast<int *>(smem + L::kOffCol);
  int *col_wk = col_sq + 128;
  long long *col_c = reinterpret_cast<long long *>(col_wk + 128);
  MergeCtl *ctl = reinterpret_cast<MergeCtl *>(smem + L::kOffCtl);
  AbortCtl *abort = &ctl->abort;

  const int t = threadIdx.x, warp = t >> 5;
  const size_t hb = (size_t)bh * a.nq;
  const int passes = a.ws.passes[bh];
  const int32_t *list_a = a.ws.list + (size_t)bh * 2 * a.nq;
  const int32_t *list_b = list_a + a.nq;
  const int row_a = ta * kMergeTile + t, row_b = tb * kMergeTile + t;
  const int ga = row_a < nA ? list_a[row_a] : -1;
  const int gb = row_b < nB ? list_b[row_b] : -1;
  const uint32_t *chi_a = a.ws.chi + (hb + (ga >= 0 ? ga : 0)) * kMergeWords;
  const uint32_t *chi_b = a.ws.chi + (hb + (gb >= 0 ? gb : 0)) * kMergeWords;

  // fp16 digit pairs of the key sizes (keys 2*i and 2*i + 1), digit p = bits [11p, 11p + 11)
  for (int i = t; i < 512; i += kMergeThreads) {
    const int j = 2 * i;
    const int s0 = j < a.nk ? max(0, __ldg(a.sizes_k + (size_t)bh * a.nk + j)) : 0;
    const int s1 = j + 1 < a.nk ? max(0, __ldg(a.sizes_k + (size_t)bh * a.nk + j + 1)) : 0;
#pragma unroll
    for (int p = 0; p < 3; ++p)
      hv2[p * 512 + i] = half_bits((s0 >> (11 * p)) & 2047) | (half_bits((s1 >> (11 * p)) & 2047) << 16);
  }
  col_sq[t] = gb >= 0 ? a.ws.gsq[hb + gb] : 0;
  col_wk[t] = gb >= 0 ? a.ws.gwk[hb + gb] : 0;
  col_c[t] = gb >= 0 ? group_cost(col_sq[t], col_wk[t], a) : 0;
  const uint32_t n_cols = passes == 1 ? 128u : (passes == 2 ? 256u : 512u);
  if (t == 0) {
    mbar_init(&ctl->done[0], 1);
    mbar_init(&ctl->done[1], 1);
    mbar_init(&ctl->fin, 1);
    abort_init(&ctl->abort, a.status);
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(&ctl->tmem_base, n_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;

  constexpr uint32_t kId = idesc_f16_f32(kMergeTile, kMergeTile);
  const int n_chunks = (a.nk + kMergeChunkKeys - 1) / kMergeChunkKeys;
  bool ok = true;
  for (int c = 0; c < n_chunks; ++c) {
    const int buf = c & 1;
    if (c >= 2) {
      const bool w = mbar_wait(&ctl->done[buf], ((c >> 1) - 1) & 1, abort, a.timeout_ns);
      ok = __syncthreads_and(w ? 1 : 0) != 0;
      if (!ok) break;
    }
    uint8_t *tile_a = smem + L::kOffA + buf * kMergeTileBytes;
    uint8_t *tile_b = smem + L::kOffB + buf * 3 * kMergeTileBytes;
    const uint64_t bits_a = ga >= 0 ? (static_cast<uint64_t>(chi_a[2 * c + 1]) << 32) | chi_a[2 * c] : 0ull;
    const uint64_t bits_b = gb >= 0 ? (static_cast<uint64_t>(chi_b[2 * c + 1]) << 32) | chi_b[2 * c] : 0ull;
    uint32_t v[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = 0x3c003c00u & pair_mask(static_cast<uint32_t>(bits_a >> (2 * i)));
    store_row_sw128(tile_a, t, v);
    for (int p = 0; p < passes; ++p) {
      const uint32_t *h = hv2 + p * 512 + c * (kMergeChunkKeys / 2);
#pragma unroll
      for (int i = 0; i < 32; ++i) v[i] = h[i] & pair_mask(static_cast<uint32_t>(bits_b >> (2 * i)));
      store_row_sw128(tile_b + p * kMergeTileBytes, t, v);
    }
    fence_proxy_async_smem();
    __syncthreads();
    if (t == 0) {
      tc_fence_after();
      const uint64_t da = smem_desc_sw128(smem_addr(tile_a), 16, 1024);
      for (int p = 0; p < passes; ++p) {
        const uint64_t db = smem_desc_sw128(smem_addr(tile_b + p * kMergeTileBytes), 16, 1024);
#pragma unroll
        for (int kk = 0; kk < kMergeChunkKeys / 16; ++kk)
          umma_bf16_ss(tmem + 128u * p, da + 2 * kk, db + 2 * kk, kId, (c > 0 || kk > 0) ? 1u : 0u);
      }
      umma_commit(&ctl->done[buf]);
    }
  }
  if (t == 0) umma_commit(&ctl->fin);
  const bool fin_t = mbar_drain(&ctl->fin, 0, a.timeout_ns);
  if (!fin_t) raise_timeout(a.status);
  const bool fin = __syncthreads_and(fin_t ? 1 : 0) != 0;
  tc_fence_after();
  if (ok && fin) {
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    const long long sqa = ga >= 0 ? a.ws.gsq[hb + ga] : 0;
    const long long wka = ga >= 0 ? a.ws.gwk[hb + ga] : 0;
    const long long ca = group_cost(sqa, wka, a);
    unsigned long long best = kNoPair;
    // the operand buffers are free now: thread t keeps its row's 32 intersections of a
    // column block at inter[i * 128 + t]
    long long *inter = reinterpret_cast<long long *>(smem + L::kOffB);
    for (int c0 = 0; c0 < kMergeTile; c0 += 32) {
      uint32_t d[32];
      tmem_ld32(tmem + lane_off + c0, d);
      tmem_ld_wait();
#pragma unroll
      for (int i = 0; i < 32; ++i) inter[i * kMergeTile + t] = static_cast<long long>(__uint_as_float(d[i]));
      for (int p = 1; p < passes; ++p) {
        tmem_ld32(tmem + lane_off + 128u * p + c0, d);
        tmem_ld_wait();
        const long long scale = p == 1 ? 2048ll : (1ll << 22);
#pragma unroll
        for (int i = 0; i < 32; ++i) inter[i * kMergeTile + t] += scale * static_cast<long long>(__uint_as_float(d[i]));
      }
      const int n_here = min(32, nB - tb * kMergeTile - c0);
      for (int i = 0; i < n_here; ++i) {
        const int b = c0 + i;
        const long long dc =
            group_cost(sqa + col_sq[b], wka + col_wk[b] - inter[i * kMergeTile + t], a) - ca - col_c[b];
        const long long dcc = min(max(dc, -(kDcBias - 1)), kDcBias - 1);
        const unsigned long long key = (static_cast<unsigned long long>(dcc + kDcBias) << 10) |
                                       static_cast<unsigned long long>(tb * kMergeTile + b);
        best = min(best, key);
      }
    }
    if (ga >= 0 && best != kNoPair) atomicMin(a.ws.best + hb + row_a, best);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, n_cols);
}

// One CTA per (batch, head): accept the disjoint pairs of round r, apply them,
// and build the next round's lists (or emit the final groups).
__global__ void __launch_bounds__(kMergeHeadThreads) merge_apply_kernel(const MergeArgs a, int r) {
  __shared__ unsigned long long win[kMergeMaxClusters];
  __shared__ int redirect[kMergeMaxClusters];
  __shared__ int s_tot[66];
  const int bh = blockIdx.x, t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const size_t hb = (size_t)bh * a.nq;
  const int nA = a.ws.nlist[2 * bh], nB = a.ws.nlist[2 * bh + 1];
  const int32_t *list_a = a.ws.list + (size_t)bh * 2 * a.nq;
  const int32_t *list_b = list_a + a.nq;
  win[t] = kNoPair;
  redirect[t] = -1;
  __syncthreads();
  if (t < nA) {
    const unsigned long long key = a.ws.best[hb + t];
    if (key != kNoPair && static_cast<long long>(key >> 10) < kDcBias)  // dC < 0
      atomicMin(&win[key & 1023u], ((key >> 10) << 10) | static_cast<unsigned long long>(t));
  }
  __syncthreads();
  for (int b = warp; b < nB; b += kMergeHeadThreads / 32) {
    const unsigned long long w = win[b];
    if (w == kNoPair) continue;
    const int ga = list_a[w & 1023u], gb = list_b[b];
    const int lead = min(ga, gb), other = max(ga, gb);
    const uint32_t word = a.ws.chi[(hb + ga) * kMergeWords + lane] | a.ws.chi[(hb + gb) * kMergeWords + lane];
    int wk = 0;
    for (uint32_t rest = word; rest; rest &= rest - 1u) {
      const int j = lane * 32 + __ffs(rest) - 1;
      wk += max(0, __ldg(a.sizes_k + (size_t)bh * a.nk + j));
    }
    wk = warp_sum_int(wk);
    const int sq = a.ws.gsq[hb + ga] + a.ws.gsq[hb + gb];
    __syncwarp();
    a.ws.chi[(hb + lead) * kMergeWords + lane] = word;
    if (lane == 0) {
      a.ws.gsq[hb + lead] = sq;
      a.ws.gwk[hb + lead] = wk;
      redirect[other] = lead;
    }
  }
  __syncthreads();
  if (t < a.nq) {
    const int l = a.ws.lead[hb + t];
    const int rd = redirect[l];
    if (rd >= 0) a.ws.lead[hb + t] = rd;
  }
  __syncthreads();
  if (r + 1 < a.rounds) merge_build_lists(a, bh, r + 1, s_tot);
  else merge_emit(a, bh);
}

}  // namespace vsa
