// a5 Micro selection inside omitted blocks (HyMoR-Attn abstract: a fine
// residual over the scattered high-value tail left inside omitted Macro
// blocks, selected online).
//
// Candidates of Micro row r (64 query rows) are the 16-key tiles t that lie in
// a key block omitted by r's Macro query block and hold a valid key.  The
// pooled score qbar64_r . kbar16_t * scale is computed for every (r, t) of an
// enabled head by an fp32 register-tiled GEMM (64 rows x 128 tiles per CTA);
// the score is stored as an order-preserving uint32 key, 0 for
// non-candidates.  Two selection modes:
//   top-k      one warp per Micro row takes the k largest keys (ties to the
//              lower tile) with k rounds of warp arg-max;
//   percentile a 3-pass radix select (11 + 11 + 10 bits, histograms built in
//              shared memory, merged with global atomics, the first pass fused
//              into the score GEMM) finds, per enabled head, the exact key of
//              rank ceil(q * M) among its M candidates; one warp per Micro row
//              then compacts the tiles strictly above it into an ascending
//              list.
// Nothing is synchronised with the host: the rank search runs on the device.
#pragma once

#include "common.cuh"

namespace vsa {

constexpr int kMicroRows = 64;
constexpr int kMicroKeys = 16;
constexpr int kScoreBM = 64;    // Micro rows per CTA
constexpr int kScoreBN = 128;   // tiles per CTA
constexpr int kScoreBK = 32;    // d per smem step
constexpr int kScoreThreads = 256;
constexpr int kHistBins = 2048;

struct MicroWs {
  int32_t *slot_of_bh;  // [B*H] slot or -1
  int32_t *bh_of_slot;  // [slots] the (batch, head) of each slot
  uint32_t *bitmap;     // [slots][n_q][bitmap_words] kept key blocks of each Macro row
  uint32_t *keys;       // [slots][n_r][n_t]
  uint32_t *hist;       // [slots][3][kHistBins]
  uint32_t *state;      // [slots][8]: M, prefix, rank-left, tau, ...
  int n_slots;
  int bitmap_words;     // max(32, ceil(n_k / 32))
  int *status;          // the launch's status word
};

constexpr int kMicroMaxKeyBlocks = 4096;

// Dense kept-block bitmap of every Macro row of the enabled heads (grid: rows x slots).
__global__ void micro_bitmap_kernel(const int32_t *__restrict__ counts, const int32_t *__restrict__ idx, int n_q,
                                    int n_k, int BH, MicroWs ws) {
  const int row = blockIdx.x;  // Macro row within the head
  const int slot = blockIdx.y;
  const int bh = ws.bh_of_slot[slot];
  if (row >= n_q) return;
  __shared__ uint32_t bits[kMicroMaxKeyBlocks / 32];
  const int W = ws.bitmap_words;
  for (int w = threadIdx.x; w < W; w += blockDim.x) bits[w] = 0u;
  __syncthreads();
  const size_t r = (size_t)bh * n_q + row;
  const int c = counts[r];
  for (int e = threadIdx.x; e < c; e += blockDim.x) {
    const int j = idx[r * n_k + e];
    if (j >= 0 && j < n_k) atomicOr(&bits[j >> 5], 1u << (j & 31));
  }
  __syncthreads();
  for (int w = threadIdx.x; w < W; w += blockDim.x) ws.bitmap[((size_t)slot * n_q + row) * W + w] = bits[w];
}

struct ScoreArgs {
  const float *q64;  // [BH, n_r, d]
  const float *k16;  // [BH, n_t, d]
  int n_r, n_t, n_q, bq, bk, n_valid;
  float scale;
  int fuse_hist;  // build the first radix histogram (percentile mode)
};

template <int D>
__global__ void __launch_bounds__(kScoreThreads) micro_score_kernel(ScoreArgs a, MicroWs ws) {
  const int slot = blockIdx.z;  // enabled heads only
  const int bh = ws.bh_of_slot[slot];
  const int r0 = blockIdx.y * kScoreBM;
  const int t0 = blockIdx.x * kScoreBN;
  __shared__ float As[kScoreBK][kScoreBM + 4];
  __shared__ float Bs[kScoreBK][kScoreBN + 4];
  __shared__ uint32_t rowbits[kScoreBM][32];
  __shared__ uint32_t hist[kHistBins];
  __shared__ uint32_t cand_count;
  const int tid = threadIdx.x;
  const float *qp = a.q64 + (size_t)bh * a.n_r * D;
  const float *kp = a.k16 + (size_t)bh * a.n_t * D;

  // kept bitmaps of the Macro rows of this CTA's Micro rows: the 32 words
  // (1024 key blocks) from the one holding the CTA's first tile, which cover
  // all of its 128 tiles
  const int per = a.bk / kMicroKeys;
  const int W = ws.bitmap_words;
  const int w0 = (t0 / per) >> 5;
  for (int i = tid; i < kScoreBM * 32; i += kScoreThreads) {
    const int rr = i >> 5, w = i & 31;
    const int r = r0 + rr;
    uint32_t v = 0xffffffffu;  // rows outside the head, words past the row: nothing is a candidate
    if (r < a.n_r && w0 + w < W) {
      const int qi = (r * kMicroRows) / a.bq;
      v = ws.bitmap[((size_t)slot * a.n_q + qi) * W + w0 + w];
    }
    rowbits[rr][w] = v;
  }
  if (a.fuse_hist) {
    for (int i = tid; i < kHistBins; i += kScoreThreads) hist[i] = 0u;
    if (tid == 0) cand_count = 0u;
  }

  const int ty = tid / 16, tx = tid % 16;  // 16 x 16 threads, 4 rows x 8 tiles each
  float acc[4][8];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;

  for (int k0 = 0; k0 < D; k0 += kScoreBK) {
    __syncthreads();
    // A: 64 rows x 32 d, transposed into As[d][row]
    for (int i = tid; i < kScoreBM * kScoreBK / 4; i += kScoreThreads) {
      const int rr = i / (kScoreBK / 4), c4 = i % (kScoreBK / 4);
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (r0 + rr < a.n_r) v = __ldg(reinterpret_cast<const float4 *>(qp + (size_t)(r0 + rr) * D + k0) + c4);
      As[c4 * 4 + 0][rr] = v.x; As[c4 * 4 + 1][rr] = v.y; As[c4 * 4 + 2][rr] = v.z; As[c4 * 4 + 3][rr] = v.w;
    }
    for (int i = tid; i < kScoreBN * kScoreBK / 4; i += kScoreThreads) {
      const int tt = i / (kScoreBK / 4), c4 = i % (kScoreBK / 4);
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (t0 + tt < a.n_t) v = __ldg(reinterpret_cast<const float4 *>(kp + (size_t)(t0 + tt) * D + k0) + c4);
      Bs[c4 * 4 + 0][tt] = v.x; Bs[c4 * 4 + 1][tt] = v.y; Bs[c4 * 4 + 2][tt] = v.z; Bs[c4 * 4 + 3][tt] = v.w;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < kScoreBK; ++kk) {
      const float4 av = *reinterpret_cast<const float4 *>(&As[kk][ty * 4]);
      const float4 b0 = *reinterpret_cast<const float4 *>(&Bs[kk][tx * 4]);
      const float4 b1 = *reinterpret_cast<const float4 *>(&Bs[kk][64 + tx * 4]);
      const float ar[4] = {av.x, av.y, av.z, av.w};
      const float2 br2[4] = {make_float2(b0.x, b0.y), make_float2(b0.z, b0.w), make_float2(b1.x, b1.y),
                             make_float2(b1.z, b1.w)};
      // packed pairs of accumulators (fma.rn.f32x2): each lane is the same
      // single-rounding fma as before, in the same order over kk
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 a2 = make_float2(ar[i], ar[i]);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float2 r = ffma2(a2, br2[j], make_float2(acc[i][2 * j], acc[i][2 * j + 1]));
          acc[i][2 * j] = r.x;
          acc[i][2 * j + 1] = r.y;
        }
      }
    }
  }

  // keys + candidate test + fused first-pass histogram
  uint32_t local_cnt = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int rr = ty * 4 + i;
    const int r = r0 + rr;
    const bool row_ok = r < a.n_r && r * kMicroRows < a.n_valid;
    uint32_t out[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int t = t0 + (j < 4 ? tx * 4 + j : 64 + tx * 4 + (j - 4));
      bool cand = row_ok && t < a.n_t && t * kMicroKeys < a.n_valid;
      if (cand) {
        const int kb = t / per;
        cand = ((rowbits[rr][(kb >> 5) - w0] >> (kb & 31)) & 1u) == 0u;
      }
      const uint32_t key = cand ? float_key(acc[i][j] * a.scale) : 0u;
      out[j] = key;
      if (a.fuse_hist) {
        // the scores of a head fall in few top-11-bit bins: lanes with the
        // same bin add once, so the shared-memory atomics do not serialise
        const unsigned active = __ballot_sync(0xffffffffu, cand);
        if (cand) {
          const uint32_t bin = key >> 21;
          const unsigned peers = __match_any_sync(active, bin);
          if (__ffs(peers) - 1 == (tid & 31)) atomicAdd(&hist[bin], static_cast<uint32_t>(__popc(peers)));
          ++local_cnt;
        }
      }
    }
    if (r < a.n_r) {
      uint32_t *dst = ws.keys + ((size_t)slot * a.n_r + r) * a.n_t + t0;
      if (t0 + kScoreBN <= a.n_t) {
        *reinterpret_cast<uint4 *>(dst + tx * 4) = make_uint4(out[0], out[1], out[2], out[3]);
        *reinterpret_cast<uint4 *>(dst + 64 + tx * 4) = make_uint4(out[4], out[5], out[6], out[7]);
      } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int tt = j < 4 ? tx * 4 + j : 64 + tx * 4 + (j - 4);
          if (t0 + tt < a.n_t) dst[tt] = out[j];
        }
      }
    }
  }
  if (a.fuse_hist) {
    atomicAdd(&cand_count, local_cnt);
    __syncthreads();
    uint32_t *gh = ws.hist + (size_t)slot * 3 * kHistBins;
    for (int i = tid; i < kHistBins; i += kScoreThreads)
      if (hist[i]) atomicAdd(&gh[i], hist[i]);
    if (tid == 0 && cand_count) atomicAdd(&ws.state[slot * 8 + 0], cand_count);
  }
}

// Radix pass p (1 or 2): histogram of the next digit of keys whose higher
// digits equal the prefix found so far.
__global__ void micro_hist_kernel(MicroWs ws, size_t per_slot, int pass) {
  const int slot = blockIdx.y;
  __shared__ uint32_t hist[kHistBins];
  for (int i = threadIdx.x; i < kHistBins; i += blockDim.x) hist[i] = 0u;
  __syncthreads();
  const uint32_t prefix = ws.state[slot * 8 + 1];
  const uint32_t *keys = ws.keys + (size_t)slot * per_slot;
  const int hi_shift = pass == 1 ? 21 : 10;
  const int lo_shift = pass == 1 ? 10 : 0;
  const uint32_t lo_mask = pass == 1 ? 0x7ffu : 0x3ffu;
  const size_t n4 = per_slot / 4;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += (size_t)gridDim.x * blockDim.x) {
    const uint4 v = reinterpret_cast<const uint4 *>(keys)[i];
    const uint32_t kv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 4; ++e)
      if (kv[e] != 0u && (kv[e] >> hi_shift) == prefix) atomicAdd(&hist[(kv[e] >> lo_shift) & lo_mask], 1u);
  }
  for (size_t i = n4 * 4 + (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < per_slot;
       i += (size_t)gridDim.x * blockDim.x) {
    const uint32_t kv = keys[i];
    if (kv != 0u && (kv >> hi_shift) == prefix) atomicAdd(&hist[(kv >> lo_shift) & lo_mask], 1u);
  }
  __syncthreads();
  uint32_t *gh = ws.hist + ((size_t)slot * 3 + pass) * kHistBins;
  for (int i = threadIdx.x; i < kHistBins; i += blockDim.x)
    if (hist[i]) atomicAdd(&gh[i], hist[i]);
}

// Find the digit holding the rank-th smallest key (one warp per slot).
// pass 0 also turns M into the nearest rank ceil(q * M) (IEEE double).
__global__ void micro_find_kernel(MicroWs ws, double q, int pass) {
  const int slot = blockIdx.x;
  const int lane = threadIdx.x;
  uint32_t *st = ws.state + slot * 8;
  const uint32_t *h = ws.hist + ((size_t)slot * 3 + pass) * kHistBins;
  const int bins = pass == 2 ? 1024 : 2048;
  uint32_t left;
  if (pass == 0) {
    const uint32_t M = st[0];
    long long rank = (long long)ceil(q * (double)M);
    if (rank < 1) rank = 1;
    if (rank > (long long)M) rank = (long long)M;
    left = M == 0 ? 0u : (uint32_t)rank;
  } else {
    left = st[2];
  }
  if (left == 0u) {  // no candidate: nothing is selected
    if (lane == 0) {
      st[2] = 0u;
      st[3] = 0xffffffffu;
      st[4] = 1u;  // empty flag
    }
    return;
  }
  // lane l holds bins [l * per, (l + 1) * per) in registers (all loads in
  // flight at once); a scan of the lanes' totals finds the lane whose bins
  // hold the rank, and that lane walks its own bins
  const int per = bins / 32;
  uint32_t c[2048 / 32];
  uint32_t tot = 0u;
#pragma unroll
  for (int i = 0; i < 2048 / 32; ++i) {
    c[i] = i < per ? h[lane * per + i] : 0u;
    tot += c[i];
  }
  uint32_t incl = tot;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  const uint32_t excl = incl - tot;
  const uint32_t ballot = __ballot_sync(0xffffffffu, incl >= left);
  int digit = -1;
  if (ballot) {
    const int first = __ffs(ballot) - 1;
    int my_digit = -1;
    uint32_t my_left = 0u;
    if (lane == first) {
      uint32_t run = excl;
#pragma unroll
      for (int i = 0; i < 2048 / 32; ++i) {
        if (my_digit < 0 && i < per && run + c[i] >= left) {
          my_digit = lane * per + i;
          my_left = left - run;
        }
        run += c[i];
      }
    }
    digit = __shfl_sync(0xffffffffu, my_digit, first);
    left = __shfl_sync(0xffffffffu, my_left, first);
  }
  if (lane == 0) {
    const uint32_t prefix = pass == 0 ? 0u : st[1];
    const uint32_t np = (pass == 0) ? (uint32_t)digit : ((prefix << (pass == 1 ? 11 : 10)) | (uint32_t)digit);
    st[1] = np;
    st[2] = left;
    if (pass == 2) {
      st[3] = np;  // the exact key of rank ceil(q * M)
      st[4] = 0u;
    }
  }
}

// Compaction: one warp per Micro row of the enabled heads (the rows of the
// other heads were zeroed by the host); tiles with key > tau (percentile) in
// ascending order.
__global__ void micro_compact_kernel(MicroWs ws, int n_r, int n_t, int BH, int row_capacity, int32_t *m_counts,
                                     int32_t *m_idx) {
  const int lane = threadIdx.x & 31;
  const size_t sw = (size_t)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  if (sw >= (size_t)ws.n_slots * n_r) return;
  const int slot = (int)(sw / n_r), r = (int)(sw % n_r);
  const size_t gw = (size_t)ws.bh_of_slot[slot] * n_r + r;
  int32_t *dst = m_idx + gw * row_capacity;
  const uint32_t *st = ws.state + slot * 8;
  const uint32_t tau = st[3];
  const bool empty = st[4] != 0u;
  const uint32_t *keys = ws.keys + ((size_t)slot * n_r + r) * n_t;
  int total = 0;
  bool overflow = false;
  if (!empty) {
    // four consecutive tiles per lane per step (n_t is a multiple of 8, rows
    // start 16-byte aligned): one 16-byte load, then an exclusive scan of the
    // lanes' counts keeps the output ascending
    for (int t0 = 0; t0 < n_t; t0 += 128) {
      const int t = t0 + 4 * lane;
      uint4 kv = make_uint4(0u, 0u, 0u, 0u);
      if (t < n_t) kv = *reinterpret_cast<const uint4 *>(keys + t);
      const uint32_t m = (kv.x > tau ? 1u : 0u) | (kv.y > tau ? 2u : 0u) | (kv.z > tau ? 4u : 0u) |
                         (kv.w > tau ? 8u : 0u);
      const int c = __popc(m);
      const int off = warp_exclusive_scan(c, lane);
      int o = total + off;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        if ((m >> i) & 1u) {
          if (o < row_capacity) dst[o] = t + i;
          else overflow = true;
          ++o;
        }
      }
      total += __shfl_sync(0xffffffffu, off + c, 31);
    }
  }
  if (__any_sync(0xffffffffu, overflow) && lane == 0) latch_status(ws.status, VSA_ERR_CAPACITY);
  if (lane == 0) m_counts[gw] = total < row_capacity ? total : row_capacity;
}

// Top-k per Micro row (k <= 32): k rounds of warp arg-max over 64-bit keys
// (score key, inverted tile index), then an ascending write of the winners.
__global__ void micro_topk_kernel(MicroWs ws, int n_r, int n_t, int BH, int topk, int row_capacity,
                                  int32_t *m_counts, int32_t *m_idx) {
  const int lane = threadIdx.x & 31;
  const size_t sw = (size_t)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  if (sw >= (size_t)ws.n_slots * n_r) return;
  const int slot = (int)(sw / n_r), r = (int)(sw % n_r);
  const size_t gw = (size_t)ws.bh_of_slot[slot] * n_r + r;
  int32_t *dst = m_idx + gw * row_capacity;
  uint32_t *keys = ws.keys + ((size_t)slot * n_r + r) * n_t;
  int chosen = -1;  // lane i holds the i-th winner
  int n_sel = 0;
  for (int round = 0; round < topk; ++round) {
    uint64_t best = 0ull;
    for (int t = lane; t < n_t; t += 32) {
      const uint32_t kv = keys[t];
      if (kv == 0u) continue;
      const uint64_t pk = ((uint64_t)kv << 32) | (uint64_t)(0xffffffffu - (uint32_t)t);
      best = pk > best ? pk : best;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const uint64_t y = __shfl_xor_sync(0xffffffffu, best, o);
      best = y > best ? y : best;
    }
    if (best == 0ull) break;
    const int t = (int)(0xffffffffu - (uint32_t)(best & 0xffffffffull));
    if (lane == round) chosen = t;
    if (lane == 0) keys[t] = 0u;  // remove the winner
    __syncwarp();
    ++n_sel;
  }
  // ascending order: rank of each winner among the winners
  int rank = 0;
  for (int i = 0; i < n_sel; ++i) {
    const int other = __shfl_sync(0xffffffffu, chosen, i);
    if (lane < n_sel && other < chosen) ++rank;
  }
  const int cap = n_sel < row_capacity ? n_sel : row_capacity;
  if (lane < n_sel && rank < row_capacity) dst[rank] = chosen;
  if (n_sel > row_capacity && lane == 0) latch_status(ws.status, VSA_ERR_CAPACITY);
  if (lane == 0) m_counts[gw] = cap;
}

}  // namespace vsa
