// a4 / a6 Block-sparse attention forward on the 5th-generation tensor cores.
//
// HyperVAttention section 2 Eq. (4): each query block attends only to its
// selected key blocks; section 4.3: the selected key blocks of a row are
// walked as one packed sequence of fixed-size tiles.  HyMoR-Attn (abstract):
// the fine Micro pass over 16-key tiles inside omitted blocks is merged with
// the Macro output by exact LSE merging; that merge is this kernel's
// epilogue when merge inputs are given.
//
// One CTA = one 128-row query tile of one (batch, head).  The tile's key
// segments (list entries of seg_keys keys; the union of two 64-row lists
// when list_rows = 64, each entry tagged with the halves that use it) are
// packed into 128-key stages.  The union is built once, before the pipeline
// starts, in shared memory (lists of up to kListStage entries; longer lists
// are merged on the fly from global memory).  Warp roles:
//   warp 0     TMA producer of Q and K: Q once, then the K boxes of each
//              stage into 2 ring slots (128B-swizzled, one box per segment
//              and 64-column chunk, or one 4 KB pair box per 16-key segment
//              at d = 128; the boxes of a stage issued by one lane each; rows
//              past n_valid arrive as zeros); it publishes each stage's
//              segment starts and box kinds in the stage info ring.
//   warp 10    TMA producer of V: the same boxes of V into 2 ring slots, at
//              the starts read from the info ring.  Two warps keep the copy
//              engine fed: with K and V from one warp the per-box issue paced
//              the Micro pass and the cluster-group pass (HunyuanVideo-like
//              Micro pass 1.62 -> 1.42 ms, Wan-1.3B-like group pass 6.32 ->
//              5.43 ms).
//   warp 1     MMA issuer (one thread): S_s = Q K_s^T into TMEM buffer S[s&1],
//              then O[s&1] += P_{s-1} V_{s-1}; tcgen05.commit frees ring slots
//              and signals the softmax.
//   warps 2-9  softmax in two groups of four warps (one warp per TMEM lane
//              quadrant): group g owns the stages s with s & 1 = g, its S
//              buffer and its own O accumulator, so one group's exponentials
//              overlap the other group's TMEM loads, maxima and stores.  A
//              thread owns one query row of its group's stages: it reads the
//              S row from TMEM, masks, keeps its group's running reference
//              max in the log2 domain, rescales its O row only when the max
//              grew by more than 2^8 (lazy rescale), and writes P as bf16
//              pairs back over the first 64 columns of the S buffer (the A
//              operand of P.V).  It keeps two row sums: of P in fp32 (for
//              LSE) and of the bf16-rounded P (to normalise O).
//              Epilogue: the two groups exchange (max, sums) through shared
//              memory, merge their partial results exactly, normalise, and
//              each writes half of the row's columns (and, if asked, merges
//              with a previous (O, LSE)).
// TMEM: S_0 [0,128), S_1 [128,256), O_0 [256, 256 + d), O_1 [384, 384 + d).
//
// Barrier phases.  A parity wait is only unambiguous when the barrier cannot
// run two phases ahead of its waiter, so every per-stage barrier is split by
// stage parity: P of stage t (p_full[t&1]) cannot be signalled again before
// the MMA issuer consumed it, because stage t+2 needs S_{t+2}, which is issued
// after that wait.  The commit that signals S_t also covers P.V of stage t-2
// (issued before S_t), so a group that sees S_t may rescale its O at once.
// The epilogue waits on mma_drain, committed once after the last MMA.
//
// Normalising O by the sum of the same bf16-rounded P that multiplied V makes
// the output an exact convex combination of the selected V rows: a softmax
// dominated by one key returns that key's V without the rounding of its
// weight.  LSE uses the fp32 sum.
#pragma once

#include "common.cuh"
#include "merge.cuh"

namespace vsa {

constexpr int kSoftmaxWarps = 8;
constexpr int kAttnThreads = 64 + 32 * kSoftmaxWarps;
constexpr int kSingleThreads = kAttnThreads + 32;  // the single-tile kernel: + the V producer (warp 10)
constexpr int kTileM = 128;
constexpr int kStageKeys = 128;
constexpr int kChunkBytes = 128 * 128;  // one 64-column bf16 chunk of a 128-row tile
constexpr int kInfoRing = 4;
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleThreshold = 8.0f;  // log2 units
// logits reach the FMA-pipe exponential at most kRescaleThreshold above the
// running reference maximum
static_assert(kRescaleThreshold <= kExp2PolyMaxInput, "exp2_poly2 is exact in range only up to 2^126");
constexpr int kListStage = 2048;  // list entries staged in shared memory per list (fast path)
constexpr int kUnionCap = 2 * kListStage;

struct AttnArgs {
  int n_pad, n_valid;
  int list_rows, seg_keys, seg_shift, idx_stride;
  const int32_t *counts;
  const int32_t *idx;
  float scale_log2;  // softmax scale * log2(e)
  void *o;
  int o_fp32;
  float *lse;
  const float *merge_o;
  const float *merge_lse;
  const int32_t *heads;  // grid row -> b * H + h, or NULL for grid row = b * H + h
  int n_bh;              // B * H
  unsigned long long timeout_ns;
  int *status;           // the launch's status word
  // Pair boxes (16-key segments, d = 128): a segment's K / V rows arrive as one
  // 4 KB box of the 5-D maps xm.k[0] / xm.v[0], laid out [row group of 8][column
  // chunk][8 rows][128 B]; a segment that holds rows in [n_valid8, n_valid)
  // comes as four 8-row boxes of xm.k[1] / xm.v[1] into the same places.
  int pair_boxes;
  int n_valid8;          // n_valid rounded down to a multiple of 8
  // Cluster-group mode (tile_list non-null; list_rows 128, seg_keys 16): tile T of
  // head bh uses list row tile_list[bh][T] (-1: no such tile, the CTA leaves at
  // once), whose entries are key clusters j < n_kc; cluster j is the K/V rows
  // [kc_off[j], kc_off[j] + kc_size[j]), walked as 16-key segments of which the
  // last may be partial.  Query and output rows per head: n_rows_q.
  const int32_t *tile_list;  // [BH][n_tiles]
  const int32_t *kc_off;     // [BH][n_kc]
  const int32_t *kc_size;    // [BH][n_kc]
  int n_kc, n_lists_bh, n_tiles, n_rows_q;
  // Pooled-rectification mode (pool_nk > 0; seg_keys 128): the keys are the bf16
  // means of the pool_nk key blocks (K / V maps of pooled rows), key block j
  // weighted by its valid key count s_j = clamp(pool_nvalid - j * pool_bk, 0,
  // pool_bk); the lists (counts / idx, list_rows query rows each) name the kept
  // blocks, which this pass skips.
  int pool_nk, pool_bk, pool_nvalid;
};

struct StageInfo {
  int start[8];   // first key row of each segment of the stage
  uint32_t mask;  // bit 2*s + h: segment s is used by query half h
  int full;       // every column of the stage is used by every row
  int tail;       // some used segment reaches past n_valid (exact per-column masks)
  uint32_t use16; // bit 8*h + q: 16-column group q is used by query half h
  uint32_t len4;  // cluster-group mode: bits [4s, 4s + 4) = 16 - valid keys of segment s
  uint32_t box4;  // bits [4s, 4s + 4): segments covered by segment s's K / V box (0: inside another's)
};

template <int D>
struct AttnSmem {
  static constexpr int kQBytes = kTileM * D * 2;
  static constexpr int kKVBytes = kStageKeys * D * 2;
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kQBytes;
  static constexpr int kOffV = kOffK + 2 * kKVBytes;
  static constexpr int kOffX = kOffV + 2 * kKVBytes;  // epilogue exchange: [2 groups][3][128] floats
  static constexpr int kOffU = kOffX + 4096;          // the tile's segment union: [kUnionCap] entries
  static constexpr int kOffL = kOffU + kUnionCap * 4; // the tile's lists, staged: [2][kListStage]
  static constexpr int kOffCtl = kOffL + 2 * kListStage * 4;
  static constexpr int kBytes = kOffCtl + 1024;  // barriers, info ring, misc
  static constexpr int kAlloc = kBytes + 1024;   // slack for 1024-byte alignment
};

struct AttnCtl {
  uint64_t q_full;
  uint64_t k_full[2], k_empty[2];
  uint64_t v_full[2], v_empty[2];
  uint64_t s_full[2], s_free[2];
  uint64_t p_full[2];               // per S buffer: P of the stage written
  uint64_t mma_drain;               // every MMA of the CTA has completed (one phase)
  uint64_t info_full[kInfoRing];
  uint64_t xbar[4];  // per lane quadrant: the two groups' final (max, sum) exchange
  uint32_t tmem_base;
  AbortCtl abort;
  int n_seg;
  int n_ent;  // cluster-group mode: key clusters of the tile's list
  int fast;  // the union sits in shared memory (lists short enough to stage)
  StageInfo info[kInfoRing];
};

// Cursor over the (union of the) sorted list(s) of a tile, walked by a whole
// warp in lockstep; lane-parallel windows of 32 entries keep the global reads
// coalesced.
struct ListCursor {
  const int32_t *p[2];
  int n[2];
  int pos[2];
  int base[2];
  int win[2];  // this lane's window entry of each list
  int nl;

  __device__ void init(const int32_t *p0, int n0, const int32_t *p1, int n1, int lists, int lane) {
    p[0] = p0; n[0] = n0; p[1] = p1; n[1] = n1; nl = lists;
    for (int h = 0; h < 2; ++h) {
      pos[h] = 0;
      base[h] = 0;
      win[h] = (h < nl && lane < n[h]) ? __ldg(p[h] + lane) : 0x7fffffff;
    }
  }
  __device__ int peek(int h, int lane) {
    if (h >= nl || pos[h] >= n[h]) return 0x7fffffff;
    if (pos[h] - base[h] >= 32) {
      base[h] = pos[h];
      const int e = base[h] + lane;
      win[h] = e < n[h] ? __ldg(p[h] + e) : 0x7fffffff;
    }
    return __shfl_sync(0xffffffffu, win[h], pos[h] - base[h]);
  }
  // Next segment of the union, or -1 at the end; *m = halves using it.
  __device__ int next(uint32_t *m, int lane) {
    const int a = peek(0, lane);
    const int b = peek(1, lane);
    if (a == 0x7fffffff && b == 0x7fffffff) return -1;
    if (nl == 1) {
      ++pos[0];
      *m = 3u;
      return a;
    }
    if (a < b) { ++pos[0]; *m = 1u; return a; }
    if (b < a) { ++pos[1]; *m = 2u; return b; }
    ++pos[0]; ++pos[1]; *m = 3u; return a;
  }
};

constexpr uint32_t kUnionDropped = 0xffffffffu;  // no real entry: segment indices stay below 2^30

// Number of entries of the ascending array p[0, n) below v.
__device__ __forceinline__ int lower_bound_smem(const int32_t *p, int n, int v) {
  int lo = 0, hi = n;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (p[mid] < v) lo = mid + 1;
    else hi = mid;
  }
  return lo;
}

// Warp-cooperative: stages one or two ascending lists (n0, n1 entries, each
// at most `stride`) in shared memory at sl and sl + stride, checks them
// (entries strictly ascending, in [0, n_max)), and writes their union to su,
// ascending, each entry = index | (lists holding it) << 30 (bit 30: list 0,
// bit 31: list 1; a lone list gets single_tag).  Two lists are merged by rank
// -- entry i of list 0 lands at i + #(list-1 entries below it), entry j of
// list 1 at j + #(list-0 entries at or below it); a list-1 entry equal to a
// list-0 entry is dropped and that list-0 entry is tagged for both -- and one
// compaction pass closes the gaps.  Returns the union size, or -1 when a
// list is invalid.  su holds n0 + n1 entries of scratch.
// Rank merge of two ascending lists already in shared memory into their
// ascending union su, each entry tagged (bits 30-31) with the lists that hold
// it (1 = A, 2 = B, 3 = both); returns the union's length.  su needs room for
// nA + nB entries until the closing compaction.
__device__ __forceinline__ int merge_staged(const int32_t *A, int nA, const int32_t *B, int nB, uint32_t *su,
                                            int lane) {
  for (int i = lane; i < nA; i += 32) {
    const int v = A[i];
    const int r = lower_bound_smem(B, nB, v);
    const bool d = r < nB && B[r] == v;
    su[i + r] = static_cast<uint32_t>(v) | ((d ? 3u : 1u) << 30);
  }
  for (int j = lane; j < nB; j += 32) {
    const int v = B[j];
    const int r = lower_bound_smem(A, nA, v);
    const bool d = r < nA && A[r] == v;
    su[j + r + (d ? 1 : 0)] = d ? kUnionDropped : (static_cast<uint32_t>(v) | (2u << 30));
  }
  __syncwarp();
  int n = 0;
  for (int k0 = 0; k0 < nA + nB; k0 += 32) {
    const int k = k0 + lane;
    const uint32_t x = k < nA + nB ? su[k] : kUnionDropped;
    const uint32_t keep = __ballot_sync(0xffffffffu, x != kUnionDropped);
    __syncwarp();
    if (x != kUnionDropped) su[n + __popc(keep & ((1u << lane) - 1u))] = x;
    n += __popc(keep);
    __syncwarp();
  }
  return n;
}

__device__ __forceinline__ int stage_union(const int32_t *g0, int n0, const int32_t *g1, int n1, int n_lists,
                                           int n_max, int32_t *sl, int stride, uint32_t *su, uint32_t single_tag,
                                           int lane) {
  const int cnt[2] = {n0, n_lists > 1 ? n1 : 0};
  const int32_t *src[2] = {g0, g1};
  for (int h = 0; h < n_lists; ++h)
    for (int e = lane; e < cnt[h]; e += 32) sl[h * stride + e] = __ldg(src[h] + e);
  __syncwarp();
  bool ok = true;
  for (int h = 0; h < n_lists; ++h) {
    const int32_t *li = sl + h * stride;
    for (int e = lane; e < cnt[h]; e += 32) {
      const int v = li[e];
      if (v < 0 || v >= n_max || (e > 0 && li[e - 1] >= v)) ok = false;
    }
  }
  if (!__all_sync(0xffffffffu, ok)) return -1;
  if (n_lists == 1) {
    for (int e = lane; e < cnt[0]; e += 32) su[e] = static_cast<uint32_t>(sl[e]) | (single_tag << 30);
    __syncwarp();
    return cnt[0];
  }
  return merge_staged(sl, cnt[0], sl + stride, cnt[1], su, lane);
}

// Warp-cooperative validation of one list (strictly ascending, in range);
// returns false on a violation.
__device__ __forceinline__ bool list_valid(const int32_t *p, int n, int n_seg_max, int lane) {
  bool ok = true;
  for (int e = lane; e < n; e += 32) {
    const int v = __ldg(p + e);
    if (v < 0 || v >= n_seg_max) ok = false;
    if (e > 0 && __ldg(p + e - 1) >= v) ok = false;
  }
  return __all_sync(0xffffffffu, ok);
}

// acc += the two bf16 values packed in pk (fp32 accumulation).
__device__ __forceinline__ float add_bf16x2_f32(float acc, uint32_t pk) {
  asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %1;\n\t"
      "add.rn.f32.bf16 %0, lo, %0;\n\tadd.rn.f32.bf16 %0, hi, %0;\n\t}"
      : "+f"(acc)
      : "r"(pk));
  return acc;
}

// Taller K / V boxes of cluster-group mode: [0] 32 rows, [1] 64 rows (a run of
// consecutive segments of one key cluster is contiguous in memory).
struct alignas(64) GroupMaps {
  CUtensorMap k[2];
  CUtensorMap v[2];
};

template <int D>
__global__ void __launch_bounds__(kSingleThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ GroupMaps xm,
                    const AttnArgs a) {
  using L = AttnSmem<D>;
  extern __shared__ uint8_t attn_smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(attn_smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  uint8_t *sQ = smem + L::kOffQ;
  uint8_t *sK = smem + L::kOffK;
  uint8_t *sV = smem + L::kOffV;
  float *sX = reinterpret_cast<float *>(smem + L::kOffX);  // [2 groups][max, sum, rounded sum][128 rows]
  AttnCtl *ctl = reinterpret_cast<AttnCtl *>(smem + L::kOffCtl);
  AbortCtl *abort = &ctl->abort;

  const int tile = blockIdx.x;
  // (batch, head) of this grid row: the caller's head list, or all of them in order.  An
  // out-of-range entry latches BAD_INDEX before any setup and the whole CTA leaves.
  const int bh = a.heads ? __ldg(a.heads + blockIdx.y) : static_cast<int>(blockIdx.y);
  if (bh < 0 || bh >= a.n_bh) {
    if (threadIdx.x == 0) latch_status(a.status, VSA_ERR_BAD_INDEX);
    return;
  }
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const bool groups = a.tile_list != nullptr;
  const bool pooled = a.pool_nk > 0;
  int group_row = 0;
  if (groups) {
    group_row = __ldg(a.tile_list + (size_t)bh * a.n_tiles + tile);
    if (group_row < 0) return;  // no tile here
    if (group_row >= a.n_lists_bh) {
      if (threadIdx.x == 0) latch_status(a.status, VSA_ERR_BAD_INDEX);
      return;
    }
  }
  const int n_lists = kTileM / a.list_rows;
  const int lists_per_bh = groups ? a.n_lists_bh : a.n_pad / a.list_rows;
  const int seg_per_stage = kStageKeys / a.seg_keys;
  const size_t lrow0 = (size_t)bh * lists_per_bh + (groups ? (size_t)group_row : (size_t)tile * n_lists);
  const int n_rows_q = groups ? a.n_rows_q : a.n_pad;
  const int q_valid = groups ? a.n_rows_q : a.n_valid;

  // ---------------------------------------------------------------- setup
  if (warp == 0) {
    if (lane == 0) {
      mbar_init(&ctl->q_full, 1);
      for (int i = 0; i < 2; ++i) {
        mbar_init(&ctl->k_full[i], 1);
        mbar_init(&ctl->k_empty[i], 1);
        mbar_init(&ctl->v_full[i], 1);
        mbar_init(&ctl->v_empty[i], 1);
        mbar_init(&ctl->s_full[i], 1);
        mbar_init(&ctl->s_free[i], 128);
        mbar_init(&ctl->p_full[i], 128);
      }
      mbar_init(&ctl->mma_drain, 1);
      for (int i = 0; i < kInfoRing; ++i) mbar_init(&ctl->info_full[i], 1);
      for (int i = 0; i < 4; ++i) mbar_init(&ctl->xbar[i], 64);
      abort_init(&ctl->abort, a.status);
      fence_barrier_init();
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
    }
    // Segment union of the tile, with list validation.  Fast path (both lists
    // fit the staging area): the lists are copied to shared memory, checked
    // there, and merged by rank into the union -- entry i of list 0 lands at
    // i + #(list-1 entries below it), entry j of list 1 at j + #(list-0
    // entries at or below it); a list-1 entry equal to a list-0 entry is
    // dropped and that list-0 entry is tagged for both halves -- then one
    // compaction pass closes the gaps.  Longer lists are walked from global
    // memory by ListCursor (count here, segments again in the producer).
    const int n_seg_max = a.n_pad / a.seg_keys;
    int cnt[2] = {0, 0};
    bool ok = true;
    for (int h = 0; h < n_lists; ++h) {
      cnt[h] = __ldg(a.counts + lrow0 + h);
      if (cnt[h] < 0 || cnt[h] > a.idx_stride) ok = false;
    }
    const bool fast = ok && cnt[0] <= kListStage && cnt[1] <= kListStage;
    int n_seg = 0;
    if (pooled) {
      // kept-block bitmaps of the tile's query blocks (one per list) in shared memory
      uint32_t *sb = reinterpret_cast<uint32_t *>(smem + L::kOffL);
      sb[lane] = 0u;
      sb[32 + lane] = 0u;
      __syncwarp();
      for (int h = 0; h < n_lists && ok; ++h) {
        const int32_t *li = a.idx + (lrow0 + h) * a.idx_stride;
        for (int e = lane; e < cnt[h]; e += 32) {
          const int j = __ldg(li + e);
          if (j < 0 || j >= a.pool_nk) ok = false;
          else atomicOr(&sb[h * 32 + (j >> 5)], 1u << (j & 31));
        }
      }
      ok = __all_sync(0xffffffffu, ok);
      __syncwarp();
      n_seg = ok ? (a.pool_nk + kStageKeys - 1) / kStageKeys : 0;
    } else if (groups) {
      // the group's key clusters: ids at sl[e], first rows at sl[kListStage + e],
      // sizes at su[kListStage + e], inclusive prefix of their 16-key segment counts at su[e]
      int32_t *sl = reinterpret_cast<int32_t *>(smem + L::kOffL);
      uint32_t *su = reinterpret_cast<uint32_t *>(smem + L::kOffU);
      ok = ok && fast;
      const int n = ok ? cnt[0] : 0;
      const int32_t *li = a.idx + lrow0 * a.idx_stride;
      for (int e = lane; e < n; e += 32) sl[e] = __ldg(li + e);
      __syncwarp();
      int carry = 0;
      for (int e0 = 0; e0 < n; e0 += 32) {
        const int e = e0 + lane;
        int segs = 0;
        if (e < n) {
          const int j = sl[e];
          if (j < 0 || j >= a.n_kc || (e > 0 && sl[e - 1] >= j)) {
            ok = false;
          } else {
            const int off = __ldg(a.kc_off + (size_t)bh * a.n_kc + j);
            const int sz = __ldg(a.kc_size + (size_t)bh * a.n_kc + j);
            if (off < 0 || sz < 0 || (long long)off + sz > a.n_pad) ok = false;
            segs = ok ? (sz + 15) >> 4 : 0;
            sl[kListStage + e] = off;
            su[kListStage + e] = static_cast<uint32_t>(ok ? sz : 0);
          }
        }
        const int incl = warp_exclusive_scan(segs, lane) + segs + carry;
        if (e < n) su[e] = static_cast<uint32_t>(incl);
        carry = __shfl_sync(0xffffffffu, incl, 31);
      }
      ok = __all_sync(0xffffffffu, ok);
      n_seg = ok ? carry : 0;
      __syncwarp();
    } else if (fast) {
      n_seg = stage_union(a.idx + lrow0 * a.idx_stride, cnt[0], a.idx + (lrow0 + 1) * a.idx_stride, cnt[1],
                          n_lists, n_seg_max, reinterpret_cast<int32_t *>(smem + L::kOffL), kListStage,
                          reinterpret_cast<uint32_t *>(smem + L::kOffU), 3u, lane);
      ok = n_seg >= 0;
    } else if (ok) {
      for (int h = 0; h < n_lists && ok; ++h)
        ok = list_valid(a.idx + (lrow0 + h) * a.idx_stride, cnt[h], n_seg_max, lane);
      if (ok && n_lists == 1) {
        n_seg = cnt[0];
      } else if (ok) {
        ListCursor cur;
        cur.init(a.idx + lrow0 * a.idx_stride, cnt[0], a.idx + (lrow0 + 1) * a.idx_stride, cnt[1], 2, lane);
        uint32_t m;
        while (cur.next(&m, lane) >= 0) ++n_seg;
      }
    }
    if (!ok) {
      n_seg = 0;
      if (lane == 0) latch_status(a.status, VSA_ERR_BAD_INDEX);
    }
    if (lane == 0) {
      ctl->n_seg = n_seg;
      ctl->n_ent = cnt[0];
      ctl->fast = fast ? 1 : 0;
    }
  } else if (warp == 1) {
    tmem_alloc(&ctl->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  const int n_seg = ctl->n_seg;
  const int n_stages = (n_seg + seg_per_stage - 1) / seg_per_stage;
  const uint32_t tmem = ctl->tmem_base;
  const uint32_t tS[2] = {tmem, tmem + 128u};
  const uint32_t tO[2] = {tmem + 256u, tmem + 384u};

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (n_stages > 0) {
      const bool fast = ctl->fast != 0;
      const uint32_t *su = reinterpret_cast<const uint32_t *>(smem + L::kOffU);
      ListCursor cur;
      if (!fast)
        cur.init(a.idx + lrow0 * a.idx_stride, __ldg(a.counts + lrow0),
                 n_lists > 1 ? a.idx + (lrow0 + 1) * a.idx_stride : nullptr,
                 n_lists > 1 ? __ldg(a.counts + lrow0 + 1) : 0, n_lists, lane);
      if (lane == 0) {
        mbar_arrive_expect_tx(&ctl->q_full, L::kQBytes);
        for (int c = 0; c < D / 64; ++c)
          tma_load_3d(sQ + c * kChunkBytes, &tm_q, &ctl->q_full, c * 64, tile * kTileM, bh);
      }
      // copy lane l < seg_per_stage * D/64 moves segment l / (D/64), column chunk l % (D/64)
      constexpr int kNC = D / 64;
      const int cp_seg = lane / kNC < 8 ? lane / kNC : 0;
      const int cp_chunk = lane % kNC;
      const bool cp_lane = lane < seg_per_stage * kNC;
      const uint32_t all = seg_per_stage == 8 ? 0xffffu : ((1u << (2 * seg_per_stage)) - 1u);
      const int g_shift = a.seg_shift - 4;  // 16-column groups per segment = 1 << g_shift
      const int n_ent = ctl->n_ent;
      int cur_e = 0, cur_k = 0;  // cluster-group mode: the next stage's first segment
      int issued = 0;
      for (int s = 0; s < n_stages; ++s) {
        const int slot = s & 1;
        const uint32_t use_par = ((s >> 1) - 1) & 1;
        // this stage's segments: lane i < seg_per_stage holds segment i's first key row
        int my_start = 0;
        uint32_t b0 = 0u, b1 = 0u;  // bit i: segment i used by query half 0 / 1
        uint32_t my_len4 = 0u;
        int my_box = 1;  // segments covered by this lane's K / V box (0: inside another lane's box)
        if (pooled) {
          my_start = s * kStageKeys;
          b0 = b1 = 1u;
        } else if (groups) {
          // lane i < seg_per_stage: segment i of the stage, counted on from the stage's
          // first segment (segment cur_k of entry cur_e); su[e] is the inclusive prefix
          // of the entries' segment counts
          const int g = s * seg_per_stage + lane;
          const bool has = lane < seg_per_stage && g < n_seg;
          int e = cur_e, k = cur_k + lane, start = 0;
          if (has) {
            const int32_t *sl = reinterpret_cast<const int32_t *>(smem + L::kOffL);
            for (;;) {
              const int ns = static_cast<int>(su[e]) - (e > 0 ? static_cast<int>(su[e - 1]) : 0);
              if (k < ns || e >= n_ent - 1) break;
              k -= ns;
              ++e;
            }
            start = sl[kListStage + e] + 16 * k;
            const int len = min(16, static_cast<int>(su[kListStage + e]) - 16 * k);
            my_len4 = static_cast<uint32_t>(16 - len) << (4 * lane);
          }
          cur_e = __shfl_sync(0xffffffffu, e, seg_per_stage - 1);
          cur_k = __shfl_sync(0xffffffffu, k, seg_per_stage - 1) + 1;
          const int start0 = __shfl_sync(0xffffffffu, start, 0);
          my_start = has ? start : start0;
          b0 = b1 = __ballot_sync(0xffffffffu, has);
          my_len4 = __reduce_or_sync(0xffffffffu, my_len4);
          // runs of consecutive segments of one entry are contiguous rows: cover each
          // run greedily with 64-, 32- and 16-row boxes
          const int e_up = __shfl_up_sync(0xffffffffu, e, 1), k_up = __shfl_up_sync(0xffffffffu, k, 1);
          const uint32_t cont = __ballot_sync(0xffffffffu, has && lane > 0 && e_up == e && k_up + 1 == k);
          const uint32_t starts = b0 & ~cont;
          if (has) {
            const uint32_t upto = (2u << lane) - 1u;
            const int rs = 31 - __clz(starts & upto);
            const uint32_t enders = ((starts | ~b0) & ~upto) | (1u << seg_per_stage);
            const int re = __ffs(enders) - 1;
            const int run = re - rs, p = lane - rs, n64 = run >> 2;
            if (p < 4 * n64) {
              my_box = (p & 3) == 0 ? 4 : 0;
            } else {
              const int q = p - 4 * n64, rem = run - 4 * n64;
              my_box = rem >= 2 ? (q == 0 ? 2 : (q == 2 ? 1 : 0)) : (q == 0 ? 1 : 0);
            }
          }
        } else if (fast) {
          const int e = s * seg_per_stage + lane;
          const bool has = lane < seg_per_stage && e < n_seg;
          const uint32_t x = has ? su[e] : 0u;
          const int seg = static_cast<int>(x & 0x3fffffffu);
          const int seg0 = __shfl_sync(0xffffffffu, seg, 0);  // a stage holds at least one segment
          my_start = (has ? seg : seg0) * a.seg_keys;
          b0 = __ballot_sync(0xffffffffu, has && ((x >> 30) & 1u));
          b1 = __ballot_sync(0xffffffffu, has && ((x >> 31) & 1u));
        } else {
          int start0 = 0, nseg = 0;
          for (int i = 0; i < seg_per_stage; ++i) {
            uint32_t m = 0u;
            const int sg = (nseg == i) ? cur.next(&m, lane) : -1;
            if (sg >= 0) {
              if (i == 0) start0 = sg * a.seg_keys;
              if (lane == i) my_start = sg * a.seg_keys;
              b0 |= (m & 1u) << i;
              b1 |= ((m >> 1) & 1u) << i;
              ++nseg;
            } else if (lane == i) {
              my_start = start0;  // repeat a loaded segment; masked out
            }
          }
        }
        const uint32_t used = b0 | b1;
        const bool tail = pooled ? false
                        : groups ? my_len4 != 0u
                                 : __any_sync(0xffffffffu, lane < seg_per_stage && ((used >> lane) & 1u) &&
                                                               my_start + a.seg_keys > a.n_valid);
        uint32_t mask = 0u, use16 = 0u;
        if (groups) {
          // both halves use every segment: spread bit i of b0 to bits 2i, 2i + 1
          uint32_t x = b0 & 0xffu;
          x = (x | (x << 4)) & 0x0f0fu;
          x = (x | (x << 2)) & 0x3333u;
          x = (x | (x << 1)) & 0x5555u;
          mask = x | (x << 1);
          use16 = (b0 & 0xffu) | ((b0 & 0xffu) << 8);
        } else {
          for (int i = 0; i < seg_per_stage; ++i)
            mask |= (((b0 >> i) & 1u) << (2 * i)) | (((b1 >> i) & 1u) << (2 * i + 1));
          for (int q = 0; q < 8; ++q)
            use16 |= (((b0 >> (q >> g_shift)) & 1u) << q) | (((b1 >> (q >> g_shift)) & 1u) << (8 + q));
        }
        const bool full = pooled || (mask == all && !tail);
        bool ok = true;
        if (s >= 2) ok = mbar_wait_warp(&ctl->k_empty[slot], use_par, abort, a.timeout_ns, lane);
        if (!ok) break;
        int st_i[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) st_i[i] = __shfl_sync(0xffffffffu, my_start, i);
        const uint32_t box4 =
            __reduce_or_sync(0xffffffffu, lane < 8 ? static_cast<uint32_t>(my_box) << (4 * lane) : 0u);
        if (lane == 0) {
          StageInfo &inf = ctl->info[s & (kInfoRing - 1)];
#pragma unroll
          for (int i = 0; i < 8; ++i) inf.start[i] = i < seg_per_stage ? st_i[i] : 0;
          inf.mask = mask;
          inf.full = full ? 1 : 0;
          inf.tail = tail ? 1 : 0;
          inf.use16 = use16;
          inf.len4 = my_len4;
          inf.box4 = box4;
          mbar_arrive(&ctl->info_full[s & (kInfoRing - 1)]);
          mbar_arrive_expect_tx(&ctl->k_full[slot], L::kKVBytes);
        }
        __syncwarp();
        const int cp_row = __shfl_sync(0xffffffffu, my_start, cp_seg);
        const int cp_box = __shfl_sync(0xffffffffu, my_box, cp_seg);
        const uint32_t cp_off = cp_chunk * kChunkBytes + cp_seg * a.seg_keys * 128;
        const CUtensorMap *map_k = cp_box == 4 ? &xm.k[1] : (cp_box == 2 ? &xm.k[0] : &tm_k);
        // pair boxes: lane i < 8 moves segment i (its own my_start) whole
        const bool pair_lane = a.pair_boxes && lane < 8;
        const bool pair_whole = my_start + 16 <= a.n_valid8 || my_start >= a.n_valid;
        if (pair_lane) {
          uint8_t *dst = sK + slot * L::kKVBytes + lane * 4096;
          if (pair_whole) {
            tma_load_5d(dst, &xm.k[0], &ctl->k_full[slot], 0, 0, 0, my_start >> 3, bh);
          } else {
            for (int q = 0; q < 4; ++q)
              tma_load_3d(dst + (q >> 1) * 2048 + (q & 1) * 1024, &xm.k[1], &ctl->k_full[slot], (q & 1) * 64,
                          my_start + 8 * (q >> 1), bh);
          }
        } else if (!a.pair_boxes && cp_lane && cp_box > 0) {
          tma_load_3d(sK + slot * L::kKVBytes + cp_off, map_k, &ctl->k_full[slot], cp_chunk * 64, cp_row, bh);
        }
        issued = s + 1;
        __syncwarp();
      }
      if (abort_raised(abort) && lane == 0) {
        // let copies still in flight land before the CTA's shared memory goes away
        mbar_drain(&ctl->q_full, 0, a.timeout_ns);
        for (int s = max(0, issued - 2); s < issued; ++s) {
          mbar_drain(&ctl->k_full[s & 1], (s >> 1) & 1, a.timeout_ns);
        }
      }
    }
  } else if (warp == 10) {
    // ---------------------------------------------------------- V producer
    // the stage's V boxes, at the starts (and box kinds) the K producer
    // published in the stage info ring.  The K producer rewrites the entry of
    // stage s for stage s + 4 only after S_{s+2} completed; S_{s+2} is issued
    // after P.V of stage s, which waited for V_s: this warp has read it.
    if (n_stages > 0) {
      constexpr int kNC = D / 64;
      const int cp_seg = lane / kNC < 8 ? lane / kNC : 0;
      const int cp_chunk = lane % kNC;
      const bool cp_lane = lane < seg_per_stage * kNC;
      int issued = 0;
      for (int s = 0; s < n_stages; ++s) {
        const int slot = s & 1;
        const uint32_t use_par = ((s >> 1) - 1) & 1;
        bool ok = mbar_wait_warp(&ctl->info_full[s & (kInfoRing - 1)], (s >> 2) & 1, abort, a.timeout_ns, lane);
        if (!ok) break;
        const StageInfo &inf = ctl->info[s & (kInfoRing - 1)];
        const int my_start = inf.start[lane & 7];
        const int cp_row = inf.start[cp_seg];
        const int cp_box = static_cast<int>((inf.box4 >> (4 * cp_seg)) & 15u);
        if (s >= 2) ok = mbar_wait_warp(&ctl->v_empty[slot], use_par, abort, a.timeout_ns, lane);
        if (!ok) break;
        if (lane == 0) mbar_arrive_expect_tx(&ctl->v_full[slot], L::kKVBytes);
        __syncwarp();
        if (!a.pair_boxes) {
          if (cp_lane && cp_box > 0) {
            const CUtensorMap *map_v = cp_box == 4 ? &xm.v[1] : (cp_box == 2 ? &xm.v[0] : &tm_v);
            tma_load_3d(sV + slot * L::kKVBytes + cp_chunk * kChunkBytes + cp_seg * a.seg_keys * 128, map_v,
                        &ctl->v_full[slot], cp_chunk * 64, cp_row, bh);
          }
        } else if (lane < 8) {
          uint8_t *dst = sV + slot * L::kKVBytes + lane * 4096;
          if (my_start + 16 <= a.n_valid8 || my_start >= a.n_valid) {
            tma_load_5d(dst, &xm.v[0], &ctl->v_full[slot], 0, 0, 0, my_start >> 3, bh);
          } else {
            for (int q = 0; q < 4; ++q)
              tma_load_3d(dst + (q >> 1) * 2048 + (q & 1) * 1024, &xm.v[1], &ctl->v_full[slot], (q & 1) * 64,
                          my_start + 8 * (q >> 1), bh);
          }
        }
        issued = s + 1;
        __syncwarp();
      }
      if (abort_raised(abort) && lane == 0)
        for (int s = max(0, issued - 2); s < issued; ++s) mbar_drain(&ctl->v_full[s & 1], (s >> 1) & 1, a.timeout_ns);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs the issuing loop in lockstep; one elected lane
    // issues each MMA and commit, so descriptors stay warp-uniform.
    if (n_stages > 0) {
      constexpr uint32_t kIdS = idesc_bf16_f32(kTileM, kStageKeys, false);
      constexpr uint32_t kIdO = idesc_bf16_f32(kTileM, D, true);
      // descriptor bases; K steps and ring slots only add to the start address field
      // pair boxes: K / V 8-row groups 2048 bytes apart, the two column chunks
      // of a group 1024 bytes apart
      const uint32_t kv_chunk = a.pair_boxes ? 1024u : static_cast<uint32_t>(kChunkBytes);
      const uint32_t kv_group = a.pair_boxes ? 2048u : 1024u;
      const uint64_t dQ = smem_desc_sw128(smem_addr(sQ), 16, 1024);
      const uint64_t dK0 = smem_desc_sw128(smem_addr(sK), 16, kv_group);
      const uint64_t dV0 = smem_desc_sw128(smem_addr(sV), kv_chunk, kv_group);
      constexpr uint64_t kSlotStep = L::kKVBytes >> 4;
      const uint32_t leader = elect_one();
      bool ok = mbar_wait_uni(&ctl->q_full, 0, abort, a.timeout_ns, lane);
      auto issue_pv = [&](int t) -> bool {
        if (!mbar_wait_uni(&ctl->p_full[t & 1], (t >> 1) & 1, abort, a.timeout_ns, lane)) return false;
        if (!mbar_wait_uni(&ctl->v_full[t & 1], (t >> 1) & 1, abort, a.timeout_ns, lane)) return false;
        tc_fence_after();
        const uint64_t dv = dV0 + (uint64_t)(t & 1) * kSlotStep;
        const uint32_t to = (t & 1) ? tO[1] : tO[0];
        const uint32_t ts = (t & 1) ? tS[1] : tS[0];
#pragma unroll
        for (int kk = 0; kk < kStageKeys / 16; ++kk) {
          // P (bf16 pairs) sits in the first 64 columns of the stage's S buffer
          umma_bf16_ts_one(to, ts + kk * 8, dv + (uint64_t)(kk * 2 * kv_group / 16), kIdO,
                           (t >= 2 || kk > 0) ? 1u : 0u, leader);
        }
        umma_commit_one(&ctl->v_empty[t & 1], leader);
        return true;
      };
      for (int s = 0; ok && s < n_stages; ++s) {
        const int slot = s & 1;
        ok = mbar_wait_uni(&ctl->k_full[slot], (s >> 1) & 1, abort, a.timeout_ns, lane);
        if (ok && s >= 2) ok = mbar_wait_uni(&ctl->s_free[slot], ((s - 2) >> 1) & 1, abort, a.timeout_ns, lane);
        if (!ok) break;
        tc_fence_after();
        const uint64_t dk = dK0 + (uint64_t)slot * kSlotStep;
        const uint32_t ts = slot ? tS[1] : tS[0];
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t offq = (uint64_t)(((kk >> 2) * kChunkBytes + (kk & 3) * 32) >> 4);
          const uint64_t offk = (uint64_t)(((kk >> 2) * kv_chunk + (kk & 3) * 32) >> 4);
          umma_bf16_ss_one(ts, dQ + offq, dk + offk, kIdS, kk > 0 ? 1u : 0u, leader);
        }
        umma_commit_one(&ctl->k_empty[slot], leader);
        umma_commit_one(&ctl->s_full[slot], leader);
        if (s >= 1) ok = issue_pv(s - 1);
      }
      if (ok) issue_pv(n_stages - 1);
      // every MMA issued by the leader has completed once mma_drain flips
      umma_commit_one(&ctl->mma_drain, leader);
      mbar_drain(&ctl->mma_drain, 0, a.timeout_ns);
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int g = (warp - 2) >> 2;            // group: stages s with s & 1 == g
    const int quad = warp & 3;
    const int row = quad * 32 + lane;         // row within the tile == TMEM lane
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const int half = row >> 6;                // query half for 64-row lists
    const uint32_t tSg = g == 0 ? tS[0] : tS[1];
    const uint32_t tOg = g == 0 ? tO[0] : tO[1];
    float m2 = -INFINITY;  // this group's running reference max of scaled logits, log2 units
    float l = 0.f;         // sum of P (fp32) over this group's stages
    float lr = 0.f;        // sum of the bf16-rounded P over this group's stages
    bool ok = true;
    const float sl2 = pooled ? 1.f : a.scale_log2;  // pooled logits arrive scaled
    const float2 sc2 = make_float2(sl2, sl2);
    for (int t = g; t < n_stages; t += 2) {
      ok = mbar_wait_warp(&ctl->info_full[t & (kInfoRing - 1)], (t >> 2) & 1, abort, a.timeout_ns, lane);
      if (ok) ok = mbar_wait_warp(&ctl->s_full[g], (t >> 1) & 1, abort, a.timeout_ns, lane);
      if (!ok) break;
      tc_fence_after();
      const StageInfo &inf = ctl->info[t & (kInfoRing - 1)];
      // the row's 128 logits: r[c][j] = S[row][32 c + j]
      uint32_t r[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(tSg + lane_off + c * 32, r[c]);
      tmem_ld_wait();
      if (!inf.full && (!inf.tail || groups)) {
        // whole 16-column groups this half does not use
        const uint32_t u = (inf.use16 >> (8 * half)) & 0xffu;
        if (u != 0xffu) {
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const bool drop = !((u >> q) & 1u);
#pragma unroll
            for (int j = 0; j < 16; ++j)
              if (drop) r[q >> 1][(q & 1) * 16 + j] = __float_as_uint(-INFINITY);
          }
        }
      }
      if (!inf.full && inf.tail && groups) {
        // partial segments (the last one of a key cluster): columns past its valid keys
        uint32_t part = inf.len4;
        while (part != 0u) {
          const int sg = (__ffs(part) - 1) >> 2;
          const int nv = 16 - static_cast<int>((part >> (4 * sg)) & 15u);
          part &= ~(0xfu << (4 * sg));
          switch (sg) {
#define VSA_MASK_SEG(K)                                                                      \
  case K: {                                                                                  \
    _Pragma("unroll") for (int j = 0; j < 16; ++j) if (j >= nv) r[(K) >> 1][((K) & 1) * 16 + j] = \
        __float_as_uint(-INFINITY);                                                          \
  } break;
            VSA_MASK_SEG(0)
            VSA_MASK_SEG(1)
            VSA_MASK_SEG(2)
            VSA_MASK_SEG(3)
            VSA_MASK_SEG(4)
            VSA_MASK_SEG(5)
            VSA_MASK_SEG(6)
            VSA_MASK_SEG(7)
#undef VSA_MASK_SEG
            default: break;
          }
        }
      } else if (!inf.full && inf.tail) {
        // a segment reaches past n_valid: valid columns as a 128-bit mask built
        // per segment (a used segment's valid keys form one prefix of it)
        uint64_t vm[2] = {0ull, 0ull};
        const uint32_t mask = inf.mask;
        const int nseg = kStageKeys >> a.seg_shift;
#pragma unroll 1
        for (int sg = 0; sg < nseg; ++sg) {
          if (!((mask >> (2 * sg + half)) & 1u)) continue;
          const int nv = min(a.seg_keys, max(0, a.n_valid - inf.start[sg]));
          const int lo = sg * a.seg_keys, hi = lo + nv;
#pragma unroll
          for (int w = 0; w < 2; ++w) {
            const int l0 = max(0, lo - 64 * w), h0 = min(64, hi - 64 * w);
            if (h0 > l0) {
              const uint64_t upto = h0 >= 64 ? ~0ull : ((1ull << h0) - 1ull);
              vm[w] |= upto & ~((1ull << l0) - 1ull);
            }
          }
        }
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (!((vm[c >> 1] >> ((c & 1) * 32 + j)) & 1ull)) r[c][j] = __float_as_uint(-INFINITY);
      }
      if (pooled) {
        // logit * scale * log2(e) + log2(s_j), -inf for kept blocks and blocks without keys
        const uint32_t *sb = reinterpret_cast<const uint32_t *>(smem + L::kOffL) + (n_lists > 1 ? half * 32 : 0);
        const uint32_t w4[4] = {sb[4 * t], sb[4 * t + 1], sb[4 * t + 2], sb[4 * t + 3]};
        const int n_full = a.pool_nvalid / a.pool_bk, rem = a.pool_nvalid - n_full * a.pool_bk;
        const int lim = n_full - kStageKeys * t;  // columns below lim are full-size blocks
        const float lb = log2f(static_cast<float>(a.pool_bk));
        const float lr = rem > 0 ? log2f(static_cast<float>(rem)) : -INFINITY;
        if (lim >= kStageKeys) {
#pragma unroll
          for (int c = 0; c < 4; ++c)
#pragma unroll
            for (int j = 0; j < 32; ++j)
              r[c][j] = ((w4[c] >> j) & 1u) ? __float_as_uint(-INFINITY)
                                            : __float_as_uint(fmaf(__uint_as_float(r[c][j]), a.scale_log2, lb));
        } else {
#pragma unroll
          for (int c = 0; c < 4; ++c)
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const int col = 32 * c + j;
              const float b = col < lim ? lb : (col == lim ? lr : -INFINITY);
              r[c][j] = ((w4[c] >> j) & 1u) ? __float_as_uint(-INFINITY)
                                            : __float_as_uint(fmaf(__uint_as_float(r[c][j]), a.scale_log2, b));
            }
        }
      }
      float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        mx[j & 3] = max3f(mx[j & 3], __uint_as_float(r[0][j]), __uint_as_float(r[1][j]));
        mx[(j + 2) & 3] = max3f(mx[(j + 2) & 3], __uint_as_float(r[2][j]), __uint_as_float(r[3][j]));
      }
      const float rmax = max3f(mx[0], mx[1], fmaxf(mx[2], mx[3]));
      const float m_new = fmaxf(m2, rmax * sl2);
      const bool need = m_new > m2 + kRescaleThreshold || (m2 == -INFINITY && m_new != -INFINITY);
      const bool any_rescale = __any_sync(0xffffffffu, need);
      float alpha = 1.f;
      if (need) {
        alpha = fast_exp2(m2 - m_new);  // exp2(-inf) = 0
        l *= alpha;
        lr *= alpha;
        m2 = m_new;
      }
      // P = exp2(s * scale * log2(e) - m2).  While m2 is -inf every logit of
      // the row is -inf (masked), so the exponent is -inf and P = 0.
      const float neg_m = m2 != -INFINITY ? -m2 : 0.f;
      const float2 nm2 = make_float2(neg_m, neg_m);
      float2 rs2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
      float rr[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int c = 0; c < 4; ++c) {
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const float2 x = ffma2(make_float2(__uint_as_float(r[c][2 * j]), __uint_as_float(r[c][2 * j + 1])), sc2, nm2);
          const float2 p = make_float2(fast_exp2(x.x), fast_exp2(x.y));
          rs2[j & 1] = fadd2(rs2[j & 1], p);
          const uint32_t pk = pack_bf16x2(p.x, p.y);
          rr[j & 3] = add_bf16x2_f32(rr[j & 3], pk);
          r[c >> 1][(c & 1) * 16 + j] = pk;  // packed in place over consumed logits
        }
      }
      const float2 rsum = fadd2(rs2[0], rs2[1]);
      l += rsum.x + rsum.y;
      lr += (rr[0] + rr[1]) + (rr[2] + rr[3]);
      if (any_rescale && t >= 2) {
        // cold path: rescale this group's O row by alpha (1 for rows whose max
        // stayed).  P.V of stage t-2 was issued before S_t, so the commit that
        // signalled S_t covers it; P.V of stage t waits for p_full below.
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(tOg + lane_off + c * 32, o);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * alpha);
          tmem_st32(tOg + lane_off + c * 32, o);
        }
      }
      tmem_st32(tSg + lane_off + 0, r[0]);
      tmem_st32(tSg + lane_off + 32, r[1]);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&ctl->s_free[g]);
      mbar_arrive(&ctl->p_full[g]);
    }

    // ---------------------------------------------------------- epilogue
    // exchange (max, sum, rounded sum) with the other group's thread of this row
    float *xs = sX;  // [2][3][128]
    xs[(g * 3 + 0) * 128 + row] = m2;
    xs[(g * 3 + 1) * 128 + row] = l;
    xs[(g * 3 + 2) * 128 + row] = lr;
    float mo = -INFINITY, lo = 0.f, lro = 0.f;
    if (ok) {
      mbar_arrive(&ctl->xbar[quad]);
      ok = mbar_wait_warp(&ctl->xbar[quad], 0, abort, a.timeout_ns, lane);
      if (ok) {
        mo = xs[((g ^ 1) * 3 + 0) * 128 + row];
        lo = xs[((g ^ 1) * 3 + 1) * 128 + row];
        lro = xs[((g ^ 1) * 3 + 2) * 128 + row];
      }
    }
    if (ok && n_stages > 0) {
      // the MMA issuer commits mma_drain after its last P.V: one phase, no ambiguity
      ok = mbar_wait_warp(&ctl->mma_drain, 0, abort, a.timeout_ns, lane);
    }
    // group 0 / 1 partial results -> exact merge
    const float m0 = g == 0 ? m2 : mo, m1 = g == 0 ? mo : m2;
    const float l0 = g == 0 ? l : lo, l1 = g == 0 ? lo : l;
    const float r0 = g == 0 ? lr : lro, r1 = g == 0 ? lro : lr;
    const float mm = fmaxf(m0, m1);
    const bool live = ok && n_stages > 0 && mm != -INFINITY;
    const float w0 = live && m0 != -INFINITY ? fast_exp2(m0 - mm) : 0.f;
    const float w1 = live && m1 != -INFINITY ? fast_exp2(m1 - mm) : 0.f;
    const float lsum = l0 * w0 + l1 * w1;
    const float rsum = r0 * w0 + r1 * w1;
    const int grow = tile * kTileM + row;
    const size_t orow = (size_t)bh * n_rows_q + grow;
    const bool row_ok = live && grow < q_valid && lsum > 0.f && rsum > 0.f;
    const float s0 = row_ok ? w0 / rsum : 0.f, s1 = row_ok ? w1 / rsum : 0.f;
    float lse = row_ok ? (mm + log2f(lsum)) * 0.69314718055994531f : -INFINITY;
    MergeWeights mw;
    mw.wa = 0.f;
    mw.wb = 1.f;
    if (a.merge_o != nullptr) {
      const float lm = grow < a.n_valid ? a.merge_lse[orow] : -INFINITY;
      mw = lse_merge_weights(lm, lse);
      lse = mw.lse;
    }
    if (g == 0) a.lse[orow] = lse;
    if (ok) tc_fence_after();
    // this group writes columns [g * D/2, (g + 1) * D/2) of the row
    constexpr int DH = D / 2;
    // tcgen05.ld is warp-collective: load when any row of the warp needs it
    const bool warp_loads = __any_sync(0xffffffffu, row_ok);
#pragma unroll 1
    for (int c = 0; c < DH / 32; ++c) {
      const int col = g * DH + c * 32;
      uint32_t oa[32], ob[32];
      if (warp_loads) {
        tmem_ld32(tO[0] + lane_off + col, oa);
        tmem_ld32(tO[1] + lane_off + col, ob);
        tmem_ld_wait();
      }
      float v[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        float x = 0.f;
        if (row_ok) {
          // a group without stages never wrote its O: its weight is 0 and its columns are not read
          x = (s0 > 0.f ? s0 * __uint_as_float(oa[j]) : 0.f) + (s1 > 0.f ? s1 * __uint_as_float(ob[j]) : 0.f);
        }
        v[j] = x;
      }
      if (a.merge_o != nullptr) {
        const float4 *mo4 = reinterpret_cast<const float4 *>(a.merge_o + orow * D + col);
#pragma unroll
        for (int q4 = 0; q4 < 8; ++q4) {
          const float4 m = mo4[q4];
          v[4 * q4 + 0] = mw.wa * m.x + mw.wb * v[4 * q4 + 0];
          v[4 * q4 + 1] = mw.wa * m.y + mw.wb * v[4 * q4 + 1];
          v[4 * q4 + 2] = mw.wa * m.z + mw.wb * v[4 * q4 + 2];
          v[4 * q4 + 3] = mw.wa * m.w + mw.wb * v[4 * q4 + 3];
        }
      }
      if (a.o_fp32) {
        float4 *dst = reinterpret_cast<float4 *>(static_cast<float *>(a.o) + orow * D + col);
#pragma unroll
        for (int q4 = 0; q4 < 8; ++q4) dst[q4] = make_float4(v[4 * q4], v[4 * q4 + 1], v[4 * q4 + 2], v[4 * q4 + 3]);
      } else {
        uint4 *dst = reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(a.o) + orow * D + col);
#pragma unroll
        for (int q8 = 0; q8 < 4; ++q8) {
          uint4 pk;
          pk.x = pack_bf16x2(v[8 * q8 + 0], v[8 * q8 + 1]);
          pk.y = pack_bf16x2(v[8 * q8 + 2], v[8 * q8 + 3]);
          pk.z = pack_bf16x2(v[8 * q8 + 4], v[8 * q8 + 5]);
          pk.w = pack_bf16x2(v[8 * q8 + 6], v[8 * q8 + 7]);
          dst[q8] = pk;
        }
      }
    }
  }

  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace vsa
