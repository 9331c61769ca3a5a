// a4 Macro pass, two query tiles per CTA sharing their K/V loads.
//
// HyperVAttention section 2 Eq. (4): each query block attends to its selected
// key blocks; section 4.3: the selected blocks of a row are walked as one
// packed sequence.  Neighbouring query blocks of a video select overlapping
// key blocks (spatio-temporal locality), so a CTA that owns two adjacent
// 128-row query tiles A and B walks the ascending union of their two lists,
// loads each union block's K and V once, and issues the S and P.V MMAs only
// for the tile(s) whose list holds that block: every MMA is useful, and each
// K/V byte feeds up to 256 query rows instead of 128.  This is the layout for
// 128-key blocks (one 128-key list entry per stage) with lists of 128 query
// rows, or (kHalf) of 64 query rows: then each tile walks the union of its two
// halves' lists and the rows of a half that did not keep a block take P = 0.
//
// Warp roles (320 threads):
//   warp 0     TMA producer: Q_A and Q_B once, then K and V of every union
//              block into 2 + 2 ring slots (rows past n_valid arrive as zeros).
//   warp 1     MMA issuer: walks the same union (warp-lockstep cursor) and,
//              per union block s, issues for each tile X that uses it
//              O_X += P_X(prev) V(prev) for X's previous block when that was
//              block s-1, then S_X = Q_X K_s^T into TMEM buffer S_X.  Blocks
//              of A and B interleave on the tensor core, so one tile's MMAs
//              run while the other tile's softmax works (ping-pong).
//   warps 2-5  softmax of tile A, warps 6-9 softmax of tile B: one thread
//              per query row walks its tile's own list, reads the S row from
//              TMEM, masks keys past n_valid, keeps the running reference max
//              in the log2 domain with lazy rescale of its TMEM O row (only
//              when the max grew by more than 2^8), writes P as bf16 pairs back
//              over the first 64 S columns (the A operand of P.V), and keeps
//              the fp32 row sum (for LSE) and the rounded-P row sum (to
//              normalise O: an exact convex combination of the V rows used).
// TMEM: S_A [0,128), S_B [128,256), O_A [256, 256 + d), O_B [384, 384 + d).
//
// P of a block goes to TMEM in two halves: p_half[X] signals keys 0-63, so the
// first half of the block's P.V runs while the softmax exponentiates keys
// 64-127, and p_full[X] signals the rest.
// Barrier phases: s_full[X], p_half[X] and p_full[X] advance once per block of tile X;
// S_X of X's next block is issued only after the MMA issuer waited p_full[X]
// of the current one, so neither can run two phases ahead of its waiter.  The
// commit that signals S_X(s) also covers P.V of X's previous block (issued
// before it), which is what a lazy rescale of O_X needs.  The K/V ring slots
// are released by one commit per union block s (into kv_free[s & 1]), issued
// after the block's S MMAs, which follow the P.V of block s-1: it frees K_s and
// V_{s-1}.  The producer waits on it for K_{s+2} and, one block later, for
// V_{s+1}; block s+2 cannot commit before K_{s+2} is loaded, so the wait stays
// unambiguous.  The issuing warp runs its loop in lockstep (waits by the
// whole warp, MMAs and commits by one elected lane), so descriptors and TMEM
// addresses stay warp-uniform; a loop run by lane 0 alone issued 8% slower.
// The issuer still does as few waits and commits per block as it can.
#pragma once

#include <type_traits>

#include "attn_fwd.cuh"

namespace vsa {

constexpr int kDualList = 1024;  // list entries staged per tile (every list of n_k <= 1024 blocks)
// Pairs j (of the 16 per 32-logit chunk) whose exponentials run on the FMA pipe
// (exp2_poly2) instead of MUFU: a 128-key row needs as many MUFU (XU) cycles
// as the tile's MMAs take, so part of the work moves to the FMA pipe.  Kernel
// time of a dense launch (8 heads, 16K tokens) by share moved: 0% 1.084 ms,
// 12.5% 1.005, 25% 1.013, 37.5% 1.018, 50% 1.068.  Masked logits come out as
// 2^-125 instead of 0 on these pairs; here the only masked keys are padding
// keys (past n_valid), whose V rows arrive as zeros, so they add nothing to O
// and vanish in any row sum that holds a real key.  (The single-tile kernel,
// which also masks keys of the other query half, keeps MUFU for every logit:
// there the split measured 2% slower.)
constexpr uint32_t kEmuPairs = 0x8080u;

template <int D, bool kHalf>
struct DualSmem {
  static constexpr int kQBytes = kTileM * D * 2;
  static constexpr int kKVBytes = kStageKeys * D * 2;
  static constexpr int kOffQ = 0;                       // Q_A, Q_B
  static constexpr int kOffK = kOffQ + 2 * kQBytes;
  static constexpr int kOffV = kOffK + 2 * kKVBytes;
  static constexpr int kOffU = kOffV + 2 * kKVBytes;          // union of the two lists [kDualList * 2]
  static constexpr int kOffL = kOffU + 2 * kDualList * 4;     // the two lists, staged [2][kDualList]
  // 64-row lists: per tile, the union of its two halves' lists, tagged with
  // the halves that kept each block [2][kDualList]
  static constexpr int kOffUX = kOffL + 2 * kDualList * 4;
  static constexpr int kOffCtl = kOffUX + (kHalf ? 2 * kDualList * 4 : 0);
  static constexpr int kBytes = kOffCtl + 512;
  static constexpr int kAlloc = kBytes + 1024;
};

struct DualCtl {
  uint64_t q_full;
  uint64_t k_full[2], v_full[2];
  uint64_t kv_free[2];  // one commit per union block s into kv_free[s & 1]: K_s and V_{s-1} are free
  uint64_t s_full[2];  // per tile
  uint64_t p_full[2];  // per tile: P of the block's keys 64-127 written (and its keys 0-63 before)
  uint64_t p_half[2];  // per tile: P of the block's keys 0-63 written
  uint64_t mma_drain;
  uint32_t tmem_base;
  AbortCtl abort;
  int n_union;
  int cnt[2];
  int fast;  // union and lists staged in shared memory
};

// kHalf: lists of 64-row query blocks (two per 128-row tile) instead of one
// list per tile.  Each tile then walks the union of its halves' lists; the
// softmax warps of a half that did not keep a block see all its keys masked
// and write P = 0 exactly for it (their rows' S is computed all the same: one
// M = 128 MMA covers both halves).  Those rows go through the same code as
// the others: a separate branch for them cost 13% in register spills.
template <int D, bool kHalf>
__global__ void __launch_bounds__(kAttnThreads, 1)
    attn_fwd_dual_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v, const AttnArgs a) {
  using L = DualSmem<D, kHalf>;
  extern __shared__ uint8_t dual_smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(dual_smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  uint8_t *sQ = smem + L::kOffQ;
  uint8_t *sK = smem + L::kOffK;
  uint8_t *sV = smem + L::kOffV;
  DualCtl *ctl = reinterpret_cast<DualCtl *>(smem + L::kOffCtl);
  AbortCtl *abort = &ctl->abort;

  const int pair = blockIdx.x;
  // (batch, head) of this grid row: the caller's head list, or all of them in order.  An
  // out-of-range entry latches BAD_INDEX before any setup and the whole CTA leaves.
  const int bh = a.heads ? __ldg(a.heads + blockIdx.y) : static_cast<int>(blockIdx.y);
  if (bh < 0 || bh >= a.n_bh) {
    if (threadIdx.x == 0) latch_status(a.status, VSA_ERR_BAD_INDEX);
    return;
  }
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_tiles = a.n_pad / kTileM;
  const int tile0 = 2 * pair;
  const bool has_b = tile0 + 1 < n_tiles;
  const int n_key_blocks = a.n_pad / kStageKeys;
  const size_t lrow0 = (size_t)bh * n_tiles + tile0;  // list row of tile A (list rows = 128)

  // ---------------------------------------------------------------- setup
  if (warp == 0) {
    if (lane == 0) {
      mbar_init(&ctl->q_full, 1);
      for (int i = 0; i < 2; ++i) {
        mbar_init(&ctl->k_full[i], 1);
        mbar_init(&ctl->kv_free[i], 1);
        mbar_init(&ctl->v_full[i], 1);
        mbar_init(&ctl->s_full[i], 1);
        mbar_init(&ctl->p_full[i], 128);
        mbar_init(&ctl->p_half[i], 128);
      }
      mbar_init(&ctl->mma_drain, 1);
      abort_init(&ctl->abort, a.status);
      fence_barrier_init();
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
    }
    int cnt[2] = {0, 0};
    bool ok = true;
    if (kHalf) {
      // four 64-row lists (A0, A1, B0, B1); the host sends only layers of at
      // most kDualList key blocks here, so every valid list fits in shared memory
      const size_t hrow0 = (size_t)bh * (a.n_pad / 64) + 2 * tile0;
      int c4[4] = {0, 0, 0, 0};
#pragma unroll
      for (int x = 0; x < 4; ++x) {
        if (x < (has_b ? 4 : 2)) {
          c4[x] = __ldg(a.counts + hrow0 + x);
          if (c4[x] < 0 || c4[x] > a.idx_stride || c4[x] > kDualList) ok = false;
        }
      }
      uint32_t *su_w = reinterpret_cast<uint32_t *>(smem + L::kOffU);
      int32_t *sl_w = reinterpret_cast<int32_t *>(smem + L::kOffL);
      uint32_t *ux_w = reinterpret_cast<uint32_t *>(smem + L::kOffUX);
#pragma unroll
      for (int x = 0; x < 2; ++x) {
        if (ok && x < (has_b ? 2 : 1)) {
          // tile x: union of its two halves, tags 1 = rows 0-63, 2 = rows 64-127
          const int n = stage_union(a.idx + (hrow0 + 2 * x) * a.idx_stride, c4[2 * x],
                                    a.idx + (hrow0 + 2 * x + 1) * a.idx_stride, c4[2 * x + 1], 2, n_key_blocks,
                                    sl_w, kDualList, su_w, 1u, lane);
          if (n < 0) {
            ok = false;
          } else {
            for (int e = lane; e < n; e += 32) ux_w[x * kDualList + e] = su_w[e];
            __syncwarp();
            cnt[x] = n;
          }
        }
      }
      int n_union = 0;
      if (ok) {
        // the union of the two tiles' unions drives the loads and the MMAs
#pragma unroll
        for (int x = 0; x < 2; ++x)
          for (int e = lane; e < cnt[x]; e += 32)
            sl_w[x * kDualList + e] = static_cast<int32_t>(ux_w[x * kDualList + e] & 0x3fffffffu);
        __syncwarp();
        if (has_b) {
          n_union = merge_staged(sl_w, cnt[0], sl_w + kDualList, cnt[1], su_w, lane);
        } else {
          for (int e = lane; e < cnt[0]; e += 32) su_w[e] = static_cast<uint32_t>(sl_w[e]) | (1u << 30);
          __syncwarp();
          n_union = cnt[0];
        }
      } else {
        if (lane == 0) latch_status(a.status, VSA_ERR_BAD_INDEX);
        cnt[0] = cnt[1] = 0;
      }
      if (lane == 0) {
        ctl->n_union = n_union;
        ctl->cnt[0] = cnt[0];
        ctl->cnt[1] = cnt[1];
        ctl->fast = 1;
      }
    } else {
      for (int x = 0; x < (has_b ? 2 : 1); ++x) {
        cnt[x] = __ldg(a.counts + lrow0 + x);
        if (cnt[x] < 0 || cnt[x] > a.idx_stride) ok = false;
      }
      // lists short enough to stage: validated and merged into the union in
      // shared memory once; otherwise validated here and walked from global
      // memory by ListCursor
      const bool fast = ok && cnt[0] <= kDualList && cnt[1] <= kDualList;
      int n_union = cnt[0] + cnt[1];  // cursor path: > 0 iff the union is not empty
      if (fast) {
        n_union = stage_union(a.idx + lrow0 * a.idx_stride, cnt[0], a.idx + (lrow0 + 1) * a.idx_stride, cnt[1],
                              has_b ? 2 : 1, n_key_blocks, reinterpret_cast<int32_t *>(smem + L::kOffL), kDualList,
                              reinterpret_cast<uint32_t *>(smem + L::kOffU), 1u, lane);
        ok = n_union >= 0;
      } else {
        for (int x = 0; x < (has_b ? 2 : 1) && ok; ++x)
          ok = list_valid(a.idx + (lrow0 + x) * a.idx_stride, cnt[x], n_key_blocks, lane);
      }
      if (!ok) {
        if (lane == 0) latch_status(a.status, VSA_ERR_BAD_INDEX);
        cnt[0] = cnt[1] = 0;
        n_union = 0;
      }
      if (lane == 0) {
        ctl->n_union = n_union;
        ctl->cnt[0] = cnt[0];
        ctl->cnt[1] = cnt[1];
        ctl->fast = fast ? 1 : 0;
      }
    }
  } else if (warp == 1) {
    tmem_alloc(&ctl->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  // The union of the two lists is walked until the cursor runs dry, so its
  // length never has to be counted up front.
  const bool any_block = ctl->n_union > 0;
  const uint32_t tmem = ctl->tmem_base;
  const uint32_t tS[2] = {tmem, tmem + 128u};
  const uint32_t tO[2] = {tmem + 256u, tmem + 384u};
  const int32_t *list[2] = {a.idx + lrow0 * a.idx_stride, a.idx + (lrow0 + 1) * a.idx_stride};
  const int cnt[2] = {ctl->cnt[0], has_b ? ctl->cnt[1] : 0};
  const bool fast = ctl->fast != 0;
  const int n_union = ctl->n_union;
  const uint32_t *su = reinterpret_cast<const uint32_t *>(smem + L::kOffU);
  const int32_t *sl = reinterpret_cast<const int32_t *>(smem + L::kOffL);
  const uint32_t *ux = reinterpret_cast<const uint32_t *>(smem + (kHalf ? L::kOffUX : L::kOffL));

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (any_block) {
      ListCursor cur;
      if (!fast) cur.init(list[0], cnt[0], has_b ? list[1] : nullptr, cnt[1], has_b ? 2 : 1, lane);
      if (lane == 0) {
        // Q is read by this CTA alone: its lines go first when L2 needs room,
        // so the K / V blocks that other CTAs of the head read again stay
        // (with O and LSE written as streaming stores, this cut the Macro
        // pass's DRAM reads on the HunyuanVideo-like layer from 3.21 to 2.94 GB)
        const uint64_t pol_q = l2_policy_evict_first();
        mbar_arrive_expect_tx(&ctl->q_full, (has_b ? 2 : 1) * L::kQBytes);
        for (int x = 0; x < (has_b ? 2 : 1); ++x)
          for (int c = 0; c < D / 64; ++c)
            tma_load_3d_hint(sQ + x * L::kQBytes + c * kChunkBytes, &tm_q, &ctl->q_full, c * 64,
                             (tile0 + x) * kTileM, bh, pol_q);
      }
      int issued = 0;
      for (int s = 0;; ++s) {
        const int slot = s & 1;
        const uint32_t use_par = ((s >> 1) - 1) & 1;
        uint32_t m = 0u;
        int blk;
        if (fast) {
          if (s >= n_union) break;
          blk = static_cast<int>(su[s] & 0x3fffffffu);
        } else {
          blk = cur.next(&m, lane);
          if (blk < 0) break;
        }
        const int start = blk * kStageKeys;
        bool ok = true;
        if (s >= 2) ok = mbar_wait_warp(&ctl->kv_free[slot], use_par, abort, a.timeout_ns, lane);  // K_{s-2} read
        if (!ok) break;
        if (lane == 0) {
          mbar_arrive_expect_tx(&ctl->k_full[slot], L::kKVBytes);
          for (int c = 0; c < D / 64; ++c)
            tma_load_3d(sK + slot * L::kKVBytes + c * kChunkBytes, &tm_k, &ctl->k_full[slot], c * 64, start, bh);
        }
        // V_{s-2} read: committed with block s-1
        if (s >= 2) ok = mbar_wait_warp(&ctl->kv_free[slot ^ 1], ((s - 1) >> 1) & 1, abort, a.timeout_ns, lane);
        if (!ok) break;
        if (lane == 0) {
          mbar_arrive_expect_tx(&ctl->v_full[slot], L::kKVBytes);
          for (int c = 0; c < D / 64; ++c)
            tma_load_3d(sV + slot * L::kKVBytes + c * kChunkBytes, &tm_v, &ctl->v_full[slot], c * 64, start, bh);
        }
        issued = s + 1;
        __syncwarp();
      }
      if (abort_raised(abort) && lane == 0) {
        mbar_drain(&ctl->q_full, 0, a.timeout_ns);
        for (int s = max(0, issued - 2); s < issued; ++s) {
          mbar_drain(&ctl->k_full[s & 1], (s >> 1) & 1, a.timeout_ns);
          mbar_drain(&ctl->v_full[s & 1], (s >> 1) & 1, a.timeout_ns);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (any_block) {
      constexpr uint32_t kIdS = idesc_bf16_f32(kTileM, kStageKeys, false);
      constexpr uint32_t kIdO = idesc_bf16_f32(kTileM, D, true);
      // Descriptor bases; a K step or ring slot only adds to the start
      // address field (bytes >> 4, which never carries out of its 14 bits
      // inside 227 KB of shared memory).
      const uint64_t dQ0 = smem_desc_sw128(smem_addr(sQ), 16, 1024);
      const uint64_t dK0 = smem_desc_sw128(smem_addr(sK), 16, 1024);
      const uint64_t dV0 = smem_desc_sw128(smem_addr(sV), kChunkBytes, 1024);
      constexpr uint64_t kQStep = L::kQBytes >> 4, kSlotStep = L::kKVBytes >> 4;
      ListCursor cur;
      if (!fast) cur.init(list[0], cnt[0], has_b ? list[1] : nullptr, cnt[1], has_b ? 2 : 1, lane);
      // The whole warp runs the issuing loop in lockstep; one elected lane
      // issues each MMA and commit.
      const uint32_t leader = elect_one();
      bool ok = mbar_wait_uni(&ctl->q_full, 0, abort, a.timeout_ns, lane);
      uint32_t prev = 0u;     // usage bits of the previous union block
      int pv_cnt[2] = {0, 0};  // P.V issued so far per tile
      // O_x += P_x(block s) V_s
      auto issue_pv = [&](auto xc, int s, bool &v_ready) -> bool {
        constexpr int x = decltype(xc)::value;
        // keys 0-63 of the block as soon as their P is in TMEM, keys 64-127 after
        if (!mbar_wait_uni(&ctl->p_half[x], pv_cnt[x] & 1, abort, a.timeout_ns, lane)) return false;
        if (!v_ready) {
          if (!mbar_wait_uni(&ctl->v_full[s & 1], (s >> 1) & 1, abort, a.timeout_ns, lane)) return false;
          v_ready = true;
        }
        tc_fence_after();
        const uint64_t dv = dV0 + (uint64_t)(s & 1) * kSlotStep;
        const uint32_t first = pv_cnt[x] > 0 ? 1u : 0u;
#pragma unroll
        for (int kk = 0; kk < kStageKeys / 32; ++kk)
          umma_bf16_ts_one(tO[x], tS[x] + kk * 8, dv + (uint64_t)(kk * 16 * 128 / 16), kIdO, kk > 0 ? 1u : first,
                           leader);
        if (!mbar_wait_uni(&ctl->p_full[x], pv_cnt[x] & 1, abort, a.timeout_ns, lane)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = kStageKeys / 32; kk < kStageKeys / 16; ++kk)
          umma_bf16_ts_one(tO[x], tS[x] + kk * 8, dv + (uint64_t)(kk * 16 * 128 / 16), kIdO, 1u, leader);
        ++pv_cnt[x];
        return true;
      };
      // S_x = Q_x K_s^T
      auto issue_s = [&](auto xc, int s) {
        constexpr int x = decltype(xc)::value;
        const uint64_t dq = dQ0 + (uint64_t)x * kQStep;
        const uint64_t dk = dK0 + (uint64_t)(s & 1) * kSlotStep;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t off = (uint64_t)(((kk >> 2) * kChunkBytes + (kk & 3) * 32) >> 4);
          umma_bf16_ss_one(tS[x], dq + off, dk + off, kIdS, kk > 0 ? 1u : 0u, leader);
        }
        umma_commit_one(&ctl->s_full[x], leader);
      };
      // one union block: P.V of a tile's block s-1 goes before its S of block
      // s (that S overwrites the TMEM buffer holding the tile's P)
      auto step = [&](int s, uint32_t use) {
        bool k_ready = false, v_ready = false;
        if (prev & 1u) ok = issue_pv(std::integral_constant<int, 0>{}, s - 1, v_ready);
        if (ok && (use & 1u)) {
          ok = mbar_wait_uni(&ctl->k_full[s & 1], (s >> 1) & 1, abort, a.timeout_ns, lane);
          k_ready = true;
          if (ok) {
            tc_fence_after();
            issue_s(std::integral_constant<int, 0>{}, s);
          }
        }
        if (ok && (prev & 2u)) ok = issue_pv(std::integral_constant<int, 1>{}, s - 1, v_ready);
        if (ok && (use & 2u)) {
          if (!k_ready) ok = mbar_wait_uni(&ctl->k_full[s & 1], (s >> 1) & 1, abort, a.timeout_ns, lane);
          if (ok) {
            tc_fence_after();
            issue_s(std::integral_constant<int, 1>{}, s);
          }
        }
        // the S MMAs of block s read K_s, the P.V of block s-1 V_{s-1}
        if (ok) umma_commit_one(&ctl->kv_free[s & 1], leader);
        prev = use;
      };
      int s = 0;
      if (fast) {
        // the union sits in shared memory (every lane reads the same entry)
        uint32_t e = n_union > 0 ? su[0] : 0u;
        for (; s < n_union && ok; ++s) {
          const uint32_t cur_e = e;
          if (s + 1 < n_union) e = su[s + 1];  // next entry, loaded while this block issues
          step(s, cur_e >> 30);
        }
      } else {
        for (;; ++s) {
          uint32_t use = 0u;
          if (cur.next(&use, lane) < 0) break;  // whole warp walks the union in lockstep
          if (!has_b) use &= 1u;  // a single-list cursor tags every block with both bits
          if (ok) step(s, use);
          prev = use;
        }
      }
      {
        bool v_ready = false;
        if (ok && (prev & 1u)) ok = issue_pv(std::integral_constant<int, 0>{}, s - 1, v_ready);
        if (ok && (prev & 2u)) ok = issue_pv(std::integral_constant<int, 1>{}, s - 1, v_ready);
        umma_commit_one(&ctl->mma_drain, leader);
        mbar_drain(&ctl->mma_drain, 0, a.timeout_ns);
      }
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int x = (warp - 2) >> 2;  // tile
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const bool tile_live = x == 0 || has_b;
    // this group's TMEM buffers and list as scalars (no runtime-indexed arrays)
    const uint32_t tSx = x == 0 ? tS[0] : tS[1];
    const uint32_t tOx = x == 0 ? tO[0] : tO[1];
    const int32_t *listx = x == 0 ? list[0] : list[1];
    float m2 = -INFINITY;  // running reference max of scaled logits, log2 units
    float l = 0.f;         // fp32 row sum of P
    float lr = 0.f;        // row sum of the bf16-rounded P
    bool ok = true;
    const float2 sc2 = make_float2(a.scale_log2, a.scale_log2);
    const int n_mine = tile_live ? (x == 0 ? cnt[0] : cnt[1]) : 0;
    const uint32_t *uxx = ux + x * kDualList;              // 64-row lists: this tile's tagged union
    const uint32_t half_tag = 1u << (30 + (quad >> 1));     // rows 0-63 are lane quadrants 0, 1
    for (int i = 0; i < n_mine; ++i) {
      int key0;
      bool mine = true;  // this warp's rows kept the block
      if (kHalf) {
        const uint32_t e = uxx[i];
        key0 = static_cast<int>(e & 0x3fffffffu) * kStageKeys;
        mine = (e & half_tag) != 0u;
      } else {
        key0 = (fast ? sl[x * kDualList + i] : __ldg(listx + i)) * kStageKeys;
      }
      ok = mbar_wait_warp(&ctl->s_full[x], i & 1, abort, a.timeout_ns, lane);
      if (!ok) break;
      tc_fence_after();
      uint32_t r[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(tSx + lane_off + c * 32, r[c]);
      tmem_ld_wait();
      // rows of the half that did not keep the block see every key masked
      const int nv = (kHalf && !mine) ? 0 : a.n_valid - key0;  // valid keys of this block
      if (nv < kStageKeys) {
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (c * 32 + j >= nv) r[c][j] = __float_as_uint(-INFINITY);
      }
      float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        mx[j & 3] = max3f(mx[j & 3], __uint_as_float(r[0][j]), __uint_as_float(r[1][j]));
        mx[(j + 2) & 3] = max3f(mx[(j + 2) & 3], __uint_as_float(r[2][j]), __uint_as_float(r[3][j]));
      }
      const float rmax = max3f(mx[0], mx[1], fmaxf(mx[2], mx[3]));
      const float m_new = fmaxf(m2, rmax * a.scale_log2);
      const bool need = m_new > m2 + kRescaleThreshold || (m2 == -INFINITY && m_new != -INFINITY);
      const bool any_rescale = __any_sync(0xffffffffu, need);
      float alpha = 1.f;
      if (need) {
        alpha = fast_exp2(m2 - m_new);  // exp2(-inf) = 0
        l *= alpha;
        lr *= alpha;
        m2 = m_new;
      }
      const float neg_m = m2 != -INFINITY ? -m2 : 0.f;
      const float2 nm2 = make_float2(neg_m, neg_m);
      float2 rs2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
      float rr[4] = {0.f, 0.f, 0.f, 0.f};
      // P of keys 0-63 (logit chunks 0, 1), packed into r[0]
#pragma unroll
      for (int c = 0; c < 2; ++c) {
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const float2 xx = ffma2(make_float2(__uint_as_float(r[c][2 * j]), __uint_as_float(r[c][2 * j + 1])), sc2, nm2);
          const float2 p = ((kEmuPairs >> j) & 1u) ? exp2_poly2(xx) : make_float2(fast_exp2(xx.x), fast_exp2(xx.y));
          rs2[j & 1] = fadd2(rs2[j & 1], p);
          const uint32_t pk = pack_bf16x2(p.x, p.y);
          rr[j & 3] = add_bf16x2_f32(rr[j & 3], pk);
          r[0][c * 16 + j] = pk;
        }
      }
      if (any_rescale && i > 0) {
        // cold path, before any P.V of this block: the commit that signalled
        // this S also covered the P.V of the tile's previous block, so O_x is
        // settled
#pragma unroll 1
        for (int c = 0; c < D / 8; ++c) {  // 8 columns at a time: the logits of keys 64-127 are still live
          uint32_t o[8];
          tmem_ld8(tOx + lane_off + c * 8, o);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 8; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * alpha);
          tmem_st8(tOx + lane_off + c * 8, o);
        }
      }
      // keys 0-63 handed to the tensor core first: their P.V overlaps the
      // exponentials of keys 64-127
      if (kHalf && !mine) {
#pragma unroll
        for (int j = 0; j < 32; ++j) r[0][j] = 0u;  // P = 0 exactly
      }
      tmem_st32(tSx + lane_off + 0, r[0]);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&ctl->p_half[x]);
#pragma unroll
      for (int c = 2; c < 4; ++c) {
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const float2 xx = ffma2(make_float2(__uint_as_float(r[c][2 * j]), __uint_as_float(r[c][2 * j + 1])), sc2, nm2);
          const float2 p = ((kEmuPairs >> j) & 1u) ? exp2_poly2(xx) : make_float2(fast_exp2(xx.x), fast_exp2(xx.y));
          rs2[j & 1] = fadd2(rs2[j & 1], p);
          const uint32_t pk = pack_bf16x2(p.x, p.y);
          rr[j & 3] = add_bf16x2_f32(rr[j & 3], pk);
          r[1][(c - 2) * 16 + j] = pk;
        }
      }
      if (kHalf && !mine) {
#pragma unroll
        for (int j = 0; j < 32; ++j) r[1][j] = 0u;
      }
      tmem_st32(tSx + lane_off + 32, r[1]);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&ctl->p_full[x]);
      if (!kHalf || mine) {
        const float2 rsum = fadd2(rs2[0], rs2[1]);
        l += rsum.x + rsum.y;
        lr += (rr[0] + rr[1]) + (rr[2] + rr[3]);
      }
    }

    // ---------------------------------------------------------- epilogue
    if (tile_live) {
      if (ok && n_mine > 0) ok = mbar_wait_warp(&ctl->mma_drain, 0, abort, a.timeout_ns, lane);
      const int grow = (tile0 + x) * kTileM + row;
      const size_t orow = (size_t)bh * a.n_pad + grow;
      const bool row_ok = ok && n_mine > 0 && grow < a.n_valid && l > 0.f && lr > 0.f;
      const float inv = row_ok ? 1.f / lr : 0.f;
      float lse = row_ok ? (m2 + log2f(l)) * 0.69314718055994531f : -INFINITY;
      MergeWeights mw;
      mw.wa = 0.f;
      mw.wb = 1.f;
      if (a.merge_o != nullptr) {
        const float lm = grow < a.n_valid ? a.merge_lse[orow] : -INFINITY;
        mw = lse_merge_weights(lm, lse);
        lse = mw.lse;
      }
      __stcs(a.lse + orow, lse);
      const bool warp_loads = __any_sync(0xffffffffu, row_ok);
      if (warp_loads) tc_fence_after();
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        if (warp_loads) {
          tmem_ld32(tOx + lane_off + c * 32, o);
          tmem_ld_wait();
        }
        float v[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = row_ok ? __uint_as_float(o[j]) * inv : 0.f;
        if (a.merge_o != nullptr) {
          const float4 *mo4 = reinterpret_cast<const float4 *>(a.merge_o + orow * D + c * 32);
#pragma unroll
          for (int q4 = 0; q4 < 8; ++q4) {
            const float4 mm = mo4[q4];
            v[4 * q4 + 0] = mw.wa * mm.x + mw.wb * v[4 * q4 + 0];
            v[4 * q4 + 1] = mw.wa * mm.y + mw.wb * v[4 * q4 + 1];
            v[4 * q4 + 2] = mw.wa * mm.z + mw.wb * v[4 * q4 + 2];
            v[4 * q4 + 3] = mw.wa * mm.w + mw.wb * v[4 * q4 + 3];
          }
        }
        if (a.o_fp32) {
          float4 *dst = reinterpret_cast<float4 *>(static_cast<float *>(a.o) + orow * D + c * 32);
#pragma unroll
          for (int q4 = 0; q4 < 8; ++q4)
            __stcs(dst + q4, make_float4(v[4 * q4], v[4 * q4 + 1], v[4 * q4 + 2], v[4 * q4 + 3]));
        } else {
          uint4 *dst = reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(a.o) + orow * D + c * 32);
#pragma unroll
          for (int q8 = 0; q8 < 4; ++q8) {
            uint4 pk;
            pk.x = pack_bf16x2(v[8 * q8 + 0], v[8 * q8 + 1]);
            pk.y = pack_bf16x2(v[8 * q8 + 2], v[8 * q8 + 3]);
            pk.z = pack_bf16x2(v[8 * q8 + 4], v[8 * q8 + 5]);
            pk.w = pack_bf16x2(v[8 * q8 + 6], v[8 * q8 + 7]);
            __stcs(dst + q8, pk);
          }
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
