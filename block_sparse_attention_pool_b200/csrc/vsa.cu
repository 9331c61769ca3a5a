// libvsa: host side of the C ABI declared in include/vsa.h.
//
// Validates arguments, builds TMA tensor maps through the driver entry point
// (no link-time dependency on libcuda), and launches the kernels of this
// directory.  It allocates no device memory and never synchronises except in
// vsa_read_device_status.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <algorithm>
#include <mutex>
#include <vector>

#include "../../include/vsa.h"
#include "attn_fwd.cuh"
#include "attn_fwd_dual.cuh"
#include "cluster.cuh"
#include "cluster_hybrid.cuh"
#include "cluster_merge.cuh"
#include "cluster_plan.cuh"
#include "common.cuh"
#include "merge.cuh"
#include "micro.cuh"
#include "pool.cuh"
#include "rectify.cuh"
#include "select.cuh"

namespace {

using vsa::AttnArgs;

constexpr unsigned long long kWaitLimitNs = 2000000000ull;  // 2 s per pipeline wait

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool shape_ok(const vsa_shape *s) {
  if (!s) return false;
  if (s->B < 1 || s->H < 1 || s->n_valid < 1 || s->n_pad < s->n_valid) return false;
  if (s->d != 64 && s->d != 128) return false;
  if (s->n_pad % 128 != 0) return false;
  if ((long long)s->B * s->H > 65535) return false;
  if ((long long)s->n_pad * s->d * s->B * s->H >= (1ll << 40)) return false;
  return true;
}

vsa_status launch_status() {
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? VSA_OK : VSA_ERR_CUDA;
}

// ---- status words ------------------------------------------------------------
// Caller-owned status words bound to streams (vsa_bind_status_word); launches
// on any other stream report into the process-wide word of the device.
constexpr int kMaxStatusBindings = 256;

struct StatusBinding {
  cudaStream_t stream;
  int device;
  int *word;
};

std::mutex &binding_mutex() {
  static std::mutex mu;
  return mu;
}

std::vector<StatusBinding> &bindings() {
  static std::vector<StatusBinding> b;
  return b;
}

// The status word that launches on `st` (of the current device) report into,
// or nullptr if no device address can be had.
int *status_word(cudaStream_t st) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return nullptr;
  {
    std::lock_guard<std::mutex> lock(binding_mutex());
    for (const StatusBinding &b : bindings())
      if (b.stream == st && b.device == dev) return b.word;
  }
  void *p = nullptr;
  if (cudaGetSymbolAddress(&p, vsa::g_status_word) != cudaSuccess) return nullptr;
  return static_cast<int *>(p);
}

// ---- tensor maps -----------------------------------------------------------

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// [BH][n_pad][d] bf16 viewed as a 3-D tensor (d, n_valid, BH): rows at or
// past n_valid are outside the tensor and arrive as zeros.  Box = 64 columns
// (128 bytes, one swizzle row) x box_rows rows x 1.
bool make_map(CUtensorMap *map, const void *base, const vsa_shape *s, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)s->d, (cuuint64_t)s->n_valid, (cuuint64_t)s->B * s->H};
  cuuint64_t strides[2] = {(cuuint64_t)s->d * 2, (cuuint64_t)s->n_pad * s->d * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// [BH][n_pad][128] bf16 as a 5-D tensor (64 columns, 8 rows, 2 column chunks,
// n_valid / 8 row groups, BH): a box of (64, 8, 2, 2, 1) moves 16 whole rows,
// written to shared memory as [row group][chunk][8 rows][128 B] (128B
// swizzle).  Only whole groups of valid rows lie inside the tensor: rows of a
// last partial group must come through the 3-D map instead.
bool make_pair_map(CUtensorMap *map, const void *base, const vsa_shape *s) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || s->d != 128 || s->n_valid < 8) return false;
  cuuint64_t dims[5] = {64, 8, 2, (cuuint64_t)(s->n_valid / 8), (cuuint64_t)s->B * s->H};
  cuuint64_t strides[4] = {(cuuint64_t)s->d * 2, 128, (cuuint64_t)8 * s->d * 2, (cuuint64_t)s->n_pad * s->d * 2};
  cuuint32_t box[5] = {64, 8, 2, 2, 1};
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void *>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// [BH][rows][d] bf16, all rows inside the tensor.
bool make_map_rows(CUtensorMap *map, const void *base, int rows, int d, int BH, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)rows, (cuuint64_t)BH};
  cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)rows * d * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int D>
vsa_status set_attn_smem() {
  using L = vsa::AttnSmem<D>;
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [] {
    attr_err = cudaFuncSetAttribute(vsa::attn_fwd_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc);
  });
  return attr_err == cudaSuccess ? VSA_OK : VSA_ERR_CUDA;
}

// Cluster-group mode: Q rows of the group layout ([BH][n_rows_q][d]), K/V in the
// key cluster permutation ([BH][n_pad][d], 16-row boxes).
template <int D>
vsa_status launch_attn_groups(const void *q, const void *k, const void *v, const vsa_shape *s, const AttnArgs &a,
                              cudaStream_t st) {
  using L = vsa::AttnSmem<D>;
  if (set_attn_smem<D>() != VSA_OK) return VSA_ERR_CUDA;
  const int BH = s->B * s->H;
  CUtensorMap mq, mk, mv;
  vsa::GroupMaps xm;
  if (!make_map_rows(&mq, q, a.n_rows_q, D, BH, vsa::kTileM) || !make_map(&mk, k, s, 16) || !make_map(&mv, v, s, 16) ||
      !make_map(&xm.k[0], k, s, 32) || !make_map(&xm.k[1], k, s, 64) || !make_map(&xm.v[0], v, s, 32) ||
      !make_map(&xm.v[1], v, s, 64))
    return VSA_ERR_CUDA;
  dim3 grid(a.n_tiles, BH);
  vsa::attn_fwd_kernel<D><<<grid, vsa::kSingleThreads, L::kAlloc, st>>>(mq, mk, mv, xm, a);
  return launch_status();
}

// Pooled-rectification pass: Q tiles of the layer, keys = the n_rows pooled rows
// ([BH][n_rows][d], the first n_k holding block means), 128-row boxes.
template <int D>
vsa_status launch_attn_pooled(const void *q, const void *kb, const void *vb, const vsa_shape *s, int n_rows,
                              const AttnArgs &a, int n_heads, cudaStream_t st) {
  using L = vsa::AttnSmem<D>;
  if (set_attn_smem<D>() != VSA_OK) return VSA_ERR_CUDA;
  const int BH = s->B * s->H;
  CUtensorMap mq, mk, mv;
  vsa::GroupMaps xm;
  if (!make_map(&mq, q, s, vsa::kTileM) || !make_map_rows(&mk, kb, n_rows, D, BH, vsa::kStageKeys) ||
      !make_map_rows(&mv, vb, n_rows, D, BH, vsa::kStageKeys))
    return VSA_ERR_CUDA;
  xm.k[0] = xm.k[1] = mk;
  xm.v[0] = xm.v[1] = mv;
  dim3 grid(s->n_pad / vsa::kTileM, n_heads);
  vsa::attn_fwd_kernel<D><<<grid, vsa::kSingleThreads, L::kAlloc, st>>>(mq, mk, mv, xm, a);
  return launch_status();
}

template <int D>
vsa_status launch_attn(const void *q, const void *k, const void *v, const vsa_shape *s, const AttnArgs &a,
                       int n_heads, cudaStream_t st) {
  using L = vsa::AttnSmem<D>;
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [] {
    attr_err = cudaFuncSetAttribute(vsa::attn_fwd_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc);
  });
  if (attr_err != cudaSuccess) return VSA_ERR_CUDA;
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, q, s, vsa::kTileM) || !make_map(&mk, k, s, a.seg_keys) || !make_map(&mv, v, s, a.seg_keys))
    return VSA_ERR_CUDA;
  dim3 grid(s->n_pad / vsa::kTileM, n_heads);
  vsa::GroupMaps xm;  // cluster-group mode's taller boxes, or the pair boxes of 16-key segments
  xm.k[0] = xm.k[1] = mk;
  xm.v[0] = xm.v[1] = mv;
  AttnArgs ap = a;
  ap.pair_boxes = 0;
  if (D == 128 && a.seg_keys == 16 && s->n_valid >= 8) {
    if (!make_pair_map(&xm.k[0], k, s) || !make_pair_map(&xm.v[0], v, s) || !make_map(&xm.k[1], k, s, 8) ||
        !make_map(&xm.v[1], v, s, 8))
      return VSA_ERR_CUDA;
    ap.pair_boxes = 1;
    ap.n_valid8 = s->n_valid / 8 * 8;
  }
  vsa::attn_fwd_kernel<D><<<grid, vsa::kSingleThreads, L::kAlloc, st>>>(mq, mk, mv, xm, ap);
  return launch_status();
}

// 128-row lists of 128-key blocks: two adjacent query tiles per CTA share
// their K/V loads (attn_fwd_dual_kernel).
template <int D, bool kHalf>
vsa_status launch_attn_dual(const void *q, const void *k, const void *v, const vsa_shape *s, const AttnArgs &a,
                            int n_heads, cudaStream_t st) {
  using L = vsa::DualSmem<D, kHalf>;
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [] {
    attr_err =
        cudaFuncSetAttribute(vsa::attn_fwd_dual_kernel<D, kHalf>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc);
  });
  if (attr_err != cudaSuccess) return VSA_ERR_CUDA;
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, q, s, vsa::kTileM) || !make_map(&mk, k, s, vsa::kStageKeys) || !make_map(&mv, v, s, vsa::kStageKeys))
    return VSA_ERR_CUDA;
  const int n_tiles = s->n_pad / vsa::kTileM;
  dim3 grid((n_tiles + 1) / 2, n_heads);
  vsa::attn_fwd_dual_kernel<D, kHalf><<<grid, vsa::kAttnThreads, L::kAlloc, st>>>(mq, mk, mv, a);
  return launch_status();
}

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

struct MicroLayout {
  int n_slots, bitmap_words;
  size_t off_slot, off_bitmap, off_keys, off_hist, off_state, total;
};

MicroLayout micro_layout(const vsa_shape *s, const vsa_micro_params *p) {
  MicroLayout L;
  int enabled = 0;
  for (int h = 0; h < s->H; ++h) enabled += (p->head_enable == nullptr || p->head_enable[h]) ? 1 : 0;
  L.n_slots = enabled * s->B;
  const size_t n_r = (size_t)s->n_pad / vsa::kMicroRows, n_t = (size_t)s->n_pad / vsa::kMicroKeys;
  const size_t n_qmax = (size_t)s->n_pad / 64;
  L.bitmap_words = std::max(32, (s->n_pad / 64 + 31) / 32);  // words of the longest kept-block bitmap (64-key blocks)
  size_t off = 0;
  L.off_slot = off;  // slot of each (batch, head), then (batch, head) of each slot
  off = align256(off + (size_t)s->B * s->H * 4 * 2);
  L.off_bitmap = off;
  off = align256(off + (size_t)L.n_slots * n_qmax * L.bitmap_words * 4);
  L.off_keys = off;
  off = align256(off + (size_t)L.n_slots * n_r * n_t * 4);
  L.off_hist = off;
  off = align256(off + (size_t)L.n_slots * 3 * vsa::kHistBins * 4);
  L.off_state = off;
  off = align256(off + (size_t)L.n_slots * 8 * 4);
  L.total = off;
  return L;
}

bool micro_params_ok(const vsa_micro_params *p) {
  if (!p) return false;
  if (p->mode == 1) return p->topk >= 1 && p->topk <= 32 && p->row_capacity >= 1;
  if (p->mode == 2) return p->percentile > 0.0 && p->percentile < 1.0 && p->row_capacity >= 1;
  return false;
}

int ilog2(int x) {
  int r = 0;
  while ((1 << r) < x) ++r;
  return r;
}

// Fixed scratch of vsa_select_micro_noalloc: reserved in every GPU that loads
// this library, for the life of the process.  In host code its name is only a
// host-side stand-in; the device address comes from cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_micro_noalloc_scratch[VSA_MICRO_NOALLOC_MAX_BYTES];

constexpr int kMicroMaxHeads = 1024;

// Device address of the fixed scratch on the current device.  Looked up on
// every call (a cheap query once the module is loaded), so the address stays
// right even after the primary context was reset and the module reloaded.
vsa_status noalloc_scratch(void **out) {
  void *p = nullptr;
  if (cudaGetSymbolAddress(&p, g_micro_noalloc_scratch) != cudaSuccess || p == nullptr) return VSA_ERR_CUDA;
  *out = p;
  return VSA_OK;
}

// One thread waits on a barrier that no one arrives at; the bounded wait gives
// up after limit_ns and latches VSA_ERR_TIMEOUT.
__global__ void selftest_wait_kernel(unsigned long long limit_ns, int *status) {
  __shared__ uint64_t bar;
  __shared__ vsa::AbortCtl abort_ctl;
  if (threadIdx.x != 0) return;
  vsa::abort_init(&abort_ctl, status);
  vsa::mbar_init(&bar, 1);
  vsa::fence_barrier_init();
  vsa::mbar_wait(&bar, 0, &abort_ctl, limit_ns);
}

// The softmax's FMA-pipe exponential on a caller's array, two values per thread.
__global__ void selftest_exp2_kernel(const float *__restrict__ x, float *__restrict__ y, int n) {
  const long long i = 2ll * ((long long)blockIdx.x * blockDim.x + threadIdx.x);
  if (i >= n) return;
  const float2 in = make_float2(x[i], i + 1 < n ? x[i + 1] : 0.f);
  const float2 out = vsa::exp2_poly2(in);
  y[i] = out.x;
  if (i + 1 < n) y[i + 1] = out.y;
}

// Per-head slot numbers handed to the device by value (no host-to-device copy
// and no host buffer that must outlive the call).
struct HeadSlots {
  int16_t slot[kMicroMaxHeads];  // rank among enabled heads, or -1
  int n_enabled;
  int H, BH;
};

__global__ void micro_slot_fill_kernel(HeadSlots hs, int32_t *slot_of_bh, int32_t *bh_of_slot) {
  const int bh = blockIdx.x * blockDim.x + threadIdx.x;
  if (bh >= hs.BH) return;
  const int b = bh / hs.H, h = bh % hs.H;
  const int r = hs.slot[h];
  const int slot = r < 0 ? -1 : b * hs.n_enabled + r;
  slot_of_bh[bh] = slot;
  if (slot >= 0) bh_of_slot[slot] = bh;
}

// Host-side checks shared by vsa_select_micro and vsa_select_micro_noalloc.
vsa_status check_micro_args(const float *q_pool64, const float *k_pool16, const int32_t *counts, const int32_t *idx,
                            const vsa_shape *shape, int bq, int bk, float scale, const vsa_micro_params *params,
                            const int32_t *m_counts, const int32_t *m_idx) {
  if (!shape_ok(shape) || !q_pool64 || !k_pool16 || !counts || !idx || !m_counts || !m_idx)
    return VSA_ERR_INVALID_ARG;
  if (!micro_params_ok(params)) return VSA_ERR_INVALID_ARG;
  if ((bq != 64 && bq != 128) || (bk != 64 && bk != 128)) return VSA_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !std::isfinite(scale)) return VSA_ERR_INVALID_ARG;
  if (!aligned16(q_pool64) || !aligned16(k_pool16)) return VSA_ERR_INVALID_ARG;
  if (shape->n_pad / 64 > vsa::kMicroMaxKeyBlocks) return VSA_ERR_UNSUPPORTED;
  if (shape->H > kMicroMaxHeads) return VSA_ERR_UNSUPPORTED;
  return VSA_OK;
}

// The Micro selection launch sequence on a scratch area laid out by L
// (caller workspace or the fixed array): slot table, then the kernels.
vsa_status launch_micro_select(const float *q_pool64, const float *k_pool16, const int32_t *counts,
                               const int32_t *idx, const vsa_shape *shape, int bq, int bk, float scale,
                               const vsa_micro_params *params, int32_t *m_counts, int32_t *m_idx, uint8_t *ws8,
                               const MicroLayout &L, cudaStream_t st) {
  const int n_q = shape->n_pad / bq, n_k = shape->n_pad / bk;
  const int BH = shape->B * shape->H;
  const int n_r = shape->n_pad / vsa::kMicroRows, n_t = shape->n_pad / vsa::kMicroKeys;
  vsa::MicroWs ws;
  ws.slot_of_bh = reinterpret_cast<int32_t *>(ws8 + L.off_slot);
  ws.bh_of_slot = ws.slot_of_bh + BH;
  ws.bitmap = reinterpret_cast<uint32_t *>(ws8 + L.off_bitmap);
  ws.keys = reinterpret_cast<uint32_t *>(ws8 + L.off_keys);
  ws.hist = reinterpret_cast<uint32_t *>(ws8 + L.off_hist);
  ws.state = reinterpret_cast<uint32_t *>(ws8 + L.off_state);
  ws.n_slots = L.n_slots;
  ws.bitmap_words = L.bitmap_words;
  ws.status = status_word(st);
  if (!ws.status) return VSA_ERR_CUDA;

  HeadSlots hs;
  int next = 0;
  for (int h = 0; h < shape->H; ++h)
    hs.slot[h] = (params->head_enable == nullptr || params->head_enable[h]) ? (int16_t)next++ : (int16_t)-1;
  hs.n_enabled = next;
  hs.H = shape->H;
  hs.BH = BH;
  micro_slot_fill_kernel<<<(BH + 255) / 256, 256, 0, st>>>(hs, ws.slot_of_bh, ws.bh_of_slot);
  // rows of the heads without the repair select nothing; the kernels below
  // run on the enabled heads' slots only
  if (cudaMemsetAsync(m_counts, 0, (size_t)BH * n_r * 4, st) != cudaSuccess) return VSA_ERR_CUDA;
  if (L.n_slots == 0) return launch_status();
  // histograms and rank-search state must start at zero on every call
  if (cudaMemsetAsync(ws8 + L.off_hist, 0, L.total - L.off_hist, st) != cudaSuccess) return VSA_ERR_CUDA;

  vsa::micro_bitmap_kernel<<<dim3(n_q, L.n_slots), 128, 0, st>>>(counts, idx, n_q, n_k, BH, ws);
  vsa::ScoreArgs sa{q_pool64, k_pool16, n_r, n_t, n_q, bq, bk, shape->n_valid, scale, params->mode == 2 ? 1 : 0};
  dim3 sg((n_t + vsa::kScoreBN - 1) / vsa::kScoreBN, (n_r + vsa::kScoreBM - 1) / vsa::kScoreBM, L.n_slots);
  if (shape->d == 128)
    vsa::micro_score_kernel<128><<<sg, vsa::kScoreThreads, 0, st>>>(sa, ws);
  else
    vsa::micro_score_kernel<64><<<sg, vsa::kScoreThreads, 0, st>>>(sa, ws);
  const unsigned rows_blocks = (unsigned)(((size_t)L.n_slots * n_r + 7) / 8);
  if (params->mode == 1) {
    vsa::micro_topk_kernel<<<rows_blocks, 256, 0, st>>>(ws, n_r, n_t, BH, params->topk, params->row_capacity,
                                                      m_counts, m_idx);
  } else {
    const size_t per_slot = (size_t)n_r * n_t;
    vsa::micro_find_kernel<<<L.n_slots, 32, 0, st>>>(ws, params->percentile, 0);
    vsa::micro_hist_kernel<<<dim3(256, L.n_slots), 256, 0, st>>>(ws, per_slot, 1);
    vsa::micro_find_kernel<<<L.n_slots, 32, 0, st>>>(ws, params->percentile, 1);
    vsa::micro_hist_kernel<<<dim3(256, L.n_slots), 256, 0, st>>>(ws, per_slot, 2);
    vsa::micro_find_kernel<<<L.n_slots, 32, 0, st>>>(ws, params->percentile, 2);
    vsa::micro_compact_kernel<<<rows_blocks, 256, 0, st>>>(ws, n_r, n_t, BH, params->row_capacity, m_counts, m_idx);
  }
  return launch_status();
}

// ---- clustering --------------------------------------------------------------

// Geometry of valid clustering parameters, or false.
bool cluster_geom(const vsa_cluster_params *p, vsa::ClusterGeom *g) {
  if (!p) return false;
  const int v[10] = {p->lattice_t, p->lattice_h, p->lattice_w, p->cell_t, p->cell_h, p->cell_w,
                     p->win_t,     p->win_h,     p->win_w,     p->iters};
  for (int i = 0; i < 10; ++i)
    if (v[i] < 1) return false;
  if (p->iters > 64) return false;
  if ((long long)p->cell_t * p->cell_h * p->cell_w > vsa::kClusterMaxTokens) return false;
  if ((long long)p->win_t * p->win_h * p->win_w > vsa::kClusterMaxWindow) return false;
  const long long n = (long long)p->lattice_t * p->lattice_h * p->lattice_w;
  if (n > (1ll << 30)) return false;
  g->T = p->lattice_t;
  g->H = p->lattice_h;
  g->W = p->lattice_w;
  g->kt = p->cell_t;
  g->kh = p->cell_h;
  g->kw = p->cell_w;
  g->CT = (g->T + g->kt - 1) / g->kt;
  g->CH = (g->H + g->kh - 1) / g->kh;
  g->CW = (g->W + g->kw - 1) / g->kw;
  g->wt = p->win_t;
  g->wh = p->win_h;
  g->ww = p->win_w;
  const long long cells = (long long)g->CT * g->CH * g->CW;
  if (cells > (1ll << 24)) return false;  // cell indices travel in 24 bits inside the assignment kernel
  g->n_cells = (int)cells;
  g->n_valid = (int)n;
  g->n_pad = 0;
  return true;
}

// Tokens of the largest reverse-window box (the member-list capacity).
int cluster_box_tokens(const vsa::ClusterGeom &g) {
  const long long t = std::min((long long)g.wt * g.kt, (long long)g.T);
  const long long h = std::min((long long)g.wh * g.kh, (long long)g.H);
  const long long w = std::min((long long)g.ww * g.kw, (long long)g.W);
  return (int)(t * h * w);
}

// The assignment kernel for windows of up to 16 * NB cells; its shared
// memory is set once per instantiation.
template <int D, int NB>
vsa_status launch_assign(const __nv_bfloat16 *x, const vsa::ClusterGeom &g, dim3 grid, const float *mu,
                         int32_t *assign, float *ratio, cudaStream_t st) {
  static const int bytes = vsa::AssignLayout<D>::bytes(16 * NB);
  static const cudaError_t attr =
      cudaFuncSetAttribute(vsa::cluster_assign_kernel<D, NB, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  static const cudaError_t attr_r =
      cudaFuncSetAttribute(vsa::cluster_assign_kernel<D, NB, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (attr != cudaSuccess || attr_r != cudaSuccess) return VSA_ERR_CUDA;
  if (ratio)
    vsa::cluster_assign_kernel<D, NB, true><<<grid, vsa::kClusterThreads, bytes, st>>>(x, g, mu, assign, ratio);
  else
    vsa::cluster_assign_kernel<D, NB, false><<<grid, vsa::kClusterThreads, bytes, st>>>(x, g, mu, assign, nullptr);
  return VSA_OK;
}

template <int D>
vsa_status launch_assign_any(const __nv_bfloat16 *x, const vsa::ClusterGeom &g, dim3 grid, const float *mu,
                             int32_t *assign, float *ratio, cudaStream_t st) {
  switch ((g.wt * g.wh * g.ww + 15) / 16) {
    case 1: return launch_assign<D, 1>(x, g, grid, mu, assign, ratio, st);
    case 2: return launch_assign<D, 2>(x, g, grid, mu, assign, ratio, st);
    case 3: return launch_assign<D, 3>(x, g, grid, mu, assign, ratio, st);
    case 4: return launch_assign<D, 4>(x, g, grid, mu, assign, ratio, st);
    case 5: return launch_assign<D, 5>(x, g, grid, mu, assign, ratio, st);
    case 6: return launch_assign<D, 6>(x, g, grid, mu, assign, ratio, st);
    case 7: return launch_assign<D, 7>(x, g, grid, mu, assign, ratio, st);
    default: return launch_assign<D, 8>(x, g, grid, mu, assign, ratio, st);
  }
}

template <int D>
vsa_status launch_cluster(const __nv_bfloat16 *x, const vsa::ClusterGeom &g, int iters, int BH, int32_t *assign,
                          float *mu, int32_t *sizes, int32_t *perm, float *ratio, cudaStream_t st) {
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  constexpr int kListMax = 128 + 4 * vsa::kClusterMaxTokens * vsa::kClusterMaxWindow;
  std::call_once(once, [] {
    attr_err = cudaFuncSetAttribute(vsa::cluster_update_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    kListMax);
    if (attr_err == cudaSuccess)
      attr_err = cudaFuncSetAttribute(vsa::cluster_perm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kListMax);
  });
  if (attr_err != cudaSuccess) return VSA_ERR_CUDA;
  const int list_smem = 128 + 4 * cluster_box_tokens(g);
  const dim3 grid(g.n_cells, BH);
  vsa::cluster_init_kernel<D><<<grid, 128, 0, st>>>(x, g, mu);
  for (int it = 0; it < iters; ++it) {
    // the last round's assignment also yields Lowe's ratio when asked
    const vsa_status as = launch_assign_any<D>(x, g, grid, mu, assign, it == iters - 1 ? ratio : nullptr, st);
    if (as != VSA_OK) return as;
    vsa::cluster_update_kernel<D><<<grid, vsa::kClusterThreads, list_smem, st>>>(x, g, assign, mu, sizes);
  }
  vsa::cluster_perm_kernel<<<grid, vsa::kClusterThreads, list_smem, st>>>(g, assign, sizes, perm);
  return launch_status();
}

bool select_params_ok(float scale, const vsa_select_params *params) {
  if (!(scale > 0.f) || !std::isfinite(scale)) return false;
  return params->k_min >= 0 && params->fixed_k >= 0 && params->n_anchor >= 0 && params->anchor_rot >= 0 &&
         std::isfinite(params->cum_mass);
}

// Selection over n_q query units x n_k key units (blocks, or clusters with
// explicit sizes), one CTA per 16 query units of one (batch, head).
vsa_status launch_select(const vsa::SelectArgs &a, int d, int BH, bool by_rank, cudaStream_t st) {
  const int n_q = a.n_q, n_k = a.n_k;
  if (n_k > 1024) {
    // rows too long for one warp: one CTA per row
    const dim3 grid(n_q, BH);
    if (d == 128)
      vsa::select_long_kernel<128><<<grid, vsa::kLongThreads, 0, st>>>(a);
    else
      vsa::select_long_kernel<64><<<grid, vsa::kLongThreads, 0, st>>>(a);
    return launch_status();
  }
  int nkp = 32;
  while (nkp < n_k) nkp <<= 1;
  const size_t smem = vsa::select_smem_bytes(d, nkp);
  dim3 grid((n_q + vsa::kSelRows - 1) / vsa::kSelRows, BH);
#define VSA_SEL_CASE(DD, NR)                                                                                  \
  {                                                                                                           \
    auto kern = by_rank ? vsa::select_blocks_kernel<DD, NR, true> : vsa::select_blocks_kernel<DD, NR, false>; \
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess) \
      return VSA_ERR_CUDA;                                                                                    \
    kern<<<grid, vsa::kSelThreads, smem, st>>>(a);                                                            \
  }
#define VSA_SEL_NR(DD)                     \
  switch (nkp / 32) {                      \
    case 1: VSA_SEL_CASE(DD, 1) break;     \
    case 2: VSA_SEL_CASE(DD, 2) break;     \
    case 4: VSA_SEL_CASE(DD, 4) break;     \
    case 8: VSA_SEL_CASE(DD, 8) break;     \
    case 16: VSA_SEL_CASE(DD, 16) break;   \
    default: VSA_SEL_CASE(DD, 32) break;   \
  }
  if (d == 128) {
    VSA_SEL_NR(128)
  } else {
    VSA_SEL_NR(64)
  }
#undef VSA_SEL_NR
#undef VSA_SEL_CASE
  return launch_status();
}

// Workspace of the cluster merging, carved from one caller buffer (256-byte
// aligned arrays).  Returns the bytes needed; fills *ws when base is non-null.
size_t merge_ws_layout(int BH, int nq, void *base, vsa::MergeWs *ws) {
  size_t off = 0;
  auto take = [&](size_t bytes) -> void * {
    void *p = base ? static_cast<char *>(base) + off : nullptr;
    off += align256(bytes);
    return p;
  };
  const size_t n = (size_t)BH * nq;
  vsa::MergeWs w;
  w.lead = static_cast<int32_t *>(take(n * 4));
  w.gsq = static_cast<int32_t *>(take(n * 4));
  w.gwk = static_cast<int32_t *>(take(n * 4));
  w.chi = static_cast<uint32_t *>(take(n * vsa::kMergeWords * 4));
  w.list = static_cast<int32_t *>(take(2 * n * 4));
  w.nlist = static_cast<int32_t *>(take((size_t)BH * 2 * 4));
  w.best = static_cast<unsigned long long *>(take(n * 8));
  w.passes = static_cast<int32_t *>(take((size_t)BH * 4));
  if (ws) *ws = w;
  return off;
}

}  // namespace

extern "C" {

const char *vsa_status_string(vsa_status s) {
  switch (s) {
    case VSA_OK: return "ok";
    case VSA_ERR_INVALID_ARG: return "invalid argument";
    case VSA_ERR_UNSUPPORTED: return "unsupported configuration";
    case VSA_ERR_CUDA: return "CUDA error";
    case VSA_ERR_CAPACITY: return "list capacity exceeded";
    case VSA_ERR_BAD_INDEX: return "invalid index in a list";
    case VSA_ERR_TIMEOUT: return "pipeline wait timed out";
    case VSA_ERR_SCRATCH_LIMIT: return "problem needs more scratch than the allocation-free entry point holds";
  }
  return "unknown status";
}

int vsa_version(void) { return 200; }

vsa_status vsa_read_device_status(void *stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int *word = status_word(st);
  if (!word) return VSA_ERR_CUDA;
  int h[2] = {0, 0};
  if (cudaStreamSynchronize(st) != cudaSuccess) return VSA_ERR_CUDA;
  if (cudaMemcpyAsync(h, word, sizeof(h), cudaMemcpyDeviceToHost, st) != cudaSuccess ||
      cudaMemsetAsync(word, 0, sizeof(h), st) != cudaSuccess || cudaStreamSynchronize(st) != cudaSuccess)
    return VSA_ERR_CUDA;
  return static_cast<vsa_status>(h[0]);
}

vsa_status vsa_bind_status_word(void *stream, int32_t *word) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (word && (reinterpret_cast<uintptr_t>(word) & 3u) != 0) return VSA_ERR_INVALID_ARG;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return VSA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(binding_mutex());
  std::vector<StatusBinding> &b = bindings();
  for (size_t i = 0; i < b.size(); ++i) {
    if (b[i].stream == st && b[i].device == dev) {
      b.erase(b.begin() + static_cast<long>(i));
      break;
    }
  }
  if (!word) return VSA_OK;
  if (b.size() >= (size_t)kMaxStatusBindings) return VSA_ERR_CAPACITY;
  if (cudaMemsetAsync(word, 0, VSA_STATUS_WORD_BYTES, st) != cudaSuccess) return VSA_ERR_CUDA;
  b.push_back({st, dev, word});
  return VSA_OK;
}

vsa_status vsa_selftest_wait_timeout(unsigned long long limit_ns, void *stream) {
  if (limit_ns < 1000ull || limit_ns > 5000000000ull) return VSA_ERR_INVALID_ARG;
  int *word = status_word(static_cast<cudaStream_t>(stream));
  if (!word) return VSA_ERR_CUDA;
  selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(limit_ns, word);
  return launch_status();
}

vsa_status vsa_selftest_exp2(const float *x, float *y, int n, void *stream) {
  if (n < 0 || (n > 0 && (!x || !y))) return VSA_ERR_INVALID_ARG;
  if (n == 0) return VSA_OK;
  const int threads = 256;
  const int blocks = (n / 2 + 1 + threads - 1) / threads;
  selftest_exp2_kernel<<<blocks, threads, 0, static_cast<cudaStream_t>(stream)>>>(x, y, n);
  return launch_status();
}

vsa_status vsa_pool_qk(const void *q, const void *k, const vsa_shape *shape, int bq, int bk, float *q_pool,
                       float *k_pool, float *q_pool64, float *k_pool16, void *stream) {
  if (!shape_ok(shape) || !q || !k || !q_pool || !k_pool) return VSA_ERR_INVALID_ARG;
  if ((bq != 64 && bq != 128) || (bk != 64 && bk != 128)) return VSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(q_pool) || !aligned16(k_pool)) return VSA_ERR_INVALID_ARG;
  vsa::PoolOut oq{q_pool, bq, q_pool64, 64};
  vsa::PoolOut ok{k_pool, bk, k_pool16, 16};
  dim3 grid(shape->n_pad / vsa::kPoolRows, shape->B * shape->H, 2);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const auto *qb = static_cast<const __nv_bfloat16 *>(q);
  const auto *kb = static_cast<const __nv_bfloat16 *>(k);
  if (shape->d == 128)
    vsa::pool_kernel<128><<<grid, vsa::kPoolThreads, 0, st>>>(qb, kb, shape->n_pad, shape->n_valid, oq, ok);
  else
    vsa::pool_kernel<64><<<grid, vsa::kPoolThreads, 0, st>>>(qb, kb, shape->n_pad, shape->n_valid, oq, ok);
  return launch_status();
}

vsa_status vsa_select_blocks(const float *q_pool, const float *k_pool, const vsa_shape *shape, int bq, int bk,
                             float scale, const vsa_select_params *params, int32_t *counts, int32_t *idx,
                             uint8_t *mask, void *stream) {
  if (!shape_ok(shape) || !q_pool || !k_pool || !params || !counts || !idx) return VSA_ERR_INVALID_ARG;
  if ((bq != 64 && bq != 128) || (bk != 64 && bk != 128)) return VSA_ERR_INVALID_ARG;
  if (!aligned16(q_pool) || !aligned16(k_pool)) return VSA_ERR_INVALID_ARG;
  if (!select_params_ok(scale, params)) return VSA_ERR_INVALID_ARG;
  const int n_q = shape->n_pad / bq, n_k = shape->n_pad / bk;
  if (n_k > vsa::kSelLongMax) return VSA_ERR_UNSUPPORTED;
  vsa::SelectArgs a{q_pool, k_pool, n_q, n_k, bq, bk, shape->n_valid, scale, params->k_min, params->fixed_k,
                    params->n_anchor, params->anchor_rot, params->cum_mass, counts, idx, mask, nullptr, nullptr};
  return launch_select(a, shape->d, shape->B * shape->H, params->fixed_k > 0, static_cast<cudaStream_t>(stream));
}

vsa_status vsa_select_clusters(const float *mu_q, const float *mu_k, const int32_t *sizes_q, const int32_t *sizes_k,
                               int batch_heads, int n_q, int n_k, int d, float scale,
                               const vsa_select_params *params, int32_t *counts, int32_t *idx, void *stream) {
  if (!mu_q || !mu_k || !sizes_q || !sizes_k || !params || !counts || !idx) return VSA_ERR_INVALID_ARG;
  if (batch_heads < 1 || batch_heads > 65535 || n_q < 1 || n_k < 1 || (d != 64 && d != 128)) return VSA_ERR_INVALID_ARG;
  if (!aligned16(mu_q) || !aligned16(mu_k)) return VSA_ERR_INVALID_ARG;
  if (!select_params_ok(scale, params) || params->n_anchor != 0) return VSA_ERR_INVALID_ARG;
  if (n_k > vsa::kSelLongMax) return VSA_ERR_UNSUPPORTED;
  vsa::SelectArgs a{mu_q, mu_k, n_q, n_k, 1, 1, 0, scale, params->k_min, params->fixed_k,
                    0, 0, params->cum_mass, counts, idx, nullptr, sizes_q, sizes_k};
  return launch_select(a, d, batch_heads, params->fixed_k > 0, static_cast<cudaStream_t>(stream));
}

vsa_status vsa_mask_to_lists(const uint8_t *mask, const vsa_shape *shape, int bq, int bk, int32_t *counts,
                             int32_t *idx, void *stream) {
  if (!shape_ok(shape) || !mask || !counts || !idx) return VSA_ERR_INVALID_ARG;
  if ((bq != 64 && bq != 128) || (bk != 64 && bk != 128)) return VSA_ERR_INVALID_ARG;
  const int n_q = shape->n_pad / bq, n_k = shape->n_pad / bk;
  const int rows = shape->B * shape->H * n_q;
  vsa::mask_to_lists_kernel<<<(rows + 7) / 8, 256, 0, static_cast<cudaStream_t>(stream)>>>(mask, rows, n_k, counts,
                                                                                          idx);
  return launch_status();
}

size_t vsa_select_micro_workspace_bytes(const vsa_shape *shape, const vsa_micro_params *params) {
  if (!shape_ok(shape) || !micro_params_ok(params)) return 0;
  return micro_layout(shape, params).total;
}

vsa_status vsa_select_micro(const float *q_pool64, const float *k_pool16, const int32_t *counts, const int32_t *idx,
                            const vsa_shape *shape, int bq, int bk, float scale, const vsa_micro_params *params,
                            int32_t *m_counts, int32_t *m_idx, void *workspace, size_t workspace_bytes,
                            void *stream) {
  const vsa_status ae =
      check_micro_args(q_pool64, k_pool16, counts, idx, shape, bq, bk, scale, params, m_counts, m_idx);
  if (ae != VSA_OK) return ae;
  if (!workspace || !aligned16(workspace)) return VSA_ERR_INVALID_ARG;
  const MicroLayout L = micro_layout(shape, params);
  if (workspace_bytes < L.total) return VSA_ERR_INVALID_ARG;
  return launch_micro_select(q_pool64, k_pool16, counts, idx, shape, bq, bk, scale, params, m_counts, m_idx,
                             static_cast<uint8_t *>(workspace), L, static_cast<cudaStream_t>(stream));
}

vsa_status vsa_select_micro_noalloc(const float *q_pool64, const float *k_pool16, const int32_t *counts,
                                    const int32_t *idx, const vsa_shape *shape, int bq, int bk, float scale,
                                    const vsa_micro_params *params, int32_t *m_counts, int32_t *m_idx,
                                    void *stream) {
  const vsa_status ae =
      check_micro_args(q_pool64, k_pool16, counts, idx, shape, bq, bk, scale, params, m_counts, m_idx);
  if (ae != VSA_OK) return ae;
  if ((long long)shape->B * shape->H > kMicroMaxHeads) return VSA_ERR_SCRATCH_LIMIT;
  const MicroLayout L = micro_layout(shape, params);
  if (L.total > VSA_MICRO_NOALLOC_MAX_BYTES) return VSA_ERR_SCRATCH_LIMIT;
  void *scratch = nullptr;
  const vsa_status se = noalloc_scratch(&scratch);
  if (se != VSA_OK) return se;
  return launch_micro_select(q_pool64, k_pool16, counts, idx, shape, bq, bk, scale, params, m_counts, m_idx,
                             static_cast<uint8_t *>(scratch), L, static_cast<cudaStream_t>(stream));
}

vsa_status vsa_block_sparse_fwd(const void *q, const void *k, const void *v, const vsa_shape *shape, int list_rows,
                                int seg_keys, const int32_t *counts, const int32_t *idx, int idx_stride, float scale,
                                void *o, int o_fp32, float *lse, const float *merge_o, const float *merge_lse,
                                void *stream) {
  if (!shape_ok(shape)) return VSA_ERR_INVALID_ARG;
  return vsa_block_sparse_fwd_heads(q, k, v, shape, list_rows, seg_keys, counts, idx, idx_stride, scale, o, o_fp32,
                                    lse, merge_o, merge_lse, nullptr, shape->B * shape->H, stream);
}

vsa_status vsa_block_sparse_fwd_heads(const void *q, const void *k, const void *v, const vsa_shape *shape,
                                      int list_rows, int seg_keys, const int32_t *counts, const int32_t *idx,
                                      int idx_stride, float scale, void *o, int o_fp32, float *lse,
                                      const float *merge_o, const float *merge_lse, const int32_t *heads, int n_heads,
                                      void *stream) {
  if (!shape_ok(shape) || !q || !k || !v || !counts || !idx || !o || !lse) return VSA_ERR_INVALID_ARG;
  const long long n_bh = (long long)shape->B * shape->H;
  if (n_heads < 0 || n_heads > n_bh || n_heads > 65535 || (heads == nullptr && n_heads != n_bh))
    return VSA_ERR_INVALID_ARG;
  if (list_rows != 64 && list_rows != 128) return VSA_ERR_INVALID_ARG;
  if (seg_keys != 16 && seg_keys != 32 && seg_keys != 64 && seg_keys != 128) return VSA_ERR_INVALID_ARG;
  if (idx_stride < 1 || !(scale > 0.f) || !std::isfinite(scale)) return VSA_ERR_INVALID_ARG;
  if ((merge_o == nullptr) != (merge_lse == nullptr)) return VSA_ERR_INVALID_ARG;
  if (merge_o && static_cast<const void *>(merge_o) == o) return VSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || (merge_o && !aligned16(merge_o)))
    return VSA_ERR_INVALID_ARG;
  AttnArgs a{};
  a.n_pad = shape->n_pad;
  a.n_valid = shape->n_valid;
  a.list_rows = list_rows;
  a.seg_keys = seg_keys;
  a.seg_shift = ilog2(seg_keys);
  a.idx_stride = idx_stride;
  a.counts = counts;
  a.idx = idx;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.o = o;
  a.o_fp32 = o_fp32 ? 1 : 0;
  a.lse = lse;
  a.merge_o = merge_o;
  a.merge_lse = merge_lse;
  a.heads = heads;
  a.n_bh = static_cast<int>(n_bh);
  a.timeout_ns = kWaitLimitNs;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (n_heads == 0) return VSA_OK;
  a.status = status_word(st);
  if (!a.status) return VSA_ERR_CUDA;
  if (list_rows == 128 && seg_keys == 128)
    return shape->d == 128 ? launch_attn_dual<128, false>(q, k, v, shape, a, n_heads, st)
                             : launch_attn_dual<64, false>(q, k, v, shape, a, n_heads, st);
  // 64-row lists of 128-key blocks: two query blocks per tile, two tiles per
  // CTA, when the tiles are whole and every list fits the staged union
  if (list_rows == 64 && seg_keys == 128 && shape->n_pad % vsa::kTileM == 0 &&
      shape->n_pad / vsa::kStageKeys <= vsa::kDualList)
    return shape->d == 128 ? launch_attn_dual<128, true>(q, k, v, shape, a, n_heads, st)
                             : launch_attn_dual<64, true>(q, k, v, shape, a, n_heads, st);
  return shape->d == 128 ? launch_attn<128>(q, k, v, shape, a, n_heads, st) : launch_attn<64>(q, k, v, shape, a, n_heads, st);
}

vsa_status vsa_lse_merge(const float *o_a, const float *lse_a, const float *o_b, const float *lse_b,
                         const vsa_shape *shape, void *o_out, int o_out_fp32, float *lse_out, void *stream) {
  if (!shape_ok(shape) || !o_a || !lse_a || !o_b || !lse_b || !o_out || !lse_out) return VSA_ERR_INVALID_ARG;
  if (!aligned16(o_a) || !aligned16(o_b) || !aligned16(o_out)) return VSA_ERR_INVALID_ARG;
  const size_t rows = (size_t)shape->B * shape->H * shape->n_pad;
  const unsigned blocks = (unsigned)((rows + 7) / 8);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (shape->d == 128)
    vsa::lse_merge_kernel<128><<<blocks, 256, 0, st>>>(o_a, lse_a, o_b, lse_b, rows, o_out, o_out_fp32, lse_out);
  else
    vsa::lse_merge_kernel<64><<<blocks, 256, 0, st>>>(o_a, lse_a, o_b, lse_b, rows, o_out, o_out_fp32, lse_out);
  return launch_status();
}


int vsa_cluster_count(const vsa_cluster_params *params) {
  vsa::ClusterGeom g;
  return cluster_geom(params, &g) ? g.n_cells : 0;
}

vsa_status vsa_cluster_tokens(const void *x, const vsa_shape *shape, const vsa_cluster_params *params,
                              int32_t *assign, float *centroids, int32_t *sizes, int32_t *perm, void *stream) {
  if (!shape_ok(shape) || !x || !assign || !centroids || !sizes || !perm) return VSA_ERR_INVALID_ARG;
  vsa::ClusterGeom g;
  if (!cluster_geom(params, &g) || g.n_valid != shape->n_valid) return VSA_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(centroids)) return VSA_ERR_INVALID_ARG;
  g.n_pad = shape->n_pad;
  const int BH = shape->B * shape->H;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const __nv_bfloat16 *xb = static_cast<const __nv_bfloat16 *>(x);
  return shape->d == 128 ? launch_cluster<128>(xb, g, params->iters, BH, assign, centroids, sizes, perm, nullptr, st)
                         : launch_cluster<64>(xb, g, params->iters, BH, assign, centroids, sizes, perm, nullptr, st);
}

vsa_status vsa_permute_rows(const void *src, const int32_t *perm, int batch_heads, int n_pad, int row_bytes,
                            int inverse, void *dst, void *stream) {
  if (!src || !perm || !dst || src == dst) return VSA_ERR_INVALID_ARG;
  if (batch_heads < 1 || n_pad < 1 || row_bytes < 4 || row_bytes % 4 != 0) return VSA_ERR_INVALID_ARG;
  const bool wide = row_bytes % 16 == 0;
  const uintptr_t mask = wide ? 15u : 3u;
  if ((reinterpret_cast<uintptr_t>(src) & mask) || (reinterpret_cast<uintptr_t>(dst) & mask) ||
      (reinterpret_cast<uintptr_t>(perm) & 3u))
    return VSA_ERR_INVALID_ARG;
  const long long rows = (long long)batch_heads * n_pad;
  const long long span = rows * row_bytes;
  const char *s8 = static_cast<const char *>(src);
  const char *d8 = static_cast<const char *>(dst);
  if (s8 < d8 + span && d8 < s8 + span) return VSA_ERR_INVALID_ARG;  // overlapping buffers
  const long long blocks = (rows + 7) / 8;
  if (blocks > 0x7fffffffll) return VSA_ERR_UNSUPPORTED;
  int *word = status_word(static_cast<cudaStream_t>(stream));
  if (!word) return VSA_ERR_CUDA;
  vsa::permute_rows_kernel<<<(unsigned)blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint32_t *>(src), perm, n_pad, rows, row_bytes / 4, inverse ? 1 : 0,
      static_cast<uint32_t *>(dst), word);
  return launch_status();
}

size_t vsa_merge_clusters_workspace_bytes(int batch_heads, int n_q) {
  if (batch_heads < 1 || n_q < 1) return 0;
  return merge_ws_layout(batch_heads, n_q, nullptr, nullptr);
}

vsa_status vsa_merge_clusters(const int32_t *sizes_q, const int32_t *sizes_k, const int32_t *counts,
                              const int32_t *idx, const uint8_t *sides, int batch_heads, int n_q, int n_k,
                              int rounds, int tau_q, int tau_k, void *workspace, size_t workspace_bytes,
                              int32_t *group_of, int32_t *g_counts, int32_t *g_idx, void *stream) {
  if (!sizes_q || !sizes_k || !counts || !idx || !workspace || !group_of || !g_counts || !g_idx)
    return VSA_ERR_INVALID_ARG;
  if (batch_heads < 1 || batch_heads > 65535 || n_q < 1 || n_k < 1 || rounds < 0 || rounds > 64)
    return VSA_ERR_INVALID_ARG;
  if (rounds > 0 && !sides) return VSA_ERR_INVALID_ARG;
  if (tau_q < 1 || tau_k < 1 || tau_q > (1 << 20) || tau_k > (1 << 20)) return VSA_ERR_INVALID_ARG;
  if (n_q > vsa::kMergeMaxClusters || n_k > vsa::kMergeMaxClusters) return VSA_ERR_UNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return VSA_ERR_INVALID_ARG;
  if (workspace_bytes < merge_ws_layout(batch_heads, n_q, nullptr, nullptr)) return VSA_ERR_INVALID_ARG;
  vsa::MergeArgs a{};
  a.sizes_q = sizes_q;
  a.sizes_k = sizes_k;
  a.counts = counts;
  a.idx = idx;
  a.sides = sides;
  a.nq = n_q;
  a.nk = n_k;
  a.rounds = rounds;
  a.tau_q = tau_q;
  a.tau_k = tau_k;
  a.inv_tau_q = 1.0f / (float)tau_q;
  a.inv_tau_k = 1.0f / (float)tau_k;
  a.group_of = group_of;
  a.g_counts = g_counts;
  a.g_idx = g_idx;
  merge_ws_layout(batch_heads, n_q, workspace, &a.ws);
  a.timeout_ns = kWaitLimitNs;
  a.status = status_word(static_cast<cudaStream_t>(stream));
  if (!a.status) return VSA_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  vsa::merge_init_kernel<<<batch_heads, vsa::kMergeHeadThreads, 0, st>>>(a);
  if (rounds > 0) {
    const int smem = vsa::MergeSmem::kAlloc;
    if (cudaFuncSetAttribute(vsa::merge_pairs_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
        cudaSuccess)
      return VSA_ERR_CUDA;
    const int tiles = (n_q + vsa::kMergeTile - 1) / vsa::kMergeTile;
    for (int r = 0; r < rounds; ++r) {
      vsa::merge_pairs_kernel<<<dim3(tiles, tiles, batch_heads), vsa::kMergeThreads, smem, st>>>(a);
      vsa::merge_apply_kernel<<<batch_heads, vsa::kMergeHeadThreads, 0, st>>>(a, r);
    }
  }
  return launch_status();
}

int vsa_cluster_rows_capacity(int n_valid, int n_q) {
  if (n_valid < 1 || n_q < 1) return 0;
  const long long rows = ((long long)n_valid + 127ll * n_q + 127) / 128 * 128;
  return rows > 0x7fffffffll ? 0 : static_cast<int>(rows);
}

vsa_status vsa_cluster_plan(const int32_t *group_of, const int32_t *sizes_q, const int32_t *perm_q,
                            const int32_t *sizes_k, int batch_heads, int n_q, int n_k, int n_valid, int n_pad,
                            int n_rows, int32_t *qmap, int32_t *qinv, int32_t *tile_list, int32_t *kc_off,
                            void *stream) {
  if (!group_of || !sizes_q || !perm_q || !sizes_k || !qmap || !qinv || !tile_list || !kc_off)
    return VSA_ERR_INVALID_ARG;
  if (batch_heads < 1 || batch_heads > 65535 || n_q < 1 || n_k < 1 || n_valid < 1 || n_pad < n_valid)
    return VSA_ERR_INVALID_ARG;
  if (n_rows < 128 || n_rows % 128 != 0) return VSA_ERR_INVALID_ARG;
  if (n_q > vsa::kPlanMaxClusters || n_k > vsa::kPlanMaxClusters) return VSA_ERR_UNSUPPORTED;
  int *word = status_word(static_cast<cudaStream_t>(stream));
  if (!word) return VSA_ERR_CUDA;
  vsa::PlanArgs a{group_of, sizes_q, perm_q, sizes_k, n_q, n_k, n_valid, n_pad, n_rows, qmap, qinv, tile_list, kc_off,
                  word};
  vsa::cluster_plan_kernel<<<batch_heads, vsa::kPlanThreads, 0, static_cast<cudaStream_t>(stream)>>>(a);
  return launch_status();
}

vsa_status vsa_gather_rows(const void *src, const int32_t *map, int batch_heads, int n_src, int n_dst,
                           int row_bytes, uint32_t fill, void *dst, void *stream) {
  if (!src || !map || !dst || src == dst) return VSA_ERR_INVALID_ARG;
  if (batch_heads < 1 || n_src < 1 || n_dst < 1 || row_bytes < 4 || row_bytes % 4 != 0) return VSA_ERR_INVALID_ARG;
  const bool wide = row_bytes % 16 == 0;
  const uintptr_t mask = wide ? 15u : 3u;
  if ((reinterpret_cast<uintptr_t>(src) & mask) || (reinterpret_cast<uintptr_t>(dst) & mask) ||
      (reinterpret_cast<uintptr_t>(map) & 3u))
    return VSA_ERR_INVALID_ARG;
  const char *s8 = static_cast<const char *>(src);
  const char *d8 = static_cast<const char *>(dst);
  const long long src_span = (long long)batch_heads * n_src * row_bytes;
  const long long dst_span = (long long)batch_heads * n_dst * row_bytes;
  if (s8 < d8 + dst_span && d8 < s8 + src_span) return VSA_ERR_INVALID_ARG;
  const long long rows = (long long)batch_heads * n_dst;
  const long long blocks = (rows + 7) / 8;
  if (blocks > 0x7fffffffll) return VSA_ERR_UNSUPPORTED;
  int *word = status_word(static_cast<cudaStream_t>(stream));
  if (!word) return VSA_ERR_CUDA;
  vsa::gather_rows_kernel<<<(unsigned)blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint32_t *>(src), map, n_src, n_dst, rows, row_bytes / 4, fill, static_cast<uint32_t *>(dst),
      word);
  return launch_status();
}

vsa_status vsa_cluster_group_fwd(const void *q_rows, const void *k, const void *v, const vsa_shape *shape,
                                 int n_rows, const int32_t *tile_list, const int32_t *kc_off,
                                 const int32_t *kc_size, int n_kc, const int32_t *counts, const int32_t *idx,
                                 int n_lists, float scale, void *o, int o_fp32, float *lse, void *stream) {
  if (!shape_ok(shape) || !q_rows || !k || !v || !tile_list || !kc_off || !kc_size || !counts || !idx || !o || !lse)
    return VSA_ERR_INVALID_ARG;
  if (n_rows < 128 || n_rows % 128 != 0 || n_kc < 1 || n_lists < 1) return VSA_ERR_INVALID_ARG;
  if (n_kc > vsa::kListStage) return VSA_ERR_UNSUPPORTED;
  if (!(scale > 0.f) || !std::isfinite(scale)) return VSA_ERR_INVALID_ARG;
  if (!aligned16(q_rows) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return VSA_ERR_INVALID_ARG;
  if ((long long)n_rows * shape->d * shape->B * shape->H >= (1ll << 40)) return VSA_ERR_UNSUPPORTED;
  AttnArgs a{};
  a.n_pad = shape->n_pad;
  a.n_valid = shape->n_valid;
  a.list_rows = 128;
  a.seg_keys = 16;
  a.seg_shift = 4;
  a.idx_stride = n_kc;
  a.counts = counts;
  a.idx = idx;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.o = o;
  a.o_fp32 = o_fp32 ? 1 : 0;
  a.lse = lse;
  a.n_bh = shape->B * shape->H;
  a.timeout_ns = kWaitLimitNs;
  a.status = status_word(static_cast<cudaStream_t>(stream));
  if (!a.status) return VSA_ERR_CUDA;
  a.tile_list = tile_list;
  a.kc_off = kc_off;
  a.kc_size = kc_size;
  a.n_kc = n_kc;
  a.n_lists_bh = n_lists;
  a.n_tiles = n_rows / 128;
  a.n_rows_q = n_rows;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return shape->d == 128 ? launch_attn_groups<128>(q_rows, k, v, shape, a, st)
                         : launch_attn_groups<64>(q_rows, k, v, shape, a, st);
}

vsa_status vsa_pool_kv_bf16(const void *k, const void *v, const vsa_shape *shape, int bk, int n_rows, void *k_bar,
                            void *v_bar, void *stream) {
  if (!shape_ok(shape) || !k || !v || !k_bar || !v_bar) return VSA_ERR_INVALID_ARG;
  if (bk != 64 && bk != 128) return VSA_ERR_INVALID_ARG;
  if (n_rows < shape->n_pad / bk || n_rows % 128 != 0) return VSA_ERR_INVALID_ARG;
  if (!aligned16(k) || !aligned16(v) || !aligned16(k_bar) || !aligned16(v_bar)) return VSA_ERR_INVALID_ARG;
  dim3 grid(n_rows, shape->B * shape->H, 2);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const __nv_bfloat16 *kb = static_cast<const __nv_bfloat16 *>(k), *vb = static_cast<const __nv_bfloat16 *>(v);
  __nv_bfloat16 *ko = static_cast<__nv_bfloat16 *>(k_bar), *vo = static_cast<__nv_bfloat16 *>(v_bar);
  if (shape->d == 128)
    vsa::pool_kv_bf16_kernel<128><<<grid, vsa::kPoolBfThreads, 0, st>>>(kb, vb, shape->n_pad, shape->n_valid, bk,
                                                                        n_rows, ko, vo);
  else
    vsa::pool_kv_bf16_kernel<64><<<grid, vsa::kPoolBfThreads, 0, st>>>(kb, vb, shape->n_pad, shape->n_valid, bk,
                                                                       n_rows, ko, vo);
  return launch_status();
}

vsa_status vsa_rectify_fwd(const void *q, const void *k_bar, const void *v_bar, const vsa_shape *shape, int bq,
                           int bk, int n_rows, const int32_t *counts, const int32_t *idx, int idx_stride,
                           float scale, const float *merge_o, const float *merge_lse, void *o, int o_fp32,
                           float *lse, const int32_t *heads, int n_heads, void *stream) {
  if (!shape_ok(shape) || !q || !k_bar || !v_bar || !counts || !idx || !o || !lse) return VSA_ERR_INVALID_ARG;
  const long long n_bh = (long long)shape->B * shape->H;
  if (n_heads < 0 || n_heads > n_bh || (heads == nullptr && n_heads != n_bh)) return VSA_ERR_INVALID_ARG;
  if ((bq != 64 && bq != 128) || (bk != 64 && bk != 128)) return VSA_ERR_INVALID_ARG;
  const int n_k = shape->n_pad / bk;
  if (n_k > 1024) return VSA_ERR_UNSUPPORTED;
  if (n_rows < n_k || n_rows % 128 != 0 || idx_stride < 1) return VSA_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !std::isfinite(scale)) return VSA_ERR_INVALID_ARG;
  if ((merge_o == nullptr) != (merge_lse == nullptr)) return VSA_ERR_INVALID_ARG;
  if (merge_o && static_cast<const void *>(merge_o) == o) return VSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_bar) || !aligned16(v_bar) || !aligned16(o) || (merge_o && !aligned16(merge_o)))
    return VSA_ERR_INVALID_ARG;
  AttnArgs a{};
  a.n_pad = shape->n_pad;
  a.n_valid = shape->n_valid;
  a.list_rows = bq;
  a.seg_keys = 128;
  a.seg_shift = 7;
  a.idx_stride = idx_stride;
  a.counts = counts;
  a.idx = idx;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.o = o;
  a.o_fp32 = o_fp32 ? 1 : 0;
  a.lse = lse;
  a.merge_o = merge_o;
  a.merge_lse = merge_lse;
  a.heads = heads;
  a.n_bh = static_cast<int>(n_bh);
  a.timeout_ns = kWaitLimitNs;
  a.status = status_word(static_cast<cudaStream_t>(stream));
  if (!a.status) return VSA_ERR_CUDA;
  a.pool_nk = n_k;
  a.pool_bk = bk;
  a.pool_nvalid = shape->n_valid;
  if (n_heads == 0) return VSA_OK;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return shape->d == 128 ? launch_attn_pooled<128>(q, k_bar, v_bar, shape, n_rows, a, n_heads, st)
                         : launch_attn_pooled<64>(q, k_bar, v_bar, shape, n_rows, a, n_heads, st);
}

vsa_status vsa_cluster_anchor(const void *x, const vsa_shape *shape, const vsa_cluster_params *params, int n_sub,
                              int32_t *assign, float *centroids, int32_t *sizes, int32_t *perm, float *ratio,
                              int32_t *subset, void *stream) {
  if (!shape_ok(shape) || !x || !assign || !centroids || !sizes || !perm || !ratio || !subset)
    return VSA_ERR_INVALID_ARG;
  vsa::ClusterGeom g;
  if (!cluster_geom(params, &g) || g.n_valid != shape->n_valid) return VSA_ERR_INVALID_ARG;
  if (params->iters < 1 || n_sub < 1 || n_sub > shape->n_valid) return VSA_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(centroids)) return VSA_ERR_INVALID_ARG;
  g.n_pad = shape->n_pad;
  const int BH = shape->B * shape->H;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const __nv_bfloat16 *xb = static_cast<const __nv_bfloat16 *>(x);
  const vsa_status r = shape->d == 128
                           ? launch_cluster<128>(xb, g, params->iters, BH, assign, centroids, sizes, perm, ratio, st)
                           : launch_cluster<64>(xb, g, params->iters, BH, assign, centroids, sizes, perm, ratio, st);
  if (r != VSA_OK) return r;
  vsa::subset_select_kernel<<<BH, vsa::kHybThreads, 0, st>>>(ratio, shape->n_valid, n_sub, subset);
  return launch_status();
}

size_t vsa_cluster_refine_workspace_bytes(const vsa_shape *shape, const vsa_cluster_params *params) {
  vsa::ClusterGeom g;
  if (!shape_ok(shape) || !cluster_geom(params, &g)) return 0;
  const size_t BH = (size_t)shape->B * shape->H;
  const size_t n_chunks = (shape->n_valid + vsa::kSortChunk - 1) / vsa::kSortChunk;
  return align256(BH * g.n_cells * n_chunks * 4) + align256(BH * g.n_cells * 4);
}

vsa_status vsa_cluster_refine(const void *x, const vsa_shape *shape, const vsa_cluster_params *params,
                              const int32_t *subset, int n_sub, int32_t *assign, float *centroids, int32_t *sizes,
                              int32_t *perm, void *workspace, size_t workspace_bytes, void *stream) {
  if (!shape_ok(shape) || !x || !subset || !assign || !centroids || !sizes || !perm || !workspace)
    return VSA_ERR_INVALID_ARG;
  vsa::ClusterGeom g;
  if (!cluster_geom(params, &g) || g.n_valid != shape->n_valid) return VSA_ERR_INVALID_ARG;
  if (n_sub < 0 || n_sub > shape->n_valid) return VSA_ERR_INVALID_ARG;
  if (g.n_cells > 4096) return VSA_ERR_UNSUPPORTED;
  if (!aligned16(x) || !aligned16(centroids) || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return VSA_ERR_INVALID_ARG;
  if (workspace_bytes < vsa_cluster_refine_workspace_bytes(shape, params)) return VSA_ERR_INVALID_ARG;
  const int BH = shape->B * shape->H;
  const int n_chunks = (shape->n_valid + vsa::kSortChunk - 1) / vsa::kSortChunk;
  int32_t *cnt = static_cast<int32_t *>(workspace);
  int32_t *changed = reinterpret_cast<int32_t *>(static_cast<char *>(workspace) +
                                                 align256((size_t)BH * g.n_cells * n_chunks * 4));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int *word = status_word(st);
  if (!word) return VSA_ERR_CUDA;
  if (cudaMemsetAsync(changed, 0, (size_t)BH * g.n_cells * 4, st) != cudaSuccess) return VSA_ERR_CUDA;
  const __nv_bfloat16 *xb = static_cast<const __nv_bfloat16 *>(x);
  if (n_sub > 0) {
    const dim3 grid((n_sub + vsa::kReTok - 1) / vsa::kReTok, BH);
    if (shape->d == 128) {
      static const cudaError_t attr = cudaFuncSetAttribute(
          vsa::reassign_tc_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, vsa::RtLayout<128>::kAlloc);
      if (attr != cudaSuccess) return VSA_ERR_CUDA;
      vsa::reassign_tc_kernel<128><<<grid, vsa::kRtThreads, vsa::RtLayout<128>::kAlloc, st>>>(
          xb, shape->n_pad, shape->n_valid, g.n_cells, centroids, subset, n_sub, assign, changed, kWaitLimitNs, word);
    } else {
      static const cudaError_t attr = cudaFuncSetAttribute(
          vsa::reassign_tc_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, vsa::RtLayout<64>::kAlloc);
      if (attr != cudaSuccess) return VSA_ERR_CUDA;
      vsa::reassign_tc_kernel<64><<<grid, vsa::kRtThreads, vsa::RtLayout<64>::kAlloc, st>>>(
          xb, shape->n_pad, shape->n_valid, g.n_cells, centroids, subset, n_sub, assign, changed, kWaitLimitNs, word);
    }
  }
  const dim3 cgrid(n_chunks, BH);
  vsa::sort_count_kernel<<<cgrid, 256, g.n_cells * 4, st>>>(assign, shape->n_valid, g.n_cells, n_chunks, cnt, word);
  vsa::sort_scan_kernel<<<BH, vsa::kHybThreads, 0, st>>>(cnt, g.n_cells, n_chunks, sizes);
  vsa::sort_scatter_kernel<<<cgrid, 32, g.n_cells * 4, st>>>(assign, shape->n_valid, shape->n_pad, g.n_cells,
                                                            n_chunks, cnt, perm);
  const dim3 ugrid(g.n_cells, BH);
  if (shape->d == 128)
    vsa::refresh_kernel<128><<<ugrid, 128, 0, st>>>(xb, shape->n_pad, g.n_cells, n_chunks, changed, cnt, sizes, perm,
                                                    centroids);
  else
    vsa::refresh_kernel<64><<<ugrid, 128, 0, st>>>(xb, shape->n_pad, g.n_cells, n_chunks, changed, cnt, sizes, perm,
                                                   centroids);
  return launch_status();
}

}  // extern "C"

#include "path.cuh"
