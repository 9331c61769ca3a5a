// The whole path behind one C call, on device buffers (vsa_path_fwd) or on
// host buffers with the copies pipelined against the compute
// (vsa_path_fwd_host).  Host orchestration only: every step runs in the
// kernels of this directory, through the same entry points a caller would use.
//
// HyperVAttention section 2 Eq. (2)-(4): pooled scores, Top-p / Min-kc
// selection, attention over the kept blocks; HyMoR-Attn (abstract): Micro
// residual in omitted blocks, merged by exact LSE.  Included once, from vsa.cu.
#pragma once

#include <cuda_runtime.h>

#include <mutex>
#include <vector>

#include "../../include/vsa.h"

namespace {

constexpr int kPathMaxHeads = 1024;

// Flattened (batch, head) indices of the heads with and without the Micro
// repair, written on the device from per-head ranks passed by value.
struct HeadSplit {
  int16_t rank[kPathMaxHeads];  // rank of head h among the heads with its flag
  uint8_t flag[kPathMaxHeads];  // 1 = Micro repair
  int n_rep, n_plain;           // heads per batch element with / without
  int H, BH;
};

__global__ void path_head_split_kernel(HeadSplit hs, int32_t *rep, int32_t *plain) {
  const int bh = blockIdx.x * blockDim.x + threadIdx.x;
  if (bh >= hs.BH) return;
  const int b = bh / hs.H, h = bh % hs.H;
  if (hs.flag[h])
    rep[b * hs.n_rep + hs.rank[h]] = bh;
  else
    plain[b * hs.n_plain + hs.rank[h]] = bh;
}

// The path's device buffers, carved from one caller workspace (256-byte
// aligned pieces).  Returns the bytes needed; fills *w when base is non-null.
struct PathBufs {
  float *q_pool, *k_pool, *q64, *k16, *o_macro, *lse_macro;
  int32_t *counts, *idx, *m_counts, *m_idx, *rep, *plain;
  void *micro_ws;
  size_t micro_ws_bytes;
  int cap;
};

bool path_params_ok(const vsa_shape *s, const vsa_path_params *p) {
  if (!shape_ok(s) || !p) return false;
  if ((p->bq != 64 && p->bq != 128) || (p->bk != 64 && p->bk != 128)) return false;
  if (!std::isfinite(p->scale) || p->scale < 0.f) return false;
  if (p->micro_mode < 0 || p->micro_mode > 2 || p->micro_capacity < 0) return false;
  if (s->H > kPathMaxHeads) return false;
  return true;
}

vsa_micro_params path_micro(const vsa_shape *s, const vsa_path_params *p, int cap) {
  vsa_micro_params m;
  m.mode = p->micro_mode;
  m.topk = p->micro_topk;
  m.percentile = p->micro_percentile;
  m.head_enable = p->micro_heads;
  m.row_capacity = cap;
  (void)s;
  return m;
}

size_t path_layout(const vsa_shape *s, const vsa_path_params *p, void *base, PathBufs *w) {
  size_t off = 0;
  auto take = [&](size_t bytes) -> void * {
    void *q = base ? static_cast<char *>(base) + off : nullptr;
    off += align256(bytes);
    return q;
  };
  const size_t BH = (size_t)s->B * s->H, d = (size_t)s->d;
  const size_t n_q = s->n_pad / p->bq, n_k = s->n_pad / p->bk;
  PathBufs b{};
  b.q_pool = static_cast<float *>(take(BH * n_q * d * 4));
  b.k_pool = static_cast<float *>(take(BH * n_k * d * 4));
  b.counts = static_cast<int32_t *>(take(BH * n_q * 4));
  b.idx = static_cast<int32_t *>(take(BH * n_q * n_k * 4));
  if (p->micro_mode != 0) {
    const size_t n_r = s->n_pad / vsa::kMicroRows, n_t = s->n_pad / vsa::kMicroKeys;
    b.cap = p->micro_capacity > 0 ? p->micro_capacity : (int)n_t;
    b.q64 = static_cast<float *>(take(BH * n_r * d * 4));
    b.k16 = static_cast<float *>(take(BH * n_t * d * 4));
    b.o_macro = static_cast<float *>(take(BH * s->n_pad * d * 4));
    b.lse_macro = static_cast<float *>(take(BH * s->n_pad * 4));
    b.m_counts = static_cast<int32_t *>(take(BH * n_r * 4));
    b.m_idx = static_cast<int32_t *>(take(BH * n_r * (size_t)b.cap * 4));
    b.rep = static_cast<int32_t *>(take(BH * 4));
    b.plain = static_cast<int32_t *>(take(BH * 4));
    const vsa_micro_params mp = path_micro(s, p, b.cap);
    b.micro_ws_bytes = vsa_select_micro_workspace_bytes(s, &mp);
    b.micro_ws = take(b.micro_ws_bytes);
  }
  if (w) *w = b;
  return off;
}

vsa_status path_run(const void *q, const void *k, const void *v, const vsa_shape *s, const vsa_path_params *p, void *o,
                    float *lse, const PathBufs &b, cudaStream_t st) {
  const float scale = p->scale > 0.f ? p->scale : 1.f / std::sqrt((float)s->d);
  const int n_k = s->n_pad / p->bk;
  const bool micro = p->micro_mode != 0;
  vsa_status e = vsa_pool_qk(q, k, s, p->bq, p->bk, b.q_pool, b.k_pool, micro ? b.q64 : nullptr,
                             micro ? b.k16 : nullptr, st);
  if (e != VSA_OK) return e;
  e = vsa_select_blocks(b.q_pool, b.k_pool, s, p->bq, p->bk, scale, &p->select, b.counts, b.idx, nullptr, st);
  if (e != VSA_OK) return e;
  if (!micro)
    return vsa_block_sparse_fwd(q, k, v, s, p->bq, p->bk, b.counts, b.idx, n_k, scale, o, p->o_fp32, lse, nullptr,
                                nullptr, st);
  // heads without the repair get their final output from the Macro pass;
  // heads with it keep an fp32 Macro output that the Micro pass merges into
  HeadSplit hs;
  int n_rep = 0, n_plain = 0;
  for (int h = 0; h < s->H; ++h) {
    const bool rep = p->micro_heads == nullptr || p->micro_heads[h] != 0;
    hs.flag[h] = rep ? 1 : 0;
    hs.rank[h] = static_cast<int16_t>(rep ? n_rep++ : n_plain++);
  }
  hs.n_rep = n_rep;
  hs.n_plain = n_plain;
  hs.H = s->H;
  hs.BH = s->B * s->H;
  path_head_split_kernel<<<(hs.BH + 255) / 256, 256, 0, st>>>(hs, b.rep, b.plain);
  if ((e = launch_status()) != VSA_OK) return e;
  if (n_plain > 0) {
    e = vsa_block_sparse_fwd_heads(q, k, v, s, p->bq, p->bk, b.counts, b.idx, n_k, scale, o, p->o_fp32, lse, nullptr,
                                   nullptr, b.plain, s->B * n_plain, st);
    if (e != VSA_OK) return e;
  }
  if (n_rep == 0) return VSA_OK;
  e = vsa_block_sparse_fwd_heads(q, k, v, s, p->bq, p->bk, b.counts, b.idx, n_k, scale, b.o_macro, 1, b.lse_macro,
                                 nullptr, nullptr, b.rep, s->B * n_rep, st);
  if (e != VSA_OK) return e;
  const vsa_micro_params mp = path_micro(s, p, b.cap);
  e = vsa_select_micro(b.q64, b.k16, b.counts, b.idx, s, p->bq, p->bk, scale, &mp, b.m_counts, b.m_idx, b.micro_ws,
                       b.micro_ws_bytes, st);
  if (e != VSA_OK) return e;
  return vsa_block_sparse_fwd_heads(q, k, v, s, vsa::kMicroRows, vsa::kMicroKeys, b.m_counts, b.m_idx, b.cap, scale,
                                    o, p->o_fp32, lse, b.o_macro, b.lse_macro, b.rep, s->B * n_rep, st);
}

// ---- host-buffer pipeline ---------------------------------------------------

// Workspace slots of the host-buffer pipeline: chunk i uses slot i % 3, so the
// copies in of chunk i+1 and out of chunk i-1 never wait for the compute of
// the chunk next to them.
constexpr int kHostSlots = 3;

// Copy streams and events of the host-buffer pipeline, created once per
// device and kept for the life of the process (no device memory).
struct HostPipe {
  cudaStream_t in = nullptr, out = nullptr;
  cudaEvent_t in_done[kHostSlots] = {}, comp_done[kHostSlots] = {}, out_done[kHostSlots] = {};
  bool ready = false;
};

constexpr int kPathMaxDevices = 64;

vsa_status host_pipe(HostPipe **out) {
  static std::mutex mu;
  static HostPipe pipes[kPathMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kPathMaxDevices) return VSA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(mu);
  HostPipe &hp = pipes[dev];
  if (!hp.ready) {
    if (cudaStreamCreateWithFlags(&hp.in, cudaStreamNonBlocking) != cudaSuccess ||
        cudaStreamCreateWithFlags(&hp.out, cudaStreamNonBlocking) != cudaSuccess)
      return VSA_ERR_CUDA;
    for (int i = 0; i < kHostSlots; ++i)
      if (cudaEventCreateWithFlags(&hp.in_done[i], cudaEventDisableTiming) != cudaSuccess ||
          cudaEventCreateWithFlags(&hp.comp_done[i], cudaEventDisableTiming) != cudaSuccess ||
          cudaEventCreateWithFlags(&hp.out_done[i], cudaEventDisableTiming) != cudaSuccess)
        return VSA_ERR_CUDA;
    hp.ready = true;
  }
  *out = &hp;
  return VSA_OK;
}

// Device workspace of the host pipeline: kHostSlots slots of chunk inputs and
// outputs, then the path workspace of one chunk.
struct HostLayout {
  size_t in_bytes, o_bytes, lse_bytes, slot_bytes, path_off, total;
};

HostLayout host_layout(const vsa_shape *s, const vsa_path_params *p, int chunk) {
  HostLayout L;
  const size_t rows = (size_t)chunk * s->n_pad;
  L.in_bytes = align256(rows * s->d * 2);
  L.o_bytes = align256(rows * s->d * (p->o_fp32 ? 4 : 2));
  L.lse_bytes = align256(rows * 4);
  L.slot_bytes = 3 * L.in_bytes + L.o_bytes + L.lse_bytes;
  L.path_off = kHostSlots * L.slot_bytes;
  // size the chunk's path workspace with every head of the chunk repaired
  vsa_shape cs = *s;
  cs.B = 1;
  cs.H = chunk;
  vsa_path_params all = *p;
  all.micro_heads = nullptr;
  L.total = L.path_off + path_layout(&cs, &all, nullptr, nullptr);
  return L;
}

}  // namespace

extern "C" {

size_t vsa_path_workspace_bytes(const vsa_shape *shape, const vsa_path_params *params) {
  if (!path_params_ok(shape, params)) return 0;
  return path_layout(shape, params, nullptr, nullptr);
}

vsa_status vsa_path_fwd(const void *q, const void *k, const void *v, const vsa_shape *shape,
                        const vsa_path_params *params, void *o, float *lse, void *workspace, size_t workspace_bytes,
                        void *stream) {
  if (!path_params_ok(shape, params) || !q || !k || !v || !o || !lse || !workspace) return VSA_ERR_INVALID_ARG;
  if (((uintptr_t)workspace & 255u) != 0) return VSA_ERR_INVALID_ARG;
  PathBufs b;
  if (path_layout(shape, params, workspace, &b) > workspace_bytes) return VSA_ERR_INVALID_ARG;
  return path_run(q, k, v, shape, params, o, lse, b, static_cast<cudaStream_t>(stream));
}

size_t vsa_path_host_workspace_bytes(const vsa_shape *shape, const vsa_path_params *params, int chunk_heads) {
  if (!path_params_ok(shape, params) || chunk_heads < 1) return 0;
  const int chunk = std::min(chunk_heads, shape->B * shape->H);
  return host_layout(shape, params, chunk).total;
}

vsa_status vsa_path_fwd_host(const void *q_host, const void *k_host, const void *v_host, const vsa_shape *shape,
                             const vsa_path_params *params, int chunk_heads, void *o_host, float *lse_host,
                             void *workspace, size_t workspace_bytes, void *stream) {
  if (!path_params_ok(shape, params) || chunk_heads < 1 || !q_host || !k_host || !v_host || !o_host || !lse_host ||
      !workspace)
    return VSA_ERR_INVALID_ARG;
  static std::mutex enqueue_mu;  // one caller at a time on the shared copy streams and events
  std::lock_guard<std::mutex> lock(enqueue_mu);
  if (((uintptr_t)workspace & 255u) != 0) return VSA_ERR_INVALID_ARG;
  const int BH = shape->B * shape->H;
  const int chunk = std::min(chunk_heads, BH);
  const HostLayout L = host_layout(shape, params, chunk);
  if (L.total > workspace_bytes) return VSA_ERR_INVALID_ARG;
  HostPipe *hp = nullptr;
  vsa_status e = host_pipe(&hp);
  if (e != VSA_OK) return e;
  cudaStream_t comp = static_cast<cudaStream_t>(stream);
  char *ws = static_cast<char *>(workspace);
  const size_t row_in = (size_t)shape->n_pad * shape->d * 2;
  const size_t row_o = (size_t)shape->n_pad * shape->d * (params->o_fp32 ? 4 : 2);
  const size_t row_lse = (size_t)shape->n_pad * 4;
  // the copy streams start after the work already queued on the caller's stream
  if (cudaEventRecord(hp->comp_done[0], comp) != cudaSuccess ||
      cudaStreamWaitEvent(hp->in, hp->comp_done[0], 0) != cudaSuccess ||
      cudaStreamWaitEvent(hp->out, hp->comp_done[0], 0) != cudaSuccess)
    return VSA_ERR_CUDA;
  // Chunk sizes: the first and the last chunk hold half as many heads, so
  // the copy in before the first compute and the compute and copy out after
  // the last copy in -- the parts nothing overlaps -- are half as long.
  std::vector<int> sizes;
  {
    const int half = std::max(1, chunk / 2);
    int left = BH;
    if (chunk >= 2 && BH > 2 * chunk) {
      sizes.push_back(half);
      left -= half;
    }
    while (left > 0) {
      const int n = std::min(chunk, left);
      sizes.push_back(n);
      left -= n;
    }
    if (chunk >= 2 && sizes.size() > 2 && sizes.back() == chunk) {
      sizes.back() = chunk - half;
      sizes.push_back(half);
    }
  }
  std::vector<uint8_t> flags((size_t)chunk);
  int i = 0;
  for (int c0 = 0; i < static_cast<int>(sizes.size()); c0 += sizes[i], ++i) {
    const int n = sizes[i];
    const int slot = i % kHostSlots;
    char *sq = ws + slot * L.slot_bytes;
    char *sk = sq + L.in_bytes, *sv = sk + L.in_bytes, *so = sv + L.in_bytes, *sl = so + L.o_bytes;
    // inputs of chunk i, once the chunk that used this slot before has been computed
    if (i >= kHostSlots && cudaStreamWaitEvent(hp->in, hp->comp_done[slot], 0) != cudaSuccess) return VSA_ERR_CUDA;
    const struct { const void *src; char *dst; } ins[3] = {{q_host, sq}, {k_host, sk}, {v_host, sv}};
    for (const auto &c : ins)
      if (cudaMemcpyAsync(c.dst, static_cast<const char *>(c.src) + (size_t)c0 * row_in, (size_t)n * row_in,
                          cudaMemcpyHostToDevice, hp->in) != cudaSuccess)
        return VSA_ERR_CUDA;
    if (cudaEventRecord(hp->in_done[slot], hp->in) != cudaSuccess) return VSA_ERR_CUDA;
    // the path on chunk i, once its inputs are in and the slot's earlier outputs are out
    if (cudaStreamWaitEvent(comp, hp->in_done[slot], 0) != cudaSuccess) return VSA_ERR_CUDA;
    if (i >= kHostSlots && cudaStreamWaitEvent(comp, hp->out_done[slot], 0) != cudaSuccess) return VSA_ERR_CUDA;
    vsa_shape cs = *shape;
    cs.B = 1;
    cs.H = n;
    vsa_path_params cp = *params;
    if (params->micro_mode != 0 && params->micro_heads != nullptr) {
      for (int j = 0; j < n; ++j) flags[j] = params->micro_heads[(c0 + j) % shape->H];
      cp.micro_heads = flags.data();
    }
    PathBufs b;
    path_layout(&cs, &cp, ws + L.path_off, &b);
    e = path_run(sq, sk, sv, &cs, &cp, so, reinterpret_cast<float *>(sl), b, comp);
    if (e != VSA_OK) return e;
    if (cudaEventRecord(hp->comp_done[slot], comp) != cudaSuccess) return VSA_ERR_CUDA;
    // outputs of chunk i back to the host
    if (cudaStreamWaitEvent(hp->out, hp->comp_done[slot], 0) != cudaSuccess) return VSA_ERR_CUDA;
    if (cudaMemcpyAsync(static_cast<char *>(o_host) + (size_t)c0 * row_o, so, (size_t)n * row_o,
                        cudaMemcpyDeviceToHost, hp->out) != cudaSuccess ||
        cudaMemcpyAsync(reinterpret_cast<char *>(lse_host) + (size_t)c0 * row_lse, sl, (size_t)n * row_lse,
                        cudaMemcpyDeviceToHost, hp->out) != cudaSuccess)
      return VSA_ERR_CUDA;
    if (cudaEventRecord(hp->out_done[slot], hp->out) != cudaSuccess) return VSA_ERR_CUDA;
  }
  // the caller's stream completes with the last copy out
  if (cudaEventRecord(hp->out_done[(i - 1) % kHostSlots], hp->out) != cudaSuccess ||
      cudaStreamWaitEvent(comp, hp->out_done[(i - 1) % kHostSlots], 0) != cudaSuccess)
    return VSA_ERR_CUDA;
  return VSA_OK;
}

}  // extern "C"
