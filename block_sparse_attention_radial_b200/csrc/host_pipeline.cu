// libbsa: the forward and backward passes on host buffers
// (bsa_attn_fwd_host, bsa_attn_bwd_host).
//
// The inputs live in host memory and the results go back to host memory. The
// problem is cut into groups of heads; each group's inputs are copied in on
// one stream, its kernels run on the caller's stream as soon as the inputs
// have landed, and its results are copied back on a third stream as soon as
// they are done. With pinned host memory the copy engines (one per direction)
// and the SMs work at the same time, so a call takes about the longest of
// the three (usually the host-to-device copy over PCIe) instead of their sum.
//
// Uses only the public entry points (bsa_attn_fwd, bsa_attn_bwd) and the CUDA
// runtime; the device staging buffers are the caller's workspace.

#include <cuda_runtime.h>

#include <cstdint>
#include <cstdio>
#include <mutex>

#include "bsa.h"

namespace {

constexpr int kMaxDevices = 64;
constexpr int kTargetGroups = 8;

// Per-device copy streams and events. An event is waited on right after each
// record, and a wait binds to the record that precedes it, so one event per
// kind serves every group.
struct PipeState {
  bool ready = false;
  cudaStream_t in = nullptr, out = nullptr;
  cudaEvent_t entry = nullptr, landed = nullptr, computed = nullptr, done = nullptr;
};
std::mutex g_pipe_mu;  // one caller at a time enqueues on the shared streams
PipeState g_pipe[kMaxDevices];

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Staging layout inside the workspace: the attention's own scratch, then q,
// k, v, out and lse for the whole problem.
struct HostLayout {
  size_t attn_ws, q, k, v, out, lse, total;
};

HostLayout host_layout(int32_t batch, int32_t heads, int32_t n, int32_t head_dim,
                       const bsa_block_lists *l) {
  HostLayout w;
  const size_t t = static_cast<size_t>(batch) * heads * n * head_dim * 2;
  w.attn_ws = align256(bsa_attn_fwd_workspace_bytes(batch, heads, l));
  w.q = w.attn_ws;
  w.k = w.q + align256(t);
  w.v = w.k + align256(t);
  w.out = w.v + align256(t);
  w.lse = w.out + align256(t);
  w.total = w.lse + align256(static_cast<size_t>(batch) * heads * n * sizeof(float));
  return w;
}

int pipe_state(PipeState **st) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return BSA_ERR_CUDA;
  PipeState &s = g_pipe[dev];
  if (!s.ready) {
    const unsigned fl = cudaEventDisableTiming;
    if (cudaStreamCreateWithFlags(&s.in, cudaStreamNonBlocking) != cudaSuccess ||
        cudaStreamCreateWithFlags(&s.out, cudaStreamNonBlocking) != cudaSuccess ||
        cudaEventCreateWithFlags(&s.entry, fl) != cudaSuccess ||
        cudaEventCreateWithFlags(&s.landed, fl) != cudaSuccess ||
        cudaEventCreateWithFlags(&s.computed, fl) != cudaSuccess ||
        cudaEventCreateWithFlags(&s.done, fl) != cudaSuccess)
      return BSA_ERR_CUDA;
    s.ready = true;
  }
  *st = &s;
  return BSA_OK;
}

#define PIPE_CUDA(call)                          \
  do {                                           \
    if ((call) != cudaSuccess) return BSA_ERR_CUDA; \
  } while (0)

// Groups of whole heads inside one batch item (a group of per-head lists is
// then a contiguous run of lists), about kTargetGroups of them in all. The
// first and the last group hold one head: the first group's copy is the
// only one no kernel overlaps, and the last group's kernel and copy back
// are the only ones no copy in overlaps.
struct HeadGroups {
  long long bh, mid;
  int heads;
  HeadGroups(int batch, int heads_) : heads(heads_) {
    bh = static_cast<long long>(batch) * heads;
    mid = bh > 2 ? (bh - 2 + kTargetGroups - 3) / (kTargetGroups - 2) : 1;
  }
  // The group starting at (b, h) slice `idx`: batch item b, first head h0,
  // hn heads; advances idx past it.
  void next(long long &idx, int &b, int &h0, int &hn) const {
    b = static_cast<int>(idx / heads);
    h0 = static_cast<int>(idx % heads);
    long long size = (idx == 0 || idx == bh - 1) ? 1 : mid;
    if (size > heads - h0) size = heads - h0;                 // stay inside the batch item
    if (idx > 0 && idx + size > bh - 1) size = bh - 1 - idx;  // keep the last head apart
    if (size < 1) size = 1;
    hn = static_cast<int>(size);
    idx += size;
  }
  // Most heads any group holds.
  int max_heads() const {
    long long m = mid < heads ? mid : heads;
    return static_cast<int>(m < 1 ? 1 : m);
  }
};

// The lists of heads [h0, h0 + hn): per-head lists are a contiguous run of
// rows (row_ptr keeps absolute offsets into col_idx); a shared list is kept.
bsa_block_lists group_lists(const bsa_block_lists *l, int h0, int hn) {
  bsa_block_lists sub = *l;
  if (l->num_lists > 1) {
    sub.num_lists = hn;
    sub.row_ptr = l->row_ptr + static_cast<size_t>(h0) * l->num_q_blocks;
  }
  return sub;
}

// Backward staging inside the workspace: the backward's own scratch, sized
// for the largest head group (every group's call reuses it in stream
// order), then q, k, v, out, dout, lse and dq, dk, dv for the whole problem.
struct BwdHostLayout {
  size_t attn_ws, q, k, v, out, dout, lse, dq, dk, dv, total;
};

BwdHostLayout bwd_host_layout(int32_t batch, int32_t heads, int32_t n, int32_t head_dim,
                              const bsa_block_lists *l) {
  BwdHostLayout w;
  const HeadGroups groups(batch, heads);
  const int hmax = groups.max_heads();
  const bsa_block_lists sub = group_lists(l, 0, hmax);
  const size_t t = align256(static_cast<size_t>(batch) * heads * n * head_dim * 2);
  w.attn_ws = align256(bsa_attn_bwd_workspace_bytes(1, hmax, n, &sub));
  w.q = w.attn_ws;
  w.k = w.q + t;
  w.v = w.k + t;
  w.out = w.v + t;
  w.dout = w.out + t;
  w.lse = w.dout + t;
  w.dq = w.lse + align256(static_cast<size_t>(batch) * heads * n * sizeof(float));
  w.dk = w.dq + t;
  w.dv = w.dk + t;
  w.total = w.dv + t;
  return w;
}

}  // namespace

extern "C" {

size_t bsa_attn_fwd_host_workspace_bytes(int32_t batch, int32_t heads, int32_t n,
                                         int32_t head_dim, const bsa_block_lists *l) {
  if (!l || batch < 1 || heads < 1 || n < 1 || head_dim < 1) return 0;
  if (bsa_attn_fwd_workspace_bytes(batch, heads, l) == 0) return 0;
  return host_layout(batch, heads, n, head_dim, l).total;
}

int bsa_attn_fwd_host(const void *q_host, const void *k_host, const void *v_host,
                      int32_t batch, int32_t heads, int32_t n, int32_t head_dim,
                      float softmax_scale, const bsa_block_lists *l, void *out_host,
                      float *lse_host, void *workspace, size_t workspace_bytes,
                      bsa_stream_t stream_) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (!q_host || !k_host || !v_host || !out_host || !l || !workspace) return BSA_ERR_INVALID_ARG;
  if (batch < 1 || heads < 1 || n < 1) return BSA_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return BSA_ERR_UNSUPPORTED;
  if (bsa_attn_fwd_workspace_bytes(batch, heads, l) == 0) return BSA_ERR_INVALID_ARG;
  const HostLayout w = host_layout(batch, heads, n, head_dim, l);
  if (workspace_bytes < w.total || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return BSA_ERR_INVALID_ARG;

  const HeadGroups groups(batch, heads);

  std::lock_guard<std::mutex> lk(g_pipe_mu);
  PipeState *ps = nullptr;
  int st = pipe_state(&ps);
  if (st != BSA_OK) return st;

  uint8_t *ws = static_cast<uint8_t *>(workspace);
  const size_t row = static_cast<size_t>(n) * head_dim * 2;  // bytes of one (b, h) slice
  const size_t lrow = static_cast<size_t>(n) * sizeof(float);

  // everything already on the caller's stream (e.g. the lists) comes first
  PIPE_CUDA(cudaEventRecord(ps->entry, stream));
  PIPE_CUDA(cudaStreamWaitEvent(ps->in, ps->entry, 0));
  PIPE_CUDA(cudaStreamWaitEvent(ps->out, ps->entry, 0));

  for (long long idx = 0; idx < groups.bh;) {
    int b, h0, hn;
    groups.next(idx, b, h0, hn);
    const size_t off = (static_cast<size_t>(b) * heads + h0) * row;
    const size_t bytes = static_cast<size_t>(hn) * row;
    PIPE_CUDA(cudaMemcpyAsync(ws + w.q + off, static_cast<const uint8_t *>(q_host) + off, bytes,
                              cudaMemcpyHostToDevice, ps->in));
    PIPE_CUDA(cudaMemcpyAsync(ws + w.k + off, static_cast<const uint8_t *>(k_host) + off, bytes,
                              cudaMemcpyHostToDevice, ps->in));
    PIPE_CUDA(cudaMemcpyAsync(ws + w.v + off, static_cast<const uint8_t *>(v_host) + off, bytes,
                              cudaMemcpyHostToDevice, ps->in));
    PIPE_CUDA(cudaEventRecord(ps->landed, ps->in));
    PIPE_CUDA(cudaStreamWaitEvent(stream, ps->landed, 0));

    const bsa_block_lists sub = group_lists(l, h0, hn);  // this group's heads' lists
    const size_t loff = (static_cast<size_t>(b) * heads + h0) * lrow;
    st = bsa_attn_fwd(ws + w.q + off, ws + w.k + off, ws + w.v + off, 1, hn, n, head_dim,
                      softmax_scale, &sub, ws + w.out + off,
                      reinterpret_cast<float *>(ws + w.lse + loff), ws, w.attn_ws, stream_);
    if (st != BSA_OK) return st;
    PIPE_CUDA(cudaEventRecord(ps->computed, stream));
    PIPE_CUDA(cudaStreamWaitEvent(ps->out, ps->computed, 0));
    PIPE_CUDA(cudaMemcpyAsync(static_cast<uint8_t *>(out_host) + off, ws + w.out + off, bytes,
                              cudaMemcpyDeviceToHost, ps->out));
    if (lse_host)
      PIPE_CUDA(cudaMemcpyAsync(reinterpret_cast<uint8_t *>(lse_host) + loff, ws + w.lse + loff,
                                static_cast<size_t>(hn) * lrow, cudaMemcpyDeviceToHost, ps->out));
  }
  // the caller's stream orders after the last copy back
  PIPE_CUDA(cudaEventRecord(ps->done, ps->out));
  PIPE_CUDA(cudaStreamWaitEvent(stream, ps->done, 0));
  return BSA_OK;
}

size_t bsa_attn_bwd_host_workspace_bytes(int32_t batch, int32_t heads, int32_t n,
                                         int32_t head_dim, const bsa_block_lists *l) {
  if (!l || batch < 1 || heads < 1 || n < 1 || head_dim < 1) return 0;
  if (bsa_attn_bwd_workspace_bytes(batch, heads, n, l) == 0) return 0;
  return bwd_host_layout(batch, heads, n, head_dim, l).total;
}

int bsa_attn_bwd_host(const void *q_host, const void *k_host, const void *v_host,
                      const void *out_host, const void *dout_host, const float *lse_host,
                      int32_t batch, int32_t heads, int32_t n, int32_t head_dim,
                      float softmax_scale, const bsa_block_lists *l, void *dq_host,
                      void *dk_host, void *dv_host, void *workspace, size_t workspace_bytes,
                      bsa_stream_t stream_) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (!q_host || !k_host || !v_host || !out_host || !dout_host || !lse_host || !l || !dq_host ||
      !dk_host || !dv_host || !workspace)
    return BSA_ERR_INVALID_ARG;
  if (batch < 1 || heads < 1 || n < 1) return BSA_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return BSA_ERR_UNSUPPORTED;
  if (bsa_attn_bwd_workspace_bytes(batch, heads, n, l) == 0) return BSA_ERR_INVALID_ARG;
  const BwdHostLayout w = bwd_host_layout(batch, heads, n, head_dim, l);
  if (workspace_bytes < w.total || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return BSA_ERR_INVALID_ARG;

  const HeadGroups groups(batch, heads);

  std::lock_guard<std::mutex> lk(g_pipe_mu);
  PipeState *ps = nullptr;
  int st = pipe_state(&ps);
  if (st != BSA_OK) return st;

  uint8_t *ws = static_cast<uint8_t *>(workspace);
  const size_t row = static_cast<size_t>(n) * head_dim * 2;  // bytes of one (b, h) slice
  const size_t lrow = static_cast<size_t>(n) * sizeof(float);
  const void *inputs[5] = {q_host, k_host, v_host, out_host, dout_host};
  const size_t staged_in[5] = {w.q, w.k, w.v, w.out, w.dout};
  void *outputs[3] = {dq_host, dk_host, dv_host};
  const size_t staged_out[3] = {w.dq, w.dk, w.dv};

  // everything already on the caller's stream (e.g. the lists) comes first
  PIPE_CUDA(cudaEventRecord(ps->entry, stream));
  PIPE_CUDA(cudaStreamWaitEvent(ps->in, ps->entry, 0));
  PIPE_CUDA(cudaStreamWaitEvent(ps->out, ps->entry, 0));

  for (long long idx = 0; idx < groups.bh;) {
    int b, h0, hn;
    groups.next(idx, b, h0, hn);
    const size_t off = (static_cast<size_t>(b) * heads + h0) * row;
    const size_t bytes = static_cast<size_t>(hn) * row;
    const size_t loff = (static_cast<size_t>(b) * heads + h0) * lrow;
    for (int i = 0; i < 5; ++i)
      PIPE_CUDA(cudaMemcpyAsync(ws + staged_in[i] + off,
                                static_cast<const uint8_t *>(inputs[i]) + off, bytes,
                                cudaMemcpyHostToDevice, ps->in));
    PIPE_CUDA(cudaMemcpyAsync(ws + w.lse + loff, reinterpret_cast<const uint8_t *>(lse_host) + loff,
                              static_cast<size_t>(hn) * lrow, cudaMemcpyHostToDevice, ps->in));
    PIPE_CUDA(cudaEventRecord(ps->landed, ps->in));
    PIPE_CUDA(cudaStreamWaitEvent(stream, ps->landed, 0));

    const bsa_block_lists sub = group_lists(l, h0, hn);  // this group's heads' lists
    st = bsa_attn_bwd(ws + w.q + off, ws + w.k + off, ws + w.v + off, ws + w.out + off,
                      ws + w.dout + off, reinterpret_cast<const float *>(ws + w.lse + loff), 1, hn,
                      n, head_dim, softmax_scale, &sub, ws + w.dq + off, ws + w.dk + off,
                      ws + w.dv + off, ws, w.attn_ws, stream_);
    if (st != BSA_OK) return st;
    PIPE_CUDA(cudaEventRecord(ps->computed, stream));
    PIPE_CUDA(cudaStreamWaitEvent(ps->out, ps->computed, 0));
    for (int i = 0; i < 3; ++i)
      PIPE_CUDA(cudaMemcpyAsync(static_cast<uint8_t *>(outputs[i]) + off,
                                ws + staged_out[i] + off, bytes, cudaMemcpyDeviceToHost,
                                ps->out));
  }
  // the caller's stream orders after the last copy back
  PIPE_CUDA(cudaEventRecord(ps->done, ps->out));
  PIPE_CUDA(cudaStreamWaitEvent(stream, ps->done, 0));
  return BSA_OK;
}

}  // extern "C"
