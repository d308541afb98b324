// host_pipeline.cu -- the DiT self-attention step for packed QKV that lives in
// page-locked host memory: host->device copies, the two kernels and the
// device->host copy of the output, overlapped chunk by chunk.
//
// End to end, the step is bound by the PCIe transfer of the packed input
// (3*D bf16 per token) and by the kernels, in about equal measure; the output
// (D per token) goes back on the other direction of the link. So:
//  - each batch element's packed rows arrive in one contiguous copy. Strided
//    copies of its Q|K part first (the norm needs every head of a token) and
//    of V by head chunks would let that element's kernels start earlier, but
//    they move only about 46 GB/s against 55 for contiguous ones on B200
//    hosts, and consecutive calls overlap anyway (below);
//  - the element's norm+RoPE starts as soon as its rows have arrived, and its
//    attention follows in chunks of heads;
//  - the output of a head chunk goes back to the host while later chunks
//    compute.
// Three internal streams per device carry the work: host->device copies,
// kernels, device->host copies (PCIe is full duplex); events carry the
// dependencies. The caller's stream waits for the last output copy, so work
// enqueued on it later sees the output written.
//
// Buffer fences. Across calls, a call's copies into qkv_dev must not start
// before the kernels of an earlier call that read the same qkv_dev are done,
// and its kernels must not write out_dev before an earlier call's copy out
// of the same out_dev is done. Each device keeps, per buffer address, an
// event recorded after that buffer's last use by this pipeline, and the next
// call on the buffer waits for it -- and for nothing else when the caller
// passes overlap_input, so that one call's input transfer runs under the
// previous call's kernels and one call's kernels do not wait for the
// previous call's last output copy. A buffer the table does not know (first
// use, or evicted) waits for all earlier kernels / output copies instead.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>
#include <vector>

#include "wan_kernels.h"

namespace wan {
namespace {

// The last use of one device buffer by the pipeline.
struct Fence {
  const void* ptr = nullptr;
  cudaEvent_t ev = nullptr;
  uint64_t stamp = 0;  // for least-recently-used eviction
};

constexpr size_t kMaxFences = 64;

// Internal streams, a reusable event pool and the buffer fences, one set per
// device. Reusing an event is safe here: every wait on an event is enqueued
// before the event is recorded again (the whole enqueue sequence runs under
// the device's mutex).
struct DeviceQueues {
  std::mutex mu;
  cudaStream_t h2d = nullptr;
  cudaStream_t compute = nullptr;
  cudaStream_t d2h = nullptr;
  std::vector<cudaEvent_t> events;
  std::vector<Fence> qkv_fences;  // after the last kernel that read the buffer
  std::vector<Fence> out_fences;  // after the last copy out of the buffer
  uint64_t clock = 0;
};

DeviceQueues g_queues[kMaxDevices];

cudaError_t new_event(cudaEvent_t* ev) { return cudaEventCreateWithFlags(ev, cudaEventDisableTiming); }

cudaError_t ensure_queues(DeviceQueues& q, size_t n_events) {
  for (cudaStream_t* s : {&q.h2d, &q.compute, &q.d2h}) {
    if (*s == nullptr) {
      cudaError_t e = cudaStreamCreateWithFlags(s, cudaStreamNonBlocking);
      if (e != cudaSuccess) return e;
    }
  }
  while (q.events.size() < n_events) {
    cudaEvent_t ev;
    cudaError_t e = new_event(&ev);
    if (e != cudaSuccess) return e;
    q.events.push_back(ev);
  }
  return cudaSuccess;
}

// The fence of `ptr`, or null when the table does not know the buffer.
const Fence* find_fence(const std::vector<Fence>& table, const void* ptr) {
  for (const Fence& f : table) {
    if (f.ptr == ptr) return &f;
  }
  return nullptr;
}

// The fence to record for `ptr`: its entry, a new one, or the least recently
// used entry taken over (that entry's buffer then counts as unknown).
cudaError_t fence_slot(std::vector<Fence>& table, const void* ptr, Fence** out) {
  Fence* f = nullptr;
  for (Fence& g : table) {
    if (g.ptr == ptr) f = &g;
  }
  if (f == nullptr && table.size() < kMaxFences) {
    Fence fresh;
    cudaError_t e = new_event(&fresh.ev);
    if (e != cudaSuccess) return e;
    table.push_back(fresh);
    f = &table.back();
  }
  if (f == nullptr) {
    f = &table[0];
    for (Fence& g : table) {
      if (g.stamp < f->stamp) f = &g;
    }
  }
  f->ptr = ptr;
  *out = f;
  return cudaSuccess;
}

#define WAN_CUDA_TRY(expr)              \
  do {                                  \
    const cudaError_t _e = (expr);      \
    if (_e != cudaSuccess) return _e;   \
  } while (0)

}  // namespace

cudaError_t enqueue_dit_attn_host(const HostStep& a, cudaStream_t user) {
  int dev = 0;
  WAN_CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  DeviceQueues& q = g_queues[dev];
  std::lock_guard<std::mutex> lock(q.mu);

  const int64_t B = a.batch, S = a.S;
  const int32_t heads = a.heads, hc = a.heads_per_chunk;
  const int32_t chunks = (heads + hc - 1) / hc;
  const size_t d = static_cast<size_t>(heads) * 128;  // channels per Q, K or V row
  const size_t row_qkv = 3 * d * 2, row_out = d * 2;  // bytes per token row
  const size_t n_events = 3 + static_cast<size_t>(B) * (1 + static_cast<size_t>(chunks));
  WAN_CUDA_TRY(ensure_queues(q, n_events));

  AttnPlan plan;
  WAN_CUDA_TRY(plan_attn_fwd(a.qkv_dev, a.out_dev, B, S, heads, a.scale, &plan));

  size_t next = 0;
  auto ev = [&]() { return q.events[next++]; };
  ++q.clock;

  // Without overlap_input, nothing of this call starts before the work
  // enqueued on the caller's stream so far.
  if (!a.overlap_input) {
    const cudaEvent_t ev_start = ev();
    WAN_CUDA_TRY(cudaEventRecord(ev_start, user));
    WAN_CUDA_TRY(cudaStreamWaitEvent(q.h2d, ev_start, 0));
    WAN_CUDA_TRY(cudaStreamWaitEvent(q.compute, ev_start, 0));
  }
  // Copies into qkv_dev wait for the kernels that last read it (an unknown
  // buffer: for every kernel enqueued so far).
  if (const Fence* f = find_fence(q.qkv_fences, a.qkv_dev)) {
    WAN_CUDA_TRY(cudaStreamWaitEvent(q.h2d, f->ev, 0));
  } else {
    const cudaEvent_t ev_tail = ev();
    WAN_CUDA_TRY(cudaEventRecord(ev_tail, q.compute));
    WAN_CUDA_TRY(cudaStreamWaitEvent(q.h2d, ev_tail, 0));
  }
  // Kernels writing out_dev wait for the copy that last read it (an unknown
  // buffer: for every output copy enqueued so far).
  if (const Fence* f = find_fence(q.out_fences, a.out_dev)) {
    WAN_CUDA_TRY(cudaStreamWaitEvent(q.compute, f->ev, 0));
  } else {
    const cudaEvent_t ev_tail = ev();
    WAN_CUDA_TRY(cudaEventRecord(ev_tail, q.d2h));
    WAN_CUDA_TRY(cudaStreamWaitEvent(q.compute, ev_tail, 0));
  }

  auto* qkv_h = static_cast<const unsigned char*>(a.qkv_host);
  auto* qkv_d = static_cast<unsigned char*>(a.qkv_dev);
  auto* out_h = static_cast<unsigned char*>(a.out_host);
  auto* out_d = static_cast<const unsigned char*>(a.out_dev);

  std::vector<cudaEvent_t> ev_in(B), ev_o(B * chunks);
  for (int64_t b = 0; b < B; ++b) {
    const size_t base = static_cast<size_t>(b) * S * row_qkv;
    WAN_CUDA_TRY(cudaMemcpyAsync(qkv_d + base, qkv_h + base, static_cast<size_t>(S) * row_qkv,
                                 cudaMemcpyHostToDevice, q.h2d));
    ev_in[b] = ev();
    WAN_CUDA_TRY(cudaEventRecord(ev_in[b], q.h2d));
  }
  for (int64_t b = 0; b < B; ++b) {
    WAN_CUDA_TRY(cudaStreamWaitEvent(q.compute, ev_in[b], 0));
    WAN_CUDA_TRY(launch_qk_norm_rope(qkv_d + static_cast<size_t>(b) * S * row_qkv, 1, a.F, a.H, a.W,
                                     heads, a.gamma_q, a.gamma_k, a.eps, a.theta, q.compute));
    for (int32_t c = 0; c < chunks; ++c) {
      AttnPlan part = plan;
      part.b0 = static_cast<int32_t>(b);
      part.nb = 1;
      part.h0 = c * hc;
      part.nh = (part.h0 + hc <= heads) ? hc : heads - part.h0;
      WAN_CUDA_TRY(launch_attn_fwd(part, q.compute, false));
      ev_o[b * chunks + c] = ev();
      WAN_CUDA_TRY(cudaEventRecord(ev_o[b * chunks + c], q.compute));
    }
  }
  Fence* fq = nullptr;
  WAN_CUDA_TRY(fence_slot(q.qkv_fences, a.qkv_dev, &fq));
  WAN_CUDA_TRY(cudaEventRecord(fq->ev, q.compute));
  fq->stamp = q.clock;

  for (int64_t b = 0; b < B; ++b) {
    for (int32_t c = 0; c < chunks; ++c) {
      const int32_t h0 = c * hc, nh = (h0 + hc <= heads) ? hc : heads - h0;
      const size_t off = static_cast<size_t>(b) * S * row_out + static_cast<size_t>(h0) * 128 * 2;
      WAN_CUDA_TRY(cudaStreamWaitEvent(q.d2h, ev_o[b * chunks + c], 0));
      WAN_CUDA_TRY(cudaMemcpy2DAsync(out_h + off, row_out, out_d + off, row_out,
                                     static_cast<size_t>(nh) * 128 * 2, S, cudaMemcpyDeviceToHost,
                                     q.d2h));
    }
  }
  Fence* fo = nullptr;
  WAN_CUDA_TRY(fence_slot(q.out_fences, a.out_dev, &fo));
  WAN_CUDA_TRY(cudaEventRecord(fo->ev, q.d2h));
  fo->stamp = q.clock;
  // The caller's stream continues once the output is on the host (the last
  // copy out follows every kernel of the call).
  WAN_CUDA_TRY(cudaStreamWaitEvent(user, fo->ev, 0));
  return cudaSuccess;
}

}  // namespace wan
