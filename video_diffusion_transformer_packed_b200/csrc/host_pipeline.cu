// host_pipeline.cu -- the DiT self-attention step for packed QKV that lives in
// page-locked host memory: host->device copies, the two kernels and the
// device->host copy of the output, overlapped chunk by chunk.
//
// What bounds the step end to end is the PCIe transfer of the packed input
// (3*D bf16 per token) and of the output (D per token), not the kernels, so
// the copies are cut along the dependencies of the path:
//  - norm+RoPE of a token needs that token's whole Q|K row (the RMS runs over
//    all heads), so each batch element's Q|K block is copied first, as one
//    strided 2D copy of the first 2*D channels of every token row;
//  - attention of head h needs Q, K and V of that head for every token of the
//    batch element, so V follows in chunks of heads, and the attention of a
//    head chunk starts as soon as its V chunk has arrived;
//  - the output of a head chunk goes back to the host while later chunks
//    compute.
// Host->device copies run on one internal stream, device->host copies on
// another (PCIe is full duplex), kernels on the caller's stream; events carry
// the dependencies. The whole sequence is ordered after earlier work on the
// caller's stream, and later work on that stream sees the output written.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>
#include <vector>

#include "wan_kernels.h"

namespace wan {
namespace {

// Internal streams and a reusable event pool, one set per device. Reusing an
// event is safe here: every wait on an event is enqueued before the event is
// recorded again (the whole enqueue sequence runs under the device's mutex).
struct DeviceQueues {
  std::mutex mu;
  cudaStream_t h2d = nullptr;
  cudaStream_t d2h = nullptr;
  std::vector<cudaEvent_t> events;
};

DeviceQueues g_queues[kMaxDevices];

cudaError_t ensure_queues(DeviceQueues& q, size_t n_events) {
  if (!q.h2d) {
    cudaError_t e = cudaStreamCreateWithFlags(&q.h2d, cudaStreamNonBlocking);
    if (e != cudaSuccess) return e;
  }
  if (!q.d2h) {
    cudaError_t e = cudaStreamCreateWithFlags(&q.d2h, cudaStreamNonBlocking);
    if (e != cudaSuccess) return e;
  }
  while (q.events.size() < n_events) {
    cudaEvent_t ev;
    cudaError_t e = cudaEventCreateWithFlags(&ev, cudaEventDisableTiming);
    if (e != cudaSuccess) return e;
    q.events.push_back(ev);
  }
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
  const size_t n_events = 2 + static_cast<size_t>(B) * (1 + 2 * static_cast<size_t>(chunks));
  WAN_CUDA_TRY(ensure_queues(q, n_events));

  AttnPlan plan;
  WAN_CUDA_TRY(plan_attn_fwd(a.qkv_dev, a.out_dev, B, S, heads, a.scale, &plan));

  size_t next = 0;
  auto ev = [&]() { return q.events[next++]; };
  const cudaEvent_t ev_start = ev();
  // Copies must not overwrite the device buffers before earlier work on the
  // caller's stream is done with them -- unless the caller vouches that no
  // earlier work uses these buffers (it alternates sets), in which case this
  // call's transfer overlaps the previous call's kernels.
  if (!a.overlap_input) {
    WAN_CUDA_TRY(cudaEventRecord(ev_start, user));
    WAN_CUDA_TRY(cudaStreamWaitEvent(q.h2d, ev_start, 0));
  }

  auto* qkv_h = static_cast<const unsigned char*>(a.qkv_host);
  auto* qkv_d = static_cast<unsigned char*>(a.qkv_dev);
  auto* out_h = static_cast<unsigned char*>(a.out_host);
  auto* out_d = static_cast<const unsigned char*>(a.out_dev);

  std::vector<cudaEvent_t> ev_qk(B), ev_v(B * chunks), ev_o(B * chunks);
  for (int64_t b = 0; b < B; ++b) {
    const size_t base = static_cast<size_t>(b) * S * row_qkv;
    // Q|K of every token: the first 2*D channels of each row.
    WAN_CUDA_TRY(cudaMemcpy2DAsync(qkv_d + base, row_qkv, qkv_h + base, row_qkv, 2 * d * 2, S,
                                   cudaMemcpyHostToDevice, q.h2d));
    ev_qk[b] = ev();
    WAN_CUDA_TRY(cudaEventRecord(ev_qk[b], q.h2d));
    for (int32_t c = 0; c < chunks; ++c) {
      const int32_t h0 = c * hc, nh = (h0 + hc <= heads) ? hc : heads - h0;
      const size_t off = base + (2 * d + static_cast<size_t>(h0) * 128) * 2;
      WAN_CUDA_TRY(cudaMemcpy2DAsync(qkv_d + off, row_qkv, qkv_h + off, row_qkv,
                                     static_cast<size_t>(nh) * 128 * 2, S, cudaMemcpyHostToDevice,
                                     q.h2d));
      ev_v[b * chunks + c] = ev();
      WAN_CUDA_TRY(cudaEventRecord(ev_v[b * chunks + c], q.h2d));
    }
  }
  for (int64_t b = 0; b < B; ++b) {
    WAN_CUDA_TRY(cudaStreamWaitEvent(user, ev_qk[b], 0));
    WAN_CUDA_TRY(launch_qk_norm_rope(qkv_d + static_cast<size_t>(b) * S * row_qkv, 1, a.F, a.H, a.W,
                                     heads, a.gamma_q, a.gamma_k, a.eps, a.theta, user));
    for (int32_t c = 0; c < chunks; ++c) {
      AttnPlan part = plan;
      part.b0 = static_cast<int32_t>(b);
      part.nb = 1;
      part.h0 = c * hc;
      part.nh = (part.h0 + hc <= heads) ? hc : heads - part.h0;
      WAN_CUDA_TRY(cudaStreamWaitEvent(user, ev_v[b * chunks + c], 0));
      WAN_CUDA_TRY(launch_attn_fwd(part, user, false));
      ev_o[b * chunks + c] = ev();
      WAN_CUDA_TRY(cudaEventRecord(ev_o[b * chunks + c], user));
    }
  }
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
  const cudaEvent_t ev_done = ev();
  WAN_CUDA_TRY(cudaEventRecord(ev_done, q.d2h));
  WAN_CUDA_TRY(cudaStreamWaitEvent(user, ev_done, 0));
  return cudaSuccess;
}

}  // namespace wan
