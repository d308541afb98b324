// wan_kernels.h -- host-side launchers of the two sm_100a kernels (internal to
// the library; the public surface is include/wan_attn.h).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>
#include <mutex>

namespace wan {

constexpr int kMaxDevices = 64;

// One-time setup of a launcher per device (function attributes such as the
// dynamic shared-memory limit are set per device): run() calls init(dev)
// once for the calling thread's current device, thread-safe, and returns
// that call's result every time after.
struct PerDeviceOnce {
  std::once_flag flag[kMaxDevices];
  cudaError_t result[kMaxDevices] = {};
  template <class F>
  cudaError_t run(F&& init, int* dev_out = nullptr) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::call_once(flag[dev], [&] { result[dev] = init(dev); });
    if (dev_out != nullptr) *dev_out = dev;
    return result[dev];
  }
};

// Q/K RMSNorm + bf16 round + 3D RoPE, in place on the packed buffer.
// Arguments are assumed validated by the ABI layer.
// With `stats` (the QKV projection's per-256-column sums of squares of the
// same buffer, [batch*S][2*heads*128/256] fp64, see launch_gemm_bf16) the kernel
// takes each row's sum from them instead of reducing it.
// With s_local > 0 the buffer holds a sequence shard: tokens [s0, s0 + s_local)
// of every batch element's F x H x W grid (positions from the grid index).
cudaError_t launch_qk_norm_rope(void* qkv, int64_t batch, int32_t F, int32_t H, int32_t W,
                                int32_t heads, const void* gamma_q, const void* gamma_k, float eps,
                                float theta, cudaStream_t stream, const double* stats = nullptr,
                                int64_t s0 = 0, int64_t s_local = 0);

// Everything the attention launch needs, prepared before anything is
// launched (tensor-map encoding can fail; a launch after a successful plan
// only fails if the runtime rejects it).
struct AttnPlan {
  alignas(64) unsigned char tmap[128];  // CUtensorMap over the packed buffer
  void* out;
  int32_t S, heads, D, q_pairs, n_kv;
  float scale_log2;
  // The (batch, head) block a launch covers: batches [b0, b0 + nb), heads
  // [h0, h0 + nh). plan_attn_fwd sets the whole buffer; a pipelined caller
  // narrows a copy of the plan per launch.
  int32_t b0, nb, h0, nh;
  // Skip-Softmax threshold (0 = dense; plan_attn_fwd sets 0).
  float skip_threshold;
  // Query rows [q_row0, q_row0 + q_rows) of every batch element attend all S
  // keys; out holds q_rows rows per batch element (plan_attn_fwd: 0 and S).
  int32_t q_row0, q_rows;
};

cudaError_t plan_attn_fwd(const void* qkv, void* out, int64_t batch, int64_t seq_len,
                          int32_t heads, float scale, AttnPlan* plan);

// Flash attention over the packed buffer. `pdl` marks the launch as a
// programmatic dependent of the previous kernel on the stream; `wait_ns`
// bounds every pipeline wait; `skip_loads` (self-test only) starts no copies,
// so that the waits run out and the kernel reports a timeout.
constexpr uint64_t kDefaultWaitNs = 1000000000ull;
cudaError_t launch_attn_fwd(const AttnPlan& plan, cudaStream_t stream, bool pdl,
                            uint64_t wait_ns = kDefaultWaitNs, bool skip_loads = false);

// One DiT self-attention step on packed QKV in page-locked host memory,
// through caller-owned device buffers of the same shapes; transfers and
// kernels overlapped chunk by chunk (host_pipeline.cu). Arguments are assumed
// validated by the ABI layer.
struct HostStep {
  const void* qkv_host;
  void* out_host;
  void* qkv_dev;
  void* out_dev;
  int64_t batch, S;
  int32_t F, H, W, heads, heads_per_chunk;
  const void* gamma_q;
  const void* gamma_k;
  float eps, theta, scale;
  bool overlap_input;  // no wait for earlier work on the stream (buffer fences only)
};
cudaError_t enqueue_dit_attn_host(const HostStep& step, cudaStream_t stream);

// FP8 (e4m3) variant (fp8_quant.cu, attn_fwd_fp8.cu). Codes of X are
// e4m3(fl32(x * inv_X)); the attention dequantises with scale_X. qk8 is
// [B][S][2D] (Q then K codes of each token), v8t [B][heads][128][s_pitch]
// (V codes transposed, zero past S; s_pitch a multiple of 16, >= S).
cudaError_t launch_quantize_fp8(const void* qkv, void* qk8, void* v8t, int64_t batch, int64_t S,
                                int32_t heads, int64_t s_pitch, float inv_q, float inv_k, float inv_v,
                                cudaStream_t stream);
cudaError_t launch_qkv_amax(const void* qkv, int64_t tokens, int32_t heads, float* amax, cudaStream_t stream);
cudaError_t launch_attn_fp8(const void* qk8, const void* v8t, void* out, int64_t batch, int64_t seq_len,
                            int32_t heads, int64_t s_pitch, float scale, float scale_q, float scale_k,
                            float scale_v, cudaStream_t stream);
cudaError_t read_and_clear_fp8_error(cudaStream_t stream, int32_t* code);

// Y[M][N] = X[M][K] W[N][K]^T in bf16 with fp32 accumulation (gemm_bf16.cu);
// N a multiple of 256, K of 64. When stats is not null, stats[row][j] (row
// length stat_cols / 256) receives the fp64 sum of squares of the bf16 outputs
// of row `row` in columns [256 j, 256 j + 256), for j < stat_cols / 256.
cudaError_t launch_gemm_bf16(const void* x, const void* w, void* y, int64_t M, int64_t N, int64_t K,
                             double* stats, int64_t stat_cols, cudaStream_t stream);
cudaError_t read_and_clear_gemm_error(cudaStream_t stream, int32_t* code);

// Synchronise the stream, then read and clear the Skip-Softmax counters:
// (32-row group, key tile) pairs skipped, and P V products skipped.
cudaError_t read_and_clear_skip_stats(cudaStream_t stream, int64_t* group_tiles, int64_t* products);

// Synchronise the stream, then read and clear a kernel's device error word.
cudaError_t read_and_clear_device_error(cudaStream_t stream, int32_t* code);
cudaError_t read_and_clear_norm_error(cudaStream_t stream, int32_t* code);

}  // namespace wan
