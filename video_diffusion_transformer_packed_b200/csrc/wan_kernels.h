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
  alignas(64) unsigned char tmap[128];     // CUtensorMap over the buffer holding Q
  alignas(64) unsigned char tmap_kv[128];  // CUtensorMap over the buffer holding K and V
  const void* q_base;                      // the buffer holding Q ([batch][S][3D])
  void* out;
  int32_t S, heads, D, q_pairs, n_kv;
  float scale_log2;
  // The (batch, head) block a launch covers: batches [b0, b0 + nb), heads
  // [h0, h0 + nh). plan_attn_fwd sets the whole buffer; a pipelined caller
  // narrows a copy of the plan per launch.
  int32_t b0, nb, h0, nh;
  // Skip-Softmax threshold (0 = dense; plan_attn_fwd sets 0).
  float skip_threshold;
  // Query rows [q_row0, q_row0 + q_rows) of every batch element; out holds
  // q_rows rows per batch element (plan_attn_fwd: 0 and S).
  int32_t q_row0, q_rows;
  // Keys [k_row0, k_row0 + k_rows) of the K/V buffer; K of head h at column
  // kv_k0 + 128 h, V at kv_v0 + 128 h (plan_attn_fwd: the packed buffer
  // itself, 0, S, D, 2D; plan_attn_kv points them elsewhere).
  int32_t k_row0, k_rows, kv_k0, kv_v0;
  // Partial mode (o_part not null): instead of out, the launch writes the
  // unnormalised fp32 O to o_part [batch][q_rows][heads][128] and (m, l) to
  // ml_part [batch][q_rows][heads][2], with O = sum_j 2^(a_j - m) v_j and
  // l = sum_j 2^(a_j - m) over the key range, a_j = scale log2(e) q . k_j.
  float* o_part;
  float* ml_part;
  // Partial mode with accumulate: (o_part, ml_part) already hold a state over
  // other keys, and the launch merges its own into it (each side rescaled to
  // the larger m) instead of overwriting it.
  bool accumulate;
};

cudaError_t plan_attn_fwd(const void* qkv, void* out, int64_t batch, int64_t seq_len,
                          int32_t heads, float scale, AttnPlan* plan);

// Points a plan's K/V source at another buffer: kv is [batch][kv_rows][pitch]
// bf16 with K and V in its last 2*heads*128 columns (pitch = 3D for a packed
// QKV buffer, 2D for a K|V buffer); the keys are rows [k_row0, k_row0 + k_rows).
cudaError_t plan_attn_kv(const void* kv, int64_t batch, int64_t kv_rows, int64_t pitch, int64_t k_row0,
                         int64_t k_rows, AttnPlan* plan);

// Merges partial attention states (attn_merge.cu): for each of n_units
// (row, head) units, (o_acc, ml_acc) := the log-sum-exp combination of itself
// and (o_part, ml_part) when o_part is not null; then, when out is not null,
// out = bf16(o_acc / l_acc). Layouts as AttnPlan's partial mode (o: 128 floats
// per unit, ml: 2 floats per unit); out: 128 bf16 per unit.
cudaError_t launch_attn_merge(float* o_acc, float* ml_acc, const float* o_part, const float* ml_part,
                              void* out, int64_t n_units, cudaStream_t stream);

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

// The library's own staging buffers for the host-buffer step (host_static.cu):
// packed QKV and output regions of one static device array, at fixed
// offsets, on the current device. The first call on a device looks the
// array's address up.
cudaError_t host_static_buffers(void** qkv_dev, void** out_dev);

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

// Y[M][N] = X[M][K] W[N][K]^T in bf16 with fp32 accumulation (gemm_bf16.cu);
// N a multiple of 256, K of 64. When stats is not null, stats[row][j] (row
// length stat_cols / 256) receives the fp64 sum of squares of the bf16 outputs
// of row `row` in columns [256 j, 256 j + 256), for j < stat_cols / 256.
cudaError_t launch_gemm_bf16(const void* x, const void* w, void* y, int64_t M, int64_t N, int64_t K,
                             double* stats, int64_t stat_cols, cudaStream_t stream);

// Device addresses (on the current device) of the words the kernels set when
// a bounded wait gives up, and of the Skip-Softmax counters ([0] (32-row
// group, key tile) pairs skipped, [1] P V products skipped). One copy of each
// per device, shared by every launch; the ABI takes and clears them
// atomically on the caller's stream.
cudaError_t attn_device_words(int** error_word, unsigned long long** skip_stats);
cudaError_t norm_error_word(int** word);
cudaError_t fp8_error_word(int** word);
cudaError_t gemm_error_word(int** word);

// Debug-bounds records of each kernel file (debug_bounds.cuh): two words,
// the first failed check and the count of failures.
cudaError_t bounds_words_norm(unsigned long long** words);
cudaError_t bounds_words_attn(unsigned long long** words);
cudaError_t bounds_words_fp8(unsigned long long** words);
cudaError_t bounds_words_quant(unsigned long long** words);
cudaError_t bounds_words_gemm(unsigned long long** words);
cudaError_t bounds_words_merge(unsigned long long** words);

}  // namespace wan
