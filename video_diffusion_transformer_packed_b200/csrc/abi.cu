// abi.cu -- the extern "C" boundary (include/wan_attn.h): argument
// validation, device check, and the launches. No allocation, no fallback.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <mutex>

#include "wan_attn.h"  // include/ is on the include path
#include "wan_kernels.h"

namespace {

constexpr int32_t kAbiVersion = 12;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Compute capability 10.0 only: the kernels are built for sm_100a.
int32_t check_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return WAN_ERR_UNSUPPORTED_DEVICE;
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
    return WAN_ERR_UNSUPPORTED_DEVICE;
  }
  return (major == 10 && minor == 0) ? WAN_OK : WAN_ERR_UNSUPPORTED_DEVICE;
}

int32_t check_heads(int32_t heads, int32_t head_dim) {
  if (head_dim != WAN_HEAD_DIM) return WAN_ERR_HEAD_DIM;
  if (heads < 1 || heads > WAN_MAX_HEADS) return WAN_ERR_SHAPE;
  return WAN_OK;
}

int32_t check_tokens(int64_t batch, int64_t seq_len, int32_t heads) {
  if (batch < 1 || seq_len < 1 || seq_len > INT32_MAX) return WAN_ERR_SHAPE;
  // Elements of the packed buffer must fit comfortably in int64, and the
  // attention grid (batch * heads * ceil(S/256)) in a 31-bit grid dimension.
  const int64_t d3 = 3 * static_cast<int64_t>(heads) * WAN_HEAD_DIM;
  if (batch > (INT64_MAX / 4) / (seq_len * d3)) return WAN_ERR_SHAPE;
  if (batch > (int64_t)INT32_MAX) return WAN_ERR_SHAPE;
  const int64_t ctas = batch * heads * ((seq_len + 255) / 256);
  if (ctas > INT32_MAX) return WAN_ERR_SHAPE;
  // TMA tensor-map limits: each dimension < 2^32 and strides < 2^40 bytes.
  if (static_cast<uint64_t>(seq_len) * static_cast<uint64_t>(d3) * 2ull >= (1ull << 40))
    return WAN_ERR_SHAPE;
  return WAN_OK;
}

int32_t check_grid(int64_t batch, int32_t F, int32_t H, int32_t W, int32_t heads, int64_t* S) {
  if (F < 1 || H < 1 || W < 1) return WAN_ERR_SHAPE;
  const int64_t s = static_cast<int64_t>(F) * H * W;
  if (s > INT32_MAX) return WAN_ERR_SHAPE;
  *S = s;
  return check_tokens(batch, s, heads);
}

int32_t check_norm_args(void* qkv, const void* gq, const void* gk, float eps, float theta) {
  if (!qkv || !gq || !gk) return WAN_ERR_NULL;
  if (!aligned16(qkv) || !aligned16(gq) || !aligned16(gk)) return WAN_ERR_ALIGN;
  if (!(std::isfinite(eps) && eps > 0.f)) return WAN_ERR_PARAM;
  if (!(std::isfinite(theta) && theta > 1.f)) return WAN_ERR_PARAM;
  return WAN_OK;
}

int32_t check_attn_args(const void* qkv, const void* out, int64_t batch, int64_t S, int32_t heads,
                        float scale) {
  if (!qkv || !out) return WAN_ERR_NULL;
  if (!aligned16(qkv) || !aligned16(out)) return WAN_ERR_ALIGN;
  if (!std::isfinite(scale)) return WAN_ERR_PARAM;
  const uint64_t d = static_cast<uint64_t>(heads) * WAN_HEAD_DIM;
  const uint64_t qkv_bytes = static_cast<uint64_t>(batch) * S * 3 * d * 2;
  const uint64_t out_bytes = static_cast<uint64_t>(batch) * S * d * 2;
  const uint64_t a0 = reinterpret_cast<uintptr_t>(qkv), a1 = a0 + qkv_bytes;
  const uint64_t b0 = reinterpret_cast<uintptr_t>(out), b1 = b0 + out_bytes;
  if (a0 < b1 && b0 < a1) return WAN_ERR_ALIAS;
  return WAN_OK;
}

// Host buffers must be page-locked (pinned or registered) so that the copies
// run asynchronously; device buffers must be memory of the current device.
int32_t check_memory_kind(const void* host_in, const void* host_out, const void* dev_a,
                          const void* dev_b) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return WAN_ERR_UNSUPPORTED_DEVICE;
  for (const void* p : {host_in, host_out}) {
    cudaPointerAttributes at;
    if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
      (void)cudaGetLastError();
      return WAN_ERR_MEMORY_KIND;
    }
    if (at.type != cudaMemoryTypeHost) return WAN_ERR_MEMORY_KIND;
  }
  for (const void* p : {dev_a, dev_b}) {
    cudaPointerAttributes at;
    if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
      (void)cudaGetLastError();
      return WAN_ERR_MEMORY_KIND;
    }
    if (at.type != cudaMemoryTypeDevice || at.device != dev) return WAN_ERR_MEMORY_KIND;
  }
  return WAN_OK;
}

bool positive_finite(float x) { return std::isfinite(x) && x > 0.f; }
bool overlaps(const void* a, uint64_t na, const void* b, uint64_t nb) {
  const uint64_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
  return a0 < b0 + nb && b0 < a0 + na;
}

#define WAN_TRY(expr)          \
  do {                         \
    const int32_t _s = (expr); \
    if (_s != WAN_OK) return _s; \
  } while (0)

// Status of a plan or launch: a kernel whose compiled register count differs
// from the one its per-warpgroup register split was written for is refused
// by the launcher with cudaErrorInvalidKernelImage, and gets its own status.
int32_t launch_status(cudaError_t e) {
  if (e == cudaSuccess) return WAN_OK;
  return e == cudaErrorInvalidKernelImage ? WAN_ERR_KERNEL_IMAGE : WAN_ERR_LAUNCH;
}

#define WAN_LAUNCH_TRY(expr) WAN_TRY(launch_status(expr))

// The kernels' device error words and the Skip-Softmax counters: one copy of
// each per device, shared by every launch on that device. They are taken
// (read and cleared in one atomic exchange each) by a one-thread kernel on
// the caller's stream, so a word set between the read and the clear cannot be
// lost; the taken values land in g_taken, which a mutex keeps to one reader
// at a time.
struct TakenWords {
  int attn, norm, fp8, gemm;
  unsigned long long skip[2];
};
__device__ TakenWords g_taken;

__global__ void take_words_kernel(int* attn, int* norm, int* fp8, int* gemm, unsigned long long* skip) {
  TakenWords t = {0, 0, 0, 0, {0ull, 0ull}};
  if (attn) t.attn = atomicExch(attn, 0);
  if (norm) t.norm = atomicExch(norm, 0);
  if (fp8) t.fp8 = atomicExch(fp8, 0);
  if (gemm) t.gemm = atomicExch(gemm, 0);
  if (skip) {
    t.skip[0] = atomicExch(&skip[0], 0ull);
    t.skip[1] = atomicExch(&skip[1], 0ull);
  }
  g_taken = t;
}

std::mutex g_take_mutex;

// errors: take the four error words; skip: take the Skip-Softmax counters.
cudaError_t take_device_words(cudaStream_t stream, bool errors, bool skip, TakenWords* out) {
  int *attn = nullptr, *norm = nullptr, *fp8 = nullptr, *gemm = nullptr;
  unsigned long long* skip_stats = nullptr;
  cudaError_t e = wan::attn_device_words(&attn, &skip_stats);
  if (e == cudaSuccess && errors) e = wan::norm_error_word(&norm);
  if (e == cudaSuccess && errors) e = wan::fp8_error_word(&fp8);
  if (e == cudaSuccess && errors) e = wan::gemm_error_word(&gemm);
  if (e != cudaSuccess) return e;
  if (!errors) attn = nullptr;
  if (!skip) skip_stats = nullptr;
  std::lock_guard<std::mutex> lock(g_take_mutex);
  take_words_kernel<<<1, 1, 0, stream>>>(attn, norm, fp8, gemm, skip_stats);
  e = cudaGetLastError();
  if (e == cudaSuccess) e = cudaMemcpyFromSymbolAsync(out, g_taken, sizeof(TakenWords), 0, cudaMemcpyDeviceToHost, stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
  return e;
}

}  // namespace

extern "C" {

const char* wan_status_string(int32_t status) {
  switch (status) {
    case WAN_OK: return "ok";
    case WAN_ERR_NULL: return "a required pointer is NULL";
    case WAN_ERR_ALIGN: return "a pointer is not 16-byte aligned";
    case WAN_ERR_SHAPE: return "batch, token grid or head count out of range";
    case WAN_ERR_HEAD_DIM: return "head_dim must be 128";
    case WAN_ERR_PARAM: return "eps, theta or scale is not finite or out of range";
    case WAN_ERR_UNSUPPORTED_DEVICE: return "the current device is not compute capability 10.0 (sm_100a)";
    case WAN_ERR_LAUNCH: return "the CUDA runtime rejected a launch";
    case WAN_ERR_DEVICE_TIMEOUT: return "a bounded wait inside the attention kernel gave up";
    case WAN_ERR_ALIAS: return "out overlaps qkv";
    case WAN_ERR_MEMORY_KIND:
      return "a host buffer is not page-locked, or a device buffer is not memory of the current device";
    case WAN_ERR_TOO_LARGE:
      return "the step does not fit wan_dit_attn_host_static's device buffer (WAN_HOST_STATIC_MAX_ELEMENTS)";
    case WAN_ERR_BOUNDS: return "a device-side index check of the debug-bounds build failed (wan_debug_bounds)";
    case WAN_ERR_KERNEL_IMAGE:
      return "a compiled attention kernel's register count differs from the one its register split was "
             "written for: rebuild the library with the CUDA toolkit it targets";
    default: return "unknown status";
  }
}

int32_t wan_abi_version(void) { return kAbiVersion; }

int32_t wan_qk_norm_rope(void* qkv, int64_t batch, int32_t F, int32_t H, int32_t W, int32_t heads,
                         int32_t head_dim, const void* gamma_q, const void* gamma_k, float eps,
                         float theta, void* stream) {
  int64_t S = 0;
  WAN_TRY(check_heads(heads, head_dim));
  WAN_TRY(check_grid(batch, F, H, W, heads, &S));
  WAN_TRY(check_norm_args(qkv, gamma_q, gamma_k, eps, theta));
  WAN_TRY(check_device());
  (void)cudaGetLastError();
  if (wan::launch_qk_norm_rope(qkv, batch, F, H, W, heads, gamma_q, gamma_k, eps, theta,
                               static_cast<cudaStream_t>(stream)) != cudaSuccess) {
    return WAN_ERR_LAUNCH;
  }
  return WAN_OK;
}

int32_t wan_self_attention(const void* qkv, void* out, int64_t batch, int64_t seq_len,
                           int32_t heads, int32_t head_dim, float scale, void* stream) {
  WAN_TRY(check_heads(heads, head_dim));
  WAN_TRY(check_tokens(batch, seq_len, heads));
  WAN_TRY(check_attn_args(qkv, out, batch, seq_len, heads, scale));
  WAN_TRY(check_device());
  (void)cudaGetLastError();
  wan::AttnPlan plan;
  WAN_LAUNCH_TRY(wan::plan_attn_fwd(qkv, out, batch, seq_len, heads, scale, &plan));
  if (wan::launch_attn_fwd(plan, static_cast<cudaStream_t>(stream), false) != cudaSuccess) {
    return WAN_ERR_LAUNCH;
  }
  return WAN_OK;
}

int32_t wan_self_attention_sparse(const void* qkv, void* out, int64_t batch, int64_t seq_len,
                                  int32_t heads, int32_t head_dim, float scale, float threshold,
                                  void* stream) {
  WAN_TRY(check_heads(heads, head_dim));
  WAN_TRY(check_tokens(batch, seq_len, heads));
  WAN_TRY(check_attn_args(qkv, out, batch, seq_len, heads, scale));
  if (!(std::isfinite(threshold) && threshold >= 0.f && threshold <= 1.f)) return WAN_ERR_PARAM;
  WAN_TRY(check_device());
  (void)cudaGetLastError();
  wan::AttnPlan plan;
  WAN_LAUNCH_TRY(wan::plan_attn_fwd(qkv, out, batch, seq_len, heads, scale, &plan));
  plan.skip_threshold = threshold;
  if (wan::launch_attn_fwd(plan, static_cast<cudaStream_t>(stream), false) != cudaSuccess) {
    return WAN_ERR_LAUNCH;
  }
  return WAN_OK;
}

int32_t wan_qkv_amax(const void* qkv, int64_t batch, int64_t seq_len, int32_t heads, int32_t head_dim,
                     float* amax, void* stream) {
  WAN_TRY(check_heads(heads, head_dim));
  WAN_TRY(check_tokens(batch, seq_len, heads));
  if (!qkv || !amax) return WAN_ERR_NULL;
  if (!aligned16(qkv) || (reinterpret_cast<uintptr_t>(amax) & 3u)) return WAN_ERR_ALIGN;
  WAN_TRY(check_device());
  (void)cudaGetLastError();
  if (wan::launch_qkv_amax(qkv, batch * seq_len, heads, amax, static_cast<cudaStream_t>(stream)) !=
      cudaSuccess) {
    return WAN_ERR_LAUNCH;
  }
  return WAN_OK;
}

namespace {
int32_t check_fp8_buffers(int64_t batch, int64_t S, int32_t heads, int64_t s_pitch, const void* qk8,
                          const void* v8t, const void* other, uint64_t other_bytes) {
  if (!qk8 || !v8t || !other) return WAN_ERR_NULL;
  if (!aligned16(qk8) || !aligned16(v8t) || !aligned16(other)) return WAN_ERR_ALIGN;
  if (s_pitch < S || s_pitch % 16 != 0 || s_pitch > (int64_t)INT32_MAX) return WAN_ERR_SHAPE;
  const uint64_t d = static_cast<uint64_t>(heads) * WAN_HEAD_DIM;
  const uint64_t qk_bytes = static_cast<uint64_t>(batch) * S * 2 * d;
  const uint64_t vt_bytes = static_cast<uint64_t>(batch) * d * s_pitch;
  if (overlaps(qk8, qk_bytes, v8t, vt_bytes) || overlaps(qk8, qk_bytes, other, other_bytes) ||
      overlaps(v8t, vt_bytes, other, other_bytes)) {
    return WAN_ERR_ALIAS;
  }
  return WAN_OK;
}
}  // namespace

int32_t wan_quantize_fp8(const void* qkv, void* qk8, void* v8t, int64_t batch, int64_t seq_len, int32_t heads,
                         int32_t head_dim, int64_t s_pitch, float inv_scale_q, float inv_scale_k,
                         float inv_scale_v, void* stream) {
  WAN_TRY(check_heads(heads, head_dim));
  WAN_TRY(check_tokens(batch, seq_len, heads));
  const uint64_t qkv_bytes = static_cast<uint64_t>(batch) * seq_len * 3 * heads * WAN_HEAD_DIM * 2;
  WAN_TRY(check_fp8_buffers(batch, seq_len, heads, s_pitch, qk8, v8t, qkv, qkv_bytes));
  if (!positive_finite(inv_scale_q) || !positive_finite(inv_scale_k) || !positive_finite(inv_scale_v)) {
    return WAN_ERR_PARAM;
  }
  WAN_TRY(check_device());
  (void)cudaGetLastError();
  if (wan::launch_quantize_fp8(qkv, qk8, v8t, batch, seq_len, heads, s_pitch, inv_scale_q, inv_scale_k,
                               inv_scale_v, static_cast<cudaStream_t>(stream)) != cudaSuccess) {
    return WAN_ERR_LAUNCH;
  }
  return WAN_OK;
}

int32_t wan_self_attention_fp8(const void* qk8, const void* v8t, void* out, int64_t batch, int64_t seq_len,
                               int32_t heads, int32_t head_dim, int64_t s_pitch, float scale, float scale_q,
                               float scale_k, float scale_v, void* stream) {
  WAN_TRY(check_heads(heads, head_dim));
  WAN_TRY(check_tokens(batch, seq_len, heads));
  const uint64_t out_bytes = static_cast<uint64_t>(batch) * seq_len * heads * WAN_HEAD_DIM * 2;
  WAN_TRY(check_fp8_buffers(batch, seq_len, heads, s_pitch, qk8, v8t, out, out_bytes));
  if (!std::isfinite(scale) || !positive_finite(scale_q) || !positive_finite(scale_k) ||
      !positive_finite(scale_v)) {
    return WAN_ERR_PARAM;
  }
  WAN_TRY(check_device());
  (void)cudaGetLastError();
  WAN_LAUNCH_TRY(wan::launch_attn_fp8(qk8, v8t, out, batch, seq_len, heads, s_pitch, scale, scale_q, scale_k,
                                      scale_v, static_cast<cudaStream_t>(stream)));
  return WAN_OK;
}

int32_t wan_linear(const void* x, const void* w, void* y, int64_t M, int64_t N, int64_t K, double* stats,
                   int64_t stat_cols, void* stream) {
  if (!x || !w || !y) return WAN_ERR_NULL;
  if (!aligned16(x) || !aligned16(w) || !aligned16(y)) return WAN_ERR_ALIGN;
  if (stats && (reinterpret_cast<uintptr_t>(stats) & 7u)) return WAN_ERR_ALIGN;
  if (M < 1 || N < 256 || K < 64 || N % 256 != 0 || K % 64 != 0) return WAN_ERR_SHAPE;
  if (M > (1LL << 31) || N > (1LL << 24) || K > (1LL << 24)) return WAN_ERR_SHAPE;
  if (stats && (stat_cols < 256 || stat_cols % 256 != 0 || stat_cols > N)) return WAN_ERR_SHAPE;
  const uint64_t xb = static_cast<uint64_t>(M) * K * 2, wb = static_cast<uint64_t>(N) * K * 2;
  const uint64_t yb = static_cast<uint64_t>(M) * N * 2;
  if (overlaps(y, yb, x, xb) || overlaps(y, yb, w, wb)) return WAN_ERR_ALIAS;
  if (stats && overlaps(stats, static_cast<uint64_t>(M) * (stat_cols / 256) * 8, y, yb)) return WAN_ERR_ALIAS;
  WAN_TRY(check_device());
  (void)cudaGetLastError();
  if (wan::launch_gemm_bf16(x, w, y, M, N, K, stats, stats ? stat_cols : 0, static_cast<cudaStream_t>(stream)) !=
      cudaSuccess) {
    return WAN_ERR_LAUNCH;
  }
  return WAN_OK;
}

int32_t wan_qk_norm_rope_stats(void* qkv, int64_t batch, int32_t F, int32_t H, int32_t W, int32_t heads,
                               int32_t head_dim, const void* gamma_q, const void* gamma_k, float eps, float theta,
                               const double* stats, void* stream) {
  int64_t S = 0;
  WAN_TRY(check_heads(heads, head_dim));
  WAN_TRY(check_grid(batch, F, H, W, heads, &S));
  WAN_TRY(check_norm_args(qkv, gamma_q, gamma_k, eps, theta));
  if (!stats) return WAN_ERR_NULL;
  if (reinterpret_cast<uintptr_t>(stats) & 7u) return WAN_ERR_ALIGN;
  if ((heads * WAN_HEAD_DIM) % 256 != 0) return WAN_ERR_SHAPE;  // whole 256-column statistic tiles
  WAN_TRY(check_device());
  (void)cudaGetLastError();
  if (wan::launch_qk_norm_rope(qkv, batch, F, H, W, heads, gamma_q, gamma_k, eps, theta,
                               static_cast<cudaStream_t>(stream), stats) != cudaSuccess) {
    return WAN_ERR_LAUNCH;
  }
  return WAN_OK;
}

int32_t wan_qk_norm_rope_shard(void* qkv, int64_t batch, int32_t F, int32_t H, int32_t W, int64_t s0,
                               int64_t s_local, int32_t heads, int32_t head_dim, const void* gamma_q,
                               const void* gamma_k, float eps, float theta, void* stream) {
  int64_t S = 0;
  WAN_TRY(check_heads(heads, head_dim));
  WAN_TRY(check_grid(batch, F, H, W, heads, &S));
  if (s0 < 0 || s_local < 1 || s0 + s_local > S) return WAN_ERR_SHAPE;
  WAN_TRY(check_norm_args(qkv, gamma_q, gamma_k, eps, theta));
  WAN_TRY(check_device());
  (void)cudaGetLastError();
  if (wan::launch_qk_norm_rope(qkv, batch, F, H, W, heads, gamma_q, gamma_k, eps, theta,
                               static_cast<cudaStream_t>(stream), nullptr, s0, s_local) != cudaSuccess) {
    return WAN_ERR_LAUNCH;
  }
  return WAN_OK;
}

int32_t wan_self_attention_rows(const void* qkv, void* out, int64_t batch, int64_t seq_len, int32_t heads,
                                int32_t head_dim, int64_t q_row0, int64_t q_rows, float scale, void* stream) {
  WAN_TRY(check_heads(heads, head_dim));
  WAN_TRY(check_tokens(batch, seq_len, heads));
  if (q_row0 < 0 || q_rows < 1 || q_row0 + q_rows > seq_len) return WAN_ERR_SHAPE;
  if (!qkv || !out) return WAN_ERR_NULL;
  if (!aligned16(qkv) || !aligned16(out)) return WAN_ERR_ALIGN;
  if (!std::isfinite(scale)) return WAN_ERR_PARAM;
  const uint64_t d = static_cast<uint64_t>(heads) * WAN_HEAD_DIM;
  if (overlaps(qkv, static_cast<uint64_t>(batch) * seq_len * 3 * d * 2, out,
               static_cast<uint64_t>(batch) * q_rows * d * 2)) {
    return WAN_ERR_ALIAS;
  }
  WAN_TRY(check_device());
  (void)cudaGetLastError();
  wan::AttnPlan plan;
  WAN_LAUNCH_TRY(wan::plan_attn_fwd(qkv, out, batch, seq_len, heads, scale, &plan));
  plan.q_row0 = static_cast<int32_t>(q_row0);
  plan.q_rows = static_cast<int32_t>(q_rows);
  if (wan::launch_attn_fwd(plan, static_cast<cudaStream_t>(stream), false) != cudaSuccess) return WAN_ERR_LAUNCH;
  return WAN_OK;
}

}  // extern "C"

namespace {
int32_t partial_attention(const void* q_qkv, int64_t q_seq_len, int64_t q_row0, int64_t q_rows, const void* kv,
                          int64_t kv_rows, int64_t kv_pitch, int64_t k_row0, int64_t k_rows, float* o, float* ml,
                          int64_t batch, int32_t heads, int32_t head_dim, float scale, bool accumulate,
                          void* stream) {
  WAN_TRY(check_heads(heads, head_dim));
  WAN_TRY(check_tokens(batch, q_seq_len, heads));
  if (!q_qkv || !kv || !o || !ml) return WAN_ERR_NULL;
  if (!aligned16(q_qkv) || !aligned16(kv) || !aligned16(o) || !aligned16(ml)) return WAN_ERR_ALIGN;
  const int64_t d = static_cast<int64_t>(heads) * WAN_HEAD_DIM;
  if (q_row0 < 0 || q_rows < 1 || q_row0 + q_rows > q_seq_len) return WAN_ERR_SHAPE;
  if (kv_rows < 1 || kv_rows > INT32_MAX || k_row0 < 0 || k_rows < 1 || k_row0 + k_rows > kv_rows) {
    return WAN_ERR_SHAPE;
  }
  // K and V are the last 2D columns of each kv row; rows are whole 16-byte units.
  if (kv_pitch < 2 * d || kv_pitch % 8 != 0 || kv_pitch > (int64_t)INT32_MAX) return WAN_ERR_SHAPE;
  if (batch > (INT64_MAX / 4) / (kv_rows * kv_pitch)) return WAN_ERR_SHAPE;
  if (static_cast<uint64_t>(kv_rows) * static_cast<uint64_t>(kv_pitch) * 2ull >= (1ull << 40)) return WAN_ERR_SHAPE;
  if (!std::isfinite(scale)) return WAN_ERR_PARAM;
  const uint64_t q_bytes = static_cast<uint64_t>(batch) * q_seq_len * 3 * d * 2;
  const uint64_t kv_bytes = static_cast<uint64_t>(batch) * kv_rows * kv_pitch * 2;
  const uint64_t o_bytes = static_cast<uint64_t>(batch) * q_rows * d * 4;
  const uint64_t ml_bytes = static_cast<uint64_t>(batch) * q_rows * heads * 8;
  if (overlaps(o, o_bytes, ml, ml_bytes) || overlaps(o, o_bytes, q_qkv, q_bytes) ||
      overlaps(o, o_bytes, kv, kv_bytes) || overlaps(ml, ml_bytes, q_qkv, q_bytes) ||
      overlaps(ml, ml_bytes, kv, kv_bytes)) {
    return WAN_ERR_ALIAS;
  }
  WAN_TRY(check_device());
  (void)cudaGetLastError();
  wan::AttnPlan plan;
  WAN_LAUNCH_TRY(wan::plan_attn_fwd(q_qkv, nullptr, batch, q_seq_len, heads, scale, &plan));
  WAN_LAUNCH_TRY(wan::plan_attn_kv(kv, batch, kv_rows, kv_pitch, k_row0, k_rows, &plan));
  plan.q_row0 = static_cast<int32_t>(q_row0);
  plan.q_rows = static_cast<int32_t>(q_rows);
  plan.o_part = o;
  plan.ml_part = ml;
  plan.accumulate = accumulate;
  WAN_LAUNCH_TRY(wan::launch_attn_fwd(plan, static_cast<cudaStream_t>(stream), false));
  return WAN_OK;
}
}  // namespace

extern "C" {

int32_t wan_self_attention_partial(const void* q_qkv, int64_t q_seq_len, int64_t q_row0, int64_t q_rows,
                                   const void* kv, int64_t kv_rows, int64_t kv_pitch, int64_t k_row0,
                                   int64_t k_rows, float* o, float* ml, int64_t batch, int32_t heads,
                                   int32_t head_dim, float scale, void* stream) {
  return partial_attention(q_qkv, q_seq_len, q_row0, q_rows, kv, kv_rows, kv_pitch, k_row0, k_rows, o, ml, batch,
                           heads, head_dim, scale, false, stream);
}

int32_t wan_self_attention_accumulate(const void* q_qkv, int64_t q_seq_len, int64_t q_row0, int64_t q_rows,
                                      const void* kv, int64_t kv_rows, int64_t kv_pitch, int64_t k_row0,
                                      int64_t k_rows, float* o, float* ml, int64_t batch, int32_t heads,
                                      int32_t head_dim, float scale, void* stream) {
  return partial_attention(q_qkv, q_seq_len, q_row0, q_rows, kv, kv_rows, kv_pitch, k_row0, k_rows, o, ml, batch,
                           heads, head_dim, scale, true, stream);
}

int32_t wan_attention_merge(float* o_acc, float* ml_acc, const float* o_part, const float* ml_part, void* out,
                            int64_t n_units, int32_t head_dim, void* stream) {
  if (head_dim != WAN_HEAD_DIM) return WAN_ERR_HEAD_DIM;
  if (!o_acc || !ml_acc) return WAN_ERR_NULL;
  if ((o_part == nullptr) != (ml_part == nullptr) || (o_part == nullptr && out == nullptr)) return WAN_ERR_NULL;
  if (!aligned16(o_acc) || !aligned16(ml_acc) || (o_part && !aligned16(o_part)) ||
      (ml_part && !aligned16(ml_part)) || (out && !aligned16(out))) {
    return WAN_ERR_ALIGN;
  }
  if (n_units < 1 || n_units > (INT64_MAX / 1024)) return WAN_ERR_SHAPE;
  const uint64_t ob = static_cast<uint64_t>(n_units) * WAN_HEAD_DIM * 4, mb = static_cast<uint64_t>(n_units) * 8;
  const uint64_t yb = static_cast<uint64_t>(n_units) * WAN_HEAD_DIM * 2;
  if (overlaps(o_acc, ob, ml_acc, mb) ||
      (o_part && (overlaps(o_part, ob, o_acc, ob) || overlaps(o_part, ob, ml_acc, mb) ||
                  overlaps(ml_part, mb, o_acc, ob) || overlaps(ml_part, mb, ml_acc, mb))) ||
      (out && (overlaps(out, yb, o_acc, ob) || overlaps(out, yb, ml_acc, mb) ||
               (o_part && (overlaps(out, yb, o_part, ob) || overlaps(out, yb, ml_part, mb)))))) {
    return WAN_ERR_ALIAS;
  }
  WAN_TRY(check_device());
  (void)cudaGetLastError();
  WAN_LAUNCH_TRY(wan::launch_attn_merge(o_acc, ml_acc, o_part, ml_part, out, n_units,
                                        static_cast<cudaStream_t>(stream)));
  return WAN_OK;
}

int32_t wan_skip_stats(void* stream, int64_t* group_tiles, int64_t* products) {
  TakenWords t;
  if (take_device_words(static_cast<cudaStream_t>(stream), false, true, &t) != cudaSuccess) return WAN_ERR_LAUNCH;
  if (group_tiles) *group_tiles = static_cast<int64_t>(t.skip[0]);
  if (products) *products = static_cast<int64_t>(t.skip[1]);
  return WAN_OK;
}

int32_t wan_dit_attn(void* qkv, void* out, int64_t batch, int32_t F, int32_t H, int32_t W,
                     int32_t heads, int32_t head_dim, const void* gamma_q, const void* gamma_k,
                     float eps, float theta, float scale, void* stream) {
  int64_t S = 0;
  WAN_TRY(check_heads(heads, head_dim));
  WAN_TRY(check_grid(batch, F, H, W, heads, &S));
  WAN_TRY(check_norm_args(qkv, gamma_q, gamma_k, eps, theta));
  WAN_TRY(check_attn_args(qkv, out, batch, S, heads, scale));
  WAN_TRY(check_device());
  (void)cudaGetLastError();
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  wan::AttnPlan plan;
  WAN_LAUNCH_TRY(wan::plan_attn_fwd(qkv, out, batch, S, heads, scale, &plan));
  if (wan::launch_qk_norm_rope(qkv, batch, F, H, W, heads, gamma_q, gamma_k, eps, theta, st) !=
      cudaSuccess) {
    return WAN_ERR_LAUNCH;
  }
  if (wan::launch_attn_fwd(plan, st, true) != cudaSuccess) {
    return WAN_ERR_LAUNCH;
  }
  return WAN_OK;
}

int32_t wan_dit_attn_host(const void* qkv_host, void* out_host, void* qkv_dev, void* out_dev,
                          int64_t batch, int32_t F, int32_t H, int32_t W, int32_t heads,
                          int32_t head_dim, const void* gamma_q, const void* gamma_k, float eps,
                          float theta, float scale, int32_t heads_per_chunk, int32_t flags, void* stream) {
  int64_t S = 0;
  WAN_TRY(check_heads(heads, head_dim));
  WAN_TRY(check_grid(batch, F, H, W, heads, &S));
  if (!qkv_host || !out_host) return WAN_ERR_NULL;
  WAN_TRY(check_norm_args(qkv_dev, gamma_q, gamma_k, eps, theta));
  WAN_TRY(check_attn_args(qkv_dev, out_dev, batch, S, heads, scale));
  if (heads_per_chunk < 0 || heads_per_chunk > heads) return WAN_ERR_PARAM;
  if (flags & ~WAN_HOST_OVERLAP_INPUT) return WAN_ERR_PARAM;
  const int32_t hc = heads_per_chunk > 0 ? heads_per_chunk
                                         : (heads < WAN_HOST_HEADS_PER_CHUNK ? heads : WAN_HOST_HEADS_PER_CHUNK);
  if (batch * ((heads + hc - 1) / hc) > WAN_HOST_MAX_PIECES) return WAN_ERR_SHAPE;
  WAN_TRY(check_device());
  WAN_TRY(check_memory_kind(qkv_host, out_host, qkv_dev, out_dev));
  (void)cudaGetLastError();
  wan::HostStep step;
  step.qkv_host = qkv_host;
  step.out_host = out_host;
  step.qkv_dev = qkv_dev;
  step.out_dev = out_dev;
  step.batch = batch;
  step.S = S;
  step.F = F;
  step.H = H;
  step.W = W;
  step.heads = heads;
  step.heads_per_chunk = hc;
  step.gamma_q = gamma_q;
  step.gamma_k = gamma_k;
  step.eps = eps;
  step.theta = theta;
  step.scale = scale;
  step.overlap_input = (flags & WAN_HOST_OVERLAP_INPUT) != 0;
  WAN_LAUNCH_TRY(wan::enqueue_dit_attn_host(step, static_cast<cudaStream_t>(stream)));
  return WAN_OK;
}

int32_t wan_dit_attn_host_static(const void* qkv_host, void* out_host, int64_t batch, int32_t F, int32_t H,
                                 int32_t W, int32_t heads, int32_t head_dim, const void* gamma_q,
                                 const void* gamma_k, float eps, float theta, float scale,
                                 int32_t heads_per_chunk, int32_t flags, void* stream) {
  int64_t S = 0;
  WAN_TRY(check_heads(heads, head_dim));
  WAN_TRY(check_grid(batch, F, H, W, heads, &S));
  if (!qkv_host || !out_host || !gamma_q || !gamma_k) return WAN_ERR_NULL;
  if (!aligned16(gamma_q) || !aligned16(gamma_k)) return WAN_ERR_ALIGN;
  if (!(std::isfinite(eps) && eps > 0.f) || !(std::isfinite(theta) && theta > 1.f)) return WAN_ERR_PARAM;
  if (!std::isfinite(scale)) return WAN_ERR_PARAM;
  if (heads_per_chunk < 0 || heads_per_chunk > heads) return WAN_ERR_PARAM;
  if (flags & ~WAN_HOST_OVERLAP_INPUT) return WAN_ERR_PARAM;
  const int32_t hc = heads_per_chunk > 0 ? heads_per_chunk
                                         : (heads < WAN_HOST_HEADS_PER_CHUNK ? heads : WAN_HOST_HEADS_PER_CHUNK);
  if (batch * ((heads + hc - 1) / hc) > WAN_HOST_MAX_PIECES) return WAN_ERR_SHAPE;
  // batch * S * heads * 128 elements must fit the library's static buffer.
  if (batch > WAN_HOST_STATIC_MAX_ELEMENTS / (S * heads * WAN_HEAD_DIM)) return WAN_ERR_TOO_LARGE;
  WAN_TRY(check_device());
  for (const void* p : {qkv_host, static_cast<const void*>(out_host)}) {
    cudaPointerAttributes at;
    if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
      (void)cudaGetLastError();
      return WAN_ERR_MEMORY_KIND;
    }
    if (at.type != cudaMemoryTypeHost) return WAN_ERR_MEMORY_KIND;
  }
  (void)cudaGetLastError();
  void* qkv_dev = nullptr;
  void* out_dev = nullptr;
  if (wan::host_static_buffers(&qkv_dev, &out_dev) != cudaSuccess) return WAN_ERR_LAUNCH;
  wan::HostStep step;
  step.qkv_host = qkv_host;
  step.out_host = out_host;
  step.qkv_dev = qkv_dev;
  step.out_dev = out_dev;
  step.batch = batch;
  step.S = S;
  step.F = F;
  step.H = H;
  step.W = W;
  step.heads = heads;
  step.heads_per_chunk = hc;
  step.gamma_q = gamma_q;
  step.gamma_k = gamma_k;
  step.eps = eps;
  step.theta = theta;
  step.scale = scale;
  step.overlap_input = (flags & WAN_HOST_OVERLAP_INPUT) != 0;
  WAN_LAUNCH_TRY(wan::enqueue_dit_attn_host(step, static_cast<cudaStream_t>(stream)));
  return WAN_OK;
}

int32_t wan_selftest_wait_timeout(const void* qkv, void* out, int64_t batch, int64_t seq_len,
                                  int32_t heads, int32_t head_dim, int64_t wait_limit_ns, void* stream) {
  WAN_TRY(check_heads(heads, head_dim));
  WAN_TRY(check_tokens(batch, seq_len, heads));
  WAN_TRY(check_attn_args(qkv, out, batch, seq_len, heads, 0.f));
  if (wait_limit_ns < 1000 || wait_limit_ns > 2000000000) return WAN_ERR_PARAM;
  WAN_TRY(check_device());
  (void)cudaGetLastError();
  wan::AttnPlan plan;
  WAN_LAUNCH_TRY(wan::plan_attn_fwd(qkv, out, batch, seq_len, heads, 0.f, &plan));
  if (wan::launch_attn_fwd(plan, static_cast<cudaStream_t>(stream), false,
                           static_cast<uint64_t>(wait_limit_ns), true) != cudaSuccess) {
    return WAN_ERR_LAUNCH;
  }
  return WAN_OK;
}

int32_t wan_debug_bounds(void* stream, int32_t* enabled, uint64_t* first_fault, uint64_t* count) {
  if (!enabled || !first_fault || !count) return WAN_ERR_NULL;
  *first_fault = 0;
  *count = 0;
#ifdef WAN_DEBUG_BOUNDS
  *enabled = 1;
  using Words = cudaError_t (*)(unsigned long long**);
  const Words files[] = {wan::bounds_words_norm, wan::bounds_words_attn, wan::bounds_words_fp8,
                         wan::bounds_words_quant, wan::bounds_words_gemm, wan::bounds_words_merge};
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return WAN_ERR_LAUNCH;
  for (Words words : files) {
    unsigned long long* w = nullptr;
    unsigned long long h[2] = {0ull, 0ull};
    if (words(&w) != cudaSuccess || cudaMemcpy(h, w, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess ||
        cudaMemset(w, 0, sizeof(h)) != cudaSuccess) {
      return WAN_ERR_LAUNCH;
    }
    if (*first_fault == 0) *first_fault = h[0];
    *count += h[1];
  }
  return *count != 0 ? WAN_ERR_BOUNDS : WAN_OK;
#else
  (void)stream;
  *enabled = 0;
  return WAN_OK;
#endif
}

int32_t wan_device_error(void* stream, int32_t* code) {
  if (!code) return WAN_ERR_NULL;
  *code = 0;
  TakenWords t;
  if (take_device_words(static_cast<cudaStream_t>(stream), true, false, &t) != cudaSuccess) return WAN_ERR_LAUNCH;
  *code = (t.attn & 0xFF) | ((t.norm & 0xFF) << 8) | ((t.fp8 & 0xFF) << 16) | ((t.gemm & 0x7F) << 24);
  return *code != 0 ? WAN_ERR_DEVICE_TIMEOUT : WAN_OK;
}

}  // extern "C"
