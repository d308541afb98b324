// qk_norm_rope.cu -- Q/K RMSNorm + bf16 rounding + 3D RoPE, in place on the
// packed [B][S][3][heads][128] bf16 buffer (sm_100a).
//
// What it computes (TensorRT-LLM PR "[visual_gen] Optimize Wan2.2 Dataflow",
// section 1 and "Fused Q/K Norm and RoPE"; the review comments on that PR for
// the reduction width and the weight index):
//   r   = 1/sqrt(mean_{c<D} x_c^2 + eps)        fp32 sum over all heads of the token
//   y_c = bf16_rne(x_c * r * gamma[c])           the bf16 point before RoPE
//   (y_2i, y_2i+1) rotated by pos_axis * theta^(-2j/d_a) in fp32, rounded to bf16
// with head dims [0,44) on the frame axis, [44,86) on rows, [86,128) on columns.
//
// Design: the op is HBM-bound (read + write of Q and K once: 8*D bytes per
// token, V untouched). Two warps own one (token, Q-or-K) row of D elements:
// thread u (0..63) of the pair holds the 16-byte vectors u, u+64, u+128, ...
// of the row in registers, so the row is read once, reduced (warp shuffles,
// then one shared-memory exchange between the two warps), and written once.
// The vector stride is 512 elements = 4 heads, so every vector of a thread
// sits at the same head offset 8*(u%16): a thread needs the sines and cosines
// of only 4 pairs per token, computed once per row.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "sm100.cuh"
#include "wan_kernels.h"

namespace wan {
namespace {

constexpr int kHeadDim = 128;
constexpr int kPairs = kHeadDim / 2;
constexpr int kWarpsPerRow = 2;
constexpr int kRowThreads = 32 * kWarpsPerRow;
constexpr int kRowsPerBlock = 4;
constexpr int kThreads = kRowThreads * kRowsPerBlock;
// Pair index where the row axis and the column axis start (split 44/42/42).
constexpr int kRowAxisPair0 = 44 / 2;
constexpr int kColAxisPair0 = (44 + 42) / 2;

struct NormRopeParams {
  uint16_t* qkv;
  const uint16_t* gamma_q;
  const uint16_t* gamma_k;
  int64_t rows;  // batch * S * 2 (Q and K rows of each token)
  int32_t S, H, W;
  int32_t D;     // heads * 128
  int32_t nvec;  // D / 8 sixteen-byte vectors per row
  float eps;
  float inv_d;
  float freq_over_pi[kPairs];  // per pair of a head: theta^(-2j/d_axis) / pi
};

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }
__device__ __forceinline__ float round_bf16(float x) {
  return __bfloat162float(__float2bfloat16_rn(x));
}

__device__ __forceinline__ uint4 ld_stream(const uint16_t* p) {
  uint4 v;
  asm volatile("ld.global.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}
__device__ __forceinline__ uint4 ld_cached(const uint16_t* p) {
  return *reinterpret_cast<const uint4*>(p);
}
__device__ __forceinline__ void st_v4(uint16_t* p, uint4 v) {
  asm volatile("st.global.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w)
               : "memory");
}

__device__ __forceinline__ float sumsq(uint32_t w) {
  float a = bf16_lo(w), b = bf16_hi(w);
  return fmaf(a, a, b * b);
}

// One 32-bit word = one pair (x0 in the low half, x1 in the high half).
__device__ __forceinline__ uint32_t norm_rotate_pair(uint32_t xw, uint32_t gw, float r, float c,
                                                     float s) {
  const float y0 = round_bf16(bf16_lo(xw) * r * bf16_lo(gw));
  const float y1 = round_bf16(bf16_hi(xw) * r * bf16_hi(gw));
  const float o0 = y0 * c - y1 * s;
  const float o1 = y0 * s + y1 * c;
  return wan::sm100::pack_bf16x2(o0, o1);
}

template <int VPL>
__global__ void __launch_bounds__(kThreads, 2) qk_norm_rope_kernel(const __grid_constant__ NormRopeParams p) {
  __shared__ float partial[kRowsPerBlock * kWarpsPerRow];
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int u = threadIdx.x % kRowThreads;  // thread index within the row's warp pair
  const int64_t row = static_cast<int64_t>(blockIdx.x) * kRowsPerBlock + threadIdx.x / kRowThreads;
  const bool active = row < p.rows;
  const int64_t tok = row >> 1;
  const int which = static_cast<int>(row & 1);  // 0: Q, 1: K
  uint16_t* x = p.qkv + tok * 3 * static_cast<int64_t>(p.D) + which * p.D;
  const uint16_t* g = which ? p.gamma_k : p.gamma_q;

  uint4 v[VPL];
  float ss = 0.f;
#pragma unroll
  for (int k = 0; k < VPL; ++k) {
    const int vi = u + kRowThreads * k;
    v[k] = (active && vi < p.nvec) ? ld_stream(x + 8 * vi) : make_uint4(0, 0, 0, 0);
  }
#pragma unroll
  for (int k = 0; k < VPL; ++k) {
    ss += sumsq(v[k].x) + sumsq(v[k].y) + sumsq(v[k].z) + sumsq(v[k].w);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if (lane == 0) partial[warp] = ss;
  __syncthreads();
  const int w0 = (warp / kWarpsPerRow) * kWarpsPerRow;
  const float total = partial[w0] + partial[w0 + 1];
  const float r = 1.0f / sqrtf(total * p.inv_d + p.eps);

  if (active) {
    // Grid position of the token (width fastest) and this thread's 4 rotations.
    const int s = static_cast<int>(tok % p.S);
    const int hw = p.H * p.W;
    const int pos_f = s / hw;
    const int pos_h = (s / p.W) % p.H;
    const int pos_w = s % p.W;
    const int pair0 = (u & 15) * 4;
    float cs[4], sn[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int pr = pair0 + i;
      const int pos = pr < kRowAxisPair0 ? pos_f : (pr < kColAxisPair0 ? pos_h : pos_w);
      sincospif(static_cast<float>(pos) * p.freq_over_pi[pr], &sn[i], &cs[i]);
    }
#pragma unroll
    for (int k = 0; k < VPL; ++k) {
      const int vi = u + kRowThreads * k;
      if (vi < p.nvec) {
        const uint4 gv = ld_cached(g + 8 * vi);
        uint4 o;
        o.x = norm_rotate_pair(v[k].x, gv.x, r, cs[0], sn[0]);
        o.y = norm_rotate_pair(v[k].y, gv.y, r, cs[1], sn[1]);
        o.z = norm_rotate_pair(v[k].z, gv.z, r, cs[2], sn[2]);
        o.w = norm_rotate_pair(v[k].w, gv.w, r, cs[3], sn[3]);
        st_v4(x + 8 * vi, o);
      }
    }
  }
  // Let a programmatically dependent launch (the attention kernel) start its
  // prologue; it still waits for this grid's completion before reading.
  wan::sm100::grid_launch_dependents();
}

template <int VPL>
cudaError_t launch_vpl(const NormRopeParams& p, cudaStream_t stream) {
  const int64_t blocks = (p.rows + kRowsPerBlock - 1) / kRowsPerBlock;
  qk_norm_rope_kernel<VPL><<<static_cast<unsigned>(blocks), kThreads, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_qk_norm_rope(void* qkv, int64_t batch, int32_t F, int32_t H, int32_t W,
                                int32_t heads, const void* gamma_q, const void* gamma_k, float eps,
                                float theta, cudaStream_t stream) {
  NormRopeParams p;
  p.qkv = static_cast<uint16_t*>(qkv);
  p.gamma_q = static_cast<const uint16_t*>(gamma_q);
  p.gamma_k = static_cast<const uint16_t*>(gamma_k);
  p.S = F * H * W;
  p.H = H;
  p.W = W;
  p.D = heads * kHeadDim;
  p.nvec = p.D / 8;
  p.rows = batch * static_cast<int64_t>(p.S) * 2;
  p.eps = eps;
  p.inv_d = 1.0f / static_cast<float>(p.D);
  const int split[3] = {44, 42, 42};
  for (int pr = 0; pr < kPairs; ++pr) {
    const int axis = pr < kRowAxisPair0 ? 0 : (pr < kColAxisPair0 ? 1 : 2);
    const int j = pr - (axis == 0 ? 0 : (axis == 1 ? kRowAxisPair0 : kColAxisPair0));
    p.freq_over_pi[pr] = static_cast<float>(
        std::pow(static_cast<double>(theta), -2.0 * j / static_cast<double>(split[axis])) / M_PI);
  }
  if (p.rows == 0) return cudaSuccess;
  const int vpl = (p.nvec + kRowThreads - 1) / kRowThreads;  // 16-byte vectors per thread
  if (vpl <= 1) return launch_vpl<1>(p, stream);
  if (vpl <= 2) return launch_vpl<2>(p, stream);
  if (vpl <= 3) return launch_vpl<3>(p, stream);
  if (vpl <= 4) return launch_vpl<4>(p, stream);
  if (vpl <= 6) return launch_vpl<6>(p, stream);
  if (vpl <= 8) return launch_vpl<8>(p, stream);
  if (vpl <= 10) return launch_vpl<10>(p, stream);
  if (vpl <= 12) return launch_vpl<12>(p, stream);
  return launch_vpl<16>(p, stream);
}

}  // namespace wan
