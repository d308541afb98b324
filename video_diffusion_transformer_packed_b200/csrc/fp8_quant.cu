// fp8_quant.cu -- the operands of the FP8 (e4m3) attention variant, from the
// packed bf16 [B][S][3][heads][128] buffer (sm_100a).
//
// The attention the pages time runs in FP8 with per-tensor scales (Neuron
// "Optimizing High-Quality Offline Video Generation" and the TensorRT-LLM PR's
// profiling of TE FP8 attention). A tensor X with scale s is stored as codes
//   c = e4m3(fl32(x * inv_s))        round to nearest even, saturating at +-448
// and stands for c * s. Q and K keep the packed token order ([B][S][2D]: Q
// then K of each token); V is stored transposed per (batch, head) --
// [B][heads][128][s_pitch], keys contiguous -- so that both products of the
// attention read K-major operands, and key columns past S hold code 0.
//
// qkv_amax_kernel gives the per-tensor absolute maxima a caller derives the
// scales from (one read of the buffer).
#include <cuda_runtime.h>

#include <cstdint>

#include "debug_bounds.cuh"
#include "sm100.cuh"
#include "wan_kernels.h"

WAN_BOUNDS_WORDS(bounds_words_quant)

namespace wan {
namespace {

constexpr int kTok = 128;      // tokens per quantisation block
constexpr int kThreads = 256;
constexpr int kVtPitch = 144;  // shared row pitch of the transposed V tile (16-byte multiple)

__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Eight bf16 values (one 16-byte vector) to eight e4m3 codes: fp32 product
// with inv, then round to nearest even with saturation.
__device__ __forceinline__ uint2 quant8(uint4 v, float inv) {
  uint2 r;
  r.x = wan::sm100::pack_e4m3x4(bf_lo(v.x) * inv, bf_hi(v.x) * inv, bf_lo(v.y) * inv, bf_hi(v.y) * inv);
  r.y = wan::sm100::pack_e4m3x4(bf_lo(v.z) * inv, bf_hi(v.z) * inv, bf_lo(v.w) * inv, bf_hi(v.w) * inv);
  return r;
}

// Block (token tile, head, batch): Q and K codes of 128 tokens written in
// place order; V codes gathered in shared memory and written transposed.
__global__ void __launch_bounds__(kThreads)
    quantize_fp8_kernel(const uint16_t* __restrict__ qkv, uint8_t* __restrict__ qk8,
                        uint8_t* __restrict__ v8t, int32_t S, int32_t heads, int64_t s_pitch,
                        float inv_q, float inv_k, float inv_v) {
  __shared__ __align__(16) uint8_t vt[128 * kVtPitch];  // [dim][token] codes
  const int s0 = blockIdx.x * kTok, h = blockIdx.y, b = blockIdx.z;
  const int64_t D = static_cast<int64_t>(heads) * 128;
  for (int idx = threadIdx.x; idx < kTok * 16; idx += kThreads) {
    const int t = idx >> 4, c = idx & 15;  // token in the tile, 8-element chunk of the head
    const int s = s0 + t;
    uint4 v = make_uint4(0, 0, 0, 0);
    const int64_t src_off = (static_cast<int64_t>(b) * S + s) * 3 * D + h * 128 + c * 8;
    const int64_t dst_off = (static_cast<int64_t>(b) * S + s) * 2 * D + h * 128 + c * 8;
    if (s < S && WAN_BOUNDS(kQuantLoad, src_off, 2 * D + 8, static_cast<int64_t>(gridDim.z) * S * 3 * D) &&
        WAN_BOUNDS(kQuantStoreQK, dst_off, D + 8, static_cast<int64_t>(gridDim.z) * S * 2 * D)) {
      const uint16_t* src = qkv + src_off;
      uint8_t* dst = qk8 + dst_off;
      const uint4 q = *reinterpret_cast<const uint4*>(src);
      const uint4 k = *reinterpret_cast<const uint4*>(src + D);
      v = *reinterpret_cast<const uint4*>(src + 2 * D);
      *reinterpret_cast<uint2*>(dst) = quant8(q, inv_q);
      *reinterpret_cast<uint2*>(dst + D) = quant8(k, inv_k);
    }
    const uint2 cv = quant8(v, inv_v);  // zeros past S: code 0
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const uint32_t w = e < 4 ? cv.x : cv.y;
      if (WAN_BOUNDS(kQuantStageV, (c * 8 + e) * kVtPitch + t, 1, 128 * kVtPitch)) {
        vt[(c * 8 + e) * kVtPitch + t] = static_cast<uint8_t>(w >> (8 * (e & 3)));
      }
    }
  }
  __syncthreads();
  // V^T rows: 128 dims x 128 tokens, 16 tokens per 16-byte store. s_pitch is
  // a multiple of 16, so a chunk is wholly inside or wholly past it.
  uint8_t* vrow = v8t + (static_cast<int64_t>(b) * heads + h) * 128 * s_pitch;
  for (int idx = threadIdx.x; idx < 128 * 8; idx += kThreads) {
    const int d = idx >> 3, c = idx & 7;
    const int64_t col = s0 + c * 16;
    if (col >= s_pitch) continue;
    if (!WAN_BOUNDS(kQuantStoreV, ((static_cast<int64_t>(b) * heads + h) * 128 + d) * s_pitch + col, 16,
                    static_cast<int64_t>(gridDim.z) * heads * 128 * s_pitch)) {
      continue;
    }
    *reinterpret_cast<uint4*>(vrow + d * s_pitch + col) =
        *reinterpret_cast<const uint4*>(&vt[d * kVtPitch + c * 16]);
  }
}

// max |x| of Q, K and V over the whole buffer into amax[0..2] (zeroed by the
// launcher); non-negative floats order like their bit patterns.
__global__ void __launch_bounds__(kThreads)
    qkv_amax_kernel(const uint16_t* __restrict__ qkv, int64_t tokens, int32_t D, float* amax) {
  const int chunks = 3 * D / 8;  // 16-byte vectors per token row
  float m[3] = {0.f, 0.f, 0.f};
  for (int64_t tok = blockIdx.x; tok < tokens; tok += gridDim.x) {
    const uint4* row = reinterpret_cast<const uint4*>(qkv + tok * 3 * static_cast<int64_t>(D));
    for (int c = threadIdx.x; c < chunks; c += kThreads) {
      if (!WAN_BOUNDS(kAmaxLoad, tok * 3 * static_cast<int64_t>(D) + 8 * c, 8, tokens * 3 * static_cast<int64_t>(D))) {
        continue;
      }
      const uint4 v = row[c];
      const int which = (c * 8) / D;
      float a = fmaxf(fmaxf(fabsf(bf_lo(v.x)), fabsf(bf_hi(v.x))), fmaxf(fabsf(bf_lo(v.y)), fabsf(bf_hi(v.y))));
      a = fmaxf(a, fmaxf(fmaxf(fabsf(bf_lo(v.z)), fabsf(bf_hi(v.z))), fmaxf(fabsf(bf_lo(v.w)), fabsf(bf_hi(v.w)))));
      m[which] = fmaxf(m[which], a);
    }
  }
#pragma unroll
  for (int w = 0; w < 3; ++w) {
    float x = m[w];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
    if ((threadIdx.x & 31) == 0) atomicMax(reinterpret_cast<int*>(&amax[w]), __float_as_int(x));
  }
}

}  // namespace

cudaError_t launch_quantize_fp8(const void* qkv, void* qk8, void* v8t, int64_t batch, int64_t S,
                                int32_t heads, int64_t s_pitch, float inv_q, float inv_k, float inv_v,
                                cudaStream_t stream) {
  const dim3 grid(static_cast<unsigned>((S + kTok - 1) / kTok), static_cast<unsigned>(heads),
                  static_cast<unsigned>(batch));
  quantize_fp8_kernel<<<grid, kThreads, 0, stream>>>(static_cast<const uint16_t*>(qkv),
                                                     static_cast<uint8_t*>(qk8), static_cast<uint8_t*>(v8t),
                                                     static_cast<int32_t>(S), heads, s_pitch, inv_q, inv_k,
                                                     inv_v);
  return cudaGetLastError();
}

cudaError_t launch_qkv_amax(const void* qkv, int64_t tokens, int32_t heads, float* amax, cudaStream_t stream) {
  cudaError_t e = cudaMemsetAsync(amax, 0, 3 * sizeof(float), stream);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t blocks = tokens < 8LL * sms ? tokens : 8LL * sms;
  qkv_amax_kernel<<<static_cast<unsigned>(blocks), kThreads, 0, stream>>>(static_cast<const uint16_t*>(qkv),
                                                                         tokens, heads * 128, amax);
  return cudaGetLastError();
}

}  // namespace wan
