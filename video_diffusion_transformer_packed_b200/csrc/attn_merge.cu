// attn_merge.cu -- merge of partial softmax-attention states (sm_100a).
//
// Context parallelism shards the token sequence; a rank's queries meet the
// keys one chunk at a time, each chunk of K/V arriving by a ring exchange
// that overlaps the attention of the previous one (AWS Neuron "Optimizing
// High-Quality Offline Video Generation", "Context parallelism" and "NKI
// kernels": ring_attention_const_max_fwd). A chunk's partial result is the
// state (O, m, l) of an online softmax over that key range,
//   O = sum_j 2^(a_j - m) v_j,   l = sum_j 2^(a_j - m),   a_j = scale log2(e) q . k_j,
// and two states over disjoint key ranges combine exactly:
//   m' = max(m1, m2),  O' = 2^(m1 - m') O1 + 2^(m2 - m') O2,  l' likewise,
// with the attention output O' / l' once every chunk is in.
//
// One warp per (row, head) unit: 128 fp32 of O as one float4 per lane, the
// (m, l) pair read by every lane (one 8-byte line). Purely HBM-bound: 2 x 512
// bytes read and 512 written per unit (+ 256 for the bf16 output).
#include <cuda_runtime.h>

#include <cstdint>

#include "debug_bounds.cuh"
#include "wan_kernels.h"

WAN_BOUNDS_WORDS(bounds_words_merge)

namespace wan {
namespace {

constexpr int kMergeThreads = 256;  // 8 units per block
constexpr int kHD = 128;

__device__ __forceinline__ uint32_t pack_bf16x2_rn(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

__global__ void __launch_bounds__(kMergeThreads)
    attn_merge_kernel(float* __restrict__ o_acc, float* __restrict__ ml_acc, const float* __restrict__ o_part,
                      const float* __restrict__ ml_part, uint16_t* __restrict__ out, int64_t n_units) {
  const int64_t unit = static_cast<int64_t>(blockIdx.x) * (kMergeThreads / 32) + (threadIdx.x >> 5);
  if (unit >= n_units) return;
  const int lane = threadIdx.x & 31;
  if (!WAN_BOUNDS(kMergeAcc, unit * kHD + 4 * lane, 4, n_units * kHD) || !WAN_BOUNDS(kMergeAcc, 2 * unit, 2, 2 * n_units)) {
    return;
  }
  float4* oa = reinterpret_cast<float4*>(o_acc + unit * kHD) + lane;
  float2 mla = reinterpret_cast<const float2*>(ml_acc)[unit];
  float4 o = *oa;
  if (o_part != nullptr && WAN_BOUNDS(kMergePart, unit * kHD + 4 * lane, 4, n_units * kHD) &&
      WAN_BOUNDS(kMergePart, 2 * unit, 2, 2 * n_units)) {
    const float2 mlp = reinterpret_cast<const float2*>(ml_part)[unit];
    const float4 op = reinterpret_cast<const float4*>(o_part + unit * kHD)[lane];
    const float m = fmaxf(mla.x, mlp.x);
    const float wa = exp2f(mla.x - m), wp = exp2f(mlp.x - m);
    o = make_float4(o.x * wa + op.x * wp, o.y * wa + op.y * wp, o.z * wa + op.z * wp, o.w * wa + op.w * wp);
    mla = make_float2(m, mla.y * wa + mlp.y * wp);
    *oa = o;
    if (lane == 0) reinterpret_cast<float2*>(ml_acc)[unit] = mla;
  }
  if (out != nullptr && WAN_BOUNDS(kMergeOut, unit * kHD + 4 * lane, 4, n_units * kHD)) {
    const float inv_l = 1.f / mla.y;
    reinterpret_cast<uint2*>(out + unit * kHD)[lane] =
        make_uint2(pack_bf16x2_rn(o.x * inv_l, o.y * inv_l), pack_bf16x2_rn(o.z * inv_l, o.w * inv_l));
  }
}

}  // namespace

cudaError_t launch_attn_merge(float* o_acc, float* ml_acc, const float* o_part, const float* ml_part,
                              void* out, int64_t n_units, cudaStream_t stream) {
  constexpr int64_t kUnitsPerBlock = kMergeThreads / 32;
  const int64_t blocks = (n_units + kUnitsPerBlock - 1) / kUnitsPerBlock;
  if (n_units < 1 || blocks > INT32_MAX || (o_part == nullptr) != (ml_part == nullptr) ||
      (o_part == nullptr && out == nullptr)) {
    return cudaErrorInvalidValue;
  }
  attn_merge_kernel<<<static_cast<unsigned>(blocks), kMergeThreads, 0, stream>>>(
      o_acc, ml_acc, o_part, ml_part, static_cast<uint16_t*>(out), n_units);
  return cudaGetLastError();
}

}  // namespace wan
