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
// token, V untouched). A persistent grid (a few CTAs per SM) walks the tokens.
// A token's Q and K rows are contiguous in the packed buffer, so one bulk
// copy (cp.async.bulk, the untiled TMA) stages both into a shared-memory
// ring several tokens ahead of the threads that consume them; the reads of
// the next tokens are in flight while the current one is computed. Warps 0-3
// take the Q row, warps 4-7 the K row: thread u (0..127) of a row holds the
// 16-byte vectors u, u+128, ... in registers, the row's sum of squares is
// reduced with warp shuffles and one shared-memory exchange, and results go
// straight to global memory with 16-byte stores (in place). The vector
// stride (1024 elements = 8 heads) keeps every vector of a thread at the
// same head offset 8*(u%16), so a thread needs the rotations of 4 pairs.
//
// Precision: the result is meant to be the correctly rounded value of the
// definition, so that it matches an exact evaluation to 1 bf16 ulp everywhere
// (a flipped rounding of y is amplified by a later near-cancelling rotation).
//  - sum of squares in fp64 (bf16 values convert to doubles by bit moves);
//  - r kept as a float pair r_hi + r_lo; y = round(x*g*r) is decided from
//    v_hi = fl(x*g*r_hi), and recomputed exactly (sign of x*g*r - midpoint,
//    with two FMAs) for the rare threads whose v_hi lies within 2 fp32 ulps
//    of a bf16 rounding midpoint;
//  - cos/sin from one fp64 sincos per thread (shared through shared memory),
//    split as a 16-significant-bit head plus a float tail: the products of
//    the 8-bit y with the heads are exact in fp32, so the rotation's only
//    rounding is in the final sums.
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
constexpr int kThreads = 256;    // warps 0-3: the Q row of a token, warps 4-7: its K row
constexpr int kRowThreads = 128;
constexpr int kMaxStages = 8;
constexpr uint32_t kStageBudget = 72 * 1024;  // ring bytes per CTA (3 CTAs fit an SM)
constexpr uint64_t kWaitLimitNs = 1000000000ull;
// Pair index where the row axis and the column axis start (split 44/42/42).
constexpr int kRowAxisPair0 = 44 / 2;
constexpr int kColAxisPair0 = (44 + 42) / 2;

__device__ int g_norm_error_word;

struct NormRopeParams {
  uint16_t* qkv;
  const uint16_t* gamma_q;
  const uint16_t* gamma_k;
  int64_t tokens;        // batch * S
  int32_t S, H, W;
  int32_t D;             // heads * 128
  int32_t nvec;          // D / 8 sixteen-byte vectors per row
  int32_t stages;        // ring depth
  uint32_t stage_bytes;  // Q row + K row = 4 * D bytes
  double eps;
  double inv_d;
  double freq[kPairs];   // per pair of a head: theta^(-2j/d_axis)
};

// Shared-memory layout behind the ring (offsets from the ring's end).
struct alignas(16) NormSmemTail {
  uint64_t full[kMaxStages];
  double partial[2][8];            // per warp sums of squares, double-buffered by token parity
  float4 rot[2][kPairs];           // (cos head, cos tail, sin head, sin tail) per pair
  int abort;
};

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr));
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

// x^2 of both bf16 halves of w accumulated in fp64. A bf16 value's double has
// the high word ((f32 bits >> 3) & 0x0FFFFFFF) + ((1023-127) << 20) and a zero
// low word (the sign is dropped, irrelevant for a square; zero and subnormal
// inputs map to ~2^-127, whose square is below 1e-76).
__device__ __forceinline__ void sumsq_f64(uint32_t w, double& acc) {
  const uint32_t hi_lo = ((w << 13) & 0x0FFFE000u) + 0x38000000u;
  const uint32_t hi_hi = ((w >> 3) & 0x0FFFE000u) + 0x38000000u;
  const double a = __hiloint2double(static_cast<int>(hi_lo), 0);
  const double b = __hiloint2double(static_cast<int>(hi_hi), 0);
  acc = fma(a, a, acc);
  acc = fma(b, b, acc);
}

// Distance (in fp32 ulps, mod 2^16) of v's low 16 bits from 0x7FFE: values
// 0..4 mean v is within 2 ulps of a bf16 rounding midpoint.
__device__ __forceinline__ uint32_t near_midpoint(float v) {
  return (__float_as_uint(v) - 0x7FFEu) & 0xFFFFu;
}

// Correctly rounded bf16 (as 16 bits) of xg * (r_hi + r_lo), given
// v_hi = fl(xg * r_hi): compares the exact product with the midpoint M above
// v_hi's truncation using two FMAs (the sign of the result is exact).
__device__ __forceinline__ uint32_t round_exact(float xg, float r_hi, float r_lo) {
  const float v_hi = xg * r_hi;
  const uint32_t t = __float_as_uint(v_hi) >> 16;  // truncation toward zero (sign-magnitude)
  const float m = __uint_as_float((t << 16) | 0x8000u);
  const float d = fmaf(xg, r_lo, fmaf(xg, r_hi, -m));
  uint32_t up;
  if (d == 0.f) {
    up = t & 1u;  // exact tie: to even
  } else {
    up = ((__float_as_uint(d) ^ __float_as_uint(xg)) >> 31) ^ 1u;  // |v| beyond |M|
  }
  return (t + up) & 0xFFFFu;
}

// Rotation of one pair with the float-pair cos/sin (c = ch + cl, s = sh + sl).
__device__ __forceinline__ uint32_t rotate_pair(uint32_t yw, const float4& cs) {
  const float y0 = bf16_lo(yw), y1 = bf16_hi(yw);
  const float o0 = fmaf(y0, cs.x, -(y1 * cs.z)) + fmaf(y0, cs.y, -(y1 * cs.w));
  const float o1 = fmaf(y0, cs.z, y1 * cs.x) + fmaf(y0, cs.w, y1 * cs.y);
  return wan::sm100::pack_bf16x2(o0, o1);
}

__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

template <int VPT>
__global__ void __launch_bounds__(kThreads) qk_norm_rope_kernel(const __grid_constant__ NormRopeParams p) {
  using namespace wan::sm100;
  extern __shared__ __align__(128) uint8_t smem[];
  NormSmemTail& tail = *reinterpret_cast<NormSmemTail*>(smem + p.stages * p.stage_bytes);
  const uint32_t ring = smem_u32(smem);
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int which = warp >> 2;  // 0: Q, 1: K
  const int u = tid & (kRowThreads - 1);
  const int64_t step = gridDim.x;

  if (tid == 0) {
    for (int s = 0; s < p.stages; ++s) mbar_init(smem_u32(&tail.full[s]), 1);
    tail.abort = 0;
    fence_mbar_init();
  }
  __syncthreads();
  int64_t n_issued = 0;  // copies started (thread 0 only): iterations 0 .. n_issued-1
  if (tid == 0) {
    for (int s = 0; s < p.stages; ++s) {
      const int64_t tok = blockIdx.x + s * step;
      if (tok < p.tokens) {
        const uint32_t bar = smem_u32(&tail.full[s]);
        mbar_arrive_expect_tx(bar, p.stage_bytes);
        bulk_load(ring + s * p.stage_bytes, p.qkv + tok * 3 * static_cast<int64_t>(p.D), p.stage_bytes, bar);
        ++n_issued;
      }
    }
  }

  int64_t i = 0;
  for (int64_t tok = blockIdx.x; tok < p.tokens; tok += step, ++i) {
    const int stage = static_cast<int>(i % p.stages);
    const uint32_t parity = static_cast<uint32_t>((i / p.stages) & 1);
    const int buf = static_cast<int>(i & 1);
    if (!mbar_wait(smem_u32(&tail.full[stage]), parity, nullptr, kWaitLimitNs)) {
      tail.abort = 1;
      atomicOr(&g_norm_error_word, 1);
    }

    // This row's vectors, out of the staged token.
    const uint32_t src = ring + stage * p.stage_bytes + which * p.D * 2;
    uint4 v[VPT];
#pragma unroll
    for (int k = 0; k < VPT; ++k) {
      const int vi = u + kRowThreads * k;
      v[k] = vi < p.nvec ? ld_shared_v4(src + 16 * vi) : make_uint4(0, 0, 0, 0);
    }

    // The token's 64 rotations: one fp64 sincos on every 4th thread.
    const int s = static_cast<int>(tok % p.S);
    if ((tid & 3) == 0) {
      const int pr = tid >> 2;
      const int pos = pr < kRowAxisPair0 ? s / (p.H * p.W)
                                         : (pr < kColAxisPair0 ? (s / p.W) % p.H : s % p.W);
      double sd, cd;
      sincos(static_cast<double>(pos) * p.freq[pr], &sd, &cd);
      const float ch = __uint_as_float(__float_as_uint(static_cast<float>(cd)) & 0xFFFFFF00u);
      const float sh = __uint_as_float(__float_as_uint(static_cast<float>(sd)) & 0xFFFFFF00u);
      tail.rot[buf][pr] = make_float4(ch, static_cast<float>(cd - static_cast<double>(ch)), sh,
                                      static_cast<float>(sd - static_cast<double>(sh)));
    }

    double acc0 = 0.0, acc1 = 0.0, acc2 = 0.0, acc3 = 0.0;
#pragma unroll
    for (int k = 0; k < VPT; ++k) {
      sumsq_f64(v[k].x, acc0);
      sumsq_f64(v[k].y, acc1);
      sumsq_f64(v[k].z, acc2);
      sumsq_f64(v[k].w, acc3);
    }
    double ss = (acc0 + acc1) + (acc2 + acc3);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if (lane == 0) tail.partial[buf][warp] = ss;
    __syncthreads();  // the stage is consumed; partial sums and rotations are visible
    if (tail.abort) break;

    if (tid == 0) {
      const int64_t next = tok + p.stages * step;
      if (next < p.tokens) {
        const uint32_t bar = smem_u32(&tail.full[stage]);
        mbar_arrive_expect_tx(bar, p.stage_bytes);
        bulk_load(ring + stage * p.stage_bytes, p.qkv + next * 3 * static_cast<int64_t>(p.D),
                  p.stage_bytes, bar);
        ++n_issued;
      }
    }

    const double* part = &tail.partial[buf][4 * which];
    const double rd = 1.0 / sqrt(((part[0] + part[1]) + (part[2] + part[3])) * p.inv_d + p.eps);
    const float r_hi = static_cast<float>(rd);
    const float r_lo = static_cast<float>(rd - static_cast<double>(r_hi));
    const int pair0 = (u & 15) * 4;
    const float4 cs0 = tail.rot[buf][pair0], cs1 = tail.rot[buf][pair0 + 1];
    const float4 cs2 = tail.rot[buf][pair0 + 2], cs3 = tail.rot[buf][pair0 + 3];
    const uint16_t* g = which ? p.gamma_k : p.gamma_q;
    uint16_t* x = p.qkv + tok * 3 * static_cast<int64_t>(p.D) + which * p.D;
#pragma unroll
    for (int k = 0; k < VPT; ++k) {
      const int vi = u + kRowThreads * k;
      if (vi < p.nvec) {
        const uint4 gv = ld_cached(g + 8 * vi);
        const uint32_t xw[4] = {v[k].x, v[k].y, v[k].z, v[k].w};
        const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w};
        uint32_t yw[4];
        uint32_t near = 0xFFFFu;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float xg0 = bf16_lo(xw[e]) * bf16_lo(gw[e]);  // exact: 8-bit x 8-bit significands
          const float xg1 = bf16_hi(xw[e]) * bf16_hi(gw[e]);
          const float v0 = xg0 * r_hi, v1 = xg1 * r_hi;
          near = min(near, min(near_midpoint(v0), near_midpoint(v1)));
          yw[e] = pack_bf16x2(v0, v1);
        }
        if (near <= 4u) {
          // Rare: some v_hi is within 2 ulps of a rounding midpoint.
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const uint32_t lo = round_exact(bf16_lo(xw[e]) * bf16_lo(gw[e]), r_hi, r_lo);
            const uint32_t hi = round_exact(bf16_hi(xw[e]) * bf16_hi(gw[e]), r_hi, r_lo);
            yw[e] = lo | (hi << 16);
          }
        }
        uint4 o;
        o.x = rotate_pair(yw[0], cs0);
        o.y = rotate_pair(yw[1], cs1);
        o.z = rotate_pair(yw[2], cs2);
        o.w = rotate_pair(yw[3], cs3);
        st_v4(x + 8 * vi, o);
      }
    }
  }
  if (tail.abort && tid == 0) {
    // Let every copy this block started land before it exits.
    for (int s2 = 0; s2 < p.stages; ++s2) {
      const int64_t uses = n_issued > s2 ? (n_issued - s2 + p.stages - 1) / p.stages : 0;
      if (uses > 0) {
        mbar_wait(smem_u32(&tail.full[s2]), static_cast<uint32_t>((uses - 1) & 1), nullptr, kWaitLimitNs);
      }
    }
  }
  // Let a programmatically dependent launch (the attention kernel) start its
  // prologue; it still waits for this grid's completion before reading.
  grid_launch_dependents();
}

template <int VPT>
cudaError_t launch_vpt(const NormRopeParams& p, uint32_t smem_bytes, cudaStream_t stream) {
  static int blocks_per_sm = -1;  // per instantiation; the smem size is fixed per instantiation
  static uint32_t configured_smem = 0;
  if (configured_smem != smem_bytes) {
    cudaError_t e = cudaFuncSetAttribute(qk_norm_rope_kernel<VPT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem_bytes));
    if (e != cudaSuccess) return e;
    int n = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, qk_norm_rope_kernel<VPT>, kThreads, smem_bytes);
    if (e != cudaSuccess) return e;
    blocks_per_sm = n > 0 ? n : 1;
    configured_smem = smem_bytes;
  }
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  const int64_t want = static_cast<int64_t>(sms) * blocks_per_sm;
  const int64_t blocks = p.tokens < want ? p.tokens : want;
  qk_norm_rope_kernel<VPT><<<static_cast<unsigned>(blocks), kThreads, smem_bytes, stream>>>(p);
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
  p.tokens = batch * static_cast<int64_t>(p.S);
  p.stage_bytes = 4u * static_cast<uint32_t>(p.D);
  int stages = static_cast<int>(kStageBudget / p.stage_bytes);
  p.stages = stages < 2 ? 2 : (stages > kMaxStages ? kMaxStages : stages);
  p.eps = static_cast<double>(eps);
  p.inv_d = 1.0 / static_cast<double>(p.D);
  const int split[3] = {44, 42, 42};
  for (int pr = 0; pr < kPairs; ++pr) {
    const int axis = pr < kRowAxisPair0 ? 0 : (pr < kColAxisPair0 ? 1 : 2);
    const int j = pr - (axis == 0 ? 0 : (axis == 1 ? kRowAxisPair0 : kColAxisPair0));
    p.freq[pr] = std::pow(static_cast<double>(theta), -2.0 * j / static_cast<double>(split[axis]));
  }
  if (p.tokens == 0) return cudaSuccess;
  const uint32_t smem_bytes = p.stages * p.stage_bytes + static_cast<uint32_t>(sizeof(NormSmemTail));
  const int vpt = (p.nvec + kRowThreads - 1) / kRowThreads;  // 16-byte vectors per thread
  switch (vpt) {
    case 1: return launch_vpt<1>(p, smem_bytes, stream);
    case 2: return launch_vpt<2>(p, smem_bytes, stream);
    case 3: return launch_vpt<3>(p, smem_bytes, stream);
    case 4: return launch_vpt<4>(p, smem_bytes, stream);
    case 5: return launch_vpt<5>(p, smem_bytes, stream);
    case 6: return launch_vpt<6>(p, smem_bytes, stream);
    case 7: return launch_vpt<7>(p, smem_bytes, stream);
    default: return launch_vpt<8>(p, smem_bytes, stream);
  }
}

cudaError_t read_and_clear_norm_error(cudaStream_t stream, int32_t* code) {
  cudaError_t e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return e;
  int v = 0;
  e = cudaMemcpyFromSymbol(&v, g_norm_error_word, sizeof(int));
  if (e != cudaSuccess) return e;
  if (v != 0) {
    const int zero = 0;
    e = cudaMemcpyToSymbol(g_norm_error_word, &zero, sizeof(int));
    if (e != cudaSuccess) return e;
  }
  *code = v;
  return cudaSuccess;
}

}  // namespace wan
