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
// token, V untouched). A persistent grid (a few CTAs per SM) walks the
// tokens, each CTA a contiguous range of them.
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
//  - cos/sin in fp64, one pair per thread of the first two warps, carried
//    from token to token by the angle-addition formulas (a CTA's tokens are
//    consecutive, so a pair's position mostly stays or steps by one) with a
//    fresh sincospi at every jump; shared through shared memory, split as a
//    16-significant-bit head plus a float tail: the products of the 8-bit y
//    with the heads are exact in fp32, so the rotation's only rounding is in
//    the final sums.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <mutex>

#include "debug_bounds.cuh"
#include "sm100.cuh"
#include "wan_kernels.h"

WAN_BOUNDS_WORDS(bounds_words_norm)

namespace wan {
namespace {

using wan::sm100::f2;
using wan::sm100::f2_split;
using wan::sm100::fma2;
using wan::sm100::mul2;

constexpr int kHeadDim = 128;
constexpr int kPairs = kHeadDim / 2;
constexpr int kThreads = 256;    // warps 0-3: the Q row of a token, warps 4-7: its K row
constexpr int kRowThreads = 128;
constexpr int kMaxStages = 8;
constexpr uint32_t kStageBudget = 48 * 1024;  // ring bytes per CTA
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
  int32_t S, H, W;       // S: tokens per batch element in this buffer
  int32_t s0;            // grid index of the buffer's first token (a sequence shard starts past 0)
  int32_t D;             // heads * 128
  int32_t nvec;          // D / 8 sixteen-byte vectors per row
  int32_t stages;        // ring depth
  uint32_t stage_bytes;  // Q row + K row = 4 * D bytes
  double eps;
  double inv_d;
  // Optional sums of squares from the QKV projection's epilogue
  // (gemm_bf16.cu): stats[token][j], j < stat_row; Q's partials are
  // j < stat_half, K's the next stat_half. Used by the kStats instantiation.
  const double* stats;
  int32_t stat_row, stat_half;
  double freq_pi[kPairs];  // per pair of a head: theta^(-2j/d_axis) / pi
};

// Cos/sin of the pairs' rotation angles, kept in shared memory from one
// token to the next (by the thread that owns the pair). A CTA walks a
// contiguous range of tokens, so a pair's axis position (frame, row or
// column of the token) mostly stays or grows by one: growing by one turns the
// angle by the pair's frequency (the angle-addition formulas in fp64, four
// multiply-adds); anything else -- the first token, a wrap to 0, a jump at a
// batch boundary, and every 64th position to bound the recurrence's rounding
// drift -- is one fp64 sincospi.
struct PairRotations {
  double2 cs[kPairs];    // (cos, sin) of pos * freq
  double2 step[kPairs];  // (cos, sin) of freq
  int pos[kPairs];       // the axis position cs belongs to; -1: none yet
};

// Shared-memory layout behind the ring (offsets from the ring's end).
struct alignas(16) NormSmemTail {
  uint64_t full[kMaxStages];
  double partial[2][8];            // per warp sums of squares, double-buffered by token parity
  // Rotation operands, for two pairs a = 4g + 2h and b = a + 1 at once, as
  // f32x2 lanes (a, b): rot[buf][h][0][g] = (ch, ch | sh, sh),
  // [1] = (-sh, -sh | cl, cl), [2] = (sl, sl | -sl, -sl) -- cos/sin heads and
  // tails. A warp reads the 16 entries of one (h, j): contiguous, no bank
  // conflicts. The table of iteration i+1 is written during iteration i.
  float4 rot[3][2][3][16];
  PairRotations rs;
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

__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

// Grid coordinates (frame, row, column) of sequence index s_glob.
struct GridPos {
  int f, r, c;
};
__device__ __forceinline__ GridPos grid_pos(const NormRopeParams& p, int s_glob) {
  const int q = s_glob / p.W;  // frame * H + row
  GridPos g;
  g.f = q / p.H;
  g.r = q - g.f * p.H;
  g.c = s_glob - q * p.W;
  return g;
}

// Moves pair pr's rotation to the grid position g and returns its (cos, sin).
__device__ __forceinline__ double2 rotation_move(const NormRopeParams& p, PairRotations& rs, int pr,
                                                 const GridPos& g) {
  const int pos = pr < kRowAxisPair0 ? g.f : (pr < kColAxisPair0 ? g.r : g.c);
  const int old = rs.pos[pr];
  double2 cs = rs.cs[pr];
  if (pos == old) return cs;
  if (pos == old + 1 && (pos & 63) != 0) {
    const double2 st = rs.step[pr];
    cs = make_double2(fma(cs.x, st.x, -cs.y * st.y), fma(cs.y, st.x, cs.x * st.y));
  } else {
    sincospi(static_cast<double>(pos) * p.freq_pi[pr], &cs.y, &cs.x);  // angle = pos * freq
  }
  rs.cs[pr] = cs;
  rs.pos[pr] = pos;
  return cs;
}

// The rotation operands of pair `pr`: cos/sin split into a 16-significant-bit
// head and a float tail, written into the pair's lane of the two-pair table
// entry.
__device__ __forceinline__ void rotation_write(double2 cs, int pr, float4 (&t)[2][3][16]) {
  const float ch = __uint_as_float(__float_as_uint(static_cast<float>(cs.x)) & 0xFFFFFF00u);
  const float sh = __uint_as_float(__float_as_uint(static_cast<float>(cs.y)) & 0xFFFFFF00u);
  const float cl = static_cast<float>(cs.x - static_cast<double>(ch));
  const float sl = static_cast<float>(cs.y - static_cast<double>(sh));
  const int g = pr >> 2, h = (pr >> 1) & 1, side = pr & 1;
  float* t0 = reinterpret_cast<float*>(&t[h][0][g]);
  float* t1 = reinterpret_cast<float*>(&t[h][1][g]);
  float* t2 = reinterpret_cast<float*>(&t[h][2][g]);
  t0[side] = ch;
  t0[2 + side] = sh;
  t1[side] = -sh;
  t1[2 + side] = cl;
  t2[side] = sl;
  t2[2 + side] = -sl;
}

// Exact products of the two bf16 halves of a and b (8-bit x 8-bit
// significands fit a float): one mixed-precision FMA per half, no unpacking.
__device__ __forceinline__ void prod_bf16x2(uint32_t a, uint32_t b, float& lo, float& hi) {
  asm("{\n\t.reg .b16 al, ah, bl, bh;\n\t"
      "mov.b32 {al, ah}, %2;\n\t"
      "mov.b32 {bl, bh}, %3;\n\t"
      "fma.rn.f32.bf16 %0, al, bl, 0f00000000;\n\t"
      "fma.rn.f32.bf16 %1, ah, bh, 0f00000000;\n\t}"
      : "=f"(lo), "=f"(hi)
      : "r"(a), "r"(b));
}

// Exact fp64 value of a non-negative float with a 16-bit significand (a
// square of a bf16): high word (bits >> 3) + ((1023-127) << 20), zero low
// word. Zero and subnormal squares map to about 2^-127, negligible next to eps.
__device__ __forceinline__ double square_to_f64(float sq) {
  return __hiloint2double(static_cast<int>(__umulhi(__float_as_uint(sq), 1u << 29) + 0x38000000u), 0);
}

// x^2 of both bf16 halves of w accumulated in fp64.
__device__ __forceinline__ void sumsq_pair(uint32_t w, double& acc_lo, double& acc_hi) {
  float s0, s1;
  prod_bf16x2(w, w, s0, s1);
  acc_lo += square_to_f64(s0);
  acc_hi += square_to_f64(s1);
}

// One pair: v = x*g*r_hi (x*g is exact) rounded to bf16. `near` keeps the
// per-16-bit-lane minimum of (low 16 bits of v) + 0x8002, which is below 8
// when v lies within a few fp32 ulps of a bf16 rounding midpoint (a carry
// from the low lane only widens the high lane's window).
__device__ __forceinline__ uint32_t norm_round(uint32_t xw, uint32_t gw, uint64_t r2, uint32_t& near) {
  float xg0, xg1;
  prod_bf16x2(xw, gw, xg0, xg1);
  const uint64_t v = mul2(f2(xg0, xg1), r2);
  float v0, v1;
  f2_split(v, v0, v1);
  const uint32_t lows = __byte_perm(__float_as_uint(v0), __float_as_uint(v1), 0x5410);
  near = __vminu2(near, lows + 0x80028002u);
  return wan::sm100::pack_bf16x2(v0, v1);
}

// Rotation of two adjacent pairs a = (y0, y1) in wa and b = (y2, y3) in wb,
// lanes (a, b) of f32x2 operations: (y0 ch - y1 sh, y0 sh + y1 ch) per pair.
// The head products (8-bit y x 16-bit head) are exact, so each head sum is
// rounded once; the tails add their (2^-16 smaller) share.
__device__ __forceinline__ void rotate2(uint32_t& wa, uint32_t& wb, const float4& t0, const float4& t1,
                                        const float4& t2) {
  const uint64_t ye = f2(bf16_lo(wa), bf16_lo(wb));  // (y0, y2)
  const uint64_t yo = f2(bf16_hi(wa), bf16_hi(wb));  // (y1, y3)
  const uint64_t ch = f2(t0.x, t0.y), sh = f2(t0.z, t0.w);
  const uint64_t nsh = f2(t1.x, t1.y), cl = f2(t1.z, t1.w);
  const uint64_t sl = f2(t2.x, t2.y), nsl = f2(t2.z, t2.w);
  uint64_t e = fma2(ye, ch, mul2(yo, nsh));
  e = fma2(yo, nsl, e);
  e = fma2(ye, cl, e);
  uint64_t o = fma2(ye, sh, mul2(yo, ch));
  o = fma2(yo, cl, o);
  o = fma2(ye, sl, o);
  float e0, e1, o0, o1;
  f2_split(e, e0, e1);
  f2_split(o, o0, o1);
  wa = wan::sm100::pack_bf16x2(e0, o0);
  wb = wan::sm100::pack_bf16x2(e1, o1);
}

template <int VPT, bool kStats>
__global__ void __launch_bounds__(kThreads, 3) qk_norm_rope_kernel(const __grid_constant__ NormRopeParams p) {
  using namespace wan::sm100;
  extern __shared__ __align__(128) uint8_t smem[];
  NormSmemTail& tail = *reinterpret_cast<NormSmemTail*>(smem + p.stages * p.stage_bytes);
  const uint32_t ring = smem_u32(smem);
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int which = warp >> 2;  // 0: Q, 1: K
  const int u = tid & (kRowThreads - 1);
  // This CTA's tokens: a contiguous range, the remainder spread one token
  // each over the first CTAs.
  const int64_t per_cta = p.tokens / gridDim.x, extra = p.tokens % gridDim.x;
  const int64_t t_begin = blockIdx.x * per_cta + (blockIdx.x < extra ? blockIdx.x : extra);
  const int64_t t_end = t_begin + per_cta + (blockIdx.x < extra ? 1 : 0);

  if (tid == 0) {
    for (int s = 0; s < p.stages; ++s) mbar_init(smem_u32(&tail.full[s]), 1);
    tail.abort = 0;
    fence_mbar_init();
  }
  __syncthreads();
  int64_t n_issued = 0;  // copies started (thread 0 only): iterations 0 .. n_issued-1
  if (tid == 0) {
    for (int s = 0; s < p.stages; ++s) {
      const int64_t tok = t_begin + s;
      if (tok < t_end &&
          WAN_BOUNDS(kNormLoad, tok * 3 * static_cast<int64_t>(p.D), 2 * p.D, p.tokens * 3 * static_cast<int64_t>(p.D))) {
        const uint32_t bar = smem_u32(&tail.full[s]);
        mbar_arrive_expect_tx(bar, p.stage_bytes);
        bulk_load(ring + s * p.stage_bytes, p.qkv + tok * 3 * static_cast<int64_t>(p.D), p.stage_bytes, bar);
        ++n_issued;
      }
    }
  }

  const uint16_t* g = which ? p.gamma_k : p.gamma_q;

  // Threads 0-63 own the rotations of pairs 0-63 and keep them, with the
  // sequence index and grid position of the next token, from one token to
  // the next (no division in the loop but at a batch boundary).
  const bool rot_thread = tid < kPairs;
  int s_next = static_cast<int>(t_begin % p.S);
  GridPos gp_next = grid_pos(p, s_next + p.s0);
  if (rot_thread) {
    double2 st;
    sincospi(p.freq_pi[tid], &st.y, &st.x);
    tail.rs.step[tid] = st;
    tail.rs.pos[tid] = -1;
    rotation_write(rotation_move(p, tail.rs, tid, gp_next), tid, tail.rot[0]);
    if (++s_next == p.S) {
      s_next = 0;
      gp_next = grid_pos(p, p.s0);
    } else if (++gp_next.c == p.W) {
      gp_next.c = 0;
      if (++gp_next.r == p.H) {
        gp_next.r = 0;
        ++gp_next.f;
      }
    }
  }
  __syncthreads();

  int stage = 0, rbuf = 0;
  uint32_t parity = 0;
  int64_t i = 0;
  for (int64_t tok = t_begin; tok < t_end; ++tok, ++i) {
    const int buf = static_cast<int>(i & 1);
    // With precomputed statistics, lane j of each warp fetches the row's j-th
    // partial sum now; the load's latency hides behind the ring wait.
    double st_part = 0.0;
    if constexpr (kStats) {
      if (lane < p.stat_half &&
          WAN_BOUNDS(kNormStats, tok * p.stat_row + which * p.stat_half + lane, 1, p.tokens * p.stat_row)) {
        st_part = p.stats[tok * p.stat_row + which * p.stat_half + lane];
      }
    }
    // The next token's rotations, ahead of time (they do not depend on the data).
    const int rnext = rbuf == 2 ? 0 : rbuf + 1;
    if (rot_thread && tok + 1 < t_end) {
      rotation_write(rotation_move(p, tail.rs, tid, gp_next), tid, tail.rot[rnext]);
      if (++s_next == p.S) {
        s_next = 0;
        gp_next = grid_pos(p, p.s0);
      } else if (++gp_next.c == p.W) {
        gp_next.c = 0;
        if (++gp_next.r == p.H) {
          gp_next.r = 0;
          ++gp_next.f;
        }
      }
    }
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
      v[k] = vi < p.nvec && WAN_BOUNDS(kNormStage, which * p.D * 2 + 16 * vi, 16, static_cast<int64_t>(p.stage_bytes))
                 ? ld_shared_v4(src + 16 * vi)
                 : make_uint4(0, 0, 0, 0);
    }

    if constexpr (!kStats) {
      double acc[8] = {0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0};
#pragma unroll
      for (int k = 0; k < VPT; ++k) {
        sumsq_pair(v[k].x, acc[0], acc[1]);
        sumsq_pair(v[k].y, acc[2], acc[3]);
        sumsq_pair(v[k].z, acc[4], acc[5]);
        sumsq_pair(v[k].w, acc[6], acc[7]);
      }
      double ss = ((acc[0] + acc[1]) + (acc[2] + acc[3])) + ((acc[4] + acc[5]) + (acc[6] + acc[7]));
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      if (lane == 0) tail.partial[buf][warp] = ss;
    }
    __syncthreads();  // the stage is consumed; partial sums and rotations are visible
    if (tail.abort) break;

    if (tid == 0) {
      const int64_t next = tok + p.stages;
      if (next < t_end &&
          WAN_BOUNDS(kNormLoad, next * 3 * static_cast<int64_t>(p.D), 2 * p.D, p.tokens * 3 * static_cast<int64_t>(p.D))) {
        const uint32_t bar = smem_u32(&tail.full[stage]);
        mbar_arrive_expect_tx(bar, p.stage_bytes);
        bulk_load(ring + stage * p.stage_bytes, p.qkv + next * 3 * static_cast<int64_t>(p.D),
                  p.stage_bytes, bar);
        ++n_issued;
      }
    }

    double total;
    if constexpr (kStats) {
      // the same fixed tree in every warp: every thread gets the same sum
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) st_part += __shfl_xor_sync(0xffffffffu, st_part, o);
      total = st_part;
    } else {
      const double* part = &tail.partial[buf][4 * which];
      total = (part[0] + part[1]) + (part[2] + part[3]);
    }
    const double rd = rsqrt(total * p.inv_d + p.eps);
    const float r_hi = static_cast<float>(rd);
    const float r_lo = static_cast<float>(rd - static_cast<double>(r_hi));
    const uint64_t r2 = f2(r_hi, r_hi);
    uint16_t* x = p.qkv + tok * 3 * static_cast<int64_t>(p.D) + which * p.D;

    // Pass A: y = bf16(x * g * r) for every pair held by this thread (written
    // over x), with the exact rounding for the rare vectors near a rounding
    // midpoint.
    uint32_t (&y)[VPT][4] = *reinterpret_cast<uint32_t(*)[VPT][4]>(v);
#pragma unroll
    for (int k = 0; k < VPT; ++k) {
      const int vi = u + kRowThreads * k;
      // gammas: L1-resident, the same channels for every token
      const uint4 gv = vi < p.nvec && WAN_BOUNDS(kNormGamma, 8 * vi, 8, p.D) ? ld_cached(g + 8 * vi) : make_uint4(0, 0, 0, 0);
      const uint32_t xw[4] = {v[k].x, v[k].y, v[k].z, v[k].w};
      const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w};
      uint32_t near = 0xFFFFFFFFu;
      uint32_t yk[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) yk[e] = norm_round(xw[e], gw[e], r2, near);
      if ((near & 0xFFF8u) == 0u || (near & 0xFFF80000u) == 0u) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const uint32_t lo = round_exact(bf16_lo(xw[e]) * bf16_lo(gw[e]), r_hi, r_lo);
          const uint32_t hi = round_exact(bf16_hi(xw[e]) * bf16_hi(gw[e]), r_hi, r_lo);
          yk[e] = lo | (hi << 16);
        }
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) y[k][e] = yk[e];
    }
    // Pass B: rotate, two pair positions (of the 4 per thread) at a time so
    // that only their cos/sin operands are live.
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const float4 t0 = tail.rot[rbuf][h][0][u & 15];
      const float4 t1 = tail.rot[rbuf][h][1][u & 15];
      const float4 t2 = tail.rot[rbuf][h][2][u & 15];
#pragma unroll
      for (int k = 0; k < VPT; ++k) rotate2(y[k][2 * h], y[k][2 * h + 1], t0, t1, t2);
    }
#pragma unroll
    for (int k = 0; k < VPT; ++k) {
      const int vi = u + kRowThreads * k;
      if (vi < p.nvec && WAN_BOUNDS(kNormStore, tok, 1, p.tokens) && WAN_BOUNDS(kNormColumn, 8 * vi, 8, p.D)) {
        st_v4(x + 8 * vi, make_uint4(y[k][0], y[k][1], y[k][2], y[k][3]));
      }
    }
    rbuf = rnext;
    if (++stage == p.stages) {
      stage = 0;
      parity ^= 1u;
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

template <int VPT, bool kStats>
cudaError_t launch_vpt(const NormRopeParams& p, uint32_t smem_bytes, cudaStream_t stream) {
  // Per device: the dynamic shared-memory limit set so far and the
  // occupancy at the last size (the size depends on the hidden width).
  struct DeviceState {
    uint32_t attr_smem = 0, occ_smem = 0;
    int blocks_per_sm = 1, sms = 0;
  };
  static std::mutex mu;
  static DeviceState state[kMaxDevices];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  int blocks_per_sm = 1, sms = 0;
  {
    std::lock_guard<std::mutex> lock(mu);
    DeviceState& st = state[dev];
    if (st.sms == 0) {
      e = cudaDeviceGetAttribute(&st.sms, cudaDevAttrMultiProcessorCount, dev);
      if (e != cudaSuccess) return e;
    }
    if (st.attr_smem < smem_bytes) {
      e = cudaFuncSetAttribute(qk_norm_rope_kernel<VPT, kStats>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(smem_bytes));
      if (e != cudaSuccess) return e;
      st.attr_smem = smem_bytes;
    }
    if (st.occ_smem != smem_bytes) {
      int n = 0;
      e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, qk_norm_rope_kernel<VPT, kStats>, kThreads, smem_bytes);
      if (e != cudaSuccess) return e;
      st.blocks_per_sm = n > 0 ? n : 1;
      st.occ_smem = smem_bytes;
    }
    blocks_per_sm = st.blocks_per_sm;
    sms = st.sms;
  }
  const int64_t want = static_cast<int64_t>(sms) * blocks_per_sm;
  const int64_t blocks = p.tokens < want ? p.tokens : want;
  qk_norm_rope_kernel<VPT, kStats><<<static_cast<unsigned>(blocks), kThreads, smem_bytes, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace

template <bool kStats>
cudaError_t launch_vpt_dispatch(int vpt, const NormRopeParams& p, uint32_t smem_bytes, cudaStream_t stream) {
  switch (vpt) {
    case 1: return launch_vpt<1, kStats>(p, smem_bytes, stream);
    case 2: return launch_vpt<2, kStats>(p, smem_bytes, stream);
    case 3: return launch_vpt<3, kStats>(p, smem_bytes, stream);
    case 4: return launch_vpt<4, kStats>(p, smem_bytes, stream);
    case 5: return launch_vpt<5, kStats>(p, smem_bytes, stream);
    case 6: return launch_vpt<6, kStats>(p, smem_bytes, stream);
    case 7: return launch_vpt<7, kStats>(p, smem_bytes, stream);
    default: return launch_vpt<8, kStats>(p, smem_bytes, stream);
  }
}

cudaError_t launch_qk_norm_rope(void* qkv, int64_t batch, int32_t F, int32_t H, int32_t W,
                                int32_t heads, const void* gamma_q, const void* gamma_k, float eps,
                                float theta, cudaStream_t stream, const double* stats, int64_t s0,
                                int64_t s_local) {
  NormRopeParams p;
  p.qkv = static_cast<uint16_t*>(qkv);
  p.gamma_q = static_cast<const uint16_t*>(gamma_q);
  p.gamma_k = static_cast<const uint16_t*>(gamma_k);
  p.S = s_local > 0 ? static_cast<int32_t>(s_local) : F * H * W;
  p.s0 = static_cast<int32_t>(s0);
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
  p.stats = stats;
  p.stat_half = p.D / 256;
  p.stat_row = 2 * p.stat_half;
  const int split[3] = {44, 42, 42};
  for (int pr = 0; pr < kPairs; ++pr) {
    const int axis = pr < kRowAxisPair0 ? 0 : (pr < kColAxisPair0 ? 1 : 2);
    const int j = pr - (axis == 0 ? 0 : (axis == 1 ? kRowAxisPair0 : kColAxisPair0));
    p.freq_pi[pr] =
        std::pow(static_cast<double>(theta), -2.0 * j / static_cast<double>(split[axis])) / M_PI;
  }
  if (p.tokens == 0) return cudaSuccess;
  const uint32_t smem_bytes = p.stages * p.stage_bytes + static_cast<uint32_t>(sizeof(NormSmemTail));
  const int vpt = (p.nvec + kRowThreads - 1) / kRowThreads;  // 16-byte vectors per thread
  if (stats != nullptr) return launch_vpt_dispatch<true>(vpt, p, smem_bytes, stream);
  return launch_vpt_dispatch<false>(vpt, p, smem_bytes, stream);
}

cudaError_t norm_error_word(int** word) {
  return cudaGetSymbolAddress(reinterpret_cast<void**>(word), g_norm_error_word);
}

}  // namespace wan
