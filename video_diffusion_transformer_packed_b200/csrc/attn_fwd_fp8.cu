// attn_fwd_fp8.cu -- the FP8 (e4m3) variant of the full bidirectional softmax
// attention, head_dim 128, fp32 accumulation, bf16 output (sm_100a).
//
// The pages time FP8 attention (Neuron "Optimizing High-Quality Offline Video
// Generation"; the TensorRT-LLM PR's TE FP8 attention profile). Operands are
// e4m3 codes with per-tensor scales (fp8_quant.cu): q = cq * sq, k = ck * sk,
// v = cv * sv. The kernel computes
//   out[b, i, h, :] = sv * sum_j p_ij cv_j / sum_j p_ij,
//   p_ij = 2^(log2(e) * scale * sq * sk * (cq_i . ck_j) - m_i)
// with both products on the tensor cores in kind::f8f6f4 (e4m3 x e4m3 -> fp32)
// and the probabilities rounded to e4m3 for the second product (the row sums
// use the fp32 probabilities).
//
// Structure as the bf16 kernel (attn_fwd.cu): one CTA per (batch, head, pair
// of 128-row query tiles); warp 8 loads with TMA (Q and K from the packed
// code buffer [B][S][2D], V from the transposed buffer [B][heads][128][s_pitch],
// so V^T tiles are K-major like the K tiles), warp 9 issues the MMAs, warps
// 0-3 and 4-7 run the online softmax of the two query tiles in ping-pong.
// The issuer's key loop is unrolled by eight, so that ring slots and barrier
// parities are constants in its instruction stream.
// An e4m3 tile of 128 x 128 is 16 KB, one 128-byte-swizzled box; a K = 32
// step advances 32 bytes inside it. P_t (128 codes per row, four per 32-bit
// column) is written over S_t in TMEM and handed over in two 64-key blocks.
// TMEM columns: S_0 [0,128), S_1 [128,256), O_0 [256,384), O_1 [384,512).
//
// Every mbarrier wait is bounded; a wait that gives up sets the block's abort
// flag and the device error word, and the block drains and exits.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <type_traits>

#include "debug_bounds.cuh"
#include "sm100.cuh"
#include "wan_kernels.h"

WAN_BOUNDS_WORDS(bounds_words_fp8)

namespace wan {
namespace {

using namespace wan::sm100;

constexpr int kBM = 128;
constexpr int kBN = 128;
constexpr int kHD = 128;
constexpr int kStages = 8;                  // K_j / V_j^T tiles in flight
constexpr int kTileBytes = kBM * kHD;       // 16 KB: one 128 x 128 e4m3 tile (one TMA box)
constexpr int kSteps = kHD / 32;            // K = 32 per kind::f8f6f4 MMA
constexpr int kPParts = 2;                  // P handed over in two 64-key blocks
constexpr int kStepsPerPart = kSteps / kPParts;
constexpr int kThreads = 384;
constexpr int kLoadWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kLaunchRegs = 168;
constexpr int kCtlRegs = 72;
constexpr int kSoftmaxRegs = 216;
static_assert(128 * kCtlRegs + 256 * kSoftmaxRegs <= kThreads * kLaunchRegs, "register split");
constexpr uint32_t kTmemCols = 512;
constexpr uint64_t kWaitLimitNs = 1000000000ull;
constexpr float kRescaleThreshold = 8.0f;

constexpr int kOffQ = 0;
constexpr int kOffKV = kOffQ + 2 * kTileBytes;
constexpr int kOffBar = kOffKV + kStages * kTileBytes;
constexpr int kNumBars = 1 + 2 * kStages + 2 + 2 * kPParts + 2 + 1;  // q, kv full/empty, s, p, o, drain
constexpr int kOffMisc = kOffBar + kNumBars * 8;                      // tmem holder, abort, issued[]
constexpr int kSmemBytes = kOffMisc + 64 + 1024;

constexpr int kErrProducer = 1, kErrMma = 2, kErrSoftmax = 4, kErrEpilogue = 8, kErrDrain = 16;

__device__ int g_attn_fp8_error_word;

struct AttnFp8Params {
  uint16_t* out;
  int32_t S, heads, D, q_pairs, n_kv;
  float scale_log2;  // scale * sq * sk * log2(e)
  float out_scale;   // sv
  uint64_t wait_ns;
  int64_t out_elems;  // elements of out: the debug-bounds extent
};

struct Bars {
  uint32_t base;
  __device__ __forceinline__ uint32_t q_full() const { return base; }
  __device__ __forceinline__ uint32_t kv_full(int s) const { return base + 8 * (1 + s); }
  __device__ __forceinline__ uint32_t kv_empty(int s) const { return base + 8 * (1 + kStages + s); }
  __device__ __forceinline__ uint32_t s_full(int t) const { return base + 8 * (1 + 2 * kStages + t); }
  __device__ __forceinline__ uint32_t p_full(int t, int part) const {
    return base + 8 * (3 + 2 * kStages + t * kPParts + part);
  }
  __device__ __forceinline__ uint32_t o_full(int t) const { return base + 8 * (3 + 2 * kStages + 2 * kPParts + t); }
  __device__ __forceinline__ uint32_t drain() const { return base + 8 * (5 + 2 * kStages + 2 * kPParts); }
};
static_assert(6 + 2 * kStages + 2 * kPParts == kNumBars, "barrier count");

__device__ __forceinline__ void flag_error(volatile int* abort, int site) {
  *abort = 1;
  atomicOr(&g_attn_fp8_error_word, site);
}

// ---------------------------------------------------------------- producer
__device__ void run_producer(const CUtensorMap* map_qk, const CUtensorMap* map_v, const AttnFp8Params& p,
                             uint32_t smem, Bars bars, volatile int* abort, int* issued, int b, int h,
                             int qp) {
  grid_dependency_wait();
  issued[kStages] = 1;
  mbar_arrive_expect_tx(bars.q_full(), 2 * kTileBytes);
  for (int t = 0; t < 2; ++t) {
    tma_load_3d(smem + kOffQ + t * kTileBytes, map_qk, bars.q_full(), h * kHD, (2 * qp + t) * kBM, b);
  }
  bool ok = true;
  const int items = 2 * p.n_kv;  // K_0, V_0^T, K_1, V_1^T, ...
  const int v_row = (b * p.heads + h) * kHD;
#pragma unroll 1
  for (int i = 0; i < items; ++i) {
    const int slot = i % kStages;
    const int use = i / kStages;
    if (use > 0 && !mbar_wait(bars.kv_empty(slot), (use - 1) & 1, abort, p.wait_ns)) {
      ok = false;
      break;
    }
    mbar_arrive_expect_tx(bars.kv_full(slot), kTileBytes);
    const uint32_t dst = smem + kOffKV + slot * kTileBytes;
    const int j = i >> 1;
    if ((i & 1) == 0) {
      tma_load_3d(dst, map_qk, bars.kv_full(slot), p.D + h * kHD, j * kBN, b);
    } else {
      tma_load_2d(dst, map_v, bars.kv_full(slot), j * kBN, v_row);
    }
    issued[slot] = use + 1;
  }
  if (!ok) flag_error(abort, kErrProducer);
}

__device__ void drain_producer(Bars bars, const int* issued) {
  for (int s = 0; s < kStages; ++s) {
    if (issued[s] > 0 && !mbar_wait(bars.kv_full(s), (issued[s] - 1) & 1, nullptr, kWaitLimitNs)) {
      atomicOr(&g_attn_fp8_error_word, kErrDrain);
    }
  }
  if (issued[kStages] && !mbar_wait(bars.q_full(), 0, nullptr, kWaitLimitNs)) {
    atomicOr(&g_attn_fp8_error_word, kErrDrain);
  }
}

// -------------------------------------------------------------- MMA issuer
__device__ void run_mma(const AttnFp8Params& p, uint32_t smem, Bars bars, volatile int* abort, uint32_t tmem) {
  constexpr uint32_t kIdesc = idesc_e4m3_f32(kBM, kBN);  // both products: M = N = 128, K-major B
  // K-major 128-byte-swizzled tiles: 8-row groups 1024 bytes apart; a K = 32
  // step adds 32 bytes (2 units of 16) to the start address.
  const uint64_t q_desc0 = smem_desc_sw128(smem + kOffQ, 16, 1024);
  const uint64_t kv_desc0 = smem_desc_sw128(smem + kOffKV, 16, 1024);

  auto qk_steps = [&](int t, int slot, int k0, int k1) {
    const uint32_t a0 = (t * kTileBytes) >> 4, b0 = (slot * kTileBytes) >> 4;
#pragma unroll
    for (int kk = k0; kk < k1; ++kk) {
      mma_f8_ss(tmem + t * 128, desc_add(q_desc0, a0 + 2 * kk), desc_add(kv_desc0, b0 + 2 * kk), kIdesc,
                kk > 0 ? 1u : 0u);
    }
  };
  // O_t += P_t V^T: P_t codes in TMEM (a K = 32 step is 8 columns), V^T tile K-major.
  auto pv_steps = [&](int t, int slot, int k0, int k1, uint32_t acc) {
    const uint32_t b0 = (slot * kTileBytes) >> 4;
#pragma unroll
    for (int kk = k0; kk < k1; ++kk) {
      mma_f8_ts(tmem + 256 + t * 128, tmem + t * 128 + kk * 8, desc_add(kv_desc0, b0 + 2 * kk), kIdesc,
                kk > 0 ? 1u : acc);
    }
  };
  auto ensure = [&](bool probed, uint32_t bar, uint32_t parity) -> bool {
    if (!probed && !mbar_wait(bar, parity, abort, p.wait_ns)) return false;
    tc_fence_after();
    return true;
  };
  auto kv_bar = [&](int i) { return bars.kv_full(i % kStages); };
  auto kv_par = [&](int i) { return static_cast<uint32_t>((i / kStages) & 1); };

  bool ok = mbar_wait(bars.q_full(), 0, abort, p.wait_ns) && mbar_wait(kv_bar(0), 0, abort, p.wait_ns);
  bool next_v = false, next_p = false;
  if (ok) {
    tc_fence_after();
    qk_steps(0, 0, 0, kSteps);
    mma_commit(bars.s_full(0));
    qk_steps(1, 0, 0, kSteps - 1);
    next_v = mbar_test(kv_bar(1), kv_par(1));
    qk_steps(1, 0, kSteps - 1, kSteps);
    mma_commit(bars.s_full(1));
    mma_commit(bars.kv_empty(0));
  }
  auto step = [&](int j, auto rc) -> bool {
    constexpr int r = decltype(rc)::value;  // j % 8
    constexpr int sv = (2 * r + 1) % kStages, sk = (2 * r + 2) % kStages;
    // phase parities of the ring slots of items 2j+1, 2j+2 and 2j+3
    constexpr uint32_t kpv = ((2 * r + 1) / kStages) & 1, kpk = ((2 * r + 2) / kStages) & 1,
                       kpn = ((2 * r + 3) / kStages) & 1;
    const bool more = j + 1 < p.n_kv;
    const uint32_t acc = j > 0 ? 1u : 0u;
    constexpr uint32_t pj = r & 1;
    if (!ensure(next_v, bars.kv_full(sv), kpv) || !ensure(next_p, bars.p_full(0, 0), pj)) {
      ok = false;
      return false;
    }
    bool probe = false;
#pragma unroll
    for (int part = 0; part < kPParts; ++part) {
      if (part > 0 && !ensure(probe, bars.p_full(0, part), pj)) { ok = false; break; }
      const int k0 = part * kStepsPerPart, k1 = k0 + kStepsPerPart;
      pv_steps(0, sv, k0, k1 - 1, acc);
      probe = part + 1 < kPParts ? mbar_test(bars.p_full(0, part + 1), pj)
                                 : (more ? mbar_test(bars.kv_full(sk), kpk) : true);
      pv_steps(0, sv, k1 - 1, k1, acc);
    }
    if (!ok) return false;
    if (more) {
      if (!ensure(probe, bars.kv_full(sk), kpk)) { ok = false; return false; }
      qk_steps(0, sk, 0, kSteps - 1);
      probe = mbar_test(bars.p_full(1, 0), pj);
      qk_steps(0, sk, kSteps - 1, kSteps);
      mma_commit(bars.s_full(0));
    } else {
      probe = mbar_test(bars.p_full(1, 0), pj);
    }
#pragma unroll
    for (int part = 0; part < kPParts; ++part) {
      if (!ensure(probe, bars.p_full(1, part), pj)) { ok = false; break; }
      const int k0 = part * kStepsPerPart, k1 = k0 + kStepsPerPart;
      pv_steps(1, sv, k0, k1 - 1, acc);
      probe = part + 1 < kPParts ? mbar_test(bars.p_full(1, part + 1), pj) : false;
      pv_steps(1, sv, k1 - 1, k1, acc);
    }
    if (!ok) return false;
    mma_commit(bars.kv_empty(sv));
    if (more) {
      qk_steps(1, sk, 0, kSteps - 1);
      next_v = mbar_test(bars.kv_full((sv + 2) % kStages), kpn);
      next_p = mbar_test(bars.p_full(0, 0), pj ^ 1u);
      qk_steps(1, sk, kSteps - 1, kSteps);
      mma_commit(bars.s_full(1));
      mma_commit(bars.kv_empty(sk));
    }
    return true;
  };
  // Key tiles in eights: K_j and V_j take ring slots 2j % 8 and (2j+1) % 8,
  // and a slot's phase parity repeats every eight key tiles, so within a
  // group every slot, descriptor offset and parity is a compile-time
  // constant of the issuing thread's instruction stream.
  static_assert(kStages == 8, "slot pattern");
#pragma unroll 1
  for (int j = 0; j < p.n_kv && ok; j += 8) {
    ok = step(j, std::integral_constant<int, 0>{});
    if (ok && j + 1 < p.n_kv) ok = step(j + 1, std::integral_constant<int, 1>{});
    if (ok && j + 2 < p.n_kv) ok = step(j + 2, std::integral_constant<int, 2>{});
    if (ok && j + 3 < p.n_kv) ok = step(j + 3, std::integral_constant<int, 3>{});
    if (ok && j + 4 < p.n_kv) ok = step(j + 4, std::integral_constant<int, 4>{});
    if (ok && j + 5 < p.n_kv) ok = step(j + 5, std::integral_constant<int, 5>{});
    if (ok && j + 6 < p.n_kv) ok = step(j + 6, std::integral_constant<int, 6>{});
    if (ok && j + 7 < p.n_kv) ok = step(j + 7, std::integral_constant<int, 7>{});
  }
  if (ok) {
    mma_commit(bars.o_full(0));
    mma_commit(bars.o_full(1));
  } else {
    flag_error(abort, kErrMma);
  }
  mma_commit(bars.drain());
  if (!mbar_wait(bars.drain(), 0, nullptr, kWaitLimitNs)) atomicOr(&g_attn_fp8_error_word, kErrDrain);
}

// 2^x on the FMA pipe for an eighth of the exponentials (MUFU ex2 gives 16
// per clock per SM, as many cycles per tile as the fp8 products need twice
// over; a larger share costs more FMA/ALU issue than it saves): x = n + f, n = round(x) by the 1.5*2^23 magic add, f in [-1/2, 1/2];
// 2^x = 2^n * p(f) with p the degree-3 minimax fit of 2^f in relative error
// (7.5e-5) that exp2_poly.py next to this file computes; 2^n is applied by
// adding n to the exponent field. x is clamped at -126 (masked keys).
constexpr uint32_t kPolyC0 = 0x3F7FFB49u, kPolyC1 = 0x3F31798Du, kPolyC2 = 0x3E786F0Du,
                   kPolyC3 = 0x3D61FBB0u;
constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23
__device__ __forceinline__ uint64_t exp2_poly2(uint64_t x2) {
  float x0, x1;
  f2_split(x2, x0, x1);
  x2 = f2(fmaxf(x0, -126.f), fmaxf(x1, -126.f));
  const uint64_t magic = f2(kMagic, kMagic);
  const uint64_t j = add2(x2, magic);
  const uint64_t f = sub2(x2, sub2(j, magic));
  uint64_t p = fma2(f2(__uint_as_float(kPolyC3), __uint_as_float(kPolyC3)), f,
                    f2(__uint_as_float(kPolyC2), __uint_as_float(kPolyC2)));
  p = fma2(p, f, f2(__uint_as_float(kPolyC1), __uint_as_float(kPolyC1)));
  p = fma2(p, f, f2(__uint_as_float(kPolyC0), __uint_as_float(kPolyC0)));
  float p0, p1, j0, j1;
  f2_split(p, p0, p1);
  f2_split(j, j0, j1);
  const float r0 = __uint_as_float(__float_as_uint(p0) + (__float_as_uint(j0) << 23));
  const float r1 = __uint_as_float(__float_as_uint(p1) + (__float_as_uint(j1) << 23));
  return f2(r0, r1);
}
// Four-key groups whose exponentials take the polynomial: one in eight.
__host__ __device__ constexpr bool poly_group(int w) { return (w & 7) == 7; }

// ----------------------------------------------------------------- softmax
__device__ void run_softmax(const AttnFp8Params& p, Bars bars, volatile int* abort, uint32_t tmem, int t,
                            int quarter, int lane, int b, int h, int qp) {
  const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
  const uint32_t tS = tmem + lane_base + t * 128;
  const uint32_t tO = tmem + lane_base + 256 + t * 128;
  const float sl2 = p.scale_log2;
  float m_run = -INFINITY;
  float l_run = 0.f;
  bool ok = true;

#pragma unroll 1
  for (int j = 0; j < p.n_kv; ++j) {
    if (!mbar_wait(bars.s_full(t), j & 1, abort, p.wait_ns)) { ok = false; break; }
    tc_fence_after();
    uint32_t sr[128];
    tmem_ld32(tS + 0, *reinterpret_cast<uint32_t(*)[32]>(sr + 0));
    tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(sr + 32));
    tmem_ld32(tS + 64, *reinterpret_cast<uint32_t(*)[32]>(sr + 64));
    tmem_ld32(tS + 96, *reinterpret_cast<uint32_t(*)[32]>(sr + 96));
    tmem_wait_ld();
    const int rem = p.S - j * kBN;
    if (rem < kBN) {
#pragma unroll
      for (int c = 0; c < 128; ++c) sr[c] = c < rem ? sr[c] : __float_as_uint(-INFINITY);
    }
    float mk[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) mk[k] = __uint_as_float(sr[k]);
#pragma unroll
    for (int c = 8; c < 128; c += 16) {
#pragma unroll
      for (int k = 0; k < 8; ++k) mk[k] = max3(mk[k], __uint_as_float(sr[c + k]), __uint_as_float(sr[c + 8 + k]));
    }
    const float mx = fmaxf(max3(mk[0], mk[1], mk[2]), max3(max3(mk[3], mk[4], mk[5]), mk[6], mk[7]));
    const float m_cand = mx * sl2;
    const bool raise = m_cand > m_run + kRescaleThreshold;
    float alpha = 1.f;
    if (raise) {
      alpha = ex2(m_run - m_cand);
      m_run = m_cand;
    }
    l_run *= alpha;
    if (j > 0 && __any_sync(0xffffffffu, raise)) {
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t o[32];
        tmem_ld32(tO + 32 * c, o);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
        tmem_st32(tO + 32 * c, o);
      }
      tmem_wait_st();
    }
    // p = 2^(s * scale_log2 - m): the fp32 values feed the row sum, their e4m3
    // codes (four keys per 32-bit TMEM column, the first key in the lowest
    // byte) feed O += P V^T.
    const uint64_t sl2_2 = f2(sl2, sl2);
    const uint64_t negm2 = f2(-m_run, -m_run);
    uint64_t sum2[4] = {f2(0.f, 0.f), f2(0.f, 0.f), f2(0.f, 0.f), f2(0.f, 0.f)};
#pragma unroll
    for (int part = 0; part < kPParts; ++part) {
      uint32_t pk[16];
#pragma unroll
      for (int w = 0; w < 16; ++w) {
        const int k4 = 64 * part + 4 * w;
        const uint64_t xa = fma2(f2(__uint_as_float(sr[k4]), __uint_as_float(sr[k4 + 1])), sl2_2, negm2);
        const uint64_t xb = fma2(f2(__uint_as_float(sr[k4 + 2]), __uint_as_float(sr[k4 + 3])), sl2_2, negm2);
        float p0, p1, p2, p3;
        if (poly_group(w)) {
          f2_split(exp2_poly2(xa), p0, p1);
          f2_split(exp2_poly2(xb), p2, p3);
        } else {
          float x0, x1, x2, x3;
          f2_split(xa, x0, x1);
          f2_split(xb, x2, x3);
          p0 = ex2(x0); p1 = ex2(x1); p2 = ex2(x2); p3 = ex2(x3);
        }
        sum2[(2 * w) & 3] = add2(sum2[(2 * w) & 3], f2(p0, p1));
        sum2[(2 * w + 1) & 3] = add2(sum2[(2 * w + 1) & 3], f2(p2, p3));
        pk[w] = pack_e4m3x4(p0, p1, p2, p3);
      }
      tmem_st16(tS + 16 * part, pk);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bars.p_full(t, part));
    }
    float sum_lo, sum_hi;
    f2_split(add2(add2(sum2[0], sum2[1]), add2(sum2[2], sum2[3])), sum_lo, sum_hi);
    l_run += sum_lo + sum_hi;
  }
  if (!ok) {
    flag_error(abort, kErrSoftmax);
    return;
  }
  if (!mbar_wait(bars.o_full(t), 0, abort, p.wait_ns)) {
    flag_error(abort, kErrEpilogue);
    return;
  }
  tc_fence_after();
  const float inv_l = p.out_scale / l_run;
  const int row = (2 * qp + t) * kBM + quarter * 32 + lane;
  uint16_t* dst = p.out + (static_cast<int64_t>(b) * p.S + row) * p.D + h * kHD;
#pragma unroll 1
  for (int c = 0; c < 4; ++c) {
    uint32_t o[32];
    tmem_ld32(tO + 32 * c, o);
    tmem_wait_ld();
    if (row < p.S &&
        WAN_BOUNDS(kFp8Out, (static_cast<int64_t>(b) * p.S + row) * p.D + h * kHD + 32 * c, 32, p.out_elems)) {
      uint4* d4 = reinterpret_cast<uint4*>(dst + 32 * c);
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        const float* f = reinterpret_cast<const float*>(o) + 8 * v;
        d4[v] = make_uint4(pack_bf16x2(f[0] * inv_l, f[1] * inv_l), pack_bf16x2(f[2] * inv_l, f[3] * inv_l),
                           pack_bf16x2(f[4] * inv_l, f[5] * inv_l), pack_bf16x2(f[6] * inv_l, f[7] * inv_l));
      }
    }
  }
}

__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_fp8_kernel(const __grid_constant__ CUtensorMap map_qk, const __grid_constant__ CUtensorMap map_v,
                        const AttnFp8Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t smem_base = smem_u32(smem);
  const Bars bars{smem_base + kOffBar};
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + kOffMisc);
  volatile int* abort = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);
  int* issued = reinterpret_cast<int*>(smem + kOffMisc + 8);  // [kStages + 1]

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int qp = blockIdx.x % p.q_pairs;
  const int bh = blockIdx.x / p.q_pairs;
  const int b = bh / p.heads;
  const int h = bh % p.heads;

  if (threadIdx.x == 0) {
    mbar_init(bars.q_full(), 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bars.kv_full(s), 1);
      mbar_init(bars.kv_empty(s), 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(bars.s_full(t), 1);
      for (int part = 0; part < kPParts; ++part) mbar_init(bars.p_full(t, part), 128);
      mbar_init(bars.o_full(t), 1);
    }
    mbar_init(bars.drain(), 1);
    *abort = 0;
    for (int s = 0; s <= kStages; ++s) issued[s] = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_holder, kTmemCols);
    tmem_relinquish();
  }
  if (warp == kLoadWarp && lane == 0) {
    tma_prefetch_desc(&map_qk);
    tma_prefetch_desc(&map_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // Read through a shuffle, so that the compiler knows the TMEM base to be
  // warp-uniform (the tcgen05 addresses derived from it stay in uniform
  // registers).
  const uint32_t tmem = __shfl_sync(0xffffffffu, *tmem_holder, 0);

  if (warp >= 8) {
    regs_decrease<kCtlRegs>();
    if (warp == kLoadWarp) {
      if (lane == 0) run_producer(&map_qk, &map_v, p, smem_base, bars, abort, issued, b, h, qp);
    } else if (warp == kMmaWarp) {
      if (lane == 0) run_mma(p, smem_base, bars, abort, tmem);
    }
    __syncwarp();
  } else {
    regs_increase<kSoftmaxRegs>();
    run_softmax(p, bars, abort, tmem, warp >> 2, warp & 3, lane, b, h, qp);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kLoadWarp && lane == 0 && *abort) drain_producer(bars, issued);
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess) {
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }
  });
  return fn;
}

}  // namespace

cudaError_t launch_attn_fp8(const void* qk8, const void* v8t, void* out, int64_t batch, int64_t seq_len,
                            int32_t heads, int64_t s_pitch, float scale, float scale_q, float scale_k,
                            float scale_v, cudaStream_t stream) {
  auto encode = encode_fn();
  if (!encode) return cudaErrorNotSupported;
  static PerDeviceOnce setup;
  const cudaError_t attr_err = setup.run([](int) {
    cudaFuncAttributes fa;
    cudaError_t e = cudaFuncGetAttributes(&fa, attn_fwd_fp8_kernel);
    if (e == cudaSuccess && fa.numRegs != kLaunchRegs) e = cudaErrorInvalidKernelImage;
    if (e == cudaSuccess) {
      e = cudaFuncSetAttribute(attn_fwd_fp8_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    }
    return e;
  });
  if (attr_err != cudaSuccess) return attr_err;

  const int32_t S = static_cast<int32_t>(seq_len);
  const int32_t D = heads * kHD;
  alignas(64) CUtensorMap map_qk, map_v;
  // Q|K codes as a 3D tensor: x = byte within the token's 2D codes, y = token, z = batch.
  cuuint64_t dims_qk[3] = {static_cast<cuuint64_t>(2 * D), static_cast<cuuint64_t>(S),
                           static_cast<cuuint64_t>(batch)};
  cuuint64_t str_qk[2] = {static_cast<cuuint64_t>(2 * D), static_cast<cuuint64_t>(2 * D) * S};
  cuuint32_t box[3] = {128, 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = encode(&map_qk, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(qk8), dims_qk, str_qk, box,
                      estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                      CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
  // V^T codes as a 2D tensor: x = key (s_pitch bytes per row), y = (batch, head, dim) row.
  cuuint64_t dims_v[2] = {static_cast<cuuint64_t>(s_pitch), static_cast<cuuint64_t>(batch) * D};
  cuuint64_t str_v[1] = {static_cast<cuuint64_t>(s_pitch)};
  r = encode(&map_v, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(v8t), dims_v, str_v, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;

  AttnFp8Params p;
  p.out = static_cast<uint16_t*>(out);
  p.S = S;
  p.heads = heads;
  p.D = D;
  p.q_pairs = (S + 2 * kBM - 1) / (2 * kBM);
  p.n_kv = (S + kBN - 1) / kBN;
  const float sc = scale > 0.f ? scale : 1.0f / sqrtf(static_cast<float>(kHD));
  p.scale_log2 = sc * scale_q * scale_k * 1.4426950408889634f;
  p.out_scale = scale_v;
  p.wait_ns = kWaitLimitNs;
  p.out_elems = batch * S * static_cast<int64_t>(D);
  const int64_t grid = batch * heads * static_cast<int64_t>(p.q_pairs);
  if (grid > INT32_MAX) return cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = stream;
  return cudaLaunchKernelEx(&cfg, attn_fwd_fp8_kernel, map_qk, map_v, p);
}

cudaError_t fp8_error_word(int** word) {
  return cudaGetSymbolAddress(reinterpret_cast<void**>(word), g_attn_fp8_error_word);
}

}  // namespace wan
