// attn_fwd.cu -- full bidirectional softmax attention over the packed Wan2.2
// QKV buffer, head_dim 128, bf16 in / bf16 out, fp32 accumulation (sm_100a).
//
//   out[b, i, h, :] = sum_j softmax_j(scale * q_i . k_j) v_j
//
// The attention is the dominant cost of a DiT block: all-pairs over the
// video tokens, S^2 work (AWS Neuron "Optimizing High-Quality Offline Video
// Generation", "Context parallelism"); Q, K and V are read straight out of
// the packed [Q | K | V] allocation with no repack (TensorRT-LLM PR
// "[visual_gen] Optimize Wan2.2 Dataflow", "Packed QKV Profiling Details").
//
// Design. A cluster of two CTAs (a CTA pair, one per SM) owns 512 query rows
// of one (batch, head): CTA v holds query tiles t = 0, 1 of 128 rows each,
// rows 512*qq + 256*t + 128*v. The tensor-core work runs as CTA-pair MMAs
// (tcgen05 cta_group::2, M = 256): the even CTA's MMA thread issues every
// MMA for both CTAs; each CTA supplies its own 128 rows of the A operand and
// HALF of the B operand -- 64 of the 128 keys of a K tile, 64 of the 128 head
// dims of a V tile -- which halves the shared-memory operand and TMA traffic
// per SM compared with single-CTA 128 x 128 MMAs (those left the tensor pipe
// waiting on shared-memory operand reads).
//   warp 8      TMA producer (both CTAs): Q tiles once, then the K_j / V_j
//               halves into an 8-slot ring of 16 KB; completion counted on the
//               even CTA's barriers (3D tensor map over [B][S][3D]; rows past
//               S read as zeros within the batch). No multicast.
//   warp 9      MMA issuer (even CTA): S_t = Q_t K_j^T into TMEM, then
//               O_t += P_t V_j with P_t read from TMEM; the two query tiles
//               ping-pong so one tile's softmax overlaps the other's MMAs.
//               Commits are multicast to both CTAs' barriers.
//   warps 0-3   softmax of tile 0, warps 4-7 of tile 1 (both CTAs): thread r
//               owns query row r (TMEM lane r); online softmax in base 2 with
//               the running max raised (and O rescaled in TMEM) only when a
//               tile's max exceeds it by more than 2^8 -- exact after the final
//               division. P is rounded to bf16 and written over S in TMEM;
//               readiness is signalled to the even CTA's barrier.
// TMEM columns (each CTA): S_0 [0,128), S_1 [128,256), O_0 [256,384), O_1 [384,512).
//
// Every mbarrier wait is bounded (wall-clock limit); a wait that gives up
// sets a block-wide abort flag and a device error word; the block then drains
// what it started, meets its partner at the final cluster barrier, frees TMEM
// and exits.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "sm100.cuh"
#include "wan_kernels.h"

namespace wan {
namespace {

using namespace wan::sm100;

constexpr int kBM = 128;  // query rows per tile (per CTA)
constexpr int kBN = 128;  // keys per iteration
constexpr int kHD = 128;  // head dim
constexpr int kPairRows = 4 * kBM;  // query rows per CTA pair
constexpr int kStages = 8;          // ring slots, each one K half or one V half
constexpr int kTileBytes = kBM * kHD * 2;  // 32 KB: one 128 x 128 bf16 Q tile
constexpr int kBoxBytes = 64 * 64 * 2;     // 8 KB: one TMA box of 64 rows x 64 columns
constexpr int kSlotBytes = 2 * kBoxBytes;  // 16 KB: a K half (64 keys x 128) or V half (128 keys x 64)
constexpr int kThreads = 384;  // 3 warpgroups: softmax tile 0, softmax tile 1, load/MMA
constexpr int kLoadWarp = 8;
constexpr int kMmaWarp = 9;
// Register split. The launch gives every thread kLaunchRegs (checked on the
// host against the compiled kernel before any launch); the load/MMA
// warpgroup gives registers back and the two softmax warpgroups take them:
// 128*kCtlRegs + 256*kSoftmaxRegs must not exceed 384*kLaunchRegs.
constexpr int kLaunchRegs = 168;
constexpr int kCtlRegs = 72;
constexpr int kSoftmaxRegs = 216;
static_assert(128 * kCtlRegs + 256 * kSoftmaxRegs <= kThreads * kLaunchRegs, "register split");
constexpr uint32_t kTmemCols = 512;
constexpr uint64_t kWaitLimitNs = 1000000000ull;  // 1 s per wait
constexpr float kRescaleThreshold = 8.0f;         // log2 of the largest tolerated growth
constexpr uint16_t kBothCtas = 0x3;

// Shared memory map (offsets from a 1024-byte aligned base; identical in
// both CTAs of a pair, which the CTA-pair MMAs rely on).
constexpr int kOffQ = 0;                              // 2 tiles
constexpr int kOffKV = kOffQ + 2 * kTileBytes;        // kStages slots
constexpr int kOffBar = kOffKV + kStages * kSlotBytes;
constexpr int kNumBars = 1 + 2 * kStages + 2 + 2 + 2 + 1;  // q, kv full/empty, s, p, o, drain
constexpr int kOffMisc = kOffBar + kNumBars * 8;
constexpr int kSmemBytes = kOffMisc + 64 + 1024;  // + alignment slack

// 2^x on the FMA pipe for part of the probabilities (the rest use MUFU ex2):
// x = n + f, n = round(x) by the 1.5*2^23 magic add, f in [-1/2, 1/2],
// 2^x = 2^n * p(f) with p the degree-3 minimax fit of 2^f in relative error
// (max 7.5e-5) produced by exp2_poly.py next to this file; 2^n is applied by
// adding n to the exponent field.
constexpr uint32_t kPolyC0 = 0x3F7FFB49u, kPolyC1 = 0x3F31798Du, kPolyC2 = 0x3E786F0Du,
                   kPolyC3 = 0x3D61FBB0u;
constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23
// Pairs of score columns whose exponentials go to the FMA pipe: 3 of every 8
// (the MUFU unit alone needs as long as the tensor core for one tile).
__host__ __device__ constexpr bool poly_pair(int e) { return (e & 7) == 2 || (e & 7) == 5 || (e & 7) == 7; }

// Error-word site codes.
constexpr int kErrProducer = 1, kErrMma = 2, kErrSoftmax = 4, kErrEpilogue = 8, kErrDrain = 16,
              kErrTmem = 32;

__device__ int g_attn_error_word;

struct AttnParams {
  uint16_t* out;
  int32_t S;
  int32_t heads;
  int32_t D;
  int32_t q_quads;  // ceil(S / 512): CTA pairs per (batch, head)
  int32_t n_kv;     // ceil(S / 128)
  float scale_log2; // scale * log2(e)
};

// Barrier addresses (32-bit shared-memory addresses, 8 bytes apart).
//  q_full, kv_full, p_full, drain: used in the even CTA (both CTAs' loads and
//    softmax threads arrive there);
//  kv_empty, s_full, o_full: in each CTA (the MMA commits are multicast).
struct Bars {
  uint32_t base;
  __device__ __forceinline__ uint32_t q_full() const { return base; }
  __device__ __forceinline__ uint32_t kv_full(int s) const { return base + 8 * (1 + s); }
  __device__ __forceinline__ uint32_t kv_empty(int s) const { return base + 8 * (1 + kStages + s); }
  __device__ __forceinline__ uint32_t s_full(int t) const { return base + 8 * (1 + 2 * kStages + t); }
  __device__ __forceinline__ uint32_t p_full(int t) const { return base + 8 * (3 + 2 * kStages + t); }
  __device__ __forceinline__ uint32_t o_full(int t) const { return base + 8 * (5 + 2 * kStages + t); }
  __device__ __forceinline__ uint32_t drain() const { return base + 8 * (7 + 2 * kStages); }
};
static_assert(8 + 2 * kStages == kNumBars, "barrier count");

__device__ __forceinline__ void flag_error(volatile int* abort, int site) {
  *abort = 1;
  atomicOr(&g_attn_error_word, site);
}

// ---------------------------------------------------------------- producer
// Both CTAs: this CTA's Q tiles, then its halves of K_j (keys 64v..64v+63 of
// the tile) and V_j (head dims 64v..64v+63), completion on the even CTA's
// barriers. The even CTA also announces the byte counts of both CTAs.
__device__ void run_producer(const CUtensorMap* tmap, const AttnParams& p, uint32_t smem,
                             Bars bars, uint32_t rank, volatile int* abort, int* issued, int b,
                             int h, int qq) {
  grid_dependency_wait();  // the packed buffer may still be written by the norm kernel
  const bool leader = rank == 0;
  const int xq = h * kHD, xk = p.D + h * kHD, xv = 2 * p.D + h * kHD + 64 * static_cast<int>(rank);
  const uint32_t q_bar = map_to_cta(bars.q_full(), 0);
  if (leader) mbar_arrive_expect_tx(bars.q_full(), 2 * 2 * kTileBytes);  // both CTAs' Q tiles
  for (int t = 0; t < 2; ++t) {
    const int row0 = kPairRows * qq + 2 * kBM * t + kBM * static_cast<int>(rank);
    for (int half = 0; half < 2; ++half) {       // head dims 0-63, 64-127
      for (int rh = 0; rh < 2; ++rh) {           // rows 0-63, 64-127
        tma_load_3d_pair(smem + kOffQ + t * kTileBytes + half * (kTileBytes / 2) + rh * kBoxBytes, tmap, q_bar,
                         xq + 64 * half, row0 + 64 * rh, b);
      }
    }
  }
  bool ok = true;
  const int items = 2 * p.n_kv;  // K_0, V_0, K_1, V_1, ...
#pragma unroll 1
  for (int i = 0; i < items; ++i) {
    const int slot = i % kStages;
    const int use = i / kStages;
    if (use > 0 && !mbar_wait(bars.kv_empty(slot), (use - 1) & 1, abort, kWaitLimitNs)) {
      ok = false;
      break;
    }
    if (leader) mbar_arrive_expect_tx(bars.kv_full(slot), 2 * kSlotBytes);  // both halves
    const uint32_t bar = map_to_cta(bars.kv_full(slot), 0);
    const uint32_t dst = smem + kOffKV + slot * kSlotBytes;
    const int key0 = (i >> 1) * kBN;
    if ((i & 1) == 0) {
      // K half: keys key0 + 64*rank .. +63, all 128 head dims (two column boxes)
      const int y = key0 + 64 * static_cast<int>(rank);
      tma_load_3d_pair(dst, tmap, bar, xk, y, b);
      tma_load_3d_pair(dst + kBoxBytes, tmap, bar, xk + 64, y, b);
    } else {
      // V half: all 128 keys (two row boxes), head dims 64*rank .. +63
      tma_load_3d_pair(dst, tmap, bar, xv, key0, b);
      tma_load_3d_pair(dst + kBoxBytes, tmap, bar, xv, key0 + 64, b);
    }
    issued[slot] = use + 1;
  }
  if (!ok) flag_error(abort, kErrProducer);
}

// After an abort, the even CTA waits (bounded, ignoring the abort flag) for
// every load phase it announced, so no bulk copy lands after the pair exits.
__device__ void drain_producer(Bars bars, const int* issued) {
  for (int s = 0; s < kStages; ++s) {
    if (issued[s] > 0 && !mbar_wait_cluster(bars.kv_full(s), (issued[s] - 1) & 1, nullptr, kWaitLimitNs)) {
      atomicOr(&g_attn_error_word, kErrDrain);
    }
  }
  if (!mbar_wait_cluster(bars.q_full(), 0, nullptr, kWaitLimitNs)) atomicOr(&g_attn_error_word, kErrDrain);
}

// -------------------------------------------------------------- MMA issuer
// Even CTA only. Descriptors name this CTA's shared memory; the partner's
// halves sit at the same offsets in its own shared memory.
__device__ void run_mma(const AttnParams& p, uint32_t smem, Bars bars, volatile int* abort,
                        uint32_t tmem) {
  constexpr uint32_t kIdescQK = idesc_bf16_f32(2 * kBM, kBN, 0);  // M = 256 over the pair
  constexpr uint32_t kIdescPV = idesc_bf16_f32(2 * kBM, kHD, 1);
  // Descriptors are built once; a step only adds a byte offset (in 16-byte
  // units) to the start-address field, which cannot carry out of its 14 bits
  // because shared-memory addresses stay below 2^18.
  //
  // S_t = Q_t K^T, K = 128 head dims in 8 steps of 16. Q_t: 128 rows, two
  // 64-column halves 16 KB apart; K half: 64 keys, two 64-column halves 8 KB
  // apart. Both 128-byte swizzled, 8-row groups 1024 bytes apart; a 16-element
  // step inside a half advances the start address by 32 bytes.
  const uint64_t q_desc0 = smem_desc_sw128(smem + kOffQ, 16, 1024);
  const uint64_t k_desc0 = smem_desc_sw128(smem + kOffKV, 16, 1024);
  // V half [key][64 dims] is an N-major B: 8-key groups 1024 bytes apart; a
  // 16-key step advances 2048 bytes; the 64 dims fill one swizzle span.
  const uint64_t v_desc0 = smem_desc_sw128(smem + kOffKV, kSlotBytes, 1024);

  auto issue_qk = [&](int t, int slot) {
    const uint32_t a0 = (t * kTileBytes) >> 4;
    const uint32_t b0 = (slot * kSlotBytes) >> 4;
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      const uint32_t aoff = ((kk >> 2) * (kTileBytes / 2) + (kk & 3) * 32) >> 4;
      const uint32_t boff = ((kk >> 2) * kBoxBytes + (kk & 3) * 32) >> 4;
      mma_ss_pair(tmem + t * 128, desc_add(q_desc0, a0 + aoff), desc_add(k_desc0, b0 + boff), kIdescQK,
                  kk > 0 ? 1u : 0u);
    }
  };
  // O_t += P_t V: P_t (bf16, 64 TMEM columns over S_t) is the A operand.
  auto issue_pv = [&](int t, int slot, uint32_t acc) {
    const uint32_t b0 = (slot * kSlotBytes) >> 4;
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      mma_ts_pair(tmem + 256 + t * 128, tmem + t * 128 + kk * 8, desc_add(v_desc0, b0 + kk * (2048 >> 4)),
                  kIdescPV, kk > 0 ? 1u : acc);
    }
  };
  auto wait_item = [&](int i) -> bool {
    return mbar_wait_cluster(bars.kv_full(i % kStages), (i / kStages) & 1, abort, kWaitLimitNs);
  };

  bool ok = mbar_wait_cluster(bars.q_full(), 0, abort, kWaitLimitNs) && wait_item(0);
  if (ok) {
    tc_fence_after();
    issue_qk(0, 0);
    mma_commit_pair(bars.s_full(0), kBothCtas);
    issue_qk(1, 0);
    mma_commit_pair(bars.s_full(1), kBothCtas);
    mma_commit_pair(bars.kv_empty(0), kBothCtas);
  }
#pragma unroll 1
  for (int j = 0; j < p.n_kv && ok; ++j) {
    const int iv = 2 * j + 1, ik = 2 * j + 2;
    const bool more = j + 1 < p.n_kv;
    const uint32_t acc = j > 0 ? 1u : 0u;
    if (!wait_item(iv) || !mbar_wait_cluster(bars.p_full(0), j & 1, abort, kWaitLimitNs)) { ok = false; break; }
    tc_fence_after();
    issue_pv(0, iv % kStages, acc);
    if (more) {
      if (!wait_item(ik)) { ok = false; break; }
      tc_fence_after();
      issue_qk(0, ik % kStages);
      mma_commit_pair(bars.s_full(0), kBothCtas);
    }
    if (!mbar_wait_cluster(bars.p_full(1), j & 1, abort, kWaitLimitNs)) { ok = false; break; }
    tc_fence_after();
    issue_pv(1, iv % kStages, acc);
    mma_commit_pair(bars.kv_empty(iv % kStages), kBothCtas);
    if (more) {
      issue_qk(1, ik % kStages);
      mma_commit_pair(bars.s_full(1), kBothCtas);
      mma_commit_pair(bars.kv_empty(ik % kStages), kBothCtas);
    }
  }
  if (ok) {
    mma_commit_pair(bars.o_full(0), kBothCtas);
    mma_commit_pair(bars.o_full(1), kBothCtas);
  } else {
    flag_error(abort, kErrMma);
  }
  // Every MMA this thread issued completes before either CTA releases TMEM.
  mma_commit_pair(bars.drain(), 0x1);
  if (!mbar_wait(bars.drain(), 0, nullptr, kWaitLimitNs)) atomicOr(&g_attn_error_word, kErrDrain);
}

// 2^x for both lanes of a packed pair on the FMA pipe (x clamped to >= -126,
// below which the result is under 2^-126 and only its smallness matters).
__device__ __forceinline__ uint64_t exp2_poly2(uint64_t x2) {
  float x0, x1;
  f2_split(x2, x0, x1);
  x2 = f2(fmaxf(x0, -126.f), fmaxf(x1, -126.f));
  const uint64_t magic = f2(kMagic, kMagic);
  const uint64_t j = add2(x2, magic);        // round(x) in the low mantissa bits
  const uint64_t f = sub2(x2, sub2(j, magic));  // x - round(x), in [-1/2, 1/2]
  uint64_t p = fma2(f2(__uint_as_float(kPolyC3), __uint_as_float(kPolyC3)), f,
                    f2(__uint_as_float(kPolyC2), __uint_as_float(kPolyC2)));
  p = fma2(p, f, f2(__uint_as_float(kPolyC1), __uint_as_float(kPolyC1)));
  p = fma2(p, f, f2(__uint_as_float(kPolyC0), __uint_as_float(kPolyC0)));
  float p0, p1, j0, j1;
  f2_split(p, p0, p1);
  f2_split(j, j0, j1);
  // the magic's own bits vanish when shifted by 23 (its lowest set bit is 2^22)
  const float r0 = __uint_as_float(__float_as_uint(p0) + (__float_as_uint(j0) << 23));
  const float r1 = __uint_as_float(__float_as_uint(p1) + (__float_as_uint(j1) << 23));
  return f2(r0, r1);
}

// ----------------------------------------------------------------- softmax
__device__ void run_softmax(const AttnParams& p, Bars bars, volatile int* abort, uint32_t tmem,
                            uint32_t rank, int t, int quarter, int lane, int b, int h, int qq) {
  const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
  const uint32_t tS = tmem + lane_base + t * 128;
  const uint32_t tO = tmem + lane_base + 256 + t * 128;
  const uint32_t p_bar = map_to_cta(bars.p_full(t), 0);  // the even CTA's barrier
  const float sl2 = p.scale_log2;
  float m_run = -INFINITY;  // running max, already in scaled log2 units
  float l_run = 0.f;
  bool ok = true;

#pragma unroll 1
  for (int j = 0; j < p.n_kv; ++j) {
    if (!mbar_wait(bars.s_full(t), j & 1, abort, kWaitLimitNs)) { ok = false; break; }
    tc_fence_after();
    uint32_t sr[128];  // raw fp32 scores of this thread's row
    tmem_ld32(tS + 0, *reinterpret_cast<uint32_t(*)[32]>(sr + 0));
    tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(sr + 32));
    tmem_ld32(tS + 64, *reinterpret_cast<uint32_t(*)[32]>(sr + 64));
    tmem_ld32(tS + 96, *reinterpret_cast<uint32_t(*)[32]>(sr + 96));
    tmem_wait_ld();
    const int rem = p.S - j * kBN;  // valid keys in this tile
    if (rem < kBN) {
#pragma unroll
      for (int c = 0; c < 128; ++c) sr[c] = c < rem ? sr[c] : __float_as_uint(-INFINITY);
    }
    // Row max as a tree (8 independent chains of 3-input maxima): a single
    // dependent chain over 128 values would put ~128 latencies on the
    // ping-pong's critical path.
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
      // O_t is quiescent here: S_t's completion implies every earlier MMA
      // (including the previous O_t += P V) has completed.
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
    // p = 2^(s * scale * log2(e) - m), two columns per packed instruction.
    const uint64_t sl2_2 = f2(sl2, sl2);
    const uint64_t negm2 = f2(-m_run, -m_run);
    uint64_t sum2[4] = {f2(0.f, 0.f), f2(0.f, 0.f), f2(0.f, 0.f), f2(0.f, 0.f)};  // 4 chains
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      uint32_t pk[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const int pe = 32 * half + e;  // pair index: columns 2pe, 2pe+1
        const uint64_t x2 = fma2(f2(__uint_as_float(sr[2 * pe]), __uint_as_float(sr[2 * pe + 1])), sl2_2, negm2);
        uint64_t p2;
        if (poly_pair(pe)) {
          p2 = exp2_poly2(x2);
        } else {
          float x0, x1;
          f2_split(x2, x0, x1);
          p2 = f2(ex2(x0), ex2(x1));
        }
        sum2[e & 3] = add2(sum2[e & 3], p2);
        float p0, p1;
        f2_split(p2, p0, p1);
        pk[e] = pack_bf16x2(p0, p1);
      }
      tmem_st32(tS + 32 * half, pk);
    }
    float sum_lo, sum_hi;
    f2_split(add2(add2(sum2[0], sum2[1]), add2(sum2[2], sum2[3])), sum_lo, sum_hi);
    const float sum = sum_lo + sum_hi;
    tmem_wait_st();
    tc_fence_before();
    mbar_arrive_cluster(p_bar);
    l_run += sum;
  }
  if (!ok) {
    flag_error(abort, kErrSoftmax);
    return;
  }
  if (!mbar_wait(bars.o_full(t), 0, abort, kWaitLimitNs)) {
    flag_error(abort, kErrEpilogue);
    return;
  }
  tc_fence_after();
  const float inv_l = 1.f / l_run;
  const int row = kPairRows * qq + 2 * kBM * t + kBM * static_cast<int>(rank) + quarter * 32 + lane;
  uint16_t* dst = p.out + (static_cast<int64_t>(b) * p.S + row) * p.D + h * kHD;
#pragma unroll 1
  for (int c = 0; c < 4; ++c) {
    uint32_t o[32];
    tmem_ld32(tO + 32 * c, o);
    tmem_wait_ld();
    if (row < p.S) {
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
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tmap, const AttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t smem_base = smem_u32(smem);
  const Bars bars{smem_base + kOffBar};
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + kOffMisc);
  volatile int* abort = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);
  int* issued = reinterpret_cast<int*>(smem + kOffMisc + 8);  // [kStages], producer-owned

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();  // 0: the even CTA, which issues the MMAs
  const int pair = blockIdx.x >> 1;
  const int qq = pair % p.q_quads;
  const int bh = pair / p.q_quads;
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
      mbar_init(bars.p_full(t), 2 * 128);  // softmax threads of both CTAs
      mbar_init(bars.o_full(t), 1);
    }
    mbar_init(bars.drain(), 1);
    *abort = 0;
    for (int s = 0; s < kStages; ++s) issued[s] = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc_pair(tmem_holder, kTmemCols);
    tmem_relinquish_pair();
  }
  if (warp == kLoadWarp && lane == 0) tma_prefetch_desc(&tmap);
  tc_fence_before();
  cluster_sync();  // both CTAs' barriers initialised and TMEM allocated
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  // The pair's MMAs address both CTAs' TMEM at the even CTA's column base.
  if (rank == 1 && threadIdx.x == 0 && ld_shared_cluster_u32(map_to_cta(smem_u32(tmem_holder), 0)) != tmem) {
    flag_error(abort, kErrTmem);
  }
  __syncthreads();
  const bool run = *abort == 0;

  if (warp >= 8) {
    regs_decrease<kCtlRegs>();
    if (run && warp == kLoadWarp) {
      if (lane == 0) run_producer(&tmap, p, smem_base, bars, rank, abort, issued, b, h, qq);
    } else if (run && warp == kMmaWarp && rank == 0) {
      if (lane == 0) run_mma(p, smem_base, bars, abort, tmem);
    }
    __syncwarp();
  } else {
    regs_increase<kSoftmaxRegs>();
    if (run) run_softmax(p, bars, abort, tmem, rank, warp >> 2, warp & 3, lane, b, h, qq);
  }

  tc_fence_before();
  __syncthreads();
  if (rank == 0 && warp == kLoadWarp && lane == 0 && *abort) drain_producer(bars, issued);
  cluster_sync();  // the partner's MMAs, loads and arrivals are all done
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, kTmemCols);
  }
}

// ------------------------------------------------------------------- host
PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
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

cudaError_t plan_attn_fwd(const void* qkv, void* out, int64_t batch, int64_t seq_len,
                          int32_t heads, float scale, AttnPlan* plan) {
  static_assert(sizeof(CUtensorMap) == sizeof(plan->tmap), "tensor map size");
  const int32_t S = static_cast<int32_t>(seq_len);
  const int32_t D = heads * kHD;
  auto encode = get_encode_fn();
  if (!encode) return cudaErrorNotSupported;

  static std::once_flag attr_once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(attr_once, [] {
    // The register split inside the kernel is only safe when the compiled
    // kernel launches with exactly kLaunchRegs registers per thread.
    cudaFuncAttributes fa;
    attr_err = cudaFuncGetAttributes(&fa, attn_fwd_kernel);
    if (attr_err == cudaSuccess && fa.numRegs != kLaunchRegs) attr_err = cudaErrorInvalidKernelImage;
    if (attr_err == cudaSuccess) {
      attr_err = cudaFuncSetAttribute(attn_fwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      kSmemBytes);
    }
  });
  if (attr_err != cudaSuccess) return attr_err;

  // Packed buffer as a 3D tensor: x = channel (3D), y = token, z = batch.
  // Boxes are 64 channels (128 bytes, the swizzle span) x 64 tokens.
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(3 * D), static_cast<cuuint64_t>(S),
                        static_cast<cuuint64_t>(batch)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(3 * D) * 2,
                           static_cast<cuuint64_t>(3 * D) * 2 * static_cast<cuuint64_t>(S)};
  cuuint32_t box[3] = {64, 64, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = encode(reinterpret_cast<CUtensorMap*>(plan->tmap), CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                      const_cast<void*>(qkv), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                      CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;

  plan->out = out;
  plan->S = S;
  plan->heads = heads;
  plan->D = D;
  plan->q_pairs = (S + kPairRows - 1) / kPairRows;  // CTA pairs per (batch, head)
  plan->n_kv = (S + kBN - 1) / kBN;
  const float sc = scale > 0.f ? scale : 1.0f / std::sqrt(static_cast<float>(kHD));
  plan->scale_log2 = sc * 1.4426950408889634f;
  plan->grid = 2 * batch * heads * static_cast<int64_t>(plan->q_pairs);  // two CTAs per pair
  return cudaSuccess;
}

cudaError_t launch_attn_fwd(const AttnPlan& plan, cudaStream_t stream, bool pdl) {
  AttnParams p;
  p.out = static_cast<uint16_t*>(plan.out);
  p.S = plan.S;
  p.heads = plan.heads;
  p.D = plan.D;
  p.q_quads = plan.q_pairs;
  p.n_kv = plan.n_kv;
  p.scale_log2 = plan.scale_log2;
  CUtensorMap tmap;
  memcpy(&tmap, plan.tmap, sizeof(tmap));

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(plan.grid));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;  // CTA pairs
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, attn_fwd_kernel, tmap, p);
}

cudaError_t read_and_clear_device_error(cudaStream_t stream, int32_t* code) {
  cudaError_t e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return e;
  int v = 0;
  e = cudaMemcpyFromSymbol(&v, g_attn_error_word, sizeof(int));
  if (e != cudaSuccess) return e;
  if (v != 0) {
    const int zero = 0;
    e = cudaMemcpyToSymbol(g_attn_error_word, &zero, sizeof(int));
    if (e != cudaSuccess) return e;
  }
  *code = v;
  return cudaSuccess;
}

}  // namespace wan
