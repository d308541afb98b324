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
// Design (one CTA = one (batch, head) and two 128-row query tiles):
//   warp 8      TMA producer: Q tiles once, then K_j / V_j tiles into a
//               4-slot shared-memory ring (128-byte swizzle, 3D tensor map
//               over [B][S][3D] so that rows past S read as zeros per batch).
//   warp 9      MMA issuer (one thread): tcgen05.mma S_t = Q_t K_j^T into
//               TMEM, then O_t += P_t V_j with P_t read from TMEM. The two
//               query tiles ping-pong: while one tile's softmax runs, the
//               tensor core works on the other tile. The key loop is unrolled
//               by four, so that ring slots and barrier parities are
//               constants in the issuer's instruction stream.
//   warps 0-3   softmax of tile 0, warps 4-7 softmax of tile 1: thread r owns
//               query row r (TMEM lane r). Online softmax in base 2; the
//               running max is only raised (and O rescaled in TMEM) when a
//               tile's max exceeds it by more than 2^8, which keeps the
//               result exact after the final division while skipping almost
//               all rescales. P is rounded to bf16 and written over S in TMEM.
// TMEM columns: S_0 [0,128), S_1 [128,256), O_0 [256,384), O_1 [384,512).
//
// Every mbarrier wait is bounded (wall-clock limit); a wait that gives up
// sets a block-wide abort flag and a device error word, and the block then
// drains its own copies and MMAs, frees TMEM and exits.
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

WAN_BOUNDS_WORDS(bounds_words_attn)

namespace wan {
namespace {

using namespace wan::sm100;

constexpr int kBM = 128;  // query rows per tile
constexpr int kBN = 128;  // keys per tile
constexpr int kHD = 128;  // head dim
constexpr int kStages = 4;
constexpr int kTileBytes = kBM * kHD * 2;  // 32 KB: one 128 x 128 bf16 tile
constexpr int kBoxBytes = kTileBytes / 2;  // 16 KB: 128 rows x 64 columns (one TMA box)
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
constexpr uint64_t kWaitLimitNs = 1000000000ull;  // 1 s per wait (the default limit)
constexpr float kRescaleThreshold = 8.0f;         // log2 of the largest tolerated growth
constexpr uint32_t kAllGroupsSkipped = 0x01010101u;  // Skip-Softmax votes of the four warps
// P_t is handed to the MMA issuer in column blocks, each with its own
// barrier: O_t += P_t V starts on the first keys while the softmax is still
// exponentiating the last ones. kPParts barriers per tile are allocated; the
// dense and partial kernels use four blocks, the Skip-Softmax kernel two (its
// skipped tiles wait on every block, so more blocks cost it more than they
// overlap).
constexpr int kPParts = 4;
template <bool kSkip>
constexpr int p_parts() { return kSkip ? 2 : 4; }
static_assert(p_parts<false>() <= kPParts && p_parts<true>() <= kPParts, "P blocks");
static_assert((64 / p_parts<false>()) % 16 == 0 && (64 / p_parts<true>()) % 16 == 0,
              "P is stored in 16-column pieces");

// Shared memory map (offsets from a 1024-byte aligned base).
constexpr int kOffQ = 0;                              // 2 tiles
constexpr int kOffKV = kOffQ + 2 * kTileBytes;        // kStages tiles
constexpr int kOffBar = kOffKV + kStages * kTileBytes;
constexpr int kNumBars = 1 + 2 * kStages + 2 + 2 * kPParts + 2 + 1;  // q, kv full/empty, s, p, o, drain
constexpr int kOffMisc = kOffBar + kNumBars * 8;  // tmem holder, abort flag, issued[], votes[8]
constexpr int kSmemBytes = kOffMisc + 64 + 1024;  // + alignment slack

// Error-word site codes.
constexpr int kErrProducer = 1, kErrMma = 2, kErrSoftmax = 4, kErrEpilogue = 8, kErrDrain = 16;

__device__ int g_attn_error_word;
// Skip-Softmax counters: [0] (32-row group, key tile) pairs skipped, [1] P V
// products skipped (all four groups of a query tile skipped the key tile).
__device__ unsigned long long g_attn_skip_stats[2];

struct AttnParams {
  uint16_t* out;
  float* o_part;   // partial mode (not null): fp32 unnormalised O instead of out
  float* ml_part;  // partial mode: (m, l) of every (row, head)
  int32_t accumulate;  // partial mode: merge into (o_part, ml_part) instead of overwriting them
  int32_t k_rows;  // keys [k_row0, k_row0 + k_rows) of the K/V map
  int32_t k_row0;
  int32_t kv_k0, kv_v0;  // columns of K and V of head 0 in the K/V map
  int32_t heads;
  int32_t D;
  int32_t q_pairs;  // ceil(q_rows / 256): CTAs per (batch, head)
  int32_t n_kv;     // ceil(k_rows / 128)
  int32_t b0, h0, nh;  // this launch covers batches [b0, ...) and heads [h0, h0 + nh)
  int32_t q_row0, q_rows;  // query rows [q_row0, q_row0 + q_rows); out holds q_rows rows per batch
  float skip_log2;     // Skip-Softmax: log2 of the threshold (used by the kSkip kernel only)
  float scale_log2; // scale * log2(e)
  uint64_t wait_ns; // limit of each pipeline wait
  int32_t skip_loads;  // self-test: the producer starts no copies, so the waits run out
  int64_t out_units;   // (row, head) units out (or o_part, ml_part) holds: the debug-bounds extent
};

// Barrier addresses (32-bit shared-memory addresses, 8 bytes apart).
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
  atomicOr(&g_attn_error_word, site);
}

// ---------------------------------------------------------------- producer
__device__ void run_producer(const CUtensorMap* tmap, const CUtensorMap* tmap_kv, const AttnParams& p,
                             uint32_t smem, Bars bars, volatile int* abort, int* issued, int b, int h, int qp) {
  grid_dependency_wait();  // the packed buffer may still be written by the norm kernel
  if (p.skip_loads) return;  // self-test of the bounded waits: nothing will arrive
  const int xq = h * kHD, xk = p.kv_k0 + h * kHD, xv = p.kv_v0 + h * kHD;
  issued[kStages] = 1;  // the Q copies
  mbar_arrive_expect_tx(bars.q_full(), 2 * kTileBytes);
  for (int t = 0; t < 2; ++t) {
    for (int half = 0; half < 2; ++half) {
      tma_load_3d(smem + kOffQ + t * kTileBytes + half * kBoxBytes, tmap, bars.q_full(),
                  xq + 64 * half, p.q_row0 + (2 * qp + t) * kBM, b);
    }
  }
  bool ok = true;
  const int items = 2 * p.n_kv;  // K_0, V_0, K_1, V_1, ...
#pragma unroll 1
  for (int i = 0; i < items; ++i) {
    const int slot = i % kStages;
    const int use = i / kStages;
    if (use > 0 && !mbar_wait(bars.kv_empty(slot), (use - 1) & 1, abort, p.wait_ns)) {
      ok = false;
      break;
    }
    mbar_arrive_expect_tx(bars.kv_full(slot), kTileBytes);
    const int x = (i & 1) ? xv : xk;
    const int y = p.k_row0 + (i >> 1) * kBN;
    const uint32_t dst = smem + kOffKV + slot * kTileBytes;
    tma_load_3d(dst, tmap_kv, bars.kv_full(slot), x, y, b);
    tma_load_3d(dst + kBoxBytes, tmap_kv, bars.kv_full(slot), x + 64, y, b);
    issued[slot] = use + 1;
  }
  if (!ok) flag_error(abort, kErrProducer);
}

// After an abort, waits (bounded, ignoring the abort flag) for every copy the
// producer started, so that no bulk copy lands after the block has exited.
__device__ void drain_producer(Bars bars, const int* issued) {
  for (int s = 0; s < kStages; ++s) {
    if (issued[s] > 0 && !mbar_wait(bars.kv_full(s), (issued[s] - 1) & 1, nullptr, kWaitLimitNs)) {
      atomicOr(&g_attn_error_word, kErrDrain);
    }
  }
  if (issued[kStages] && !mbar_wait(bars.q_full(), 0, nullptr, kWaitLimitNs)) {
    atomicOr(&g_attn_error_word, kErrDrain);
  }
}

// -------------------------------------------------------------- MMA issuer
template <bool kSkip>
__device__ void run_mma(const AttnParams& p, uint32_t smem, Bars bars, volatile int* abort,
                        uint32_t tmem, const volatile uint32_t* votes) {
  constexpr uint32_t kIdescQK = idesc_bf16_f32(kBM, kBN, 0);
  constexpr uint32_t kIdescPV = idesc_bf16_f32(kBM, kHD, 1);
  // Descriptors are built once; a step only adds a byte offset (in 16-byte
  // units) to the start-address field, which cannot carry out of its 14 bits
  // because shared-memory addresses stay below 2^18.
  const uint64_t q_desc0 = smem_desc_sw128(smem + kOffQ, 16, 1024);
  const uint64_t k_desc0 = smem_desc_sw128(smem + kOffKV, 16, 1024);
  // V [key][dim] is an N-major B: 8-key groups 1024 bytes apart, the two
  // 64-dim halves one box (16 KB) apart; a 16-key step advances 2048 bytes.
  const uint64_t v_desc0 = smem_desc_sw128(smem + kOffKV, kBoxBytes, 1024);

  // MMA steps [k0, k1) of one 128 x 128 x 128 product; a step is K = 16.
  // S_t = Q_t K^T: each 64-dim half of a tile is one 128-byte-swizzled box,
  // and a 16-element step inside a box advances the start address by 32 bytes.
  auto qk_steps = [&](int t, int slot, int k0, int k1) {
    const uint32_t a0 = (t * kTileBytes) >> 4;
    const uint32_t b0 = (slot * kTileBytes) >> 4;
#pragma unroll
    for (int kk = k0; kk < k1; ++kk) {
      const uint32_t off = ((kk >> 2) * kBoxBytes + (kk & 3) * 32) >> 4;
      mma_ss(tmem + t * 128, desc_add(q_desc0, a0 + off), desc_add(k_desc0, b0 + off), kIdescQK,
             kk > 0 ? 1u : 0u);
    }
  };
  // O_t += P_t V: P_t (bf16, 64 TMEM columns over S_t) is the A operand.
  auto pv_steps = [&](int t, int slot, int k0, int k1, uint32_t acc) {
    const uint32_t b0 = (slot * kTileBytes) >> 4;
#pragma unroll
    for (int kk = k0; kk < k1; ++kk) {
      mma_ts(tmem + 256 + t * 128, tmem + t * 128 + kk * 8, desc_add(v_desc0, b0 + kk * (2048 >> 4)),
             kIdescPV, kk > 0 ? 1u : acc);
    }
  };
  // The tensor core's instruction queue holds little more than one MMA, so
  // every barrier check between two groups of MMAs would leave it idle for a
  // shared-memory round trip. Instead the next group's barrier is probed
  // (non-blocking) just before the current group's last MMA, whose issue the
  // thread waits for anyway; the blocking wait runs only when the probe
  // found the phase still open.
  auto ensure = [&](bool probed, uint32_t bar, uint32_t parity) -> bool {
    if (!probed && !mbar_wait(bar, parity, abort, p.wait_ns)) return false;
    tc_fence_after();
    return true;
  };
  constexpr int kParts = p_parts<kSkip>();
  constexpr int kStepsPerPart = 8 / kParts;
  auto kv_bar = [&](int i) { return bars.kv_full(i % kStages); };
  auto kv_par = [&](int i) { return static_cast<uint32_t>((i / kStages) & 1); };

  bool ok = mbar_wait(bars.q_full(), 0, abort, p.wait_ns) && mbar_wait(kv_bar(0), 0, abort, p.wait_ns);
  bool next_v = false, next_p = false;  // probes of V_j and P_0(j) part 0
  uint32_t n_pv_skipped = 0;
  if (ok) {
    tc_fence_after();
    qk_steps(0, 0, 0, 8);
    mma_commit(bars.s_full(0));
    qk_steps(1, 0, 0, 7);
    next_v = mbar_test(kv_bar(1), kv_par(1));
    qk_steps(1, 0, 7, 8);
    mma_commit(bars.s_full(1));
    mma_commit(bars.kv_empty(0));
  }
  auto step = [&](int j, auto rc) -> bool {
    constexpr int r = decltype(rc)::value;  // j % 4
    constexpr int sv = (2 * r + 1) % kStages, sk = (2 * r + 2) % kStages;
    // phase parities of the ring slots for items 2j+1, 2j+2, 2j+3
    constexpr uint32_t kpv = ((2 * r + 1) / kStages) & 1, kpk = ((2 * r + 2) / kStages) & 1,
                       kpn = ((2 * r + 3) / kStages) & 1;
    const bool more = j + 1 < p.n_kv;
    const uint32_t acc = j > 0 ? 1u : 0u;
    constexpr uint32_t pj = r & 1;
    if (!ensure(next_v, bars.kv_full(sv), kpv) || !ensure(next_p, bars.p_full(0, 0), pj)) {
      ok = false;
      return false;
    }
    // O_0 += P_0 V_j, one block of P at a time.
    bool probe = false;
    if (kSkip && votes[0] == kAllGroupsSkipped) {
      // Every warp of query tile 0 skipped key tile j: no product. The other
      // blocks' arrivals are still awaited, so that the warps' stores of
      // P = 0 are done before S_0 is rewritten.
#pragma unroll
      for (int part = 1; part < kParts; ++part) {
        if (!ensure(false, bars.p_full(0, part), pj)) { ok = false; break; }
      }
      ++n_pv_skipped;
    } else {
#pragma unroll
      for (int part = 0; part < kParts; ++part) {
        if (part > 0 && !ensure(probe, bars.p_full(0, part), pj)) { ok = false; break; }
        const int k0 = part * kStepsPerPart, k1 = k0 + kStepsPerPart;
        pv_steps(0, sv, k0, k1 - 1, acc);
        probe = part + 1 < kParts ? mbar_test(bars.p_full(0, part + 1), pj)
                                   : (more ? mbar_test(bars.kv_full(sk), kpk) : true);
        pv_steps(0, sv, k1 - 1, k1, acc);
      }
    }
    if (!ok) return false;
    if (more) {
      // S_0 = Q_0 K_{j+1}^T
      if (!ensure(probe, bars.kv_full(sk), kpk)) { ok = false; return false; }
      qk_steps(0, sk, 0, 7);
      probe = mbar_test(bars.p_full(1, 0), pj);
      qk_steps(0, sk, 7, 8);
      mma_commit(bars.s_full(0));
    } else {
      probe = mbar_test(bars.p_full(1, 0), pj);
    }
    // O_1 += P_1 V_j
    if (!ensure(probe, bars.p_full(1, 0), pj)) { ok = false; return false; }
    if (kSkip && votes[1] == kAllGroupsSkipped) {
#pragma unroll
      for (int part = 1; part < kParts; ++part) {
        if (!ensure(false, bars.p_full(1, part), pj)) { ok = false; break; }
      }
      ++n_pv_skipped;
    } else {
#pragma unroll
      for (int part = 0; part < kParts; ++part) {
        if (part > 0 && !ensure(probe, bars.p_full(1, part), pj)) { ok = false; break; }
        const int k0 = part * kStepsPerPart, k1 = k0 + kStepsPerPart;
        pv_steps(1, sv, k0, k1 - 1, acc);
        probe = part + 1 < kParts ? mbar_test(bars.p_full(1, part + 1), pj) : false;
        pv_steps(1, sv, k1 - 1, k1, acc);
      }
    }
    if (!ok) return false;
    mma_commit(bars.kv_empty(sv));
    if (more) {
      // S_1 = Q_1 K_{j+1}^T; probe what the next iteration starts with.
      qk_steps(1, sk, 0, 7);
      next_v = mbar_test(bars.kv_full((sv + 2) % kStages), kpn);
      next_p = mbar_test(bars.p_full(0, 0), pj ^ 1u);
      qk_steps(1, sk, 7, 8);
      mma_commit(bars.s_full(1));
      mma_commit(bars.kv_empty(sk));
    }
    return true;
  };
  // Key tiles in fours: K_j and V_j take ring slots 2j % 4 and (2j+1) % 4,
  // and a slot's phase parity repeats every four key tiles, so within a
  // group every slot, descriptor offset and parity is a compile-time
  // constant. The issuing thread is on the critical path (an MMA group starts
  // only as fast as it forms the descriptors and barrier addresses), and this
  // form issues the same MMAs with about a tenth fewer cycles per key tile.
  static_assert(kStages == 4, "slot pattern");
#pragma unroll 1
  for (int j = 0; j < p.n_kv && ok; j += 4) {
    ok = step(j, std::integral_constant<int, 0>{});
    if (ok && j + 1 < p.n_kv) ok = step(j + 1, std::integral_constant<int, 1>{});
    if (ok && j + 2 < p.n_kv) ok = step(j + 2, std::integral_constant<int, 2>{});
    if (ok && j + 3 < p.n_kv) ok = step(j + 3, std::integral_constant<int, 3>{});
  }
  if (kSkip && n_pv_skipped) atomicAdd(&g_attn_skip_stats[1], n_pv_skipped);
  if (ok) {
    mma_commit(bars.o_full(0));
    mma_commit(bars.o_full(1));
  } else {
    flag_error(abort, kErrMma);
  }
  // Every MMA this thread issued completes before TMEM can be released.
  mma_commit(bars.drain());
  if (!mbar_wait(bars.drain(), 0, nullptr, kWaitLimitNs)) atomicOr(&g_attn_error_word, kErrDrain);
}

// ----------------------------------------------------------------- softmax
template <bool kSkip, bool kPartial>
__device__ void run_softmax(const AttnParams& p, Bars bars, volatile int* abort, uint32_t tmem,
                            int t, int quarter, int lane, int b, int h, int qp,
                            volatile uint8_t* votes) {
  constexpr int kParts = p_parts<kSkip>();
  constexpr int kPairsPerPart = 64 / kParts;  // bf16 pairs (TMEM columns) per block
  const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
  const uint32_t tS = tmem + lane_base + t * 128;
  const uint32_t tO = tmem + lane_base + 256 + t * 128;
  const float sl2 = p.scale_log2;
  float m_run = -INFINITY;  // running max, already in scaled log2 units
  float l_run = 0.f;
  float m_true = -INFINITY;  // exact running max (Skip-Softmax decisions)
  const bool row_valid = (2 * qp + t) * kBM + quarter * 32 + lane < p.q_rows;
  uint32_t n_skipped = 0;
  bool ok = true;

#pragma unroll 1
  for (int j = 0; j < p.n_kv; ++j) {
    if (!mbar_wait(bars.s_full(t), j & 1, abort, p.wait_ns)) { ok = false; break; }
    tc_fence_after();
    uint32_t sr[128];  // raw fp32 scores of this thread's row
    tmem_ld32(tS + 0, *reinterpret_cast<uint32_t(*)[32]>(sr + 0));
    tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(sr + 32));
    tmem_ld32(tS + 64, *reinterpret_cast<uint32_t(*)[32]>(sr + 64));
    tmem_ld32(tS + 96, *reinterpret_cast<uint32_t(*)[32]>(sr + 96));
    tmem_wait_ld();
    const int rem = p.k_rows - j * kBN;  // valid keys in this tile
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
    if constexpr (kSkip) {
      // Skip-Softmax, threshold mode: the warp's 32 rows skip this key tile
      // when each row's largest weight in it is below threshold x the row's
      // running maximum weight (a row past S never votes to skip). The rows
      // get P = 0, since the tile's O += P V still runs when another warp of
      // the query tile keeps it; the MMA issuer drops the product when all
      // four warps skip.
      const bool row_skip = row_valid && m_cand < m_true + p.skip_log2;
      m_true = fmaxf(m_true, m_cand);
      const bool warp_skip = __all_sync(0xffffffffu, row_skip);
      if (lane == 0) votes[t * 4 + quarter] = warp_skip ? 1 : 0;
      if (warp_skip) {
        uint32_t z[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) z[e] = 0u;
        tmem_st32(tS, z);
        tmem_st32(tS + 32, z);
        tmem_wait_st();
        tc_fence_before();
#pragma unroll
        for (int part = 0; part < kParts; ++part) mbar_arrive(bars.p_full(t, part));
        ++n_skipped;
        continue;
      }
    }
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
    // The row sum adds the bf16-rounded p that the P V product multiplies, so
    // that the output is a convex combination of V rows: summing the fp32 p
    // instead leaves a dominant weight's rounding error (up to 2^-9 of it)
    // uncorrected in the output.
    const uint64_t sl2_2 = f2(sl2, sl2);
    const uint64_t negm2 = f2(-m_run, -m_run);
    float sums[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};  // 8 chains
#pragma unroll
    for (int part = 0; part < kParts; ++part) {
      uint32_t pk[kPairsPerPart];
#pragma unroll
      for (int e = 0; e < kPairsPerPart; ++e) {
        const int pe = kPairsPerPart * part + e;  // pair index: columns 2pe, 2pe+1
        const uint64_t x2 = fma2(f2(__uint_as_float(sr[2 * pe]), __uint_as_float(sr[2 * pe + 1])), sl2_2, negm2);
        float x0, x1;
        f2_split(x2, x0, x1);
        const float p0 = ex2(x0), p1 = ex2(x1);
        pk[e] = pack_bf16x2(p0, p1);
        add_bf16x2_f32(pk[e], sums[2 * (e & 3)], sums[2 * (e & 3) + 1]);
      }
#pragma unroll
      for (int c = 0; c < kPairsPerPart / 16; ++c) {
        tmem_st16(tS + kPairsPerPart * part + 16 * c, *reinterpret_cast<uint32_t(*)[16]>(pk + 16 * c));
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bars.p_full(t, part));
    }
    l_run += ((sums[0] + sums[1]) + (sums[2] + sums[3])) + ((sums[4] + sums[5]) + (sums[6] + sums[7]));
  }
  if (kSkip && lane == 0 && n_skipped) atomicAdd(&g_attn_skip_stats[0], n_skipped);
  if (!ok) {
    flag_error(abort, kErrSoftmax);
    return;
  }
  if (!mbar_wait(bars.o_full(t), 0, abort, p.wait_ns)) {
    flag_error(abort, kErrEpilogue);
    return;
  }
  tc_fence_after();
  const int row = (2 * qp + t) * kBM + quarter * 32 + lane;  // within this launch's query rows
  const int64_t unit = (static_cast<int64_t>(b) * p.q_rows + row) * p.heads + h;
  if constexpr (kPartial) {
    // Partial mode: the unnormalised state of this key range, for a merge;
    // with `accumulate`, merged here into the state already in (o_part,
    // ml_part): both sides rescaled to the larger reference max.
    float4* dst = reinterpret_cast<float4*>(p.o_part + unit * kHD);
    float w_new = 1.f, w_old = 0.f;
    float2 ml = make_float2(m_run, l_run);
    const bool in_o = row < p.q_rows && WAN_BOUNDS(kAttnPartO, unit * kHD, kHD, p.out_units * kHD);
    const bool in_ml = row < p.q_rows && WAN_BOUNDS(kAttnPartML, unit, 1, p.out_units);
    if (p.accumulate && in_ml) {
      const float2 acc = reinterpret_cast<const float2*>(p.ml_part)[unit];
      const float m = fmaxf(acc.x, m_run);
      w_old = exp2f(acc.x - m);
      w_new = exp2f(m_run - m);
      ml = make_float2(m, acc.y * w_old + l_run * w_new);
    }
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
      uint32_t o[32];
      tmem_ld32(tO + 32 * c, o);
      tmem_wait_ld();
      if (in_o) {
#pragma unroll
        for (int v = 0; v < 8; ++v) {
          float4 r = make_float4(__uint_as_float(o[4 * v]), __uint_as_float(o[4 * v + 1]),
                                 __uint_as_float(o[4 * v + 2]), __uint_as_float(o[4 * v + 3]));
          if (p.accumulate) {
            const float4 a = dst[8 * c + v];
            r = make_float4(a.x * w_old + r.x * w_new, a.y * w_old + r.y * w_new, a.z * w_old + r.z * w_new,
                            a.w * w_old + r.w * w_new);
          }
          dst[8 * c + v] = r;
        }
      }
    }
    if (in_ml) reinterpret_cast<float2*>(p.ml_part)[unit] = ml;
    return;
  } else {
  const float inv_l = 1.f / l_run;
  uint16_t* dst = p.out + unit * kHD;
#pragma unroll 1
  for (int c = 0; c < 4; ++c) {
    uint32_t o[32];
    tmem_ld32(tO + 32 * c, o);
    tmem_wait_ld();
    if (row < p.q_rows && WAN_BOUNDS(kAttnOut, unit * kHD + 32 * c, 32, p.out_units * kHD)) {
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
}

template <bool kSkip, bool kPartial>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tmap, const __grid_constant__ CUtensorMap tmap_kv,
                    const AttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t smem_base = smem_u32(smem);
  const Bars bars{smem_base + kOffBar};
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + kOffMisc);
  volatile int* abort = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);
  int* issued = reinterpret_cast<int*>(smem + kOffMisc + 8);  // [kStages + 1], producer-owned
  // Skip-Softmax votes: byte [t * 4 + w] = warp w of query tile t skipped the current key tile.
  uint8_t* votes = smem + kOffMisc + 32;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int qp = blockIdx.x % p.q_pairs;
  const int bh = blockIdx.x / p.q_pairs;
  const int b = p.b0 + bh / p.nh;
  const int h = p.h0 + bh % p.nh;

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
    for (int v = 0; v < 8; ++v) votes[v] = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_holder, kTmemCols);
    tmem_relinquish();
  }
  if (warp == kLoadWarp && lane == 0) {
    tma_prefetch_desc(&tmap);
    tma_prefetch_desc(&tmap_kv);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // Read through a shuffle, so that the compiler knows the TMEM base to be
  // warp-uniform: the tcgen05 addresses derived from it are then formed in
  // uniform registers instead of being moved there before every MMA.
  const uint32_t tmem = __shfl_sync(0xffffffffu, *tmem_holder, 0);

  if (warp >= 8) {
    regs_decrease<kCtlRegs>();
    if (warp == kLoadWarp) {
      if (lane == 0) run_producer(&tmap, &tmap_kv, p, smem_base, bars, abort, issued, b, h, qp);
    } else if (warp == kMmaWarp) {
      if (lane == 0) {
        run_mma<kSkip>(p, smem_base, bars, abort, tmem, reinterpret_cast<const volatile uint32_t*>(votes));
      }
    }
    __syncwarp();
  } else {
    regs_increase<kSoftmaxRegs>();
    run_softmax<kSkip, kPartial>(p, bars, abort, tmem, warp >> 2, warp & 3, lane, b, h, qp, votes);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kLoadWarp && lane == 0 && *abort) drain_producer(bars, issued);
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
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


// A 3D tensor map over a [batch][rows][pitch] bf16 buffer: x = channel,
// y = token, z = batch. Boxes are 64 channels (128 bytes, the swizzle span) x
// 128 tokens; rows past `rows` read as zeros within the batch element.
cudaError_t encode_rows_map(void* map, const void* base, int64_t pitch, int64_t rows, int64_t batch) {
  auto encode = get_encode_fn();
  if (!encode) return cudaErrorNotSupported;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(pitch), static_cast<cuuint64_t>(rows),
                        static_cast<cuuint64_t>(batch)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(pitch) * 2,
                           static_cast<cuuint64_t>(pitch) * 2 * static_cast<cuuint64_t>(rows)};
  cuuint32_t box[3] = {64, kBM, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = encode(reinterpret_cast<CUtensorMap*>(map), CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                      const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                      CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

}  // namespace

cudaError_t plan_attn_fwd(const void* qkv, void* out, int64_t batch, int64_t seq_len,
                          int32_t heads, float scale, AttnPlan* plan) {
  static_assert(sizeof(CUtensorMap) == sizeof(plan->tmap), "tensor map size");
  static_assert(sizeof(CUtensorMap) == sizeof(plan->tmap_kv), "tensor map size");
  const int32_t S = static_cast<int32_t>(seq_len);
  const int32_t D = heads * kHD;

  static PerDeviceOnce setup;
  const cudaError_t attr_err = setup.run([](int) {
    // The register split inside the kernel is only safe when the compiled
    // kernel launches with exactly kLaunchRegs registers per thread.
    for (auto kernel : {attn_fwd_kernel<false, false>, attn_fwd_kernel<true, false>, attn_fwd_kernel<false, true>}) {
      cudaFuncAttributes fa;
      cudaError_t e = cudaFuncGetAttributes(&fa, kernel);
      if (e == cudaSuccess && fa.numRegs != kLaunchRegs) e = cudaErrorInvalidKernelImage;
      if (e == cudaSuccess) e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
      if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
  });
  if (attr_err != cudaSuccess) return attr_err;

  // Q, K and V all come from the packed buffer: one map serves both roles.
  const cudaError_t e = encode_rows_map(plan->tmap, qkv, 3 * static_cast<int64_t>(D), S, batch);
  if (e != cudaSuccess) return e;
  memcpy(plan->tmap_kv, plan->tmap, sizeof(plan->tmap));

  plan->out = out;
  plan->S = S;
  plan->heads = heads;
  plan->D = D;
  plan->q_pairs = (S + 2 * kBM - 1) / (2 * kBM);
  plan->n_kv = (S + kBN - 1) / kBN;
  const float sc = scale > 0.f ? scale : 1.0f / std::sqrt(static_cast<float>(kHD));
  plan->scale_log2 = sc * 1.4426950408889634f;
  plan->skip_threshold = 0.f;
  plan->q_row0 = 0;
  plan->q_rows = S;
  plan->b0 = 0;
  plan->nb = static_cast<int32_t>(batch);
  plan->h0 = 0;
  plan->nh = heads;
  plan->k_row0 = 0;
  plan->k_rows = S;
  plan->kv_k0 = D;
  plan->kv_v0 = 2 * D;
  plan->o_part = nullptr;
  plan->ml_part = nullptr;
  plan->accumulate = false;
  return cudaSuccess;
}

cudaError_t plan_attn_kv(const void* kv, int64_t batch, int64_t kv_rows, int64_t pitch, int64_t k_row0,
                         int64_t k_rows, AttnPlan* plan) {
  const int64_t D = plan->D;
  if (pitch < 2 * D || pitch % 8 != 0 || k_row0 < 0 || k_rows < 1 || k_row0 + k_rows > kv_rows ||
      kv_rows > INT32_MAX) {
    return cudaErrorInvalidValue;
  }
  const cudaError_t e = encode_rows_map(plan->tmap_kv, kv, pitch, kv_rows, batch);
  if (e != cudaSuccess) return e;
  plan->k_row0 = static_cast<int32_t>(k_row0);
  plan->k_rows = static_cast<int32_t>(k_rows);
  plan->kv_k0 = static_cast<int32_t>(pitch - 2 * D);
  plan->kv_v0 = static_cast<int32_t>(pitch - D);
  plan->n_kv = static_cast<int32_t>((k_rows + kBN - 1) / kBN);
  return cudaSuccess;
}

cudaError_t launch_attn_fwd(const AttnPlan& plan, cudaStream_t stream, bool pdl, uint64_t wait_ns,
                            bool skip_loads) {
  AttnParams p;
  p.out = static_cast<uint16_t*>(plan.out);
  p.o_part = plan.o_part;
  p.ml_part = plan.ml_part;
  p.accumulate = plan.accumulate ? 1 : 0;
  p.k_rows = plan.k_rows;
  p.k_row0 = plan.k_row0;
  p.kv_k0 = plan.kv_k0;
  p.kv_v0 = plan.kv_v0;
  p.heads = plan.heads;
  p.D = plan.D;
  p.n_kv = plan.n_kv;
  p.b0 = plan.b0;
  p.h0 = plan.h0;
  p.nh = plan.nh;
  p.q_row0 = plan.q_row0;
  p.q_rows = plan.q_rows;
  p.out_units = static_cast<int64_t>(plan.b0 + plan.nb) * plan.q_rows * plan.heads;
  p.q_pairs = (plan.q_rows + 2 * kBM - 1) / (2 * kBM);
  p.scale_log2 = plan.scale_log2;
  p.skip_log2 = plan.skip_threshold > 0.f ? log2f(plan.skip_threshold) : -INFINITY;
  p.wait_ns = wait_ns;
  p.skip_loads = skip_loads ? 1 : 0;
  CUtensorMap tmap, tmap_kv;
  memcpy(&tmap, plan.tmap, sizeof(tmap));
  memcpy(&tmap_kv, plan.tmap_kv, sizeof(tmap_kv));

  cudaLaunchConfig_t cfg = {};
  const int64_t grid = static_cast<int64_t>(plan.nb) * plan.nh * p.q_pairs;
  if (plan.nb < 1 || plan.nh < 1 || plan.h0 < 0 || plan.b0 < 0 || plan.h0 + plan.nh > plan.heads ||
      plan.q_row0 < 0 || plan.q_rows < 1 || static_cast<int64_t>(plan.q_row0) + plan.q_rows > plan.S ||
      plan.k_row0 < 0 || plan.k_rows < 1 || plan.n_kv != (plan.k_rows + kBN - 1) / kBN ||
      (plan.o_part != nullptr) != (plan.ml_part != nullptr) ||
      (plan.o_part != nullptr && plan.skip_threshold > 0.f) || (plan.accumulate && plan.o_part == nullptr) ||
      grid > INT32_MAX) {
    return cudaErrorInvalidValue;
  }
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  if (plan.skip_threshold > 0.f) return cudaLaunchKernelEx(&cfg, attn_fwd_kernel<true, false>, tmap, tmap_kv, p);
  if (plan.o_part != nullptr) return cudaLaunchKernelEx(&cfg, attn_fwd_kernel<false, true>, tmap, tmap_kv, p);
  return cudaLaunchKernelEx(&cfg, attn_fwd_kernel<false, false>, tmap, tmap_kv, p);
}

cudaError_t attn_device_words(int** error_word, unsigned long long** skip_stats) {
  cudaError_t e = cudaGetSymbolAddress(reinterpret_cast<void**>(error_word), g_attn_error_word);
  if (e != cudaSuccess) return e;
  return cudaGetSymbolAddress(reinterpret_cast<void**>(skip_stats), g_attn_skip_stats);
}


}  // namespace wan
