// gemm_bf16.cu -- Y = X W^T for the DiT block's projections (bf16 in, fp32
// accumulation, bf16 out), with an optional epilogue statistic for the Q/K
// RMSNorm that follows the QKV projection (sm_100a).
//
// The QKV projection produces the packed [Q | K | V] buffer the attention
// path reads (TensorRT-LLM PR "[visual_gen] Optimize Wan2.2 Dataflow": the
// fused QKV projection output stays packed), and the Neuron page's qkv_cte
// kernel fuses that projection with the distributed Q/K RMSNorm and RoPE
// ("NKI kernels"). The norm needs the sum of squares over a token's whole
// hidden width, which no output tile of a GEMM holds; so the epilogue here
// fuses the part that does fit: for each output row and each 256-column tile
// inside the first `stat_cols` columns (Q and K), the sum of squares of the
// bf16-rounded outputs in fp64 (squares of bf16 values are exact), written to
// stats[row][tile]. The norm+RoPE pass then reads those instead of reducing.
//
//   X: [M][K] bf16 (activations, K contiguous)    W: [N][K] bf16 (weights, as a Linear layer stores them)
//   Y: [M][N] bf16                                 stats: [M][stat_cols / 256] fp64
//
// Design: a persistent grid (one CTA per SM) walks 256 x 256 output tiles,
// grouped 16 M-blocks at a time so that the tiles a wave works on share their
// X and W blocks in L2. A CTA computes a tile as two 128 x 256 halves that
// share each W block (tcgen05.mma M = 128, N = 256, K = 16, both operands
// K-major from 128-byte-swizzled shared memory): per K step of 64 one 32 KB X
// block and one 32 KB W block arrive by TMA into a 3-stage ring. The two fp32
// accumulators take all 512 TMEM columns. Warp 4 loads, warp 5 issues the
// MMAs, warps 0-3 (one TMEM lane = one output row each) convert, store and
// reduce the statistic; the next tile's MMAs wait for the accumulators to be
// read out (the epilogue is a few per cent of a tile's MMA time at K = 5120).
// Every wait is bounded; a wait that gives up sets the block's abort flag and
// a device error word, and the block drains and exits.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "debug_bounds.cuh"
#include "sm100.cuh"
#include "wan_kernels.h"

WAN_BOUNDS_WORDS(bounds_words_gemm)

namespace wan {
namespace {

using namespace wan::sm100;

constexpr int kTileM = 256;  // two 128-row halves
constexpr int kTileN = 256;
constexpr int kKStep = 64;   // K elements per stage: one 128-byte swizzle span
constexpr int kStages = 3;
constexpr int kHalfBytes = 128 * kKStep * 2;    // 16 KB: 128 rows x 64 bf16
constexpr int kABytes = kTileM * kKStep * 2;    // 32 KB
constexpr int kBBytes = kTileN * kKStep * 2;    // 32 KB
constexpr int kStageBytes = kABytes + kBBytes;  // 64 KB
constexpr int kGroupM = 16;                     // M-blocks per raster group
constexpr int kThreads = 192;                   // warps 0-3 epilogue, 4 load, 5 MMA
constexpr int kLoadWarp = 4;
constexpr int kMmaWarp = 5;
constexpr uint32_t kTmemCols = 512;
constexpr uint64_t kWaitLimitNs = 2000000000ull;

constexpr int kOffRing = 0;
constexpr int kOffBar = kOffRing + kStages * kStageBytes;
constexpr int kNumBars = 2 * kStages + 3;  // full/empty per stage, acc_full, acc_empty, drain
constexpr int kOffMisc = kOffBar + kNumBars * 8;
constexpr int kSmemBytes = kOffMisc + 32 + 1024;

constexpr int kErrLoad = 1, kErrMma = 2, kErrEpilogue = 4;

__device__ int g_gemm_error_word;

struct GemmParams {
  uint16_t* y;
  double* stats;     // may be null
  int64_t M, N, K;
  int32_t stat_tiles;  // 256-column tiles covered by the statistic (stats row length)
  int32_t m_blocks, n_blocks, k_steps;
  int64_t tiles;
};

struct Bars {
  uint32_t base;
  __device__ __forceinline__ uint32_t full(int s) const { return base + 8 * s; }
  __device__ __forceinline__ uint32_t empty(int s) const { return base + 8 * (kStages + s); }
  __device__ __forceinline__ uint32_t acc_full() const { return base + 8 * (2 * kStages); }
  __device__ __forceinline__ uint32_t acc_empty() const { return base + 8 * (2 * kStages + 1); }
  __device__ __forceinline__ uint32_t drain() const { return base + 8 * (2 * kStages + 2); }
};

__device__ __forceinline__ void tile_coords(const GemmParams& p, int64_t t, int& mb, int& nb) {
  const int64_t per_group = static_cast<int64_t>(kGroupM) * p.n_blocks;
  const int64_t g = t / per_group;
  const int64_t r = t - g * per_group;
  const int64_t m0 = g * kGroupM;
  const int64_t gm = (p.m_blocks - m0) < kGroupM ? (p.m_blocks - m0) : kGroupM;  // last group may be short
  mb = static_cast<int>(m0 + r % gm);
  nb = static_cast<int>(r / gm);
}

__device__ __forceinline__ void flag_error(volatile int* abort, int site) {
  *abort = 1;
  atomicOr(&g_gemm_error_word, site);
}

__global__ void __launch_bounds__(kThreads, 1)
    gemm_bf16_kernel(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_w,
                     const GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t base = smem_u32(smem);
  const Bars bars{base + kOffBar};
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + kOffMisc);
  volatile int* abort = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);
  int64_t* loads_issued = reinterpret_cast<int64_t*>(smem + kOffMisc + 8);  // producer-owned
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bars.full(s), 1);
      mbar_init(bars.empty(s), 1);
    }
    mbar_init(bars.acc_full(), 1);
    mbar_init(bars.acc_empty(), 128);
    mbar_init(bars.drain(), 1);
    *abort = 0;
    *loads_issued = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_holder, kTmemCols);
    tmem_relinquish();
  }
  if (warp == kLoadWarp && lane == 0) {
    tma_prefetch_desc(&map_x);
    tma_prefetch_desc(&map_w);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == kLoadWarp) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      int64_t it = 0;
      bool ok = true;
      for (int64_t t = blockIdx.x; t < p.tiles && ok; t += gridDim.x) {
        int mb, nb;
        tile_coords(p, t, mb, nb);
        for (int ks = 0; ks < p.k_steps; ++ks, ++it) {
          const int slot = static_cast<int>(it % kStages);
          const int64_t use = it / kStages;
          if (use > 0 && !mbar_wait(bars.empty(slot), static_cast<uint32_t>((use - 1) & 1), abort, kWaitLimitNs)) {
            ok = false;
            break;
          }
          const uint32_t dst = base + kOffRing + slot * kStageBytes;
          mbar_arrive_expect_tx(bars.full(slot), kStageBytes);
          const int k0 = ks * kKStep;
          tma_load_2d(dst, &map_x, bars.full(slot), k0, mb * kTileM);
          tma_load_2d(dst + kHalfBytes, &map_x, bars.full(slot), k0, mb * kTileM + 128);
          tma_load_2d(dst + kABytes, &map_w, bars.full(slot), k0, nb * kTileN);
          tma_load_2d(dst + kABytes + kHalfBytes, &map_w, bars.full(slot), k0, nb * kTileN + 128);
          *loads_issued = it + 1;
        }
      }
      if (!ok) flag_error(abort, kErrLoad);
    }
  } else if (warp == kMmaWarp) {
    if (lane == 0) {
      // --------------------------------------------------------- MMA issuer
      constexpr uint32_t kIdesc = idesc_bf16_f32(128, kTileN, 0);
      const uint64_t desc0 = smem_desc_sw128(base + kOffRing, 16, 1024);
      int64_t it = 0;
      int64_t tiles_done = 0;
      bool ok = true;
      for (int64_t t = blockIdx.x; t < p.tiles && ok; t += gridDim.x, ++tiles_done) {
        // the accumulators must have been read out by the epilogue
        if (tiles_done > 0 &&
            !mbar_wait(bars.acc_empty(), static_cast<uint32_t>((tiles_done - 1) & 1), abort, kWaitLimitNs)) {
          ok = false;
          break;
        }
        tc_fence_after();
        bool ready = false;  // probe result for the stage of step `it`
        for (int ks = 0; ks < p.k_steps; ++ks, ++it) {
          const int slot = static_cast<int>(it % kStages);
          if (!ready && !mbar_wait(bars.full(slot), static_cast<uint32_t>((it / kStages) & 1), abort, kWaitLimitNs)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = (slot * kStageBytes) >> 4;
          const uint32_t a1 = a0 + (kHalfBytes >> 4);
          const uint32_t b0 = a0 + (kABytes >> 4);
#pragma unroll
          for (int kk = 0; kk < kKStep / 16; ++kk) {
            const uint32_t acc = (ks > 0 || kk > 0) ? 1u : 0u;
            if (kk == kKStep / 16 - 1) {
              // probe the next step's stage while this step's last MMAs wait for queue room
              const int64_t nx = it + 1;
              ready = ks + 1 < p.k_steps &&
                      mbar_test(bars.full(static_cast<int>(nx % kStages)), static_cast<uint32_t>((nx / kStages) & 1));
            }
            mma_ss(tmem, desc_add(desc0, a0 + 2 * kk), desc_add(desc0, b0 + 2 * kk), kIdesc, acc);
            mma_ss(tmem + 256, desc_add(desc0, a1 + 2 * kk), desc_add(desc0, b0 + 2 * kk), kIdesc, acc);
          }
          mma_commit(bars.empty(slot));
        }
        if (!ok) break;
        mma_commit(bars.acc_full());
      }
      if (!ok) flag_error(abort, kErrMma);
      // every MMA this thread issued completes before TMEM can be released
      mma_commit(bars.drain());
      if (!mbar_wait(bars.drain(), 0, nullptr, kWaitLimitNs)) atomicOr(&g_gemm_error_word, kErrMma);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    int64_t tiles_done = 0;
    for (int64_t t = blockIdx.x; t < p.tiles; t += gridDim.x, ++tiles_done) {
      int mb, nb;
      tile_coords(p, t, mb, nb);
      if (!mbar_wait(bars.acc_full(), static_cast<uint32_t>(tiles_done & 1), abort, kWaitLimitNs)) {
        flag_error(abort, kErrEpilogue);
        break;
      }
      tc_fence_after();
      const bool stat = p.stats != nullptr && nb < p.stat_tiles;
#pragma unroll 1
      for (int half = 0; half < 2; ++half) {
        const int64_t row = static_cast<int64_t>(mb) * kTileM + half * 128 + threadIdx.x;
        uint16_t* yrow = p.y + row * p.N + static_cast<int64_t>(nb) * kTileN;
        double ss = 0.0;
#pragma unroll 1
        for (int c = 0; c < kTileN / 32; ++c) {
          uint32_t v[32];
          tmem_ld32(tmem + lane_base + half * 256 + 32 * c, v);
          tmem_wait_ld();
          uint32_t w[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            w[e] = pack_bf16x2(__uint_as_float(v[2 * e]), __uint_as_float(v[2 * e + 1]));
          }
          if (stat) {
            // squares of bf16 values are exact in fp32 (16-bit significands)
            // and move to fp64 by bit arithmetic: high word (bits >> 3) +
            // ((1023 - 127) << 20), low word 0. A zero square maps to 2^-127
            // (as in the norm kernel's own sum), negligible next to eps.
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const float lo = __uint_as_float(w[e] << 16), hi = __uint_as_float(w[e] & 0xFFFF0000u);
              ss += __hiloint2double(static_cast<int>(__umulhi(__float_as_uint(lo * lo), 1u << 29) + 0x38000000u), 0);
              ss += __hiloint2double(static_cast<int>(__umulhi(__float_as_uint(hi * hi), 1u << 29) + 0x38000000u), 0);
            }
          }
          if (row < p.M && WAN_BOUNDS(kGemmY, row * p.N + static_cast<int64_t>(nb) * kTileN + 32 * c, 32,
                                      static_cast<int64_t>(p.M) * p.N)) {
            uint4* dst = reinterpret_cast<uint4*>(yrow + 32 * c);
#pragma unroll
            for (int q = 0; q < 4; ++q) dst[q] = make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
          }
        }
        if (stat && row < p.M &&
            WAN_BOUNDS(kGemmStats, row * p.stat_tiles + nb, 1, static_cast<int64_t>(p.M) * p.stat_tiles)) {
          p.stats[row * p.stat_tiles + nb] = ss;
        }
      }
      tc_fence_before();
      mbar_arrive(bars.acc_empty());
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kLoadWarp && lane == 0 && *abort) {
    // let every copy this block started land before it exits
    const int64_t n = *loads_issued;
    for (int s = 0; s < kStages; ++s) {
      const int64_t uses = n > s ? (n - s + kStages - 1) / kStages : 0;
      if (uses > 0 && !mbar_wait(bars.full(s), static_cast<uint32_t>((uses - 1) & 1), nullptr, kWaitLimitNs)) {
        atomicOr(&g_gemm_error_word, kErrLoad);
      }
    }
  }
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

PFN_cuTensorMapEncodeTiled_v12000 gemm_encode_fn() {
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

cudaError_t launch_gemm_bf16(const void* x, const void* w, void* y, int64_t M, int64_t N, int64_t K,
                             double* stats, int64_t stat_cols, cudaStream_t stream) {
  auto encode = gemm_encode_fn();
  if (!encode) return cudaErrorNotSupported;
  static PerDeviceOnce setup;
  static int sms_of[kMaxDevices];
  int dev = 0;
  const cudaError_t attr_err = setup.run(
      [](int d) {
        cudaError_t e = cudaFuncSetAttribute(gemm_bf16_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
        if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms_of[d], cudaDevAttrMultiProcessorCount, d);
        return e;
      },
      &dev);
  if (attr_err != cudaSuccess) return attr_err;
  const int sms = sms_of[dev];
  alignas(64) CUtensorMap map_x, map_w;
  cuuint32_t box[2] = {kKStep, 128};
  cuuint32_t estr[2] = {1, 1};
  cuuint64_t dims_x[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(M)};
  cuuint64_t str_x[1] = {static_cast<cuuint64_t>(K) * 2};
  CUresult r = encode(&map_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(x), dims_x, str_x, box, estr,
                      CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
  cuuint64_t dims_w[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(N)};
  r = encode(&map_w, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(w), dims_w, str_x, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
  GemmParams p;
  p.y = static_cast<uint16_t*>(y);
  p.stats = stats;
  p.M = M;
  p.N = N;
  p.K = K;
  p.stat_tiles = static_cast<int32_t>(stat_cols / kTileN);
  p.m_blocks = static_cast<int32_t>((M + kTileM - 1) / kTileM);
  p.n_blocks = static_cast<int32_t>(N / kTileN);
  p.k_steps = static_cast<int32_t>(K / kKStep);
  p.tiles = static_cast<int64_t>(p.m_blocks) * p.n_blocks;
  const int64_t grid = p.tiles < sms ? p.tiles : sms;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = stream;
  return cudaLaunchKernelEx(&cfg, gemm_bf16_kernel, map_x, map_w, p);
}

cudaError_t gemm_error_word(int** word) {
  return cudaGetSymbolAddress(reinterpret_cast<void**>(word), g_gemm_error_word);
}

}  // namespace wan
