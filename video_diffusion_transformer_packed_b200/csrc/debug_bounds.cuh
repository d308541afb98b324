// debug_bounds.cuh -- device-side index checks of the debug-bounds build.
//
// Built with -DWAN_DEBUG_BOUNDS (build.py --debug-bounds, which writes
// libwanattn_debug.so next to the release library), every instrumented
// global- or shared-memory access first checks its element range
// [off, off + n) against the extent of the buffer it addresses, as the
// launch parameters define that extent. A failed check records the first
// failure of the translation unit (site and offset) in a device word, counts
// it, and the caller skips the access: nothing traps and the kernel runs on,
// so the context stays usable and the host reads the record through
// wan_debug_bounds. In the release build the check is the constant true and
// the compiler removes it.
//
// The library is built without relocatable device code, so every translation
// unit that uses the checks keeps its own words (WAN_BOUNDS_WORDS defines
// them with an accessor of the given name); the ABI reads all of them.
#pragma once

#include <cuda_runtime.h>

#include <cstdint>

namespace wan {
namespace bounds {

// Sites: which access failed (the high byte of a fault record).
enum Site : uint32_t {
  kNormLoad = 1,     // norm+RoPE: bulk copy of a token's Q|K rows
  kNormStage = 2,    // norm+RoPE: 16-byte vector read out of a ring stage
  kNormStore = 3,    // norm+RoPE: 16-byte store of a result vector (token)
  kNormColumn = 4,   // norm+RoPE: the vector's columns inside the Q or K row
  kNormGamma = 5,    // norm+RoPE: 16-byte gamma vector
  kNormStats = 6,    // norm+RoPE: a precomputed partial sum of squares
  kAttnOut = 7,      // attention: 16-byte store into out
  kAttnPartO = 8,    // attention, partial mode: a row's fp32 O
  kAttnPartML = 9,   // attention, partial mode: a row's (m, l)
  kFp8Out = 10,      // FP8 attention: 16-byte store into out
  kQuantLoad = 11,   // FP8 quantisation: 16-byte read of Q, K or V
  kQuantStoreQK = 12,  // FP8 quantisation: 8-byte store of Q or K codes
  kQuantStageV = 13,   // FP8 quantisation: a V code into the transpose tile
  kQuantStoreV = 14,   // FP8 quantisation: 16-byte store of V^T codes
  kAmaxLoad = 15,      // amax: 16-byte read of the packed buffer
  kGemmY = 16,         // GEMM: 16-byte store into Y
  kGemmStats = 17,     // GEMM: a partial sum of squares
  kMergeAcc = 18,      // merge: the running (O, m, l)
  kMergePart = 19,     // merge: a partial (O, m, l)
  kMergeOut = 20,      // merge: 16-byte store of the finalised output
};

constexpr int kOffsetBits = 56;

// Fault record: site in bits 56..63, the element offset's low 56 bits below
// (a negative offset keeps its two's-complement low bits). 0 means none.
__host__ __device__ constexpr uint64_t encode(uint32_t site, int64_t off) {
  return (static_cast<uint64_t>(site) << kOffsetBits) |
         (static_cast<uint64_t>(off) & ((uint64_t{1} << kOffsetBits) - 1));
}
__host__ __device__ constexpr uint32_t site_of(uint64_t record) {
  return static_cast<uint32_t>(record >> kOffsetBits);
}
__host__ __device__ constexpr int64_t offset_of(uint64_t record) {
  // sign-extend the 56-bit field
  return static_cast<int64_t>(record << (64 - kOffsetBits)) >> (64 - kOffsetBits);
}

// True when [off, off + n) lies inside [0, extent). Otherwise words[0] gets
// the record (if it is still 0), words[1] counts the failure, and false is
// returned. Host code (a test of this logic) uses plain memory operations.
__host__ __device__ inline bool check(unsigned long long* words, uint32_t site, int64_t off, int64_t n,
                                      int64_t extent) {
  if (off >= 0 && n >= 0 && off <= extent - n) return true;
#ifdef __CUDA_ARCH__
  atomicCAS(&words[0], 0ull, static_cast<unsigned long long>(encode(site, off)));
  atomicAdd(&words[1], 1ull);
#else
  if (words[0] == 0) words[0] = encode(site, off);
  words[1] += 1;
#endif
  return false;
}

}  // namespace bounds
}  // namespace wan

// The words of this translation unit and a host accessor `name` for them.
#define WAN_BOUNDS_WORDS(name)                                                   \
  namespace wan {                                                                \
  namespace {                                                                    \
  __device__ unsigned long long g_bounds_words[2];                               \
  }                                                                              \
  cudaError_t name(unsigned long long** words) {                                 \
    return cudaGetSymbolAddress(reinterpret_cast<void**>(words), g_bounds_words); \
  }                                                                              \
  }

#ifdef WAN_DEBUG_BOUNDS
#define WAN_BOUNDS(site, off, n, extent) \
  (::wan::bounds::check(::wan::g_bounds_words, ::wan::bounds::site, (off), (n), (extent)))
#else
#define WAN_BOUNDS(site, off, n, extent) (true)
#endif
