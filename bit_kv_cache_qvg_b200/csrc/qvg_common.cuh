// qvg_common.cuh -- device helpers and kernel parameter blocks shared by the
// sm_100a kernels of the QVG codec.  All arithmetic that decides a stored bit
// is spelled out with explicit-rounding intrinsics (__fsub_rn, __ddiv_rn, ...)
// so that no multiply-add contraction changes a result.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace qvg {

constexpr int kD = 128;            // channels per token handled by the kernels
constexpr int kMaxK = 256;         // centroids per block (uint8 assignments)
constexpr int kMaxT = 8;           // residual stages
// Shared memory the fused dequantisation gives to centroid tables (whole
// stages; three of K = 256 at bf16); later stages are read through L2.
constexpr int kDqTableSmemBytes = 200 * 1024;

enum : int { kBF16 = 0, kFP32 = 1 };

// ---------------------------------------------------------------- storage
template <int DT> struct Store;
template <> struct Store<kBF16> {
  using T = __nv_bfloat16;
  static constexpr int bytes = 2;
  __device__ static __forceinline__ float ld(const T* p) { return __bfloat162float(*p); }
  __device__ static __forceinline__ T from_f32(float x) { return __float2bfloat16_rn(x); }
};
template <> struct Store<kFP32> {
  using T = float;
  static constexpr int bytes = 4;
  __device__ static __forceinline__ float ld(const T* p) { return *p; }
  __device__ static __forceinline__ T from_f32(float x) { return x; }
};

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t b16) {
  return __uint_as_float(b16 << 16);
}

// bf16 nearest to a double, ties to even, in a single rounding (no
// intermediate fp32).  Written from the format: keep 7 of the 52 stored
// mantissa bits in the normal range; in the subnormal range (|x| < 2^-126)
// the value is an integer multiple of 2^-133.
__device__ __forceinline__ uint16_t f64_to_bf16_rne(double x) {
  unsigned long long u = (unsigned long long)__double_as_longlong(x);
  const uint16_t sign = (uint16_t)((u >> 48) & 0x8000u);
  const unsigned long long a = u & 0x7FFFFFFFFFFFFFFFull;
  if (a > 0x7FF0000000000000ull) return 0x7FC0;                       // NaN
  if (a >= 0x3810000000000000ull) {                                    // >= 2^-126
    const unsigned long long r = a + ((1ull << 44) - 1ull) + ((a >> 45) & 1ull);
    const int e = (int)(r >> 52) - 1023;
    if (e > 127) return sign | 0x7F80;                                 // overflow / inf
    return sign | (uint16_t)((e + 127) << 7) | (uint16_t)((r >> 45) & 0x7F);
  }
  const double scaled = __dmul_rn(__longlong_as_double((long long)a), 0x1p133);
  return sign | (uint16_t)__double2ll_rn(scaled);
}

// FP8 E4M3 (satfinite, round to nearest even) via the hardware conversion.
__device__ __forceinline__ uint8_t f32_to_e4m3(float x) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(x));
  return (uint8_t)(r & 0xFF);
}

__device__ __forceinline__ float e4m3_to_f32(uint8_t c) {
  uint32_t h2;
  const uint16_t in = (uint16_t)c;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(in));
  return __half2float(__ushort_as_half((unsigned short)(h2 & 0xFFFF)));
}

// ---------------------------------------------------------------- params
// One batch of W blocks ("units") of the quantiser, N tokens each.
struct UnitBatch {
  int W;            // units in this batch
  int64_t N;        // tokens per unit
  int K;            // centroids
  int dtype;        // kBF16 / kFP32
};

// One chunk of a cache whose chunks have their own settings (the adaptive
// cache): its tokens, stage count, group size and where its arrays start.
struct ChunkDesc {
  int64_t o;            // first token of the chunk (per head)
  int64_t n;            // tokens of the chunk (per head)
  int64_t scale_off;    // byte offset of its [H][n][d/G] scale (and zero) bytes
  int64_t assign_off;   // byte offset of its [T][H][n] assignments
  int64_t table_off;    // element offset of its [T][H][K][d] centroid tables
  int32_t T;            // stages
  int32_t G;            // group size
};

// Dequantiser: a set of (chunk, head) units.  A unit's tokens are
// [chunk_off[c], chunk_off[c+1]) of head h.  Packed arrays are stored chunk by
// chunk: chunk c holds H*n_c tokens starting at token row H*chunk_off[c]
// (head-major inside the chunk), its assignments [T][H][n_c] start at byte
// T*H*chunk_off[c], and its tables [T][H][K][d] start at table c.  Output row
// of (h, token) is h*y_head_stride + chunk_off[c] + i.
struct DequantParams {
  const uint8_t* codes;
  const uint8_t* scale;
  const uint8_t* zero;
  const uint8_t* assign;
  const void* centroids;
  void* Y;
  const int64_t* chunk_off;   // device [n_chunks+1], or nullptr: one chunk of N tokens
  const ChunkDesc* desc;      // device [n_chunks] per-chunk layouts (adaptive cache), or nullptr
  int64_t N;                  // tokens (single-chunk case)
  int64_t y_head_stride;      // tokens between heads in Y
  int n_chunks;
  int H;
  int K;
  int T;
  int G;
  int t_smem;                 // stages whose tables are staged in shared memory
  int sym;                    // 1: one scale byte per group, value s*(u - 2); zero unused
};

}  // namespace qvg
