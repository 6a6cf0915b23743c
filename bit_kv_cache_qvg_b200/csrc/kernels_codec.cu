// kernels_codec.cu -- memory-bound codec kernels for sm_100a:
//   * qvg_dequant_fused: unpack 2-bit codes, dequantise with the E4M3 group
//     scale and zero point, add every stage's centroid in reverse stage order,
//     write the storage dtype -- one pass, values kept in registers (m.163.com
//     article on Quant VideoGen, section 五, fused dequantisation kernel;
//     gist.science/de, Technische Zusammenfassung 2C "Fused Kernel").
//   * qvg_residual / qvg_residual_quant: R(t) = round(R(t-1) - C(t)[pi(t)])
//     (section 三, centroid subtraction), and for the last stage the per-group
//     min/max 2-bit quantisation with E4M3 scale and zero point (section 五).
//
// Thread layout shared by all three: 8 threads per token, thread j owns the
// two 8-channel chunks j and j+8 (channels 8j..8j+7 and 64+8j..64+8j+7).  The
// 8 threads of a token therefore read and write 128 contiguous bytes per
// instruction (coalesced), read centroid rows from shared memory without bank
// conflicts, and a group of G channels is reduced with xor-shuffles over
// G/8 threads.
#include "qvg_common.cuh"
#include "qvg_launch.h"

namespace qvg {
namespace {

// ---------------------------------------------------------------- 8-value IO
template <int DT> struct Vec8;

template <> struct Vec8<kBF16> {
  __device__ static __forceinline__ void load(const void* p, float (&v)[8]) {
    const uint4 w = *reinterpret_cast<const uint4*>(p);
    const uint32_t x[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      v[2 * e] = __uint_as_float(x[e] << 16);
      v[2 * e + 1] = __uint_as_float(x[e] & 0xFFFF0000u);
    }
  }
  // Round 8 fp32 values to bf16 (nearest even) and store 16 bytes.
  __device__ static __forceinline__ void store(void* p, const float (&v)[8]) {
    uint32_t x[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const __nv_bfloat162 b = __floats2bfloat162_rn(v[2 * e], v[2 * e + 1]);
      x[e] = *reinterpret_cast<const uint32_t*>(&b);
    }
    *reinterpret_cast<uint4*>(p) = make_uint4(x[0], x[1], x[2], x[3]);
  }
  // Round to bf16 (nearest even, two values per conversion) and return the
  // rounded values as fp32.
  __device__ static __forceinline__ void round(float (&v)[8]) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const __nv_bfloat162 b = __floats2bfloat162_rn(v[2 * e], v[2 * e + 1]);
      const uint32_t x = *reinterpret_cast<const uint32_t*>(&b);
      v[2 * e] = __uint_as_float(x << 16);
      v[2 * e + 1] = __uint_as_float(x & 0xFFFF0000u);
    }
  }
};

template <> struct Vec8<kFP32> {
  __device__ static __forceinline__ void load(const void* p, float (&v)[8]) {
    const float4 a = reinterpret_cast<const float4*>(p)[0];
    const float4 b = reinterpret_cast<const float4*>(p)[1];
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  }
  __device__ static __forceinline__ void store(void* p, const float (&v)[8]) {
    reinterpret_cast<float4*>(p)[0] = make_float4(v[0], v[1], v[2], v[3]);
    reinterpret_cast<float4*>(p)[1] = make_float4(v[4], v[5], v[6], v[7]);
  }
  __device__ static __forceinline__ void round(float (&)[8]) {}
};

// ---------------------------------------------------------------- packed pairs
// Two values as a bf16 pair word (low half first), each cut to its 16 high
// bits: exact for values that are already bf16.  For fp32 values (STICKY) the
// cut keeps the exponent, and the lowest kept bit is set when a cut bit was
// set, so a nonzero value never becomes zero (the channel-range checks need
// the exponents only).
template <bool STICKY>
__device__ __forceinline__ uint32_t bf16_pair_bits(float lo, float hi) {
  const uint32_t a = __float_as_uint(lo), b = __float_as_uint(hi);
  uint32_t w = __byte_perm(a, b, 0x7632);
  if (STICKY) w |= ((a & 0xFFFFu) != 0u ? 1u : 0u) | ((b & 0xFFFFu) != 0u ? 0x10000u : 0u);
  return w;
}
// Lane-wise bf16 maximum; a NaN lane yields the other operand.
__device__ __forceinline__ uint32_t bf16x2_max(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
// Two fp32 values operated on with the f32x2 instructions (float2 intrinsics:
// each lane of the pair is rounded as a separate IEEE fp32 operation).
__device__ __forceinline__ float2 f2(float lo, float hi) { return make_float2(lo, hi); }
// the two bf16 values of a 32-bit word (low half first) as fp32
__device__ __forceinline__ float2 bf16x2_to_f2(uint32_t w) {
  return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}

// ---------------------------------------------------------------- dequant
// Eight lanes per token: lane l of the eight owns channels 8l..8l+7 and
// 64+8l..64+8l+7 (bytes 2l, 2l+1, 16+2l, 17+2l of the token's 32-byte code
// row); for each centroid row the eight lanes read 128 contiguous bytes per
// half, so the shared-memory tables are read without bank conflicts, and
// they write two coalesced 128-byte halves of the output row.  Each group of
// eight lanes walks kDqU tokens per step and keeps the codes, scale/zero bytes
// and assignments of the next kDqDepth - 1 steps in flight, every byte in a
// register of its own, so that nothing waits on a load before the step that
// uses it.  E4M3 bytes are decoded by the hardware conversion; a nibble of
// codes (two channels) maps to a pair of floats through a 16-entry table.
// Fewer threads than the SM holds leave each more registers for the bytes in
// flight, which is what the kernel is short of.
constexpr int kDqThreads = 640;
constexpr int kDqWarps = kDqThreads / 32;
constexpr int kDqStreams = 4 * kDqWarps;        // token streams per block (8 lanes each)

// tokens per stream per step, and steps whose loads are in flight (fewer
// when more assignment bytes are held per token)
template <int TT> constexpr int dq_unroll() { return 2; }
template <int TT> constexpr int dq_depth() { return 2; }

template <int DT> struct Oct;                   // a lane's 8 channels of a row
template <> struct Oct<kBF16> {
  __device__ static __forceinline__ void add(const char* row, float2 (&y)[4]) {
    const uint4 w = *reinterpret_cast<const uint4*>(row);
    y[0] = __fadd2_rn(y[0], bf16x2_to_f2(w.x));
    y[1] = __fadd2_rn(y[1], bf16x2_to_f2(w.y));
    y[2] = __fadd2_rn(y[2], bf16x2_to_f2(w.z));
    y[3] = __fadd2_rn(y[3], bf16x2_to_f2(w.w));
  }
  __device__ static __forceinline__ void store(char* row, const float2 (&y)[4]) {
    uint32_t x[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const __nv_bfloat162 b = __float22bfloat162_rn(y[e]);
      x[e] = *reinterpret_cast<const uint32_t*>(&b);
    }
    *reinterpret_cast<uint4*>(row) = make_uint4(x[0], x[1], x[2], x[3]);
  }
};
template <> struct Oct<kFP32> {
  __device__ static __forceinline__ void add(const char* row, float2 (&y)[4]) {
    const float4 a = reinterpret_cast<const float4*>(row)[0];
    const float4 b = reinterpret_cast<const float4*>(row)[1];
    y[0] = __fadd2_rn(y[0], f2(a.x, a.y));
    y[1] = __fadd2_rn(y[1], f2(a.z, a.w));
    y[2] = __fadd2_rn(y[2], f2(b.x, b.y));
    y[3] = __fadd2_rn(y[3], f2(b.z, b.w));
  }
  __device__ static __forceinline__ void store(char* row, const float2 (&y)[4]) {
    reinterpret_cast<float4*>(row)[0] = make_float4(y[0].x, y[0].y, y[1].x, y[1].y);
    reinterpret_cast<float4*>(row)[1] = make_float4(y[2].x, y[2].y, y[3].x, y[3].y);
  }
};

// Two E4M3 bytes (low byte first) as fp32 values, through the hardware
// conversion to f16 (exact for every finite E4M3 value) and then to fp32.
__device__ __forceinline__ float2 e4m3x2_to_f2(uint32_t pair16) {
  uint32_t h;
  asm("{\n\t.reg .b16 a;\n\tcvt.u16.u32 a, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, a;\n\t}" : "=r"(h) : "r"(pair16));
  float lo, hi;
  asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %2;\n\tcvt.f32.f16 %0, l;\n\tcvt.f32.f16 %1, h;\n\t}"
      : "=f"(lo), "=f"(hi)
      : "r"(h));
  return make_float2(lo, hi);
}

// TT = number of stages when it is <= 4 (assignments fetched a step ahead
// with the codes), or -1 for the generic runtime-T loop.
template <int DT, int TT, bool SYM>
__global__ void __launch_bounds__(kDqThreads, 1)
qvg_dequant_fused(const DequantParams p, const int splits) {
  constexpr int ESZ = Store<DT>::bytes;
  constexpr int TR = TT <= 0 ? 1 : TT;
  constexpr int kDqU = dq_unroll<TT>();
  constexpr int kDqDepth = dq_depth<TT>();
  extern __shared__ __align__(16) unsigned char smem[];

  const int unit = blockIdx.x / splits;
  const int part = blockIdx.x % splits;
  const int h = unit % p.H;
  const int c = unit / p.H;
  int64_t o_c = 0, n_c = p.N;
  int T = TT < 0 ? p.T : TT, G = p.G;
  const int K = p.K;
  const int64_t tab_elems = (int64_t)K * kD;
  const size_t tab_bytes = (size_t)tab_elems * ESZ;
  // where the unit's scale/zero bytes, assignments and tables start
  int64_t sc_row0, as0, tab0;
  if (p.desc != nullptr) {                       // per-chunk layouts (generic instance only)
    const ChunkDesc dsc = p.desc[c];
    o_c = dsc.o; n_c = dsc.n; T = dsc.T; G = dsc.G;
    sc_row0 = dsc.scale_off / (kD / G) + (int64_t)h * n_c;   // in rows of d/G bytes
    as0 = dsc.assign_off + (int64_t)h * n_c;
    tab0 = dsc.table_off;
  } else {
    if (p.chunk_off != nullptr) {
      o_c = p.chunk_off[c];
      n_c = p.chunk_off[c + 1] - o_c;
    }
    sc_row0 = (int64_t)p.H * o_c + (int64_t)h * n_c;
    as0 = (int64_t)T * p.H * o_c + (int64_t)h * n_c;
    tab0 = (int64_t)c * T * p.H * tab_elems;
  }
  const int t_smem = min(p.t_smem, T);
  const int64_t per = (n_c + splits - 1) / splits;
  const int64_t i_begin = (int64_t)part * per;
  const int64_t i_end = min(n_c, i_begin + per);
  const char* tables = static_cast<const char*>(p.centroids) + tab0 * ESZ;
  float2* nlut = reinterpret_cast<float2*>(smem + (size_t)p.t_smem * tab_bytes);  // nibble -> two codes
  if (i_end <= i_begin) return;                                                  // uniform over the block
  // the symmetric mode reads the codes as u - 2
  if (threadIdx.x < 16)
    nlut[threadIdx.x] = SYM ? make_float2((float)(threadIdx.x & 3u) - 2.0f, (float)(threadIdx.x >> 2) - 2.0f)
                            : make_float2((float)(threadIdx.x & 3u), (float)(threadIdx.x >> 2));
  for (int t = 0; t < t_smem; ++t) {
    const uint4* src = reinterpret_cast<const uint4*>(tables + ((int64_t)t * p.H + h) * tab_bytes);
    uint4* dst = reinterpret_cast<uint4*>(smem + (size_t)t * tab_bytes);
    const int n16 = (int)(tab_bytes / 16);
    for (int x = threadIdx.x; x < n16; x += blockDim.x) dst[x] = src[x];
  }
  __syncthreads();

  const int ql = threadIdx.x & 7;                // lane within the token's eight
  const int stream = threadIdx.x >> 3;           // this group's token stream
  const int ng = kD / G;
  const int g0 = (8 * ql) / G, g1 = (64 + 8 * ql) / G;   // groups of the two 8-channel halves
  const int nt = (int)(i_end - i_begin);         // tokens of this block (< 2^31)
  const int64_t row0 = (int64_t)p.H * o_c + (int64_t)h * n_c + i_begin;
  // per-lane base pointers; a token t of the block is an int offset from them
  const uint16_t* cbp = reinterpret_cast<const uint16_t*>(p.codes + row0 * (kD / 4)) + ql;
  const uint8_t* scp = p.scale + (sc_row0 + i_begin) * ng;
  const uint8_t* zrp = p.zero + (sc_row0 + i_begin) * ng;
  const uint8_t* ap = p.assign + as0 + i_begin;
  const int64_t asg_t = (int64_t)p.H * n_c;
  char* yp = static_cast<char*>(p.Y) + ((int64_t)h * p.y_head_stride + o_c + i_begin) * kD * ESZ + 8 * ql * ESZ;
  const int step = kDqStreams * kDqU;

  // codes (two 16-bit words), scale/zero bytes of both halves and (TT > 0)
  // assignments of tokens t0..t0+kDqU-1 (past the block's end: token 0 again;
  // nothing is stored for those), each in a register of its own: they are
  // combined only by the step that uses them
  struct Pre {
    uint32_t c0, c1, s0, z0, s1, z1;
    uint32_t k[TR];
  };
  auto load = [&](int t0, Pre (&pr)[kDqU]) {
#pragma unroll
    for (int u = 0; u < kDqU; ++u) {
      const int t = t0 + u < nt ? t0 + u : 0;
      pr[u].c0 = cbp[t * (kD / 8)];
      pr[u].c1 = cbp[t * (kD / 8) + 8];
      pr[u].s0 = scp[t * ng + g0];
      pr[u].s1 = scp[t * ng + g1];
      pr[u].z0 = SYM ? 0u : (uint32_t)zrp[t * ng + g0];
      pr[u].z1 = SYM ? 0u : (uint32_t)zrp[t * ng + g1];
#pragma unroll
      for (int tt = 0; tt < TR; ++tt) pr[u].k[tt] = TT > 0 ? (uint32_t)ap[tt * asg_t + t] : 0u;
    }
  };
  auto process = [&](int tb, const Pre (&pr)[kDqU]) {
#pragma unroll
    for (int u = 0; u < kDqU; ++u) {
      const int t = tb + u;
      const uint32_t cb = pr[u].c0 | (pr[u].c1 << 16);
      // y = s*q + m (exact in fp32: E4M3 operands, q <= 3), two channels per
      // op; the symmetric mode multiplies, y = s*(u - 2) (exact, and with the
      // sign of zero that product has)
      float2 y0[4], y1[4];
      {
        const float2 g0v = e4m3x2_to_f2(pr[u].s0 | (pr[u].z0 << 8));
        const float2 g1v = e4m3x2_to_f2(pr[u].s1 | (pr[u].z1 << 8));
        const float2 sp0 = f2(g0v.x, g0v.x), sp1 = f2(g1v.x, g1v.x);
        if (SYM) {
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            y0[e] = __fmul2_rn(sp0, nlut[(cb >> (4 * e)) & 0xFu]);
            y1[e] = __fmul2_rn(sp1, nlut[(cb >> (16 + 4 * e)) & 0xFu]);
          }
        } else {
          const float2 mp0 = f2(g0v.y, g0v.y), mp1 = f2(g1v.y, g1v.y);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            y0[e] = __ffma2_rn(sp0, nlut[(cb >> (4 * e)) & 0xFu], mp0);
            y1[e] = __ffma2_rn(sp1, nlut[(cb >> (16 + 4 * e)) & 0xFu], mp1);
          }
        }
      }
      // centroids of stage T, T-1, ..., 1, in that order
#pragma unroll
      for (int tt = 0; tt < (TT < 0 ? kMaxT : (TT == 0 ? 0 : TR)); ++tt) {
        const int st = (TT >= 0 ? TT : T) - 1 - tt;   // a constant in the fixed-T instances
        if (TT < 0 && st < 0) break;
        int k = TT > 0 ? (int)pr[u].k[st] : (int)ap[st * asg_t + (t < nt ? t : 0)];
        k = min(k, K - 1);
        // shared and global rows on separate paths, so that the shared one is
        // addressed as shared memory (st < t_smem is uniform over the block)
        if (st < t_smem) {
          const char* r = reinterpret_cast<const char*>(smem) + (st * (int)tab_elems + k * kD + 8 * ql) * ESZ;
          Oct<DT>::add(r, y0);
          Oct<DT>::add(r + 64 * ESZ, y1);
        } else {
          const char* r = tables + (((int64_t)st * p.H + h) * tab_elems + (int64_t)k * kD + 8 * ql) * ESZ;
          Oct<DT>::add(r, y0);
          Oct<DT>::add(r + 64 * ESZ, y1);
        }
      }
      if (t < nt) {
        char* yr = yp + (int64_t)t * (kD * ESZ);
        Oct<DT>::store(yr, y0);
        Oct<DT>::store(yr + 64 * ESZ, y1);
      }
    }
  };
  // kDqDepth steps of per-token bytes held: step d of a round is loaded
  // kDqDepth steps before it is processed
  Pre pre[kDqDepth][kDqU];
  const int t_first = stream * kDqU;
#pragma unroll
  for (int d = 0; d < kDqDepth; ++d) load(t_first + d * step, pre[d]);
  for (int t0 = t_first; t0 < nt; t0 += kDqDepth * step) {
#pragma unroll
    for (int d = 0; d < kDqDepth; ++d) {
      const int tb = t0 + d * step;
      if (tb < nt) process(tb, pre[d]);
      load(tb + kDqDepth * step, pre[d]);
    }
  }
}

template <int DT, bool SYM>
static cudaError_t launch_dq_t(const DequantParams& p, int blocks, int splits, size_t smem, cudaStream_t s) {
  const void* fn;
  switch (p.T) {
    case 0: fn = reinterpret_cast<const void*>(qvg_dequant_fused<DT, 0, SYM>); break;
    case 1: fn = reinterpret_cast<const void*>(qvg_dequant_fused<DT, 1, SYM>); break;
    case 2: fn = reinterpret_cast<const void*>(qvg_dequant_fused<DT, 2, SYM>); break;
    case 3: fn = reinterpret_cast<const void*>(qvg_dequant_fused<DT, 3, SYM>); break;
    case 4: fn = reinterpret_cast<const void*>(qvg_dequant_fused<DT, 4, SYM>); break;
    default: fn = reinterpret_cast<const void*>(qvg_dequant_fused<DT, -1, SYM>); break;
  }
  cudaError_t e = ensure_dynamic_smem(fn, smem);
  if (e != cudaSuccess) return e;
  switch (p.T) {
    case 0: qvg_dequant_fused<DT, 0, SYM><<<blocks, kDqThreads, smem, s>>>(p, splits); break;
    case 1: qvg_dequant_fused<DT, 1, SYM><<<blocks, kDqThreads, smem, s>>>(p, splits); break;
    case 2: qvg_dequant_fused<DT, 2, SYM><<<blocks, kDqThreads, smem, s>>>(p, splits); break;
    case 3: qvg_dequant_fused<DT, 3, SYM><<<blocks, kDqThreads, smem, s>>>(p, splits); break;
    case 4: qvg_dequant_fused<DT, 4, SYM><<<blocks, kDqThreads, smem, s>>>(p, splits); break;
    default: qvg_dequant_fused<DT, -1, SYM><<<blocks, kDqThreads, smem, s>>>(p, splits); break;
  }
  return cudaGetLastError();
}

// ---------------------------------------------------------------- residual / quant
constexpr int kRqThreads = 512;
constexpr int kRqTokPerIter = kRqThreads / 8;

__device__ __forceinline__ float grp_min(float v, int G) {
  if (G >= 16) v = fminf(v, __shfl_xor_sync(0xffffffffu, v, 1));
  if (G >= 32) v = fminf(v, __shfl_xor_sync(0xffffffffu, v, 2));
  if (G >= 64) v = fminf(v, __shfl_xor_sync(0xffffffffu, v, 4));
  return v;
}
__device__ __forceinline__ float grp_max(float v, int G) {
  if (G >= 16) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 1));
  if (G >= 32) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 2));
  if (G >= 64) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 4));
  return v;
}

__device__ __forceinline__ float min3f(float a, float b, float c) {
  float r;
  asm("min.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
// min and max of 8 values
__device__ __forceinline__ void minmax8(const float (&r)[8], float& lo, float& hi) {
  lo = min3f(min3f(r[0], r[1], r[2]), min3f(r[3], r[4], r[5]), fminf(r[6], r[7]));
  hi = max3f(max3f(r[0], r[1], r[2]), max3f(r[3], r[4], r[5]), fmaxf(r[6], r[7]));
}

// E4M3 code -> value and -> correctly rounded reciprocal (0 where the value
// is 0 or NaN), built once per block in shared memory.
struct E4m3Tables {
  float dec[256];
  float rcp[256];
};

// Quantise one 8-channel chunk given its group's (lo, hi); returns the 16-bit
// packed codes and the scale/zero bytes.  q = clamp(rint(fl((r - m) / s)), 0, 3)
// and s = E4M3(fl(span / 3)), every quotient the IEEE fp32 one: it is formed
// as q0 = x * y with y = RN(1/divisor), then corrected once,
// q = fma(fma(-divisor, q0, x), y, q0) (Markstein's method), which returns
// the IEEE quotient for every E4M3 divisor and every normal quotient (an
// exhaustive host check covers all fp32 inputs); a subnormal quotient gives
// code 0 and E4M3 0 either way.  Clamping to [0, 3] before rounding gives the
// same code (the boundaries -0.5 and 3.5 clamp to the same code on both
// sides); rounding to nearest even is an add and a subtract of 1.5 * 2^23;
// the codes are packed with fused multiply-adds by 4^e, exact in fp32.  Pairs
// of channels go through the packed f32x2 instructions (each lane one IEEE
// fp32 operation).
__device__ __forceinline__ uint32_t quant_chunk(const float (&r)[8], float lo, float hi, const E4m3Tables& tab,
                                                uint8_t& sc_out, uint8_t& zc_out) {
  constexpr float kThird = 0x1.555556p-2f;  // RN(1/3)
  constexpr float kRound = 12582912.0f;     // 1.5 * 2^23
  lo = __fadd_rn(lo, 0.0f);                 // -0 -> +0
  hi = __fadd_rn(hi, 0.0f);
  const uint8_t zc = f32_to_e4m3(lo);
  const float m = tab.dec[zc];
  const float span = __fsub_rn(hi, m);
  const float t0 = __fmul_rn(span, kThird);
  const uint8_t scb = f32_to_e4m3(__fmaf_rn(__fmaf_rn(-3.0f, t0, span), kThird, t0));
  const float s = tab.dec[scb];
  sc_out = scb;
  zc_out = zc;
  // s = 0 needs no branch: y = 0 makes every quotient +-0, hence code 0
  const float y = tab.rcp[scb];
  const float2 nm2 = f2(-m, -m), y2 = f2(y, y), ns2 = f2(-s, -s), k2 = f2(kRound, kRound), nk2 = f2(-kRound, -kRound);
  float2 pk2 = f2(0.0f, 0.0f);
#pragma unroll
  for (int e = 0; e < 8; e += 2) {
    const float2 d2 = __fadd2_rn(f2(r[e], r[e + 1]), nm2);
    const float2 q02 = __fmul2_rn(d2, y2);
    const float2 t2 = __ffma2_rn(__ffma2_rn(ns2, q02, d2), y2, q02);
    const float2 tc = f2(fminf(fmaxf(t2.x, 0.0f), 3.0f), fminf(fmaxf(t2.y, 0.0f), 3.0f));
    const float2 q2 = __fadd2_rn(__fadd2_rn(tc, k2), nk2);
    pk2 = __ffma2_rn(q2, f2((float)(1 << (2 * e)), (float)(1 << (2 * e + 2))), pk2);
  }
  const float pk = __fadd_rn(pk2.x, pk2.y);
  return __float_as_uint(__fadd_rn(pk, 8388608.0f)) & 0xFFFFu;   // 2^23: integer in the low bits
}

// The symmetric mode (one E4M3 byte per group): s = E4M3(max |r|),
// q = clamp(rint(fl(r / s)), -2, 1), stored u = q + 2, packed as in
// quant_chunk.  The quotient is the IEEE one by the same Markstein
// correction (the divisor is again an E4M3 value); rounding to nearest even
// is the add and subtract of 1.5 * 2^23 (exact for |q| <= 2), and u = q + 2
// is added after rounding.  s = 0 makes every quotient +-0, hence u = 2.
__device__ __forceinline__ uint32_t quant_chunk_sym(const float (&r)[8], float lo, float hi, const E4m3Tables& tab,
                                                    uint8_t& sc_out) {
  constexpr float kRound = 12582912.0f;     // 1.5 * 2^23
  const float amax = fmaxf(fabsf(lo), fabsf(hi));
  const uint8_t scb = f32_to_e4m3(amax);
  const float s = tab.dec[scb];
  sc_out = scb;
  const float y = tab.rcp[scb];
  const float2 y2 = f2(y, y), ns2 = f2(-s, -s), k2 = f2(kRound, kRound), nk2 = f2(-kRound, -kRound);
  const float2 two2 = f2(2.0f, 2.0f);
  float2 pk2 = f2(0.0f, 0.0f);
#pragma unroll
  for (int e = 0; e < 8; e += 2) {
    const float2 d2 = f2(r[e], r[e + 1]);
    const float2 q02 = __fmul2_rn(d2, y2);
    const float2 t2 = __ffma2_rn(__ffma2_rn(ns2, q02, d2), y2, q02);
    const float2 tc = f2(fminf(fmaxf(t2.x, -2.0f), 1.0f), fminf(fmaxf(t2.y, -2.0f), 1.0f));
    const float2 u2 = __fadd2_rn(__fadd2_rn(__fadd2_rn(tc, k2), nk2), two2);
    pk2 = __ffma2_rn(u2, f2((float)(1 << (2 * e)), (float)(1 << (2 * e + 2))), pk2);
  }
  const float pk = __fadd_rn(pk2.x, pk2.y);
  return __float_as_uint(__fadd_rn(pk, 8388608.0f)) & 0xFFFFu;   // 2^23: integer in the low bits
}

// GT > 0 fixes the group size at compile time (the quantising pass is
// instantiated for every supported G, so its group reductions and stores fold
// to straight-line code); GT = 0 reads it from the parameters.
template <int DT, bool QUANT, bool HAS_C, int GT, bool SYM>
__global__ void __launch_bounds__(kRqThreads)
qvg_residual_quant(const ResidualParams p, const int64_t per_block) {
  constexpr int ESZ = Store<DT>::bytes;
  extern __shared__ __align__(16) unsigned char smem[];
  const int u = blockIdx.y;
  const int64_t t0 = (int64_t)blockIdx.x * per_block;
  const int64_t t1 = min(p.N, t0 + per_block);
  if (HAS_C) {
    const uint4* src = reinterpret_cast<const uint4*>(static_cast<const char*>(p.C) + (int64_t)u * p.K * kD * ESZ);
    uint4* dst = reinterpret_cast<uint4*>(smem);
    const int n16 = p.K * kD * ESZ / 16;
    for (int x = threadIdx.x; x < n16; x += blockDim.x) dst[x] = src[x];
    __syncthreads();
  }
  // E4M3 decode and reciprocal tables for the quantiser
  __shared__ E4m3Tables s_tab;
  if (QUANT) {
    for (int c = threadIdx.x; c < 256; c += blockDim.x) {
      const float v = e4m3_to_f32((uint8_t)c);
      s_tab.dec[c] = v;
      s_tab.rcp[c] = (v == 0.0f || v != v) ? 0.0f : __frcp_rn(v);
    }
    __syncthreads();
  }
  // largest |value| per channel of the values this pass hands to the next
  // k-means (fixed-point scale of the centroid sums), and the smallest
  // nonzero |value| (whether every value fits that fixed point), when asked
  __shared__ uint32_t s_chmax[kD];
  __shared__ uint32_t s_chmin[kD];
  const bool want_max = !QUANT && p.chmax != nullptr;
  if (want_max) {
    for (int x = threadIdx.x; x < kD; x += blockDim.x) { s_chmax[x] = 0u; s_chmin[x] = 0u; }
    __syncthreads();
  }
  // Both extremes are kept on packed bf16 pairs (two channels per 32-bit
  // word; for fp32 data the words keep each value's exponent, see
  // bf16_pair_bits, which is all the fixed-point scale and its check use):
  //   xw = max of |v| (bf16 max of the sign-cleared word);
  //   nw = max of (|v| + 0x7FFF) per half: zero gives 0x7FFF, a NaN that the
  //        max ignores, and a nonzero h gives 0x8000 | (h - 1), i.e. -(h - 1),
  //        so the maximum is minus (smallest nonzero |v| - 1 ulp); no half
  //        carries into the other (each sum is at most 0xFFFE).
  uint32_t xw[8], nw[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) { xw[e] = 0u; nw[e] = 0x7FFF7FFFu; }
  const int j = threadIdx.x & 7;
  const int G = GT > 0 ? GT : p.G;
  const int ng = kD / G;
  const char* Rin = static_cast<const char*>(p.R_in) + (int64_t)u * p.N * kD * ESZ;
  // The loop bound is uniform across the warp (4 tokens per warp per
  // iteration) so that the group shuffles below always run on all 32 lanes;
  // lanes past the end work on a valid token and store nothing.
  const int64_t warp_tok = (threadIdx.x >> 5) * 4;
  for (int64_t ib = t0 + warp_tok; ib < t1; ib += kRqTokPerIter) {
    const int64_t iv = ib + ((threadIdx.x >> 3) & 3);
    const bool valid = iv < t1;
    const int64_t i = valid ? iv : ib;
    float r0[8], r1[8];
    Vec8<DT>::load(Rin + (i * kD + 8 * j) * ESZ, r0);
    Vec8<DT>::load(Rin + (i * kD + 64 + 8 * j) * ESZ, r1);
    if (HAS_C) {
      int k = p.pi[(int64_t)u * p.N + i];
      k = k < p.K ? k : p.K - 1;
      float c0[8], c1[8];
      const char* crow = reinterpret_cast<const char*>(smem) + (int64_t)k * kD * ESZ;
      Vec8<DT>::load(crow + 8 * j * ESZ, c0);
      Vec8<DT>::load(crow + (64 + 8 * j) * ESZ, c1);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        r0[e] = __fsub_rn(r0[e], c0[e]);
        r1[e] = __fsub_rn(r1[e], c1[e]);
      }
      Vec8<DT>::round(r0);
      Vec8<DT>::round(r1);
    }
    if (!QUANT) {
      if (valid && p.R_out != nullptr) {
        char* Ro = static_cast<char*>(p.R_out) + ((int64_t)u * p.N + i) * kD * ESZ;
        Vec8<DT>::store(Ro + 8 * j * ESZ, r0);
        Vec8<DT>::store(Ro + (64 + 8 * j) * ESZ, r1);
      }
      float s2 = 0.0f;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        s2 = __fmaf_rn(r0[e], r0[e], s2);
        s2 = __fmaf_rn(r1[e], r1[e], s2);
      }
      s2 += __shfl_xor_sync(0xffffffffu, s2, 1);
      s2 += __shfl_xor_sync(0xffffffffu, s2, 2);
      s2 += __shfl_xor_sync(0xffffffffu, s2, 4);
      if (valid && j == 0 && p.rnorm2 != nullptr) p.rnorm2[(int64_t)u * p.N + i] = s2;
      if (want_max) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const uint32_t a0 = bf16_pair_bits<DT == kFP32>(r0[2 * e], r0[2 * e + 1]) & 0x7FFF7FFFu;
          const uint32_t a1 = bf16_pair_bits<DT == kFP32>(r1[2 * e], r1[2 * e + 1]) & 0x7FFF7FFFu;
          xw[e] = bf16x2_max(xw[e], a0);
          xw[4 + e] = bf16x2_max(xw[4 + e], a1);
          nw[e] = bf16x2_max(nw[e], a0 + 0x7FFF7FFFu);
          nw[4 + e] = bf16x2_max(nw[4 + e], a1 + 0x7FFF7FFFu);
        }
      }
    } else {
      float lo0, hi0, lo1, hi1;
      minmax8(r0, lo0, hi0);
      minmax8(r1, lo1, hi1);
      if (G == 128) {
        lo0 = lo1 = fminf(lo0, lo1);
        hi0 = hi1 = fmaxf(hi0, hi1);
      }
      const int Gs = G > 64 ? 64 : G;
      lo0 = grp_min(lo0, Gs); hi0 = grp_max(hi0, Gs);
      lo1 = grp_min(lo1, Gs); hi1 = grp_max(hi1, Gs);
      uint8_t s0, z0 = 0, s1, z1 = 0;
      const uint32_t q0 = SYM ? quant_chunk_sym(r0, lo0, hi0, s_tab, s0) : quant_chunk(r0, lo0, hi0, s_tab, s0, z0);
      const uint32_t q1 = SYM ? quant_chunk_sym(r1, lo1, hi1, s_tab, s1) : quant_chunk(r1, lo1, hi1, s_tab, s1, z1);
      if (!valid) continue;
      const int64_t row = (int64_t)u * p.N + i;
      uint8_t* cr = p.codes + row * (kD / 4);
      *reinterpret_cast<uint16_t*>(cr + 2 * j) = (uint16_t)q0;
      *reinterpret_cast<uint16_t*>(cr + 16 + 2 * j) = (uint16_t)q1;
      if ((8 * j) % G == 0) {
        p.scale[row * ng + (8 * j) / G] = s0;
        if (!SYM) p.zero[row * ng + (8 * j) / G] = z0;
      }
      if (G < 128 && (64 + 8 * j) % G == 0) {
        p.scale[row * ng + (64 + 8 * j) / G] = s1;
        if (!SYM) p.zero[row * ng + (64 + 8 * j) / G] = z1;
      }
    }
  }
  if (want_max) {
    // lanes j, j+8, j+16, j+24 hold the same channels (invalid lanes repeat a
    // valid token, so they never raise a maximum)
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      xw[e] = bf16x2_max(xw[e], __shfl_xor_sync(0xffffffffu, xw[e], 8));
      xw[e] = bf16x2_max(xw[e], __shfl_xor_sync(0xffffffffu, xw[e], 16));
      nw[e] = bf16x2_max(nw[e], __shfl_xor_sync(0xffffffffu, nw[e], 8));
      nw[e] = bf16x2_max(nw[e], __shfl_xor_sync(0xffffffffu, nw[e], 16));
    }
    // chmax holds fp32 bits of the largest |v|; chmin holds 0x7FFFFFFF minus
    // the fp32 bits of the smallest nonzero |v|, so that an atomic maximum
    // finds it and zero means "no nonzero value"
    if ((threadIdx.x & 31) < 8) {
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const int c0 = (e < 4 ? 8 * j + 2 * e : 64 + 8 * j + 2 * (e - 4));
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          const uint32_t x = (xw[e] >> (16 * hf)) & 0xFFFFu;
          const uint32_t n = (nw[e] >> (16 * hf)) & 0xFFFFu;
          atomicMax(&s_chmax[c0 + hf], x << 16);
          if ((n & 0x7FFFu) <= 0x7F80u)        // not the NaN of an all-zero channel
            atomicMax(&s_chmin[c0 + hf], 0x7FFFFFFFu - ((((n & 0x7FFFu) + 1u)) << 16));
        }
      }
    }
    __syncthreads();
    for (int x = threadIdx.x; x < kD; x += blockDim.x) {
      if (s_chmax[x] != 0u) atomicMax(&p.chmax[(int64_t)u * kD + x], s_chmax[x]);
      if (s_chmin[x] != 0u) atomicMax(&p.chmin[(int64_t)u * kD + x], s_chmin[x]);
    }
  }
}

// ---------------------------------------------------------------- range statistic
// The adaptive cache's per-chunk statistic: over every block, token and
// group of G channels, the sum of the E4M3 codes of the group's range
// fl32(max - min).  Sixteen threads per token, thread c owning channels
// 8c .. 8c+7; a group's extremes are combined over its G/8 threads by
// xor-shuffles, and its first thread adds the code.  Adding +0 maps a -0
// range to +0 (the code of a zero range is 0).
template <int DT>
__global__ void __launch_bounds__(256)
qvg_range_stat(const void* X, int64_t rows, int G, unsigned long long* out) {
  constexpr int ESZ = Store<DT>::bytes;
  const int c = threadIdx.x & 15;
  const int64_t row = (int64_t)blockIdx.x * 16 + (threadIdx.x >> 4);
  const bool valid = row < rows;
  float v[8];
  Vec8<DT>::load(static_cast<const char*>(X) + ((valid ? row : 0) * kD + 8 * c) * ESZ, v);
  float lo, hi;
  minmax8(v, lo, hi);
  for (int w = 1; w < G / 8; w <<= 1) {
    lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, w));
    hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, w));
  }
  uint32_t code = 0;
  if (valid && (c % (G / 8)) == 0) code = f32_to_e4m3(__fadd_rn(__fsub_rn(hi, lo), 0.0f));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) code += __shfl_xor_sync(0xffffffffu, code, off);
  __shared__ uint32_t part[8];
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = code;
  __syncthreads();
  if (threadIdx.x == 0) {
    unsigned long long sum = 0;
    for (int w = 0; w < 8; ++w) sum += part[w];
    atomicAdd(out, sum);
  }
}

// ---------------------------------------------------------------- centroid init
template <int DT>
__global__ void __launch_bounds__(256)
qvg_init_centroids(const void* src, int64_t src_unit_stride, void* C, float* cn, int K) {
  constexpr int ESZ = Store<DT>::bytes;
  const int u = blockIdx.y;
  const int k = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (k >= K) return;
  const char* s = static_cast<const char*>(src) + ((int64_t)u * src_unit_stride + (int64_t)k * kD) * ESZ;
  char* d = static_cast<char*>(C) + ((int64_t)u * K + k) * kD * ESZ;
  double acc = 0.0;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const int jj = lane * 4 + e;
    float v;
    if (DT == kBF16) {
      const uint16_t b = reinterpret_cast<const uint16_t*>(s)[jj];
      reinterpret_cast<uint16_t*>(d)[jj] = b;
      v = bf16_bits_to_f32(b);
    } else {
      v = reinterpret_cast<const float*>(s)[jj];
      reinterpret_cast<float*>(d)[jj] = v;
    }
    acc = __dadd_rn(acc, __dmul_rn((double)v, (double)v));
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc = __dadd_rn(acc, __shfl_xor_sync(0xffffffffu, acc, off));
  if (lane == 0) cn[(int64_t)u * K + k] = __double2float_rn(acc);
}

template <typename F>
cudaError_t set_smem(F* f, size_t bytes) {
  return ensure_dynamic_smem(reinterpret_cast<const void*>(f), bytes);
}

}  // namespace

cudaError_t launch_dequant(const DequantParams& p, int dtype, cudaStream_t s) {
  const int esz = dtype == kBF16 ? 2 : 4;
  const size_t smem = (size_t)p.t_smem * p.K * kD * esz + 16 * sizeof(float2);
  const int units = p.n_chunks * p.H;
  if (units == 0) return cudaSuccess;
  if (p.desc != nullptr) {                       // per-chunk layouts: the generic instance
    DequantParams q = p;
    q.T = -1;                                    // selects it below; the kernel reads each chunk's T
    const int splits = 1;
    return dtype == kBF16 ? (p.sym ? launch_dq_t<kBF16, true>(q, units * splits, splits, smem, s)
                                   : launch_dq_t<kBF16, false>(q, units * splits, splits, smem, s))
                          : (p.sym ? launch_dq_t<kFP32, true>(q, units * splits, splits, smem, s)
                                   : launch_dq_t<kFP32, false>(q, units * splits, splits, smem, s));
  }
  const int sms = device_sm_count();
  // One resident block per SM: split blocks along tokens until the grid is
  // about four waves, so that the last one is short and every block stages
  // its tables once for a few thousand tokens.
  int splits = (4 * sms + units - 1) / units;
  const int64_t ntok = p.chunk_off ? 0 : p.N;
  if (ntok > 0) {
    const int64_t max_splits = (ntok + 1023) / 1024;
    if (splits > max_splits) splits = (int)max_splits;
  } else if (splits > 8) {
    splits = 8;
  }
  if (splits < 1) splits = 1;
  const int blocks = units * splits;
  if (p.sym)
    return dtype == kBF16 ? launch_dq_t<kBF16, true>(p, blocks, splits, smem, s)
                          : launch_dq_t<kFP32, true>(p, blocks, splits, smem, s);
  return dtype == kBF16 ? launch_dq_t<kBF16, false>(p, blocks, splits, smem, s)
                        : launch_dq_t<kFP32, false>(p, blocks, splits, smem, s);
}

template <int DT, bool Q, bool C, int GT, bool SYM>
static cudaError_t launch_rq_g(const ResidualParams& p, dim3 grid, int64_t per, size_t smem, cudaStream_t s) {
  cudaError_t e = set_smem(qvg_residual_quant<DT, Q, C, GT, SYM>, smem);
  if (e != cudaSuccess) return e;
  qvg_residual_quant<DT, Q, C, GT, SYM><<<grid, kRqThreads, smem, s>>>(p, per);
  return cudaGetLastError();
}

template <int DT, bool Q, bool C, bool SYM>
static cudaError_t launch_rq_mode(const ResidualParams& p, dim3 grid, int64_t per, size_t smem, cudaStream_t s) {
  switch (p.G) {
    case 8: return launch_rq_g<DT, Q, C, 8, SYM>(p, grid, per, smem, s);
    case 16: return launch_rq_g<DT, Q, C, 16, SYM>(p, grid, per, smem, s);
    case 32: return launch_rq_g<DT, Q, C, 32, SYM>(p, grid, per, smem, s);
    case 64: return launch_rq_g<DT, Q, C, 64, SYM>(p, grid, per, smem, s);
    case 128: return launch_rq_g<DT, Q, C, 128, SYM>(p, grid, per, smem, s);
    default: return launch_rq_g<DT, Q, C, 0, SYM>(p, grid, per, smem, s);
  }
}

// The quantising pass takes the instance of its group size and scale mode;
// the others use neither.
template <int DT, bool Q, bool C>
static cudaError_t launch_rq(const ResidualParams& p, dim3 grid, int64_t per, size_t smem, cudaStream_t s) {
  if (!Q) return launch_rq_g<DT, Q, C, 0, false>(p, grid, per, smem, s);
  return p.sym ? launch_rq_mode<DT, Q, C, true>(p, grid, per, smem, s)
               : launch_rq_mode<DT, Q, C, false>(p, grid, per, smem, s);
}

cudaError_t launch_residual(const ResidualParams& p, int dtype, bool quant, cudaStream_t s) {
  const int esz = dtype == kBF16 ? 2 : 4;
  const bool has_c = p.C != nullptr;
  const size_t smem = has_c ? (size_t)p.K * kD * esz : 0;
  const int sms = device_sm_count();
  // About eight blocks per SM (four waves at two resident blocks per SM), so
  // that the last wave is short; each block stages the table once.
  int64_t splits = (8 * (int64_t)sms + p.W - 1) / p.W;
  const int64_t min_tok = 256;
  if (splits * min_tok > p.N) splits = (p.N + min_tok - 1) / min_tok;
  if (splits < 1) splits = 1;
  const int64_t per = (p.N + splits - 1) / splits;
  const dim3 grid((unsigned)splits, (unsigned)p.W);
  if (dtype == kBF16) {
    if (quant) return has_c ? launch_rq<kBF16, true, true>(p, grid, per, smem, s)
                            : launch_rq<kBF16, true, false>(p, grid, per, smem, s);
    return has_c ? launch_rq<kBF16, false, true>(p, grid, per, smem, s)
                 : launch_rq<kBF16, false, false>(p, grid, per, smem, s);
  }
  if (quant) return has_c ? launch_rq<kFP32, true, true>(p, grid, per, smem, s)
                          : launch_rq<kFP32, true, false>(p, grid, per, smem, s);
  return has_c ? launch_rq<kFP32, false, true>(p, grid, per, smem, s)
               : launch_rq<kFP32, false, false>(p, grid, per, smem, s);
}

cudaError_t launch_range_stat(const void* X, int64_t rows, int G, int dtype, unsigned long long* out,
                              cudaStream_t s) {
  if (rows <= 0) return cudaSuccess;
  const unsigned grid = (unsigned)((rows + 15) / 16);
  if (dtype == kBF16) qvg_range_stat<kBF16><<<grid, 256, 0, s>>>(X, rows, G, out);
  else qvg_range_stat<kFP32><<<grid, 256, 0, s>>>(X, rows, G, out);
  return cudaGetLastError();
}

cudaError_t launch_init_centroids(const void* src, int64_t src_unit_stride, void* C,
                                  float* cn, int W, int K, int dtype, cudaStream_t s) {
  const dim3 grid((unsigned)((K + 7) / 8), (unsigned)W);
  if (dtype == kBF16) qvg_init_centroids<kBF16><<<grid, 256, 0, s>>>(src, src_unit_stride, C, cn, K);
  else qvg_init_centroids<kFP32><<<grid, 256, 0, s>>>(src, src_unit_stride, C, cn, K);
  return cudaGetLastError();
}

}  // namespace qvg
