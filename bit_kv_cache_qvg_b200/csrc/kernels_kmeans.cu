// kernels_kmeans.cu -- k-means steps of semantic-aware smoothing (m.163.com
// article on Quant VideoGen, section 三: tokens grouped by k-means, the group
// mean is the centroid) on sm_100a CUDA cores:
//   * qvg_assign_exact: the assignment of a token (or of a list of flagged
//     tokens) decided exactly.  fp32 screening distances g_k = |c_k|^2 - 2 r.c_k
//     for all centroids, then the exact fp64 squared distance (channels in
//     ascending order, separate subtract / multiply / add) for every centroid
//     whose screening value lies within the rounding-error bound of the
//     minimum; ties go to the lowest index.
//   * qvg_kmeans_update: per 2048-token segment a stable counting sort of the
//     tokens by centroid, fp64 sums of each centroid's tokens in ascending
//     order, then a fixed-order reduction over segments, the mean (one fp64
//     divide) and one rounding to the storage dtype; an empty centroid keeps
//     its value.  The reduction order never depends on scheduling, so the
//     result is deterministic.
#include "qvg_common.cuh"
#include "qvg_launch.h"

namespace qvg {
namespace {

// ---------------------------------------------------------------- assign
constexpr int kAsThreads = 256;
constexpr int kAsWarps = kAsThreads / 32;
constexpr float kExactGamma = 1.52587890625e-05f;   // 2^-16

// Screening error bound.  For any centroid at least as close as the true
// nearest one, |c_k| <= |r| + sqrt(D_min); the fp32 dot product of 128 terms
// is within gamma * |r| * |c_k| of the exact value with gamma = 2^-16 (twice
// the classical 128 * 2^-24 bound), |c_k|^2 is rounded once (2^-24 relative)
// and the final fused multiply-add once more.  Any centroid whose screening
// value is within twice that bound of the minimum is decided exactly.
__device__ __forceinline__ float screening_threshold(float gmin, float rn2, float gamma) {
  const float nr = sqrtf(fmaxf(rn2, 0.0f)) * 1.0001f;
  const float dmin = fmaxf(rn2 + gmin, 0.0f);
  const float cb = 1.02f * nr + sqrtf(dmin);
  const float E = 2.0f * gamma * nr * cb + 1.2e-7f * cb * cb + 1.2e-7f * fabsf(gmin) + 1e-30f;
  return gmin + 2.0f * E;
}

template <int DT>
__global__ void __launch_bounds__(kAsThreads)
qvg_assign_exact(const AssignParams p) {
  using ST = typename Store<DT>::T;
  constexpr int ESZ = Store<DT>::bytes;
  extern __shared__ __align__(16) unsigned char smem[];
  const int u = blockIdx.y;
  const int K = p.K;
  const int Kp = (K + 31) & ~31;
  const int NM = Kp / 32;                       // centroid slots per lane (<= 8)
  // Rows handled by this block: e = (blockIdx.x * warps + warp) + k * (gridDim.x * warps).
  const int64_t n_rows = p.list ? (int64_t)p.list_count[u] : p.N;
  if ((int64_t)blockIdx.x * kAsWarps >= n_rows) return;   // nothing for this block
  // Transposed table [kD][Ks] with a padded row stride Ks (Kp + 2 values for
  // bf16, Kp + 1 for fp32) so that writing it column by column and reading it
  // row by row are both free of bank conflicts.
  const int Ks = Kp + (ESZ == 2 ? 2 : 1);
  ST* Ct = reinterpret_cast<ST*>(smem);
  float* cn_s = reinterpret_cast<float*>(smem + (((size_t)kD * Ks * ESZ + 15) & ~size_t(15)));
  float* rbuf = cn_s + kMaxK;                   // [warps][kD]

  // Stage the table: each thread moves one 16-byte piece of a centroid row
  // (consecutive threads take consecutive centroids of the same piece, so the
  // transposed shared-memory writes are conflict-free).
  const ST* Cg = static_cast<const ST*>(p.C) + (int64_t)u * K * kD;
  constexpr int kPer16 = 16 / ESZ;                       // values per 16-byte piece
  for (int x = threadIdx.x; x < Kp * (kD / kPer16); x += blockDim.x) {
    const int k = x % Kp, piece = x / Kp;
    ST v[kPer16];
    if (k < K) {
      *reinterpret_cast<uint4*>(v) = *reinterpret_cast<const uint4*>(Cg + (int64_t)k * kD + piece * kPer16);
    } else {
#pragma unroll
      for (int e = 0; e < kPer16; ++e) v[e] = Store<DT>::from_f32(0.0f);
    }
#pragma unroll
    for (int e = 0; e < kPer16; ++e) Ct[(piece * kPer16 + e) * Ks + k] = v[e];
  }
  for (int k = threadIdx.x; k < Kp; k += blockDim.x)
    cn_s[k] = k < K ? p.cn[(int64_t)u * K + k] : __int_as_float(0x7f800000);
  __syncthreads();

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float* rw = rbuf + warp * kD;
  const char* Rg = static_cast<const char*>(p.R) + (int64_t)u * p.N * kD * ESZ;
  const int64_t stride = (int64_t)gridDim.x * kAsWarps;

  for (int64_t e = (int64_t)blockIdx.x * kAsWarps + warp; e < n_rows; e += stride) {
    const int64_t i = p.list ? (int64_t)p.list[(int64_t)u * p.N + e] : e;
    // row -> shared (fp32, exact)
    const char* rrow = Rg + i * kD * ESZ;
    if (DT == kBF16) {
      const uint2 w = *reinterpret_cast<const uint2*>(rrow + lane * 8);
      rw[4 * lane + 0] = __uint_as_float(w.x << 16);
      rw[4 * lane + 1] = __uint_as_float(w.x & 0xFFFF0000u);
      rw[4 * lane + 2] = __uint_as_float(w.y << 16);
      rw[4 * lane + 3] = __uint_as_float(w.y & 0xFFFF0000u);
    } else {
      const float4 w = *reinterpret_cast<const float4*>(rrow + lane * 16);
      rw[4 * lane + 0] = w.x; rw[4 * lane + 1] = w.y; rw[4 * lane + 2] = w.z; rw[4 * lane + 3] = w.w;
    }
    __syncwarp();
    float dot[8];
#pragma unroll
    for (int m = 0; m < 8; ++m) dot[m] = 0.0f;
#pragma unroll 4
    for (int jj = 0; jj < kD; ++jj) {
      const float rj = rw[jj];
      const ST* crow = Ct + jj * Ks + lane;
#pragma unroll
      for (int m = 0; m < 8; ++m)
        if (m < NM) dot[m] = __fmaf_rn(rj, Store<DT>::ld(crow + 32 * m), dot[m]);
    }
    float g[8];
    float gmin = __int_as_float(0x7f800000);
#pragma unroll
    for (int m = 0; m < 8; ++m) {
      g[m] = (m < NM) ? __fmaf_rn(-2.0f, dot[m], cn_s[lane + 32 * m]) : __int_as_float(0x7f800000);
      gmin = fminf(gmin, g[m]);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) gmin = fminf(gmin, __shfl_xor_sync(0xffffffffu, gmin, off));
    const float thr = screening_threshold(gmin, p.rnorm2[(int64_t)u * p.N + i], kExactGamma);

    double bestD = __longlong_as_double(0x7ff0000000000000ll);
    int bestK = 0x7fffffff;
#pragma unroll
    for (int m = 0; m < 8; ++m) {
      if (m < NM && g[m] <= thr) {
        const int k = lane + 32 * m;
        double D = 0.0;
        for (int jj = 0; jj < kD; ++jj) {
          const double diff = __dsub_rn((double)rw[jj], (double)Store<DT>::ld(Ct + jj * Ks + k));
          D = __dadd_rn(D, __dmul_rn(diff, diff));
        }
        if (D < bestD) { bestD = D; bestK = k; }
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const double oD = __shfl_xor_sync(0xffffffffu, bestD, off);
      const int oK = __shfl_xor_sync(0xffffffffu, bestK, off);
      if (oD < bestD || (oD == bestD && oK < bestK)) { bestD = oD; bestK = oK; }
    }
    if (lane == 0) p.pi[(int64_t)u * p.N + i] = (uint8_t)bestK;
    __syncwarp();
  }
}

// ---------------------------------------------------------------- listed near-ties
constexpr int kCandWarps = 8;

// Exact squared distance, fp64, channels in ascending order (one subtract,
// multiply and add per channel), centroid row read from global memory.
template <int DT>
__device__ __forceinline__ double exact_dist(const float* rw, const char* crow) {
  double D = 0.0;
#pragma unroll 2
  for (int j0 = 0; j0 < kD; j0 += 8) {
    float c[8];
    if (DT == kBF16) {
      const uint4 w = *reinterpret_cast<const uint4*>(crow + j0 * 2);
      const uint32_t x[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        c[2 * e] = __uint_as_float(x[e] << 16);
        c[2 * e + 1] = __uint_as_float(x[e] & 0xFFFF0000u);
      }
    } else {
      const float4 a = *reinterpret_cast<const float4*>(crow + j0 * 4);
      const float4 b = *reinterpret_cast<const float4*>(crow + j0 * 4 + 16);
      c[0] = a.x; c[1] = a.y; c[2] = a.z; c[3] = a.w; c[4] = b.x; c[5] = b.y; c[6] = b.z; c[7] = b.w;
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const double diff = __dsub_rn((double)rw[j0 + e], (double)c[e]);
      D = __dadd_rn(D, __dmul_rn(diff, diff));
    }
  }
  return D;
}

template <int DT>
__global__ void __launch_bounds__(kCandWarps * 32)
qvg_assign_candidates(const void* R, const void* C, const int K, const int64_t N, const uint2* list,
                      const uint32_t* list_count, uint8_t* pi) {
  constexpr int ESZ = Store<DT>::bytes;
  __shared__ float rbuf[kCandWarps][kD];
  const int u = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t n_rows = min((int64_t)list_count[u], N);
  const int64_t stride = (int64_t)gridDim.x * kCandWarps;
  float* rw = rbuf[warp];
  const char* Ru = static_cast<const char*>(R) + (int64_t)u * N * kD * ESZ;
  const char* Cu = static_cast<const char*>(C) + (int64_t)u * K * kD * ESZ;
  const uint32_t all = (K + 31) / 32 >= 32 ? 0xFFFFFFFFu : ((1u << ((K + 31) / 32)) - 1u);
  for (int64_t e = (int64_t)blockIdx.x * kCandWarps + warp; e < n_rows; e += stride) {
    const uint2 ent = list[(int64_t)u * N + e];
    const int64_t tok = ent.x;
    if (tok >= N) continue;                    // warp-uniform; never true for listed tokens
    uint32_t chunks = ent.y & all;
    if (chunks == 0) chunks = all;
    const char* rrow = Ru + tok * kD * ESZ;
    if (DT == kBF16) {
      const uint2 w = *reinterpret_cast<const uint2*>(rrow + lane * 8);
      rw[4 * lane + 0] = __uint_as_float(w.x << 16);
      rw[4 * lane + 1] = __uint_as_float(w.x & 0xFFFF0000u);
      rw[4 * lane + 2] = __uint_as_float(w.y << 16);
      rw[4 * lane + 3] = __uint_as_float(w.y & 0xFFFF0000u);
    } else {
      const float4 w = *reinterpret_cast<const float4*>(rrow + lane * 16);
      rw[4 * lane + 0] = w.x; rw[4 * lane + 1] = w.y; rw[4 * lane + 2] = w.z; rw[4 * lane + 3] = w.w;
    }
    __syncwarp();
    double bestD = __longlong_as_double(0x7ff0000000000000ll);
    int bestK = 0x7fffffff;
    // chunks in ascending order; lane takes centroid 32*chunk + lane
    while (chunks) {
      const int c = __ffs(chunks) - 1;
      chunks &= chunks - 1;
      const int k = c * 32 + lane;
      if (k < K) {
        const double D = exact_dist<DT>(rw, Cu + (int64_t)k * kD * ESZ);
        if (D < bestD) { bestD = D; bestK = k; }
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const double oD = __shfl_xor_sync(0xffffffffu, bestD, off);
      const int oK = __shfl_xor_sync(0xffffffffu, bestK, off);
      if (oD < bestD || (oD == bestD && oK < bestK)) { bestD = oD; bestK = oK; }
    }
    if (lane == 0) pi[(int64_t)u * N + tok] = (uint8_t)bestK;
    __syncwarp();
  }
}

// ---------------------------------------------------------------- update
constexpr int kUpThreads = 512;
constexpr int kUpWarps = kUpThreads / 32;
constexpr int kTokPerWarp = kSeg / kUpWarps;      // 128
constexpr int kRounds = kTokPerWarp / 32;         // 4
constexpr int kBatch = 8;                         // rows in flight per warp

// Exact widening of a bf16 / fp32 value to fp64 with integer operations (the
// exponent is rebiased, the significand shifted); zero, subnormal, infinite
// and NaN inputs take the conversion instruction.
__device__ __forceinline__ double widen_bf16(uint32_t b) {
  const uint32_t e = (b >> 7) & 0xFFu;
  if (e == 0u || e == 0xFFu) return (double)__uint_as_float(b << 16);
  const unsigned long long bits = ((unsigned long long)(b & 0x8000u) << 48) |
                                  ((unsigned long long)(e + 896u) << 52) |
                                  ((unsigned long long)(b & 0x7Fu) << 45);
  return __longlong_as_double((long long)bits);
}
__device__ __forceinline__ double widen_f32(uint32_t f) {
  const uint32_t e = (f >> 23) & 0xFFu;
  if (e == 0u || e == 0xFFu) return (double)__uint_as_float(f);
  const unsigned long long bits = ((unsigned long long)(f & 0x80000000u) << 32) |
                                  ((unsigned long long)(e + 896u) << 52) |
                                  ((unsigned long long)(f & 0x7FFFFFu) << 29);
  return __longlong_as_double((long long)bits);
}

// Lane's four channels of a row as raw 32-bit words (bf16 pairs or fp32).
template <int DT>
__device__ __forceinline__ void load4raw(const char* row, int lane, uint32_t (&w)[4]) {
  if (DT == kBF16) {
    const uint2 x = *reinterpret_cast<const uint2*>(row + lane * 8);
    w[0] = x.x & 0xFFFFu; w[1] = x.x >> 16; w[2] = x.y & 0xFFFFu; w[3] = x.y >> 16;
  } else {
    const uint4 x = *reinterpret_cast<const uint4*>(row + lane * 16);
    w[0] = x.x; w[1] = x.y; w[2] = x.z; w[3] = x.w;
  }
}
template <int DT>
__device__ __forceinline__ double widen(uint32_t w) {
  return DT == kBF16 ? widen_bf16(w) : widen_f32(w);
}

template <int DT>
__device__ __forceinline__ void load4(const char* row, int lane, float (&v)[4]) {
  if (DT == kBF16) {
    const uint2 w = *reinterpret_cast<const uint2*>(row + lane * 8);
    v[0] = __uint_as_float(w.x << 16);
    v[1] = __uint_as_float(w.x & 0xFFFF0000u);
    v[2] = __uint_as_float(w.y << 16);
    v[3] = __uint_as_float(w.y & 0xFFFF0000u);
  } else {
    const float4 w = *reinterpret_cast<const float4*>(row + lane * 16);
    v[0] = w.x; v[1] = w.y; v[2] = w.z; v[3] = w.w;
  }
}

template <int DT>
__global__ void __launch_bounds__(kUpThreads, 2)
qvg_update_partial(const UpdateParams p) {
  constexpr int ESZ = Store<DT>::bytes;
  constexpr int kMaxC = 2 * kSeg;                  // contributions per segment
  __shared__ uint16_t hist[kUpWarps][kMaxK];      // per-warp counts, then offsets
  __shared__ int tot[kMaxK];
  __shared__ int start[kMaxK];
  __shared__ int dsum[kMaxK];
  __shared__ uint16_t sorted[kMaxC];              // token | 0x8000 when subtracted
  __shared__ uint8_t sorted_k[kMaxC];
  __shared__ int wsum[kMaxK / 32];
  __shared__ double2 piece[kUpWarps][kD / 2];     // first run of each warp when it continues a centroid

  const int u = blockIdx.y, sgi = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t seg0 = (int64_t)sgi * kSeg;
  const int seg_len = (int)min((int64_t)kSeg, p.N - seg0);
  const uint8_t* pn = p.pi + (int64_t)u * p.N + seg0;
  const uint8_t* po = p.pi_old ? p.pi_old + (int64_t)u * p.N + seg0 : nullptr;

  for (int x = threadIdx.x; x < kUpWarps * kMaxK; x += blockDim.x) (&hist[0][0])[x] = 0;
  for (int x = threadIdx.x; x < kMaxK; x += blockDim.x) dsum[x] = 0;
  __syncthreads();

  // 1. Stable per-warp ranks of the contributions.  Warp w owns tokens
  //    [w*128, w*128+128); its contributions are taken in a fixed order:
  //    pass 0 = subtractions (old centroid), pass 1 = additions (new centroid).
  // the warp's 128 assignments (and the previous ones), loaded up front:
  // round r of lane l is token w*128 + r*32 + l
  uint8_t an[kRounds], ao[kRounds];
#pragma unroll
  for (int r = 0; r < kRounds; ++r) {
    const int tok = warp * kTokPerWarp + r * 32 + lane;
    an[r] = tok < seg_len ? pn[tok] : 0;
    ao[r] = (po != nullptr && tok < seg_len) ? po[tok] : 0;
  }
  int key[2][kRounds], rank[2][kRounds];
#pragma unroll
  for (int ps = 0; ps < 2; ++ps) {
#pragma unroll
    for (int r = 0; r < kRounds; ++r) {
      const int tok = warp * kTokPerWarp + r * 32 + lane;
      bool valid = tok < seg_len;
      int k = 0;
      if (valid) {
        const int kn = an[r];
        if (po == nullptr) { valid = ps == 1; k = kn; }
        else {
          const int ko = ao[r];
          valid = ko != kn;
          k = ps == 0 ? ko : kn;
        }
      }
      key[ps][r] = valid ? k : 0x10000 + lane;           // invalid keys never match
      const unsigned mask = __match_any_sync(0xffffffffu, key[ps][r]);
      const int before = __popc(mask & ((1u << lane) - 1u));
      const int base = valid ? hist[warp][k] : 0;
      __syncwarp();
      if (valid && before == 0) {
        hist[warp][k] = (uint16_t)(base + __popc(mask));
        atomicAdd(&dsum[k], ps == 0 ? -__popc(mask) : __popc(mask));
      }
      __syncwarp();
      rank[ps][r] = base + before;
    }
  }
  __syncthreads();

  // 2. Exclusive prefix over (k, w): offsets of each warp's run of centroid k.
  if (threadIdx.x < kMaxK) {
    const int k = threadIdx.x;
    int run = 0;
    for (int w = 0; w < kUpWarps; ++w) {
      const int c = hist[w][k];
      hist[w][k] = (uint16_t)run;
      run += c;
    }
    tot[k] = run;
    int v = run;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int o = __shfl_up_sync(0xffffffffu, v, off);
      if (lane >= off) v += o;
    }
    if (lane == 31) wsum[k >> 5] = v;
    start[k] = v - run;
  }
  __syncthreads();
  if (threadIdx.x < kMaxK) {
    const int k = threadIdx.x;
    int add = 0;
    for (int w = 0; w < (k >> 5); ++w) add += wsum[w];
    start[k] += add;
    if (k < p.K) {
      const int64_t o = ((int64_t)u * p.nseg + sgi) * p.K + k;
      p.ncontrib[o] = tot[k];
      p.dcount[o] = dsum[k];
    }
  }
  __syncthreads();
  const int total = start[kMaxK - 1] + tot[kMaxK - 1];

  // 3. Scatter into centroid order (stable within a centroid).
#pragma unroll
  for (int ps = 0; ps < 2; ++ps) {
#pragma unroll
    for (int r = 0; r < kRounds; ++r) {
      const int k = key[ps][r];
      if (k < 0x10000) {
        const int tok = warp * kTokPerWarp + r * 32 + lane;
        const int pos = start[k] + hist[warp][k] + rank[ps][r];
        sorted[pos] = (uint16_t)(tok | (ps == 0 ? 0x8000 : 0));
        sorted_k[pos] = (uint8_t)k;
      }
    }
  }
  __syncthreads();

  // 4. Each warp sums an equal share of the sorted contributions (lane owns 4
  //    channels) run by run.  A run holding all of a centroid's contributions
  //    is written out directly; a warp's first run that continues a centroid
  //    from the previous warp is parked in shared memory; a last run that
  //    continues into the next warp is completed by this warp after the
  //    barrier, adding the parked pieces in warp order.
  const char* R = static_cast<const char*>(p.R) + ((int64_t)u * p.N + seg0) * kD * ESZ;
  double* part = p.partial + ((int64_t)u * p.nseg + sgi) * p.K * kD;
  const int share = (total + kUpWarps - 1) / kUpWarps;
  const int r0 = min(total, warp * share);
  const int r1 = min(total, r0 + share);
  int cur = -1, cur_begin = r0;
  double a0 = 0.0, a1 = 0.0, a2 = 0.0, a3 = 0.0;
  int own_k = -1;
  double o0 = 0.0, o1 = 0.0, o2 = 0.0, o3 = 0.0;
  auto emit = [&](int k, int run_begin, int run_end) {
    const int cb = start[k], ce = start[k] + tot[k];
    if (cb >= run_begin && ce <= run_end) {            // all of the centroid's contributions
      double2* dst = reinterpret_cast<double2*>(part + (int64_t)k * kD + lane * 4);
      dst[0] = make_double2(a0, a1);
      dst[1] = make_double2(a2, a3);
    } else if (cb < run_begin) {                        // continues a centroid: park it
      piece[warp][lane * 2] = make_double2(a0, a1);
      piece[warp][lane * 2 + 1] = make_double2(a2, a3);
    } else {                                            // starts here, continues past r1
      own_k = k; o0 = a0; o1 = a1; o2 = a2; o3 = a3;
    }
  };
  for (int b = r0; b < r1; b += kBatch) {
    uint32_t v[kBatch][4];
    int kk[kBatch];
    bool neg[kBatch];
#pragma unroll
    for (int q = 0; q < kBatch; ++q) {
      const int pos = min(b + q, r1 - 1);
      kk[q] = sorted_k[pos];
      const int e = sorted[pos];
      neg[q] = (e & 0x8000) != 0;
      load4raw<DT>(R + (int64_t)(e & 0x7FFF) * kD * ESZ, lane, v[q]);
    }
#pragma unroll
    for (int q = 0; q < kBatch; ++q) {
      if (b + q < r1) {
        if (kk[q] != cur) {
          if (cur >= 0) emit(cur, cur_begin, b + q);
          cur = kk[q];
          cur_begin = b + q;
          a0 = a1 = a2 = a3 = 0.0;
        }
        // a subtraction adds the negated value (a sign flip, exact)
        const double x0 = widen<DT>(v[q][0]), x1 = widen<DT>(v[q][1]);
        const double x2 = widen<DT>(v[q][2]), x3 = widen<DT>(v[q][3]);
        a0 = __dadd_rn(a0, neg[q] ? -x0 : x0);
        a1 = __dadd_rn(a1, neg[q] ? -x1 : x1);
        a2 = __dadd_rn(a2, neg[q] ? -x2 : x2);
        a3 = __dadd_rn(a3, neg[q] ? -x3 : x3);
      }
    }
  }
  if (cur >= 0) emit(cur, cur_begin, r1);
  __syncthreads();
  if (own_k >= 0) {
    const int last_w = min(kUpWarps - 1, (start[own_k] + tot[own_k] - 1) / share);
    for (int w = warp + 1; w <= last_w; ++w) {
      const double2 x = piece[w][lane * 2], y = piece[w][lane * 2 + 1];
      o0 = __dadd_rn(o0, x.x); o1 = __dadd_rn(o1, x.y);
      o2 = __dadd_rn(o2, y.x); o3 = __dadd_rn(o3, y.y);
    }
    double2* dst = reinterpret_cast<double2*>(part + (int64_t)own_k * kD + lane * 4);
    dst[0] = make_double2(o0, o1);
    dst[1] = make_double2(o2, o3);
  }
}

// Running sums += segment sums (segments in order), counts += changes, then
// the mean of every non-empty centroid, rounded once to the storage dtype.
template <int DT>
__global__ void __launch_bounds__(256)
qvg_update_finalize(const UpdateParams p) {
  const int u = blockIdx.y;
  const int k = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (k >= p.K) return;
  const int64_t seg_stride = (int64_t)p.K * kD;
  const int* nc = p.ncontrib + (int64_t)u * p.nseg * p.K + k;
  const int* dc = p.dcount + (int64_t)u * p.nseg * p.K + k;
  const double* part = p.partial + ((int64_t)u * p.nseg * p.K + k) * kD + lane * 4;
  double2* Sk = reinterpret_cast<double2*>(p.S + ((int64_t)u * p.K + k) * kD + lane * 4);
  const bool full = p.pi_old == nullptr;
  double a0 = 0.0, a1 = 0.0, a2 = 0.0, a3 = 0.0;
  long long n = 0;
  if (!full) {
    const double2 x = Sk[0], y = Sk[1];
    a0 = x.x; a1 = x.y; a2 = y.x; a3 = y.y;
    n = p.n[(int64_t)u * p.K + k];
  }
  bool any = false;
  for (int s0 = 0; s0 < p.nseg; s0 += 32) {
    const int sl = s0 + lane;
    const int c = sl < p.nseg ? nc[(int64_t)sl * p.K] : 0;
    int d = sl < p.nseg ? dc[(int64_t)sl * p.K] : 0;
    unsigned m = __ballot_sync(0xffffffffu, c > 0);
    any |= m != 0;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) d += __shfl_xor_sync(0xffffffffu, d, off);
    n += d;
    // segments in ascending order, four loads in flight
    while (m) {
      int idx[4];
      double2 x[4], y[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        idx[q] = m ? __ffs(m) - 1 : -1;
        if (m) m &= m - 1;
        if (idx[q] >= 0) {
          const double2* src = reinterpret_cast<const double2*>(part + (int64_t)(s0 + idx[q]) * seg_stride);
          x[q] = src[0];
          y[q] = src[1];
        }
      }
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        if (idx[q] >= 0) {
          a0 = __dadd_rn(a0, x[q].x); a1 = __dadd_rn(a1, x[q].y);
          a2 = __dadd_rn(a2, y[q].x); a3 = __dadd_rn(a3, y[q].y);
        }
      }
    }
  }
  if (full || any) {
    Sk[0] = make_double2(a0, a1);
    Sk[1] = make_double2(a2, a3);
    if (lane == 0) p.n[(int64_t)u * p.K + k] = n;
  }
  if (n <= 0 || !(full || any)) return;   // empty keeps its centroid; unchanged needs no update
  const double dn = (double)n;
  const double a[4] = {a0, a1, a2, a3};
  double sq = 0.0;
  if (DT == kBF16) {
    uint16_t b[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      b[e] = f64_to_bf16_rne(__ddiv_rn(a[e], dn));
      const double c = (double)bf16_bits_to_f32(b[e]);
      sq = __dadd_rn(sq, __dmul_rn(c, c));
    }
    uint2 w;
    w.x = (uint32_t)b[0] | ((uint32_t)b[1] << 16);
    w.y = (uint32_t)b[2] | ((uint32_t)b[3] << 16);
    *reinterpret_cast<uint2*>(static_cast<char*>(p.C) + (((int64_t)u * p.K + k) * kD + lane * 4) * 2) = w;
  } else {
    float f[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      f[e] = __double2float_rn(__ddiv_rn(a[e], dn));
      sq = __dadd_rn(sq, __dmul_rn((double)f[e], (double)f[e]));
    }
    *reinterpret_cast<float4*>(static_cast<char*>(p.C) + (((int64_t)u * p.K + k) * kD + lane * 4) * 4) =
        make_float4(f[0], f[1], f[2], f[3]);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) sq = __dadd_rn(sq, __shfl_xor_sync(0xffffffffu, sq, off));
  if (lane == 0) p.cn[(int64_t)u * p.K + k] = __double2float_rn(sq);
}

}  // namespace

size_t assign_exact_smem_bytes(int K, int dtype) {
  const int Kp = (K + 31) & ~31;
  const int esz = dtype == kBF16 ? 2 : 4;
  const int Ks = Kp + (esz == 2 ? 2 : 1);
  return (((size_t)kD * Ks * esz + 15) & ~size_t(15)) + kMaxK * sizeof(float) + kAsWarps * kD * sizeof(float);
}

cudaError_t launch_assign_exact(const AssignParams& p, int dtype, cudaStream_t s) {
  const size_t smem = assign_exact_smem_bytes(p.K, dtype);
  const int sms = device_sm_count();
  // Every row (or every listed row) is visited by a grid-stride loop; blocks
  // whose first row is past the (device-side) row count exit before staging
  // the table.  List mode expects few rows: about one block per SM in total.
  // In list mode the listed rows are unevenly spread over the blocks (V
  // blocks with large outliers list more near-ties), so every block gets up
  // to 32 CTAs; CTAs beyond a block's count return at once.
  int64_t bpu = p.list ? 32 : (3 * (int64_t)sms + p.W - 1) / p.W;
  const int64_t max_bpu = (p.N + kAsWarps - 1) / kAsWarps;
  if (bpu > max_bpu) bpu = max_bpu;
  if (bpu < 1) bpu = 1;
  const dim3 grid((unsigned)bpu, (unsigned)p.W);
  cudaError_t e;
  if (dtype == kBF16) {
    e = ensure_dynamic_smem(reinterpret_cast<const void*>(qvg_assign_exact<kBF16>), smem);
    if (e != cudaSuccess) return e;
    qvg_assign_exact<kBF16><<<grid, kAsThreads, smem, s>>>(p);
  } else {
    e = ensure_dynamic_smem(reinterpret_cast<const void*>(qvg_assign_exact<kFP32>), smem);
    if (e != cudaSuccess) return e;
    qvg_assign_exact<kFP32><<<grid, kAsThreads, smem, s>>>(p);
  }
  return cudaGetLastError();
}

cudaError_t launch_assign_candidates(const void* R, const void* C, int K, int64_t N, int W,
                                     const uint2* list, const uint32_t* list_count, uint8_t* pi,
                                     cudaStream_t s) {
  // listed tokens are few and unevenly spread over the blocks: up to 32 CTAs
  // per block, those past a block's count return at once
  const dim3 grid(32u, (unsigned)W);
  qvg_assign_candidates<kBF16><<<grid, kCandWarps * 32, 0, s>>>(R, C, K, N, list, list_count, pi);
  return cudaGetLastError();
}

cudaError_t launch_update_partial(const UpdateParams& p, int dtype, cudaStream_t s) {
  const dim3 g1((unsigned)p.nseg, (unsigned)p.W);
  if (dtype == kBF16) qvg_update_partial<kBF16><<<g1, kUpThreads, 0, s>>>(p);
  else qvg_update_partial<kFP32><<<g1, kUpThreads, 0, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_update_finalize(const UpdateParams& p, int dtype, cudaStream_t s) {
  const dim3 g2((unsigned)((p.K + 7) / 8), (unsigned)p.W);
  if (dtype == kBF16) qvg_update_finalize<kBF16><<<g2, 256, 0, s>>>(p);
  else qvg_update_finalize<kFP32><<<g2, 256, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace qvg
