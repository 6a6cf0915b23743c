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
qvg_assign_exact(const AssignParams p, const int per_block, const float gamma) {
  using ST = typename Store<DT>::T;
  constexpr int ESZ = Store<DT>::bytes;
  extern __shared__ __align__(16) unsigned char smem[];
  const int u = blockIdx.y;
  const int K = p.K;
  const int Kp = (K + 31) & ~31;
  const int NM = Kp / 32;                       // centroid slots per lane (<= 8)
  ST* Ct = reinterpret_cast<ST*>(smem);         // [kD][Kp] transposed table
  float* cn_s = reinterpret_cast<float*>(smem + (size_t)kD * Kp * ESZ);
  float* rbuf = cn_s + kMaxK;                   // [warps][kD]

  const int64_t n_rows = p.list ? (int64_t)p.list_count[u] : p.N;
  const int64_t e0 = (int64_t)blockIdx.x * per_block;
  const int64_t e1 = min(n_rows, e0 + per_block);
  if (e0 >= e1) return;                         // nothing listed for this block
  const ST* Cg = static_cast<const ST*>(p.C) + (int64_t)u * K * kD;
  for (int x = threadIdx.x; x < Kp * kD; x += blockDim.x) {
    const int k = x / kD, jj = x % kD;
    Ct[jj * Kp + k] = k < K ? Cg[(int64_t)k * kD + jj] : Store<DT>::from_f32(0.0f);
  }
  for (int k = threadIdx.x; k < Kp; k += blockDim.x)
    cn_s[k] = k < K ? p.cn[(int64_t)u * K + k] : __int_as_float(0x7f800000);
  __syncthreads();

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float* rw = rbuf + warp * kD;
  const char* Rg = static_cast<const char*>(p.R) + (int64_t)u * p.N * kD * ESZ;

  for (int64_t e = e0 + warp; e < e1; e += kAsWarps) {
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
      const ST* crow = Ct + jj * Kp + lane;
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
    const float thr = screening_threshold(gmin, p.rnorm2[(int64_t)u * p.N + i], gamma);

    double bestD = __longlong_as_double(0x7ff0000000000000ll);
    int bestK = 0x7fffffff;
#pragma unroll
    for (int m = 0; m < 8; ++m) {
      if (m < NM && g[m] <= thr) {
        const int k = lane + 32 * m;
        double D = 0.0;
        for (int jj = 0; jj < kD; ++jj) {
          const double diff = __dsub_rn((double)rw[jj], (double)Store<DT>::ld(Ct + jj * Kp + k));
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

// ---------------------------------------------------------------- update
constexpr int kUpThreads = 1024;
constexpr int kUpWarps = kUpThreads / 32;
constexpr int kTokPerWarp = kSeg / kUpWarps;      // 64
constexpr int kRounds = kTokPerWarp / 32;         // 2

template <int DT>
__global__ void __launch_bounds__(kUpThreads)
qvg_update_partial(const UpdateParams p) {
  constexpr int ESZ = Store<DT>::bytes;
  __shared__ uint16_t hist[kUpWarps][kMaxK];      // per-warp counts, then offsets
  __shared__ int tot[kMaxK];
  __shared__ int start[kMaxK];
  __shared__ uint16_t sorted[kSeg];
  __shared__ int wsum[kMaxK / 32];

  const int u = blockIdx.y, sgi = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t seg0 = (int64_t)sgi * kSeg;
  const int seg_len = (int)min((int64_t)kSeg, p.N - seg0);
  const uint8_t* pi = p.pi + (int64_t)u * p.N + seg0;

  for (int x = threadIdx.x; x < kUpWarps * kMaxK; x += blockDim.x) (&hist[0][0])[x] = 0;
  __syncthreads();

  // Stable per-warp ranks: tokens of warp w are [w*64, w*64+64) of the segment.
  int key[kRounds], rank[kRounds];
#pragma unroll
  for (int r = 0; r < kRounds; ++r) {
    const int tok = warp * kTokPerWarp + r * 32 + lane;
    const bool valid = tok < seg_len;
    key[r] = valid ? (int)pi[tok] : 0x10000 + lane;     // invalid keys never match
    const unsigned mask = __match_any_sync(0xffffffffu, key[r]);
    const int before = __popc(mask & ((1u << lane) - 1u));
    const int base = valid ? hist[warp][key[r]] : 0;
    __syncwarp();
    if (valid && before == 0) hist[warp][key[r]] = (uint16_t)(base + __popc(mask));
    __syncwarp();
    rank[r] = base + before;
  }
  __syncthreads();

  // Exclusive prefix over (k, w): offsets of each warp's run of centroid k.
  if (threadIdx.x < kMaxK) {
    const int k = threadIdx.x;
    int run = 0;
    for (int w = 0; w < kUpWarps; ++w) {
      const int c = hist[w][k];
      hist[w][k] = (uint16_t)run;
      run += c;
    }
    tot[k] = run;
    // block-wide exclusive scan of tot over k (256 threads = 8 warps)
    int v = run;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int o = __shfl_up_sync(0xffffffffu, v, off);
      if (lane >= off) v += o;
    }
    if (lane == 31) wsum[k >> 5] = v;
    start[k] = v - run;            // exclusive within the warp
  }
  __syncthreads();
  if (threadIdx.x < kMaxK) {
    const int k = threadIdx.x;
    int add = 0;
    for (int w = 0; w < (k >> 5); ++w) add += wsum[w];
    start[k] += add;
  }
  __syncthreads();

#pragma unroll
  for (int r = 0; r < kRounds; ++r) {
    const int tok = warp * kTokPerWarp + r * 32 + lane;
    if (tok < seg_len) {
      const int k = key[r];
      sorted[start[k] + hist[warp][k] + rank[r]] = (uint16_t)tok;
    }
  }
  __syncthreads();

  // Per-centroid fp64 sums in ascending token order; lane owns 4 channels.
  const char* R = static_cast<const char*>(p.R) + ((int64_t)u * p.N + seg0) * kD * ESZ;
  double* part = p.partial + ((int64_t)u * p.nseg + sgi) * p.K * kD;
  int* cnt = p.counts + ((int64_t)u * p.nseg + sgi) * p.K;
  for (int k = warp; k < p.K; k += kUpWarps) {
    const int n = tot[k];
    if (lane == 0) cnt[k] = n;
    if (n == 0) continue;
    const int s0 = start[k];
    double a0 = 0.0, a1 = 0.0, a2 = 0.0, a3 = 0.0;
    for (int b = 0; b < n; b += 8) {
      float v[8][4];
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const int tok = sorted[s0 + min(b + q, n - 1)];
        const char* row = R + (int64_t)tok * kD * ESZ;
        if (DT == kBF16) {
          const uint2 w = *reinterpret_cast<const uint2*>(row + lane * 8);
          v[q][0] = __uint_as_float(w.x << 16);
          v[q][1] = __uint_as_float(w.x & 0xFFFF0000u);
          v[q][2] = __uint_as_float(w.y << 16);
          v[q][3] = __uint_as_float(w.y & 0xFFFF0000u);
        } else {
          const float4 w = *reinterpret_cast<const float4*>(row + lane * 16);
          v[q][0] = w.x; v[q][1] = w.y; v[q][2] = w.z; v[q][3] = w.w;
        }
      }
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        if (b + q < n) {
          a0 = __dadd_rn(a0, (double)v[q][0]);
          a1 = __dadd_rn(a1, (double)v[q][1]);
          a2 = __dadd_rn(a2, (double)v[q][2]);
          a3 = __dadd_rn(a3, (double)v[q][3]);
        }
      }
    }
    double2* dst = reinterpret_cast<double2*>(part + (int64_t)k * kD + lane * 4);
    dst[0] = make_double2(a0, a1);
    dst[1] = make_double2(a2, a3);
  }
}

template <int DT>
__global__ void __launch_bounds__(256)
qvg_update_finalize(const UpdateParams p) {
  const int u = blockIdx.y;
  const int k = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (k >= p.K) return;
  int64_t n = 0;
  for (int s = 0; s < p.nseg; ++s) n += p.counts[((int64_t)u * p.nseg + s) * p.K + k];
  if (n == 0) return;                           // empty: keep the previous centroid
  double a[4] = {0.0, 0.0, 0.0, 0.0};
  for (int s = 0; s < p.nseg; ++s) {
    if (p.counts[((int64_t)u * p.nseg + s) * p.K + k] == 0) continue;
    const double2* src = reinterpret_cast<const double2*>(
        p.partial + (((int64_t)u * p.nseg + s) * p.K + k) * kD + lane * 4);
    const double2 x = src[0], y = src[1];
    a[0] = __dadd_rn(a[0], x.x); a[1] = __dadd_rn(a[1], x.y);
    a[2] = __dadd_rn(a[2], y.x); a[3] = __dadd_rn(a[3], y.y);
  }
  const double dn = (double)n;
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

cudaError_t launch_assign_exact(const AssignParams& p, int dtype, cudaStream_t s) {
  const int Kp = (p.K + 31) & ~31;
  const int esz = dtype == kBF16 ? 2 : 4;
  const size_t smem = (size_t)kD * Kp * esz + kMaxK * sizeof(float) + kAsWarps * kD * sizeof(float);
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // rows per block: enough blocks to fill the GPU, at least 64 rows each
  int64_t blocks_per_unit = (4 * (int64_t)sms + p.W - 1) / p.W;
  const int64_t max_rows = p.N;
  if (blocks_per_unit * 64 > max_rows) blocks_per_unit = (max_rows + 63) / 64;
  if (blocks_per_unit < 1) blocks_per_unit = 1;
  const int per = (int)((max_rows + blocks_per_unit - 1) / blocks_per_unit);
  const dim3 grid((unsigned)blocks_per_unit, (unsigned)p.W);
  const float gamma = 1.52587890625e-05f;   // 2^-16
  cudaError_t e;
  if (dtype == kBF16) {
    e = cudaFuncSetAttribute(qvg_assign_exact<kBF16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    qvg_assign_exact<kBF16><<<grid, kAsThreads, smem, s>>>(p, per, gamma);
  } else {
    e = cudaFuncSetAttribute(qvg_assign_exact<kFP32>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    qvg_assign_exact<kFP32><<<grid, kAsThreads, smem, s>>>(p, per, gamma);
  }
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
