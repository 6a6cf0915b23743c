// kernels_kmeans.cu -- k-means steps of semantic-aware smoothing (m.163.com
// article on Quant VideoGen, section 三: tokens grouped by k-means, the group
// mean is the centroid) on sm_100a CUDA cores:
//   * qvg_assign_exact: the assignment of a token (or of a list of flagged
//     tokens) decided exactly.  fp32 screening distances g_k = |c_k|^2 - 2 r.c_k
//     for all centroids, then the exact fp64 squared distance (channels in
//     ascending order, separate subtract / multiply / add) for every centroid
//     whose screening value lies within the rounding-error bound of the
//     minimum; ties go to the lowest index.
//   * qvg_kmeans_update: exact centroid sums in 64-bit fixed point (so the
//     order of the adds cannot change them), the mean (one fp64 divide) and
//     one rounding to the storage dtype; an empty centroid keeps its value.
//     After the first iteration only the tokens whose assignment changed are
//     read.
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
      rw[4 * lane + 0] = (double)__uint_as_float(w.x << 16);
      rw[4 * lane + 1] = (double)__uint_as_float(w.x & 0xFFFF0000u);
      rw[4 * lane + 2] = (double)__uint_as_float(w.y << 16);
      rw[4 * lane + 3] = (double)__uint_as_float(w.y & 0xFFFF0000u);
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
// multiply and add per channel), token row as fp64 in shared memory, centroid
// row read from global memory.
template <int DT>
__device__ __forceinline__ double exact_dist(const double* rw, const char* crow) {
  double D = 0.0;
#pragma unroll 2
  for (int j0 = 0; j0 < kD; j0 += 8) {
    double c[8];
    if (DT == kBF16) {
      const uint4 w = *reinterpret_cast<const uint4*>(crow + j0 * 2);
      const uint32_t x[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        c[2 * e] = (double)__uint_as_float(x[e] << 16);
        c[2 * e + 1] = (double)__uint_as_float(x[e] & 0xFFFF0000u);
      }
    } else {
      const float4 a = *reinterpret_cast<const float4*>(crow + j0 * 4);
      const float4 b = *reinterpret_cast<const float4*>(crow + j0 * 4 + 16);
      c[0] = a.x; c[1] = a.y; c[2] = a.z; c[3] = a.w; c[4] = b.x; c[5] = b.y; c[6] = b.z; c[7] = b.w;
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const double diff = __dsub_rn(rw[j0 + e], c[e]);
      D = __dadd_rn(D, __dmul_rn(diff, diff));
    }
  }
  return D;
}

// Every listed token of the wave is dealt out over all warps of the grid
// (one resident wave of CTAs): the listed tokens are unevenly spread over the
// blocks, so a split per block would leave most warps idle while a few walk a
// long list.  Each CTA forms the prefix of the blocks' list counts, and a warp
// finds the block of its entry by binary search.
constexpr int kCandMaxWave = 1024;

template <int DT>
__global__ void __launch_bounds__(kCandWarps * 32)
qvg_assign_candidates(const void* R, const void* C, const int K, const int64_t N, const int W, const uint2* list,
                      const uint32_t* list_count, uint8_t* pi) {
  constexpr int ESZ = Store<DT>::bytes;
  __shared__ double rbuf[kCandWarps][kD];
  __shared__ int64_t s_pre[kCandMaxWave + 1];    // s_pre[u] = listed entries of blocks 0 .. u-1
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp == 0) {
    const int per = (W + 31) / 32;
    const int b0 = min(W, lane * per), b1 = min(W, b0 + per);
    int64_t sum = 0;
    for (int u = b0; u < b1; ++u) sum += min((int64_t)list_count[u], N);
    int64_t incl = sum;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int64_t o = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += o;
    }
    int64_t run = incl - sum;
    for (int u = b0; u < b1; ++u) {
      s_pre[u] = run;
      run += min((int64_t)list_count[u], N);
    }
    if (lane == 31) s_pre[W] = incl;
  }
  __syncthreads();
  const int64_t total = s_pre[W];
  const int64_t stride = (int64_t)gridDim.x * kCandWarps;
  double* rw = rbuf[warp];
  const uint32_t all = (K + 7) / 8 >= 32 ? 0xFFFFFFFFu : ((1u << ((K + 7) / 8)) - 1u);
  for (int64_t g = (int64_t)blockIdx.x * kCandWarps + warp; g < total; g += stride) {
    int lo = 0, hi = W - 1;                      // the last block u with s_pre[u] <= g
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s_pre[mid] <= g) lo = mid; else hi = mid - 1;
    }
    const int u = lo;
    const int64_t e = g - s_pre[u];
    const char* Ru = static_cast<const char*>(R) + (int64_t)u * N * kD * ESZ;
    const char* Cu = static_cast<const char*>(C) + (int64_t)u * K * kD * ESZ;
    const uint2 ent = list[(int64_t)u * N + e];
    const int64_t tok = ent.x;
    if (tok >= N) continue;                    // warp-uniform; never true for listed tokens
    uint32_t groups = ent.y & all;
    if (groups == 0) groups = all;
    const char* rrow = Ru + tok * kD * ESZ;
    if (DT == kBF16) {
      const uint2 w = *reinterpret_cast<const uint2*>(rrow + lane * 8);
      rw[4 * lane + 0] = (double)__uint_as_float(w.x << 16);
      rw[4 * lane + 1] = (double)__uint_as_float(w.x & 0xFFFF0000u);
      rw[4 * lane + 2] = (double)__uint_as_float(w.y << 16);
      rw[4 * lane + 3] = (double)__uint_as_float(w.y & 0xFFFF0000u);
    } else {
      const float4 w = *reinterpret_cast<const float4*>(rrow + lane * 16);
      rw[4 * lane + 0] = w.x; rw[4 * lane + 1] = w.y; rw[4 * lane + 2] = w.z; rw[4 * lane + 3] = w.w;
    }
    __syncwarp();
    double bestD = __longlong_as_double(0x7ff0000000000000ll);
    int bestK = 0x7fffffff;
    // groups in ascending order, four per round: lane l takes centroid
    // 8*g + (l % 8) of the (l / 8)-th group of the round, so each lane meets
    // its centroids in ascending order
    while (groups) {
      int gsel = -1;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int g8 = groups ? __ffs(groups) - 1 : -1;
        if (groups) groups &= groups - 1;
        if (q == (lane >> 3)) gsel = g8;
      }
      const int k = gsel * 8 + (lane & 7);
      if (gsel >= 0 && k < K) {
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
// Centroid sums in 64-bit fixed point.  For channel c of the stage input let
// m_c be its largest magnitude over the block, e_c = floor(log2 m_c), and
// L_c = e_c + k - 62 with 2^k > N.  A value is converted to the integer
// v / 2^L_c, which is exact for every value that is a multiple of 2^L_c:
// all bf16 values within 39 binades of m_c when N < 2^16 (fp32: 23 binades).
// No sum of the block's integers can leave the int64 range, integer addition
// is associative, so the sums are exact and do not depend on the order in
// which tokens are added -- the update may use atomics and still be
// deterministic -- and S * 2^L_c equals the fp64 sum taken in any order
// whenever that sum is itself exact.  (A channel with a value below the
// window takes an exact 320-bit sum in the centroid kernel instead; see
// exact_member_sum.)  The mean is one fp64 divide of the sum
// (converted exactly, or rounded once if it needs more than 53 bits) by the
// member count, rounded once to the storage dtype.
//
// Three launches per iteration:
//   bucket    (one CTA per block): the block's entries -- every token on the
//             first iteration; later, every token whose assignment changed,
//             once for the centroid it joined (+) and once for the one it left
//             (-) -- are counted per centroid and written to a list bucketed by
//             centroid; per-centroid offsets and member-count changes go to
//             global memory (on the first iteration the running sums are
//             cleared here).
//   sum       (several CTAs per block): each warp walks a contiguous piece of
//             the list, gathers rows two batches ahead, converts them to fixed
//             point and accumulates them in registers while the centroid stays
//             the same; each run is added to the running sums with 64-bit
//             integer atomics (exact, so the order does not matter).
//   centroids (a warp per centroid): every centroid with entries gets its new
//             count and, if non-empty, its mean and squared norm.
constexpr int kBucketThreads = 1024;
constexpr size_t kBucketStageBytes = 192 * 1024;   // largest staged pair of assignment arrays
constexpr int kScan = 8;              // assignments per thread per scan step (loads in flight)
constexpr int kSumThreads = 256;
constexpr int kSumWarps = kSumThreads / 32;
constexpr int kSumSlices = 8;         // sum CTAs per block

// List entry: token (bits 0-22), centroid (23-30), subtract flag (31).
constexpr uint32_t kEntTok = 0x7FFFFFu;
constexpr int kEntKShift = 23;
constexpr uint32_t kEntSub = 1u << 31;
constexpr uint32_t kEntNone = 0xFFFFFFFFu;   // never a real entry (token 2^23-1 is out of range)

// L_c of a channel from the bits of its largest magnitude (0 for an all-zero
// channel), clamped so that 2^-L_c is a normal float.
__device__ __forceinline__ int fix_exponent(uint32_t maxbits, int log2n) {
  const int e = maxbits == 0u ? 0 : (int)((maxbits >> 23) & 0xFFu) - 127;
  const int L = e + log2n - 62;
  return L < -126 ? -126 : L;
}

// Assignments of tokens c + j*blockDim.x + threadIdx.x, j < kScan: new (kn)
// and previous (ko; -1 on a full pass).  Past the end both read -1, so
// kn == ko marks "nothing to do" for unchanged and missing tokens alike.
// Indices are clamped to K - 1: every stored assignment is below K, but after
// a device-side timeout the assignments of the abandoned tiles were never
// written, and the clamp keeps every later access of this call in bounds.
__device__ __forceinline__ void load_assignments(const uint8_t* piu, const uint8_t* pio, int64_t N, int64_t c,
                                                 int K, int (&kn)[kScan], int (&ko)[kScan]) {
#pragma unroll
  for (int j = 0; j < kScan; ++j) {
    const int64_t t = c + (int64_t)j * blockDim.x + threadIdx.x;
    kn[j] = t < N ? min((int)piu[t], K - 1) : -1;
    ko[j] = (t < N && pio != nullptr) ? min((int)pio[t], K - 1) : -1;
  }
}

// Copy the N assignment bytes at g into shared memory at s + (g mod 16), so
// that token t sits at s[(g mod 16) + t]: 16-byte loads over the aligned
// middle, single bytes for the ragged ends (nothing outside [g, g + N) is
// read).  The caller synchronises.
__device__ __forceinline__ void stage_assignments(const uint8_t* g, int64_t N, uint8_t* s) {
  const int off = (int)(reinterpret_cast<uintptr_t>(g) & 15u);
  const int64_t b0 = (int64_t)((16 - off) & 15) < N ? (int64_t)((16 - off) & 15) : N;   // first aligned token
  const int64_t n16 = (N - b0) / 16;
  const int64_t b1 = b0 + 16 * n16;                             // first token of the tail
  const uint4* src = reinterpret_cast<const uint4*>(g + b0);
  uint4* dst = reinterpret_cast<uint4*>(s + off + b0);
  for (int64_t x = threadIdx.x; x < n16; x += blockDim.x) dst[x] = src[x];
  if (threadIdx.x < b0) s[off + threadIdx.x] = g[threadIdx.x];
  if (threadIdx.x < N - b1) s[off + b1 + threadIdx.x] = g[b1 + threadIdx.x];
  // the bytes before the first token and up to the next 4-byte boundary
  // after the last are zero, so that whole words can be compared
  if (threadIdx.x < off) s[threadIdx.x] = 0;
  const int64_t end = off + N, end4 = (end + 3) & ~int64_t(3);
  if (threadIdx.x < end4 - end) s[end + threadIdx.x] = 0;
}

// Warp-aggregated shared-memory add of `v` to counter[key] (lanes with the
// same key are combined; `key` < 0 takes part in no add).  Returns, for
// returning adds, the slot of this lane: old value + rank among its peers.
__device__ __forceinline__ int warp_add(int* counter, int key, int v, bool want_slot) {
  const unsigned peers = __match_any_sync(0xffffffffu, key);
  const int lane = threadIdx.x & 31;
  const int leader = __ffs(peers) - 1;
  const int rank = __popc(peers & ((1u << lane) - 1u));
  int base = 0;
  if (key >= 0 && lane == leader) base = atomicAdd(counter + key, v * __popc(peers));
  if (want_slot) base = __shfl_sync(0xffffffffu, base, leader);
  return base + rank;
}

template <int DT>
__global__ void __launch_bounds__(kBucketThreads, 1)
qvg_update_bucket(const UpdateParams p) {
  __shared__ int hist[kMaxK];
  __shared__ int dcnt[kMaxK];
  __shared__ int cursor[kMaxK];      // next slot for an added row (from the bucket's start, upward)
  __shared__ int cursor_sub[kMaxK];  // next slot for a removed row (from the bucket's end, downward)
  const int u = blockIdx.x;
  const int K = p.K;
  const int64_t N = p.N;
  const bool full = p.pi_old == nullptr;
  for (int x = threadIdx.x; x < kMaxK; x += blockDim.x) { hist[x] = 0; dcnt[x] = 0; }
  if (full) {                                  // the running sums restart from zero
    longlong2* S = reinterpret_cast<longlong2*>(p.S + (int64_t)u * K * kD);
    for (int x = threadIdx.x; x < K * kD / 2; x += blockDim.x) S[x] = make_longlong2(0, 0);
  }
  __syncthreads();
  const uint8_t* piu = p.pi + (int64_t)u * N;
  const uint8_t* pio = full ? nullptr : p.pi_old + (int64_t)u * N;
  // When the block's assignments fit in shared memory they are staged there
  // once (a few wide loads per thread instead of a round trip per scan step
  // and pass), and both passes read them from there.
  extern __shared__ __align__(16) uint8_t s_pi[];
  const int64_t pad = (N + 31) & ~int64_t(15);
  const int a_off = (int)(reinterpret_cast<uintptr_t>(piu) & 15u);
  // Incremental passes over staged arrays whose tokens sit at the same byte
  // offset compare four tokens per 32-bit word, so that the (many) unchanged
  // tokens cost one compare per four.
  const bool words = p.stage_pi && !full && a_off == (int)(reinterpret_cast<uintptr_t>(pio) & 15u);
  if (p.stage_pi) {
    stage_assignments(piu, N, s_pi);
    if (!full) stage_assignments(pio, N, s_pi + pad);
    piu = s_pi + a_off;
    if (!full) pio = s_pi + pad + (reinterpret_cast<uintptr_t>(pio) & 15u);
  }
  __syncthreads();
  const uint32_t* wn = reinterpret_cast<const uint32_t*>(s_pi);
  const uint32_t* wo = reinterpret_cast<const uint32_t*>(s_pi + pad);
  const int64_t n_words = (a_off + N + 3) / 4;
  // changed tokens of word g: calls f(token, new centroid, old centroid)
  auto word_changes = [&](int64_t g, auto&& f) {
    const uint32_t xn = wn[g], xo = wo[g];
    if (xn == xo) return;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int bn = (int)((xn >> (8 * j)) & 0xFFu), bo = (int)((xo >> (8 * j)) & 0xFFu);
      const int64_t t = 4 * g + j - a_off;
      if (bn != bo && t >= 0 && t < N) f((uint32_t)t, min(bn, K - 1), min(bo, K - 1));
    }
  };
  const int64_t step = (int64_t)kScan * blockDim.x;
  if (words) {
    for (int64_t g = threadIdx.x; g < n_words; g += blockDim.x)
      word_changes(g, [&](uint32_t, int kn, int ko) {
        if (kn == ko) return;
        atomicAdd(hist + kn, 1);
        atomicAdd(hist + ko, 1);
        atomicAdd(dcnt + kn, 1);
        atomicAdd(dcnt + ko, -1);
      });
  }
  for (int64_t c = 0; c < N && !words; c += step) {
    int kn[kScan], ko[kScan];
    load_assignments(piu, pio, N, c, K, kn, ko);
#pragma unroll
    for (int j = 0; j < kScan; ++j) {
      const bool ch = kn[j] != ko[j];
      if (full) {
        // every token has an entry; neighbours often share a centroid, so
        // lanes with the same key are combined into one add
        warp_add(hist, ch ? kn[j] : -1, 1, false);
      } else if (ch) {
        // few tokens change: plain adds by the lanes that did
        atomicAdd(hist + kn[j], 1);
        atomicAdd(hist + ko[j], 1);
        atomicAdd(dcnt + kn[j], 1);
        atomicAdd(dcnt + ko[j], -1);
      }
    }
  }
  __syncthreads();
  // exclusive prefix over the counts (warp 0; 8 per lane)
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    int v[8], sum = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) { v[i] = lane * 8 + i < K ? hist[lane * 8 + i] : 0; sum += v[i]; }
    int incl = sum;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int o = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += o;
    }
    int run = incl - sum;
    int* off_u = p.off + (int64_t)u * (K + 1);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int k = lane * 8 + i;
      if (k < K) { cursor[k] = run; cursor_sub[k] = -(run + v[i]); off_u[k] = run; }
      run += v[i];
    }
    if (lane == 31) off_u[K] = run;
  }
  for (int k = threadIdx.x; k < K; k += blockDim.x)
    p.cnt[(int64_t)u * K + k] = full ? hist[k] : dcnt[k];
  __syncthreads();
  uint32_t* list = p.list + (int64_t)u * 2 * N;    // capacity 2N entries per block
  if (words) {
    for (int64_t g = threadIdx.x; g < n_words; g += blockDim.x)
      word_changes(g, [&](uint32_t t, int kn, int ko) {
        if (kn == ko) return;
        list[atomicAdd(cursor + kn, 1)] = t | ((uint32_t)kn << kEntKShift);
        list[-atomicAdd(cursor_sub + ko, 1) - 1] = t | ((uint32_t)ko << kEntKShift) | kEntSub;
      });
  }
  for (int64_t c = 0; c < N && !words; c += step) {
    int kn[kScan], ko[kScan];
    load_assignments(piu, pio, N, c, K, kn, ko);
#pragma unroll
    for (int j = 0; j < kScan; ++j) {
      const bool ch = kn[j] != ko[j];
      const uint32_t t = (uint32_t)(c + (int64_t)j * blockDim.x + threadIdx.x);
      if (full) {
        const int sa = warp_add(cursor, ch ? kn[j] : -1, 1, true);
        if (ch) list[sa] = t | ((uint32_t)kn[j] << kEntKShift);
      } else if (ch) {
        list[atomicAdd(cursor + kn[j], 1)] = t | ((uint32_t)kn[j] << kEntKShift);
        // cursor_sub holds minus the end of the free region: slot = end - 1 - (count so far)
        list[-atomicAdd(cursor_sub + ko[j], 1) - 1] = t | ((uint32_t)ko[j] << kEntKShift) | kEntSub;
      }
    }
  }
}

__device__ __forceinline__ void cp_async_row(void* smem_dst, const void* gsrc, int bytes) {
  const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst));
  if (bytes == 16)
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(gsrc) : "memory");
  else
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(d), "l"(gsrc) : "memory");
}
__device__ __forceinline__ void cp_async_commit_group() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait_groups() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// Each warp walks its piece of the list two rows at a time, one per
// half-warp (16 lanes x 8 channels), with a ring of kSumRing row pairs in
// shared memory filled by cp.async (every lane copies, and later reads back,
// its own 8 channels of a row), so that many rows are in flight without
// holding registers.  Within a bucket the added rows come first and the
// removed rows last, so a run (one centroid, its added rows then its removed
// rows, with their signs) is summed in registers and applied when it ends;
// each half-warp keeps its own run.
constexpr int kSumRing = 16;

template <int DT>
__global__ void __launch_bounds__(kSumThreads, 3)
qvg_update_sum(const UpdateParams p) {
  constexpr int ESZ = Store<DT>::bytes;
  constexpr int LANE_BYTES = 8 * ESZ;            // a lane's 8 channels
  constexpr int ROW = kD * ESZ;
  extern __shared__ __align__(16) unsigned char smem[];
  const int u = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int half = lane >> 4, hl = lane & 15;    // row of the pair, lane within the half
  const int64_t N = p.N;
  const int E = p.off[(int64_t)u * (p.K + 1) + p.K];
  // this warp's piece of the block's list
  const int64_t part = (int64_t)blockIdx.x * kSumWarps + warp, parts = (int64_t)gridDim.x * kSumWarps;
  const int e0 = (int)(E * part / parts), e1 = (int)(E * (part + 1) / parts);
  const int n = e1 - e0;
  if (n <= 0) return;
  const int npairs = (n + 1) >> 1;
  float to_fix[8];
  // For bf16 rows the scaling by 2^-L is also an integer add of -L to the
  // exponent field of each half of a pair word, valid when L <= 0 for every
  // channel of the lane: a normal value is scaled exactly, a zero becomes at
  // most 2^-1 and rounds to 0, and a bf16 subnormal can only occur in a
  // channel that the centroid kernel sums exactly instead.  The warp takes
  // that path when all its lanes qualify (the sums are the same either way).
  uint32_t shiftw[4];
  bool lane_fast = true;
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const int L = fix_exponent(p.chmax[(int64_t)u * kD + 8 * hl + e], p.log2n);
    to_fix[e] = __int_as_float((127 - L) << 23);
    lane_fast &= L <= 0;
    const uint32_t part = (uint32_t)(L <= 0 ? -L : 0) << ((e & 1) ? 23 : 7);
    if ((e & 1) == 0) shiftw[e >> 1] = part; else shiftw[e >> 1] |= part;
  }
  const bool fast = DT == kBF16 && __all_sync(0xffffffffu, lane_fast);
  const uint32_t* list = p.list + (int64_t)u * 2 * N + e0;
  const char* Ru = static_cast<const char*>(p.R) + (int64_t)u * N * ROW + hl * LANE_BYTES;
  unsigned char* ring = smem + (size_t)warp * kSumRing * 2 * ROW + half * ROW + hl * LANE_BYTES;
  // S keeps channel c at (c % 8) * 16 + c / 8, so that the adds of a
  // half-warp (lane hl owns channels 8*hl ... 8*hl + 7) to one channel slot e
  // land on 128 contiguous bytes
  long long* Su = p.S + (int64_t)u * p.K * kD + hl;

  // entries in groups of 32 (16 pairs), one per lane; two groups held, the
  // next loaded one group ahead of the issue pointer
  uint32_t ge0 = lane < n ? list[lane] : kEntNone;
  uint32_t ge1 = 32 + lane < n ? list[32 + lane] : kEntNone;
  auto issue = [&](int jp, int slot) {           // rows 2jp and 2jp+1 into ring slot
    const int r = 2 * jp + half;                  // this half's row (entry index)
    const uint32_t ent = __shfl_sync(0xffffffffu, (r >> 5) & 1 ? ge1 : ge0, r & 31);
    if (r < n) {
      const char* src = Ru + (int64_t)(ent & kEntTok) * ROW;
      unsigned char* dst = ring + slot * 2 * ROW;
      if (DT == kBF16) {
        cp_async_row(dst, src, 16);
      } else {
        cp_async_row(dst, src, 16);
        cp_async_row(dst + 16, src + 16, 16);
      }
    }
  };
#pragma unroll
  for (int r = 0; r < kSumRing; ++r) {
    if (r < npairs) issue(r, r);
    cp_async_commit_group();
  }
  long long run[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) run[e] = 0;
  uint32_t run_key = 0xFFFFFFFFu;                 // centroid of this half's open run
  auto flush = [&]() {
    if (run_key != 0xFFFFFFFFu) {
      long long* a = Su + (int64_t)run_key * kD;
#pragma unroll
      for (int e = 0; e < 8; ++e) atomicAdd(reinterpret_cast<unsigned long long*>(a + 16 * e), (unsigned long long)run[e]);
    }
  };
  for (int jp = 0; jp < npairs; ++jp) {
    cp_async_wait_groups<kSumRing - 1>();
    if ((jp & 15) == 0 && jp >= 16) {              // entering group g = jp/16: fetch group g+1
      const int nxt = 2 * jp + 32 + lane;
      const uint32_t x = nxt < n ? list[nxt] : kEntNone;
      if (((jp >> 4) + 1) & 1) ge1 = x; else ge0 = x;
    }
    const int r = 2 * jp + half;
    const uint32_t ent = __shfl_sync(0xffffffffu, (r >> 5) & 1 ? ge1 : ge0, r & 31);
    const int slot = jp % kSumRing;
    if (r < n && fast) {
      // bf16 rows, exponent-add scaling: the sign of a subtracted row is one
      // xor per pair word, the scaling one integer add per pair word
      const uint4 w = *reinterpret_cast<const uint4*>(ring + slot * 2 * ROW);
      const uint32_t key = (ent >> kEntKShift) & 0xFFu;
      const uint32_t sgn = (ent & kEntSub) ? 0x80008000u : 0u;
      if (key != run_key) {
        flush();
        run_key = key;
#pragma unroll
        for (int e = 0; e < 8; ++e) run[e] = 0;
      }
      const uint32_t x[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint32_t xs = (x[e] ^ sgn) + shiftw[e];
        run[2 * e] += __float2ll_rn(__uint_as_float(xs << 16));
        run[2 * e + 1] += __float2ll_rn(__uint_as_float(xs & 0xFFFF0000u));
      }
    } else if (r < n) {
      float v[8];
      const unsigned char* src = ring + slot * 2 * ROW;
      if (DT == kBF16) {
        const uint4 w = *reinterpret_cast<const uint4*>(src);
        const uint32_t x[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          v[2 * e] = __uint_as_float(x[e] << 16);
          v[2 * e + 1] = __uint_as_float(x[e] & 0xFFFF0000u);
        }
      } else {
        const float4 a = reinterpret_cast<const float4*>(src)[0];
        const float4 b = reinterpret_cast<const float4*>(src)[1];
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
      }
      // A run is one centroid: its added rows, then its removed rows (the
      // bucket order), summed with their signs and applied once.
      const uint32_t key = (ent >> kEntKShift) & 0xFFu;
      const float sg = (ent & kEntSub) ? -1.0f : 1.0f;
      if (key != run_key) {
        flush();
        run_key = key;
#pragma unroll
        for (int e = 0; e < 8; ++e) run[e] = 0;
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) run[e] += __float2ll_rn(__fmul_rn(__fmul_rn(v[e], sg), to_fix[e]));
    }
    // refill the slot just read with the pair kSumRing ahead
    if (jp + kSumRing < npairs) issue(jp + kSumRing, slot);
    cp_async_commit_group();
  }
  flush();
  cp_async_wait_groups<0>();
}

// ---------------------------------------------------------------- sums beyond the fixed-point window
// A channel whose smallest nonzero |value| in the block has a quantum below
// 2^L_c (more than about 39 binades under the channel's largest magnitude for
// bf16) does not fit the 64-bit fixed point.  For such a channel the centroid
// kernel forms each member sum exactly from scratch, in a 320-bit
// two's-complement integer (ten 32-bit limbs, least significant first) that
// counts units of 2^-149: every fp32 or bf16 value is a whole number of units
// below 2^277, and fewer than 2^23 of them sum to less than 2^300.
constexpr int kWideLimbs = 10;
struct Wide320 {
  uint32_t w[kWideLimbs];
};

__device__ __forceinline__ void wide_clear(Wide320& a) {
#pragma unroll
  for (int j = 0; j < kWideLimbs; ++j) a.w[j] = 0u;
}

// a += b, or a -= b when `sub`, limb by limb with the carry (borrow) in 64 bits.
__device__ __forceinline__ void wide_accumulate(Wide320& a, const Wide320& b, bool sub) {
  uint64_t c = 0;
#pragma unroll
  for (int j = 0; j < kWideLimbs; ++j) {
    if (!sub) {
      const uint64_t t = (uint64_t)a.w[j] + b.w[j] + c;
      a.w[j] = (uint32_t)t;
      c = t >> 32;
    } else {
      const uint64_t t = (uint64_t)a.w[j] - b.w[j] - c;
      a.w[j] = (uint32_t)t;
      c = (t >> 63) & 1u;
    }
  }
}

// a += v for an fp32 value v (bf16 values are widened exactly): |v| is
// M * 2^(P - 149) with M the significand (implicit bit included) and P the
// biased exponent minus one (zero for subnormals), so M lands at bit P.
__device__ __forceinline__ void wide_add_value(Wide320& a, float v) {
  const uint32_t bits = __float_as_uint(v);
  const uint32_t E = (bits >> 23) & 0xFFu;
  const uint32_t M = E ? ((bits & 0x7FFFFFu) | 0x800000u) : (bits & 0x7FFFFFu);
  if (M == 0u) return;
  const int P = E ? (int)E - 1 : 0;
  const int L0 = P >> 5, sh = P & 31;
  Wide320 b;
#pragma unroll
  for (int j = 0; j < kWideLimbs; ++j)
    b.w[j] = j == L0 ? (M << sh) : (j == L0 + 1 && sh ? (M >> (32 - sh)) : 0u);
  wide_accumulate(a, b, (bits >> 31) != 0u);
}

// The integer's value (units of 2^-149) rounded once to the nearest double,
// ties to even.
__device__ __forceinline__ double wide_to_double(Wide320 a) {
  const bool neg = (a.w[kWideLimbs - 1] >> 31) != 0u;
  if (neg) {                                   // magnitude: ~a + 1
    uint64_t c = 1;
#pragma unroll
    for (int j = 0; j < kWideLimbs; ++j) {
      const uint64_t t = (uint64_t)(~a.w[j]) + c;
      a.w[j] = (uint32_t)t;
      c = t >> 32;
    }
  }
  int top = -1;                                // highest set bit
#pragma unroll
  for (int j = kWideLimbs - 1; j >= 0; --j)
    if (top < 0 && a.w[j] != 0u) top = 32 * j + 31 - __clz(a.w[j]);
  if (top < 0) return 0.0;
  // the 64 bits [start, start + 64) of the magnitude (bits below 0 read as 0)
  auto window = [&](int start) {
    uint64_t r = 0;
#pragma unroll
    for (int j = 0; j < kWideLimbs; ++j) {
      const int pos = 32 * j - start;          // where limb j's bit 0 lands
      if (pos > -32 && pos < 64) r |= pos >= 0 ? ((uint64_t)a.w[j] << pos) : ((uint64_t)a.w[j] >> (-pos));
    }
    return r;
  };
  double mag;
  if (top <= 52) {                             // fewer than 54 bits: exact
    mag = __dmul_rn((double)window(0), 0x1p-149);
  } else {
    const int start = top - 63;                // bit 63 of the window is the top bit
    const uint64_t w = window(start);
    bool sticky = false;                       // any set bit below `start`
#pragma unroll
    for (int j = 0; j < kWideLimbs; ++j) {
      const int lo = 32 * j;
      if (lo + 32 <= start) sticky |= a.w[j] != 0u;
      else if (lo < start) sticky |= (a.w[j] & ((1u << (start - lo)) - 1u)) != 0u;
    }
    uint64_t mant = w >> 11;                   // 53 bits
    const uint64_t rest = w & 0x7FFull;
    int e2 = start + 11 - 149;                 // the value is mant * 2^e2
    if (rest > 0x400ull || (rest == 0x400ull && (sticky || (mant & 1ull)))) ++mant;
    if (mant == (1ull << 53)) { mant >>= 1; ++e2; }
    mag = __dmul_rn((double)mant, __longlong_as_double((long long)(1023 + e2) << 52));
  }
  return neg ? -mag : mag;
}

// The exact sum of channel c over the tokens of block u assigned to
// centroid k, rounded once to fp64 (the whole warp scans the assignments).
template <int DT>
__device__ double exact_member_sum(const UpdateParams& p, int u, int k, int c) {
  constexpr int ESZ = Store<DT>::bytes;
  const int lane = threadIdx.x & 31;
  const uint8_t* piu = p.pi + (int64_t)u * p.N;
  const char* Ru = static_cast<const char*>(p.R) + (int64_t)u * p.N * kD * ESZ;
  Wide320 acc;
  wide_clear(acc);
  for (int64_t i = lane; i < p.N; i += 32) {
    if ((int)piu[i] != k) continue;
    const float v = DT == kBF16 ? bf16_bits_to_f32(reinterpret_cast<const uint16_t*>(Ru)[i * kD + c])
                                : reinterpret_cast<const float*>(Ru)[i * kD + c];
    wide_add_value(acc, v);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    Wide320 o;
#pragma unroll
    for (int j = 0; j < kWideLimbs; ++j) o.w[j] = __shfl_xor_sync(0xffffffffu, acc.w[j], off);
    wide_accumulate(acc, o, false);
  }
  return wide_to_double(acc);
}

// A warp per centroid: new count; for a non-empty centroid the mean of the
// exact sum, rounded once to the storage dtype, and its squared norm.
template <int DT>
__global__ void __launch_bounds__(256)
qvg_update_centroids(const UpdateParams p) {
  const int u = blockIdx.y;
  const int k = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (k >= p.K) return;
  const bool full = p.pi_old == nullptr;
  const int* off_u = p.off + (int64_t)u * (p.K + 1);
  // every load of the warp is issued before any of them is used: the bucket
  // bounds, the count (change), the 128 sums and the channel ranges
  const int o0 = off_u[k], o1 = off_u[k + 1];
  const int cnt = p.cnt[(int64_t)u * p.K + k];
  const int n_old = full ? 0 : p.n[(int64_t)u * p.K + k];
  // channel c = 4 * lane + e sits at (c % 8) * 16 + c / 8 of the centroid's sums
  const long long* Sg = p.S + ((int64_t)u * p.K + k) * kD + (4 * (lane & 1)) * 16 + (lane >> 1);
  const long long sum[4] = {Sg[0], Sg[16], Sg[32], Sg[48]};
  const uint4 cmax = *reinterpret_cast<const uint4*>(p.chmax + (int64_t)u * kD + 4 * lane);
  const uint4 cmin = *reinterpret_cast<const uint4*>(p.chmin + (int64_t)u * kD + 4 * lane);
  if (!full && o1 == o0) return;                     // no entries: unchanged
  const int n = cnt + n_old;
  if (lane == 0) p.n[(int64_t)u * p.K + k] = n;
  if (n <= 0) return;                                // an empty centroid keeps its value
  const uint32_t cmax_e[4] = {cmax.x, cmax.y, cmax.z, cmax.w};
  const uint32_t cmin_e[4] = {cmin.x, cmin.y, cmin.z, cmin.w};
  const double dn = (double)n;
  double sq = 0.0;
  double mean[4];
  uint32_t wide = 0;                     // this lane's channels outside the fixed-point window
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const int L = fix_exponent(cmax_e[e], p.log2n);
    const double scale = __longlong_as_double((long long)(1023 + L) << 52);
    mean[e] = __ddiv_rn(__dmul_rn(__ll2double_rn(sum[e]), scale), dn);
    // the quantum of the smallest nonzero value, 2^(e_min - p) with p the
    // stored fraction bits, must be at least 2^L for the sum to be exact
    const uint32_t inv = cmin_e[e];
    if (inv != 0u) {
      const uint32_t mb = 0x7FFFFFFFu - inv;
      const int emin = (int)((mb >> 23) & 0xFFu) == 0 ? -126 : (int)((mb >> 23) & 0xFFu) - 127;
      if (emin - (DT == kBF16 ? 7 : 23) < L) wide |= 1u << e;
    }
  }
  // rare: exact sums for those channels (every lane of the warp takes part)
  unsigned any = __ballot_sync(0xffffffffu, wide != 0u);
  while (any) {
    const int src = __ffs(any) - 1;
    any &= any - 1u;
    const uint32_t wb = __shfl_sync(0xffffffffu, wide, src);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if ((wb >> e) & 1u) {
        const double exact = exact_member_sum<DT>(p, u, k, 4 * src + e);
        if (lane == src) mean[e] = __ddiv_rn(exact, dn);
      }
    }
  }
  if (DT == kBF16) {
    uint16_t h[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      h[e] = f64_to_bf16_rne(mean[e]);
      const double c = (double)bf16_bits_to_f32(h[e]);
      sq = __dadd_rn(sq, __dmul_rn(c, c));
    }
    uint2 w;
    w.x = (uint32_t)h[0] | ((uint32_t)h[1] << 16);
    w.y = (uint32_t)h[2] | ((uint32_t)h[3] << 16);
    *reinterpret_cast<uint2*>(static_cast<char*>(p.C) + (((int64_t)u * p.K + k) * kD + lane * 4) * 2) = w;
  } else {
    float f[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      f[e] = __double2float_rn(mean[e]);
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
  // one resident wave: four 8-warp CTAs per SM deal out the wave's listed tokens
  if (W < 1 || W > kCandMaxWave) return cudaErrorInvalidValue;
  const unsigned grid = (unsigned)(4 * device_sm_count());
  qvg_assign_candidates<kBF16><<<grid, kCandWarps * 32, 0, s>>>(R, C, K, N, W, list, list_count, pi);
  return cudaGetLastError();
}

cudaError_t launch_update_bucket(const UpdateParams& p, int dtype, cudaStream_t s) {
  UpdateParams q = p;
  const size_t pad = (size_t)((p.N + 31) & ~int64_t(15));
  const size_t smem = 2 * pad;
  q.stage_pi = smem <= kBucketStageBytes;
  const size_t dyn = q.stage_pi ? smem : 0;
  const void* fn = dtype == kBF16 ? reinterpret_cast<const void*>(qvg_update_bucket<kBF16>)
                                  : reinterpret_cast<const void*>(qvg_update_bucket<kFP32>);
  cudaError_t e = ensure_dynamic_smem(fn, dyn);
  if (e != cudaSuccess) return e;
  if (dtype == kBF16) qvg_update_bucket<kBF16><<<(unsigned)p.W, kBucketThreads, dyn, s>>>(q);
  else qvg_update_bucket<kFP32><<<(unsigned)p.W, kBucketThreads, dyn, s>>>(q);
  return cudaGetLastError();
}

cudaError_t launch_update_sum(const UpdateParams& p, int dtype, cudaStream_t s) {
  const dim3 grid((unsigned)kSumSlices, (unsigned)p.W);
  const size_t smem = (size_t)kSumWarps * kSumRing * 2 * kD * (dtype == kBF16 ? 2 : 4);
  const void* fn = dtype == kBF16 ? reinterpret_cast<const void*>(qvg_update_sum<kBF16>)
                                  : reinterpret_cast<const void*>(qvg_update_sum<kFP32>);
  const cudaError_t e = ensure_dynamic_smem(fn, smem);
  if (e != cudaSuccess) return e;
  if (dtype == kBF16) qvg_update_sum<kBF16><<<grid, kSumThreads, smem, s>>>(p);
  else qvg_update_sum<kFP32><<<grid, kSumThreads, smem, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_update_centroids(const UpdateParams& p, int dtype, cudaStream_t s) {
  const dim3 grid((unsigned)((p.K + 7) / 8), (unsigned)p.W);
  if (dtype == kBF16) qvg_update_centroids<kBF16><<<grid, 256, 0, s>>>(p);
  else qvg_update_centroids<kFP32><<<grid, 256, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace qvg
