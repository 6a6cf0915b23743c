// kernel_assign_tc.cu -- qvg_kmeans_assign: the k-means assignment step of
// semantic-aware smoothing (m.163.com article on Quant VideoGen, section 三)
// as a tensor-core contraction on sm_100a.
//
// For a tile of 128 tokens R (bf16) and the block's K <= 256 centroids C
// (bf16), tcgen05.mma (kind::f16, M=128, N=Kpad, fp32 accumulate) computes the
// 128 x Kpad dot products r_i . c_k into tensor memory.  The epilogue warps
// read them back with tcgen05.ld as h_ik = r_i . c_k - |c_k|^2/2 (a ninth MMA
// K-step adds the bias; argmax_k h_ik = argmin_k |r_i - c_k|^2) and keep, per
// token, the maxima of the 32 eight-column groups and of the 8 position
// classes within a group.  If a second group or a second position class comes
// within the rounding-error bound of the maximum, the token is appended to a
// per-block list that an exact fp64 pass (qvg_assign_candidates) decides;
// otherwise the maximum's column is the assignment.
//
// Data movement: the centroid table is loaded once per CTA with TMA (128-byte
// swizzle, K-major), token tiles stream through a 3-stage TMA ring; no
// multicast.  Warp roles: warp 0 = TMA producer, warp 1 = MMA issuer (one
// elected thread) and TMEM owner, warps 2-9 = epilogue (two warps per TMEM
// lane quarter, taking alternate tiles).  Two TMEM accumulators (2 x 256
// columns) let the epilogue of tile i overlap the MMAs of tile i+1.  Every
// mbarrier wait is bounded; on timeout the kernel records an error in the
// status word, drains, frees TMEM and returns.
#include <cuda.h>

#include "qvg_common.cuh"
#include "qvg_launch.h"

namespace qvg {
namespace {

constexpr int kTcThreads = 320;     // 10 warps
constexpr int kStages = 3;
constexpr int kTileM = 128;
constexpr int kAStageBytes = kTileM * kD * 2;     // 32 KB: two 16 KB K-halves
constexpr int kAHalfBytes = kTileM * 128;         // 128 rows x 128 B
constexpr uint64_t kWaitLimitNs = 2000000000ull;   // 2 s of wall time per wait
constexpr uint32_t kStatusTimeout = 1u;

struct __align__(8) TcSmemBarriers {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t b_full;
  uint64_t tmem_full[2];
  uint64_t tmem_empty[2];
  uint32_t tmem_base;
  int abort_flag;
};

// ---------------------------------------------------------------- PTX helpers
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

// Bounded wait for the phase of `parity` to complete: gives up after
// `limit_ns` of wall time and returns false.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
  const uint32_t addr = smem_u32(bar);
  uint64_t t0 = 0;
  for (uint32_t it = 0;; ++it) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(addr), "r"(parity)
        : "memory");
    if (done) return true;
    if ((it & 63u) == 0u) {
      const uint64_t now = globaltimer_ns();
      if (t0 == 0) t0 = now;
      else if (now - t0 > limit_ns) return false;
    }
  }
}

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, int x, int y, int z,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
      : "memory");
}

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups
// 1024 bytes apart (SBO), leading offset unused (1), descriptor version 1.
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFF);
  d |= (uint64_t)1 << 16;                 // LBO (16-byte units)
  d |= (uint64_t)(1024 >> 4) << 32;       // SBO
  d |= (uint64_t)1 << 46;                 // version
  d |= (uint64_t)2 << 61;                 // SWIZZLE_128B
  return d;
}

// Descriptor of a K-major operand without swizzle: 8x16-byte core matrices,
// the two 8-element K halves 128 bytes apart (LBO), 8-row groups 256 bytes
// apart (SBO).
__device__ __forceinline__ uint64_t umma_desc_noswz(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFF);
  d |= (uint64_t)(128 >> 4) << 16;        // LBO
  d |= (uint64_t)(256 >> 4) << 32;        // SBO
  d |= (uint64_t)1 << 46;                 // version
  return d;                               // layout type 0: no swizzle
}
// Byte offset of element (row, k), k < 16, in that layout.
__device__ __forceinline__ int noswz_offset(int row, int k) {
  return (row >> 3) * 256 + (k >> 3) * 128 + (row & 7) * 16 + (k & 7) * 2;
}

// Instruction descriptor: kind::f16, A = B = bf16, D = f32, both K-major.
__host__ __device__ constexpr uint32_t umma_idesc_bf16(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void umma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// 32 lanes x 32 consecutive 32-bit columns -> 32 registers per thread
// (asynchronous: the registers are valid after tmem_wait_ld).
__device__ __forceinline__ void tmem_ld32_async(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
        "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
        "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
        "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
// Wait for this thread's tensor-memory loads; the buffer's registers pass
// through the asm so that no use of them can be scheduled before the wait.
__device__ __forceinline__ void tmem_wait_ld(uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.wait::ld.sync.aligned;"
      : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
        "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
        "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]),
        "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]),
        "+r"(r[29]), "+r"(r[30]), "+r"(r[31])
      :
      : "memory");
}


struct TcParams {
  const float* rnorm2;      // [W][N]
  const float* cn;          // [W][K]
  uint8_t* pi;              // [W][N]
  uint2* list;              // [W][N] {token, mask of 8-centroid groups holding the candidates}
  uint32_t* list_count;     // [W]
  uint32_t* status;         // workspace status word
  unsigned long long* flagged;
  int64_t N;
  int K;
  int Npad;                 // K rounded up to 32 (MMA N)
  int tiles_per_unit;
  int tiles_per_cta;
  float gamma;              // relative error bound of the tensor-core dot products
  // Test hook of the bounded waits (fault injection on the host side): the
  // CTA of block 0, tile range 0 waits at most `hook_wait_ns` and, when
  // `hook_withhold` >= 0, its producer stops before issuing that tile, so
  // that the waits on it run out.  Off: hook_withhold = -1, hook_wait_ns = 0.
  int hook_withhold;
  uint64_t hook_wait_ns;
};


__device__ __forceinline__ int aborted(const TcSmemBarriers* b) {
  return *reinterpret_cast<const volatile int*>(&b->abort_flag);
}
__device__ __forceinline__ void set_abort(TcSmemBarriers* b) {
  *reinterpret_cast<volatile int*>(&b->abort_flag) = 1;
}

__device__ __forceinline__ float max3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}


// NCH > 0 fixes the number of 32-column chunks at compile time (8 for
// K = 256), so the epilogue's chunk guards fold away; NCH = 0 reads it from
// the padded centroid count.
template <int NCH>
__global__ void __launch_bounds__(kTcThreads, 1)
qvg_kmeans_assign(const __grid_constant__ CUtensorMap tmR, const __grid_constant__ CUtensorMap tmC,
                  const TcParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int u = blockIdx.y;
  const int t_begin = blockIdx.x * p.tiles_per_cta;
  const int t_end = min(p.tiles_per_unit, t_begin + p.tiles_per_cta);
  if (t_begin >= t_end) return;
  const int ntiles = t_end - t_begin;

  const int Npad = p.Npad;
  uint8_t* sB = smem;                                           // 2 x Npad x 128 B
  uint8_t* sA = smem + 2 * Npad * 128;                          // kStages x 32 KB (1024-aligned)
  uint8_t* sAx = sA + kStages * kAStageBytes;                   // 128 x 16 bf16: [1 1 1 0 ...]
  uint8_t* sBx = sAx + kTileM * 32;                             // Npad x 16 bf16: -|c|^2/2 in 3 pieces
  TcSmemBarriers* bars = reinterpret_cast<TcSmemBarriers*>(sBx + Npad * 32);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) { mbar_init(&bars->full[s], 1); mbar_init(&bars->empty[s], 1); }
    mbar_init(&bars->b_full, 1);
    for (int a = 0; a < 2; ++a) { mbar_init(&bars->tmem_full[a], 1); mbar_init(&bars->tmem_empty[a], 4); }
    bars->abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(
                     smem_u32(&bars->tmem_base)));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  // Extra K step of the MMA: A rows [1, 1, 1, 0, ...] times B rows
  // [b0, b1, b2, 0, ...] with b0 + b1 + b2 = -|c_k|^2 / 2 (three bf16 pieces
  // of the fp32 value; the most negative bf16 for padded centroids) adds -|c_k|^2/2 to every
  // dot product, so the accumulator holds r.c_k - |c_k|^2/2.
  for (int x = threadIdx.x; x < kTileM * 16; x += blockDim.x) {
    const int r = x >> 4, k = x & 15;
    *reinterpret_cast<uint16_t*>(sAx + noswz_offset(r, k)) = k < 3 ? (uint16_t)0x3F80 : (uint16_t)0;
  }
  for (int x = threadIdx.x; x < Npad * 16; x += blockDim.x) {
    const int c = x >> 4, k = x & 15;
    uint16_t bits = 0;
    if (k < 3) {
      if (c >= p.K) {
        bits = k == 0 ? (uint16_t)0xFF7F : (uint16_t)0;           // -3.39e38: never the maximum
      } else {
        const float v = -0.5f * p.cn[(int64_t)u * p.K + c];
        const __nv_bfloat16 b0 = __float2bfloat16_rn(v);
        const float r1 = __fsub_rn(v, __bfloat162float(b0));
        const __nv_bfloat16 b1 = __float2bfloat16_rn(r1);
        const __nv_bfloat16 b2 = __float2bfloat16_rn(__fsub_rn(r1, __bfloat162float(b1)));
        const __nv_bfloat16 pick = k == 0 ? b0 : (k == 1 ? b1 : b2);
        bits = *reinterpret_cast<const uint16_t*>(&pick);
      }
    }
    *reinterpret_cast<uint16_t*>(sBx + noswz_offset(c, k)) = bits;
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // visible to the tensor core
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  // The test hook applies to the CTA of block 0 that starts at tile 0 only.
  const bool hooked = p.hook_wait_ns != 0 && u == 0 && blockIdx.x == 0;
  const uint64_t wait_ns = hooked ? p.hook_wait_ns : kWaitLimitNs;
  const int withhold = hooked ? p.hook_withhold : -1;

  if (warp == 0) {
    // ---------------- TMA producer
    if (lane == 0) {
      mbar_expect_tx(&bars->b_full, (uint32_t)(2 * Npad * 128));
      tma_load_3d(sB, &tmC, 0, 0, u, &bars->b_full);
      tma_load_3d(sB + Npad * 128, &tmC, 64, 0, u, &bars->b_full);
      int issued = 0;
      bool stopped = false;
      for (int i = 0; i < ntiles; ++i) {
        const int s = i % kStages;
        const uint32_t ph = (uint32_t)(i / kStages) & 1u;
        if (!mbar_wait(&bars->empty[s], ph ^ 1u, wait_ns) || aborted(bars)) { set_abort(bars); stopped = true; break; }
        if (i == withhold) { stopped = true; break; }   // test hook: this tile is never loaded
        uint8_t* a = sA + s * kAStageBytes;
        const int row = (t_begin + i) * kTileM;
        mbar_expect_tx(&bars->full[s], (uint32_t)kAStageBytes);
        tma_load_3d(a, &tmR, 0, row, u, &bars->full[s]);
        tma_load_3d(a + kAHalfBytes, &tmR, 64, row, u, &bars->full[s]);
        ++issued;
      }
      if (stopped) {              // drain: wait (bounded) for the loads in flight
        for (int i = (issued > kStages ? issued - kStages : 0); i < issued; ++i)
          mbar_wait(&bars->full[i % kStages], (uint32_t)(i / kStages) & 1u, wait_ns);
        mbar_wait(&bars->b_full, 0, wait_ns);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc = umma_idesc_bf16(kTileM, Npad);
      const uint32_t b_addr = smem_u32(sB);
      const uint32_t ax_addr = smem_u32(sAx), bx_addr = smem_u32(sBx);
      bool ok = mbar_wait(&bars->b_full, 0, wait_ns);
      int issued = 0;
      for (int i = 0; ok && i < ntiles; ++i) {
        const int s = i % kStages;
        const uint32_t ph = (uint32_t)(i / kStages) & 1u;
        const int acc = i & 1;
        const uint32_t aph = (uint32_t)(i >> 1) & 1u;
        if (!mbar_wait(&bars->tmem_empty[acc], aph ^ 1u, wait_ns)) { ok = false; break; }
        if (!mbar_wait(&bars->full[s], ph, wait_ns)) { ok = false; break; }
        if (aborted(bars)) { ok = false; break; }
        tc_fence_after();
        const uint32_t a_addr = smem_u32(sA + s * kAStageBytes);
        const uint32_t d_tmem = tmem + (uint32_t)(acc * 256);
#pragma unroll
        for (int k = 0; k < kD / 16; ++k) {
          const uint32_t koff = (uint32_t)((k & 3) * 32);
          const uint64_t ad = umma_desc_sw128(a_addr + (k >> 2) * kAHalfBytes + koff);
          const uint64_t bd = umma_desc_sw128(b_addr + (k >> 2) * Npad * 128 + koff);
          umma_bf16(d_tmem, ad, bd, idesc, k > 0 ? 1u : 0u);
        }
        umma_bf16(d_tmem, umma_desc_noswz(ax_addr), umma_desc_noswz(bx_addr), idesc, 1u);
        umma_commit(&bars->empty[s]);
        umma_commit(&bars->tmem_full[acc]);
        ++issued;
      }
      if (!ok) {
        set_abort(bars);
        // the last MMAs issued must finish before the CTA frees tensor memory
        if (issued > 0) mbar_wait(&bars->tmem_full[(issued - 1) & 1], (uint32_t)((issued - 1) >> 1) & 1u, wait_ns);
      }
    }
  } else {
    // ---------------- epilogue (warps 2..9)
    // Warp (q, h) may read TMEM lane quarter q = warp % 4 (its 32 rows) and
    // owns accumulator h: it takes the tiles i with i % 2 == h, all columns.
    // The two warps of a quarter share an SM sub-partition and alternate
    // tiles, so each decides its rows alone (no exchange between warps).
    const int q = warp & 3;
    const int hc = (warp - 2) >> 2;
    const int row = q * 32 + lane;
    const int nch = NCH > 0 ? NCH : (Npad >> 5);   // 32-column chunks (>= 1)
    float rn2_next = 0.0f;
    {
      const int64_t tok = (int64_t)(t_begin + hc) * kTileM + row;
      if (hc < ntiles && tok < p.N) rn2_next = p.rnorm2[(int64_t)u * p.N + tok];
    }
    for (int i = hc; i < ntiles; i += 2) {
      const int acc = hc;
      const uint32_t aph = (uint32_t)(i >> 1) & 1u;
      const float rn2 = rn2_next;
      {   // prefetch the squared row norm of this warp's next tile
        const int64_t tok = (int64_t)(t_begin + i + 2) * kTileM + row;
        if (i + 2 < ntiles && tok < p.N) rn2_next = p.rnorm2[(int64_t)u * p.N + tok];
      }
      const bool ok = !aborted(bars) && mbar_wait(&bars->tmem_full[acc], aph, wait_ns);
      if (!ok) set_abort(bars);
      tc_fence_after();
      // h_k = r.c_k - |c_k|^2/2; the largest h is the nearest centroid.  Column
      // k = 8g + j lies in group g (8 consecutive columns) and position class
      // j.  The maxima of the 32 groups and of the 8 position classes are
      // kept; they are exact maxima of the accumulator values, formed with
      // three-input max instructions (about one per value).  A column other
      // than the winner w lies outside w's group or outside w's position
      // class, so the larger of the best other group and the best other
      // position class is exactly the runner-up value.  The next 32-column
      // chunk's tensor-memory load is in flight while the current one is
      // processed.
      const float kNegBig = -3.0e38f;
      float gmax[32], pmax[8];
#pragma unroll
      for (int g = 0; g < 32; ++g) gmax[g] = kNegBig;
#pragma unroll
      for (int j = 0; j < 8; ++j) pmax[j] = kNegBig;
      if (ok) {
        const uint32_t tbase = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * 256);
        uint32_t ra[32], rb[32];
        tmem_ld32_async(tbase, ra);
        tmem_wait_ld(ra);
        auto chunk = [&](const uint32_t (&r)[32], int ci) {
#pragma unroll
          for (int e = 0; e < 32; e += 8) {
            float v[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) v[j] = __uint_as_float(r[e + j]);
            gmax[ci * 4 + (e >> 3)] = max3f(max3f(v[0], v[1], v[2]), max3f(v[3], v[4], v[5]), fmaxf(v[6], v[7]));
          }
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            pmax[j] = max3f(pmax[j], __uint_as_float(r[j]), __uint_as_float(r[8 + j]));
            pmax[j] = max3f(pmax[j], __uint_as_float(r[16 + j]), __uint_as_float(r[24 + j]));
          }
        };
#pragma unroll
        for (int ci = 0; ci < 8; ci += 2) {
          if (ci < nch) {
            if (ci + 1 < nch) tmem_ld32_async(tbase + (uint32_t)((ci + 1) * 32), rb);
            chunk(ra, ci);
            tmem_wait_ld(rb);
          }
          if (ci + 1 < nch) {
            if (ci + 2 < nch) tmem_ld32_async(tbase + (uint32_t)((ci + 2) * 32), ra);
            chunk(rb, ci + 1);
            tmem_wait_ld(ra);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->tmem_empty[acc]);
      const int64_t tok = (int64_t)(t_begin + i) * kTileM + row;
      const bool valid = ok && tok < p.N && !aborted(bars);
      const int64_t gi = (int64_t)u * p.N + tok;
      bool flag = false;
      uint32_t groups = 0;
      if (valid) {
        const float M = max3f(max3f(pmax[0], pmax[1], pmax[2]), max3f(pmax[3], pmax[4], pmax[5]),
                              fmaxf(pmax[6], pmax[7]));
        // Error bound E of every h that can compete (fp32 tensor-core sums of
        // 128 exact products and the three pieces of -|c|^2/2):
        // gamma * (|r| |c| + |c|^2 / 2), where |c| <= |r| + sqrt(D_min) for
        // every centroid at least as near as the nearest.  A column whose h is
        // below thr = M - 2E cannot be the exact maximum; the extra
        // 2^-23 |M| covers the rounding of thr itself.
        const float nr = sqrtf(fmaxf(rn2, 0.0f)) * 1.0001f;
        const float cb = 1.02f * nr + sqrtf(fmaxf(rn2 - 2.0f * M, 0.0f));
        const float E = p.gamma * (nr * cb + 0.5f * cb * cb) + 6.0e-8f * cb * cb + 1e-30f;
        const float thr = M - (2.0f * E + 1.2e-7f * fabsf(M));
        uint32_t mp = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) mp |= pmax[j] >= thr ? (1u << j) : 0u;
#pragma unroll
        for (int g = 0; g < 32; ++g) groups |= gmax[g] >= thr ? (1u << g) : 0u;
        // one group and one position class reach thr: the winner is certain
        // (both masks hold M's column unless M is not a number)
        const bool unique = mp != 0u && groups != 0u && (mp & (mp - 1u)) == 0u && (groups & (groups - 1u)) == 0u;
        if (unique) {
          p.pi[gi] = (uint8_t)(8 * (__ffs(groups) - 1) + (__ffs(mp) - 1));
        } else {
          flag = true;   // the groups that reach thr hold every candidate
        }
      }
      // every lane of the warp takes part in the list append
      const unsigned fm = __ballot_sync(0xffffffffu, flag);
      if (fm) {
        const int leader = __ffs(fm) - 1;
        uint32_t base = 0;
        if (lane == leader) {
          base = atomicAdd(&p.list_count[u], (uint32_t)__popc(fm));
          atomicAdd(p.flagged, (unsigned long long)__popc(fm));
        }
        base = __shfl_sync(0xffffffffu, base, leader);
        if (flag) p.list[(int64_t)u * p.N + base + __popc(fm & ((1u << lane) - 1u))] = make_uint2((uint32_t)tok, groups);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (aborted(bars) && threadIdx.x == 0) atomicOr(p.status, kStatusTimeout);
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem));
  }
}

// ---------------------------------------------------------------- host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
  }
  return fn;
}

// 3-D bf16 map over [W][rows][128]: box = 64 channels (128 B, swizzled) x box_rows x 1.
bool make_map(CUtensorMap* m, const void* base, int64_t rows, int W, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)kD, (cuuint64_t)rows, (cuuint64_t)W};
  const cuuint64_t strides[2] = {(cuuint64_t)kD * 2, (cuuint64_t)rows * kD * 2};
  const cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

size_t assign_tc_smem_bytes(int K) {
  const int Npad = (K + 31) & ~31;
  return 1024 + 2 * (size_t)Npad * 128 + (size_t)kStages * kAStageBytes + kTileM * 32 + (size_t)Npad * 32 +
         sizeof(TcSmemBarriers);
}

cudaError_t launch_assign_tc(const AssignTcParams& a, cudaStream_t s) {
  CUtensorMap mR, mC;
  const int Npad = (a.K + 31) & ~31;
  if (!make_map(&mR, a.R, a.N, a.W, kTileM) || !make_map(&mC, a.C, a.K, a.W, Npad))
    return cudaErrorInvalidValue;
  TcParams p{};
  p.rnorm2 = a.rnorm2; p.cn = a.cn; p.pi = a.pi; p.list = a.list; p.list_count = a.list_count;
  p.status = a.status; p.flagged = a.flagged; p.N = a.N; p.K = a.K; p.Npad = Npad;
  p.tiles_per_unit = (int)((a.N + kTileM - 1) / kTileM);
  const int sms = device_sm_count();
  int splits = sms / a.W;
  if (splits < 1) splits = 1;
  p.tiles_per_cta = (p.tiles_per_unit + splits - 1) / splits;
  if (p.tiles_per_cta < 2) p.tiles_per_cta = 2;
  splits = (p.tiles_per_unit + p.tiles_per_cta - 1) / p.tiles_per_cta;
  p.gamma = a.gamma;
  p.hook_withhold = a.hook_withhold;
  p.hook_wait_ns = a.hook_wait_ns;
  const size_t smem = assign_tc_smem_bytes(a.K);
  const bool full = Npad == 256;
  const void* fn = full ? reinterpret_cast<const void*>(qvg_kmeans_assign<8>)
                        : reinterpret_cast<const void*>(qvg_kmeans_assign<0>);
  cudaError_t e = ensure_dynamic_smem(fn, smem);
  if (e != cudaSuccess) return e;
  if (full)
    qvg_kmeans_assign<8><<<dim3((unsigned)splits, (unsigned)a.W), kTcThreads, smem, s>>>(mR, mC, p);
  else
    qvg_kmeans_assign<0><<<dim3((unsigned)splits, (unsigned)a.W), kTcThreads, smem, s>>>(mR, mC, p);
  return cudaGetLastError();
}

}  // namespace qvg
