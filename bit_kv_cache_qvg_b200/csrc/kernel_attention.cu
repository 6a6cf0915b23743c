// kernel_attention.cu -- qvg_attention: softmax attention of a block of
// queries over a compressed K/V cache, with the reconstruction fused into
// the attention's K/V load (the consumer of the m.163.com article on Quant
// VideoGen, section 五: the key cache is kept before the rotary embedding,
// which is applied after dequantisation, and the fused kernel keeps the
// reconstructed values on chip instead of writing them out; gist.science/de,
// Technische Zusammenfassung 2C, "Fused Kernel").
//
//   O = softmax(rope(Q) rope(K^)^T / sqrt(d)) V^
//
// where K^ and V^ are the cache's reconstructions (the values
// qvg_dequantize writes, bit for bit), rope is the RoFormer rotary embedding
// (channel pair (2i, 2i+1) of a token at position p turned by
// p * base^(-2i/d)), the cached tokens sit at positions 0 .. Nk-1 and the
// queries at the given positions.  No mask.
//
// One CTA = one head x 256 queries (two query tiles of 128) x a range of the
// cache's tiles of 128 tokens; 24 warps in three roles:
//   * warps 8-23 (96 registers each, moved from the softmax warps by
//     setmaxnreg) dequantise each K and V tile (unpack, scale, add every
//     stage's centroid in reverse order, round to bf16 -- the arithmetic of
//     qvg_dequant_fused), apply the rotary embedding to K, and store both
//     into a two-stage ring in shared memory in the tensor core's K-major
//     operand layout (128-byte swizzle): K rows (keys) with the channels
//     contiguous, V transposed (channels) with the keys contiguous.  A
//     thread's per-token bytes of the next step are loaded during the
//     current one (at most two stages);
//   * the first thread of each query tile's group issues S = Q' K'^T
//     (tcgen05.mma kind::f16, M = N = K = 128, fp32 accumulators in tensor
//     memory) when a stage is full, and O += P V (P read from tensor memory)
//     when the group's softmax is done;
//   * warps 0-3 and 4-7 (48 registers each; one per tensor-memory lane
//     quarter, a thread per query) run the online softmax of the two query
//     tiles (base-2 exponentials against a reference maximum that rises only
//     when a row's maximum exceeds it by more than 8), write P in bf16 over
//     their S columns and, rarely, rescale O in tensor memory.
// The two query tiles' groups run independently, so one group's softmax
// overlaps the other's products.
//
// Pairs: two CTAs of a cluster hold neighbouring blocks of 256 queries; each
// reconstructs 64 keys of every tile and stores them into both CTAs' ring
// stage through distributed shared memory, and a stage is freed by a commit
// multicast to the pair once the products of both CTAs have read it.
//
// Cuts: the cache of a query block is cut into ranges so that the grid fills
// the SMs.  Inside a cluster (split CTAs per query block) each CTA leaves its
// unnormalised O with its row maximum and sum in shared memory and the
// cluster merges them through distributed shared memory; over clusters
// (gsplit ranges) they go to the caller's workspace and qvg_attention_merge
// combines them (the usual rescaling of partial softmax sums).  With no cut,
// O / l is written directly.
//
// The rotary (cos, sin) pairs come from a table of every position, formed
// in fp64 and rounded to fp32 (qvg_rope_tables).  Every mbarrier wait is
// bounded; on expiry the kernel records QVG_ERR_DEVICE_TIMEOUT in the status
// word at the start of the tables buffer and stops.  No TMA and no
// multicast loads: the operands are written by the threads that reconstruct
// them.
#include <cuda.h>

#include <atomic>
#include <type_traits>

#include "qvg_common.cuh"
#include "qvg_launch.h"

namespace qvg {
namespace {

constexpr int kAtThreads = 768;                 // 24 warps
constexpr int kAtQTiles = 2;                    // query tiles per CTA (each reconstructed K/V tile serves both)
constexpr int kAtSoftmaxThreads = 256;          // warps 0-7: softmax of the two query tiles (threads 0 and 128 issue the MMAs)
constexpr int kAtReconThreads = 512;            // warps 8-23: reconstruction into the K/V ring
constexpr int kAtTile = 128;                    // queries per query tile, cached tokens per tile
constexpr int kAtOpBytes = kAtTile * kD * 2;    // one 128 x 128 bf16 operand: 32 KB
constexpr uint64_t kAtWaitNs = 2000000000ull;   // 2 s per bounded wait
constexpr int kAtMaxSplit = 8;                  // CTAs per cluster, at most (the portable cluster size)
constexpr int kAtMaxGlobalSplit = 16;           // ranges of a global split, at most
constexpr int kMaxDevices = 64;

struct AttnParams {
  const uint8_t* codes[2];        // K, V: [H][Nk][d/4]
  const uint8_t* scale[2];        // [H][Nk][d/G]
  const uint8_t* zero[2];         // [H][Nk][d/G] (asymmetric mode)
  const uint8_t* assign[2];       // [T][H][Nk]
  const __nv_bfloat16* tab[2];    // [T][H][K][d]
  const __nv_bfloat16* Q;         // [H][Nq][d], before the rotary embedding
  const int64_t* qpos;            // [Nq] query positions
  const float2* rope;             // [max_pos + 1][d/2]: (cos, sin) of p theta_i
  float* O;                       // [H][Nq][d]
  uint32_t* status;
  int64_t max_pos;                // largest position the tables cover
  int64_t Nk, Nq;
  int H, K, T, G, sym;
  int split;                      // cluster CTAs (per query block) over ranges of the cache's tiles
  int pair;                       // 2: two CTAs (two query blocks) share each tile's reconstruction
  int gsplit;                     // ranges of the cache merged through global memory (1: none)
  float* part_O;                  // [gsplit][H][Nq][d]: unnormalised O of each range
  float2* part_ml;                // [gsplit][H][Nq]: (row maximum, row sum) of each range
  float sl;                       // log2(e) / sqrt(d)
};

struct __align__(8) AtBars {
  uint64_t s_done[2];       // S product of query tile g complete (tcgen05.commit)
  uint64_t o_done[2];       // O product of query tile g complete (tcgen05.commit)
  uint64_t kv_full[2];      // ring stage reconstructed (lane 0 of every reconstruction warp of each CTA that writes it)
  uint64_t kv_empty[2];     // ring stage free again: the O products of every CTA that read it completed
  uint32_t tmem_base;
  int abort_flag;
};

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ bool bar_wait(uint64_t* bar, uint32_t parity) {
  const uint32_t addr = smem_addr(bar);
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
      uint64_t now;
      asm volatile("mov.u64 %0, %globaltimer;" : "=l"(now));
      if (t0 == 0) t0 = now;
      else if (now - t0 > kAtWaitNs) return false;
    }
  }
}

// bar_wait that also gives up as soon as another role of the CTA has
// recorded an abort (so that no role waits out the full limit for a
// partner that has stopped).
__device__ __forceinline__ bool bar_wait_or_abort(uint64_t* bar, uint32_t parity, const volatile int* abort_flag) {
  const uint32_t addr = smem_addr(bar);
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
      if (*abort_flag) return false;
      uint64_t now;
      asm volatile("mov.u64 %0, %globaltimer;" : "=l"(now));
      if (t0 == 0) t0 = now;
      else if (now - t0 > kAtWaitNs) return false;
    }
  }
}
// bar_wait_or_abort with acquire at cluster scope: the barrier also takes
// arrivals (and the writes they release) from the other CTA of a pair.
__device__ __forceinline__ bool bar_wait_cluster(uint64_t* bar, uint32_t parity, const volatile int* abort_flag) {
  const uint32_t addr = smem_addr(bar);
  uint64_t t0 = 0;
  for (uint32_t it = 0;; ++it) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(addr), "r"(parity)
        : "memory");
    if (done) return true;
    if ((it & 63u) == 0u) {
      if (*abort_flag) return false;
      uint64_t now;
      asm volatile("mov.u64 %0, %globaltimer;" : "=l"(now));
      if (t0 == 0) t0 = now;
      else if (now - t0 > kAtWaitNs) return false;
    }
  }
}
// Named barrier over `count` threads with an OR of `pred` (every participant
// gets the same answer).
__device__ __forceinline__ bool named_bar_or(int id, int count, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(id), "r"(count)
      : "memory");
  return r != 0;
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}
// arrive on a barrier of another CTA of the cluster (shared::cluster
// address), releasing this thread's earlier writes at cluster scope
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr_of_bar) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr_of_bar) : "memory");
}
__device__ __forceinline__ void st_cluster_v4(uint32_t a, uint4 v) {
  asm volatile("st.shared::cluster.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(a), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}
__device__ __forceinline__ void st_cluster_b32(uint32_t a, uint32_t v) {
  asm volatile("st.shared::cluster.b32 [%0], %1;" ::"r"(a), "r"(v) : "memory");
}

// Shared-memory operand descriptor, K-major, 128-byte swizzle: a 128 x 128
// bf16 operand is two 64-column halves of 128 rows x 128 bytes (16 KB apart),
// and in each 8-row group of 1,024 bytes (SBO) the 16-byte chunk c of row r
// sits at chunk position c ^ (r mod 8).  The swizzle spreads a warp's stores
// of one chunk column over all banks.
__device__ __forceinline__ uint64_t op_desc(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFF);
  d |= (uint64_t)1 << 16;                 // LBO (unused with this swizzle)
  d |= (uint64_t)(1024 >> 4) << 32;       // SBO
  d |= (uint64_t)1 << 46;                 // version
  d |= (uint64_t)2 << 61;                 // SWIZZLE_128B
  return d;
}
constexpr int kAtHalfBytes = kAtTile * 128;     // one 64-column half of an operand
// Byte offset of element (row, k) of a 128 x 128 operand (k even for the
// 4-byte stores, a multiple of 8 for the 16-byte ones).
__device__ __forceinline__ int op_off(int row, int k) {
  return (k >> 6) * kAtHalfBytes + row * 128 + ((((k & 63) >> 3) ^ (row & 7)) << 4) + (k & 7) * 2;
}
// Descriptor of K-step kk (16 columns) of the operand at saddr.
__device__ __forceinline__ uint64_t op_desc_k(uint32_t saddr, int kk) {
  return op_desc(saddr + (uint32_t)((kk >> 2) * kAtHalfBytes + (kk & 3) * 32));
}

// kind::f16, A = B = bf16, D = f32, both K-major, M = N = 128.
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(128 >> 3) << 17) |
                            ((uint32_t)(128 >> 4) << 24);

__device__ __forceinline__ void mma(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(a), "l"(b), "r"(kIdesc), "r"(accumulate)
      : "memory");
}
// The same product with A read from tensor memory (lane i = row i, K
// elements packed two per 32-bit column, the lower half first).
__device__ __forceinline__ void mma_ta(uint32_t tmem_d, uint32_t tmem_a, uint64_t b, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(tmem_d),
      "r"(tmem_a), "l"(b), "r"(kIdesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_addr(bar))
               : "memory");
}
// the same arrival on the barrier at this offset in every CTA of `mask`
// (bit i = cluster rank i)
__device__ __forceinline__ void mma_commit_mc(uint64_t* bar, uint16_t mask) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          smem_addr(bar)),
      "h"(mask)
      : "memory");
}
__device__ __forceinline__ void fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tld32(uint32_t taddr, uint32_t (&r)[32]) {
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
  // the registers pass through the wait so that no use moves above it
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

__device__ __forceinline__ void tld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  // the registers pass through the wait so that no use moves above it
  asm volatile(
      "tcgen05.wait::ld.sync.aligned;"
      : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
        "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15])
      :
      : "memory");
}
__device__ __forceinline__ void tst16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};"
      ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
__device__ __forceinline__ void tst8(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};"
               ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
               : "memory");
}

__device__ __forceinline__ float exp2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Distributed shared memory of the CTA's cluster: the address of the same
// shared-memory location in CTA `rank`, loads from it, and the cluster-wide
// barrier (every thread of every CTA arrives; release/acquire order the
// shared-memory writes before it with the reads after it).
__device__ __forceinline__ uint32_t cluster_addr(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}
__device__ __forceinline__ float4 ld_cluster_f4(uint32_t a) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0,%1,%2,%3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(a) : "memory");
  return v;
}
__device__ __forceinline__ float2 ld_cluster_f2(uint32_t a) {
  float2 v;
  asm volatile("ld.shared::cluster.v2.f32 {%0,%1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(a) : "memory");
  return v;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  const __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&b);
}

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

// (cos, sin) of the rotary angle of pair i at position pos (positions outside
// [0, max_pos] are clamped, so the reads stay in bounds).
__device__ __forceinline__ float2 rope_cs(const AttnParams& p, int64_t pos, int i) {
  pos = pos < 0 ? 0 : (pos > p.max_pos ? p.max_pos : pos);
  return __ldg(p.rope + pos * (kD / 2) + i);
}

// Reconstruction of channels c0 .. c0+7 of the NR tokens tok0 .. tok0+NR-1
// (those below Nk) of cache `which` (0 = K, 1 = V) of head h: y = s*q + m
// (or s*(u - 2)), plus the centroids of stages T, ..., 1 in that order, each
// an fp32 add, then one rounding to bf16 -- the arithmetic of
// qvg_dequant_fused.  The results are fp32 values of the rounded bf16
// numbers (zero for tokens past the end).  In three steps, so that a thread
// can issue the loads of several blocks before it waits for any: the
// per-token codes, scale/zero bytes and assignments; the centroid rows they
// select (TT > 0, a fixed stage count of at most 4); the arithmetic.
template <int TT, int NR>
struct ReconBlock {
  static constexpr int TR = TT > 0 ? TT : 1;
  int tok0, c0, which;
  uint32_t code[NR], sz[NR];
  int kk[NR][TR];
  uint4 rows[NR][TR];

  // the head's streams (the same for the whole CTA), then 32-bit offsets
  // within them (a block has fewer than 2^23 tokens)
  __device__ __forceinline__ void load_tokens(const AttnParams& p, int w, int h, int t0, int ch) {
    which = w; tok0 = t0; c0 = ch;
    const int ng = kD / p.G;
    const int64_t hN = (int64_t)h * p.Nk;
    const uint8_t* codes = p.codes[w] + hN * (kD / 4) + c0 / 4;
    const uint8_t* scl = p.scale[w] + hN * ng + c0 / p.G;
    const uint8_t* zr = p.zero[w] + hN * ng + c0 / p.G;
    const uint8_t* asg = p.assign[w] + hN;
    const int64_t asg_stage = (int64_t)p.H * p.Nk;
#pragma unroll
    for (int r = 0; r < NR; ++r) {
      const uint32_t tok = (uint32_t)(tok0 + r < p.Nk ? tok0 + r : p.Nk - 1);   // past the end: a valid token, result unused
      code[r] = __ldg(reinterpret_cast<const unsigned short*>(codes + tok * (kD / 4)));
      sz[r] = (uint32_t)__ldg(scl + tok * (uint32_t)ng) | (p.sym ? 0u : ((uint32_t)__ldg(zr + tok * (uint32_t)ng) << 8));
#pragma unroll
      for (int t = 0; t < TR; ++t)
        if (TT > 0) kk[r][t] = min((int)__ldg(asg + t * asg_stage + tok), p.K - 1);
    }
  }
  // the per-token part of another block (loaded one step ahead)
  __device__ __forceinline__ void take_tokens(const ReconBlock& o) {
    which = o.which; tok0 = o.tok0; c0 = o.c0;
#pragma unroll
    for (int r = 0; r < NR; ++r) {
      code[r] = o.code[r];
      sz[r] = o.sz[r];
#pragma unroll
      for (int t = 0; t < TR; ++t) kk[r][t] = o.kk[r][t];
    }
  }
  __device__ __forceinline__ void load_rows(const AttnParams& p, int h) {
    if (TT <= 0) return;
    const __nv_bfloat16* tab = p.tab[which] + (int64_t)h * p.K * kD + c0;
    const int64_t tab_stage = (int64_t)p.H * p.K * kD;
#pragma unroll
    for (int r = 0; r < NR; ++r)
#pragma unroll
      for (int t = 0; t < TR; ++t)
        rows[r][t] = __ldg(reinterpret_cast<const uint4*>(tab + t * tab_stage + (uint32_t)kk[r][t] * kD));
  }
  __device__ __forceinline__ void finish(const AttnParams& p, const float2* nlut, int h, float (&y)[NR][8]) const {
    const int T = TT >= 0 ? TT : p.T;
#pragma unroll
    for (int r = 0; r < NR; ++r) {
      // y = s*q + m (or s*(u - 2)), exact in fp32, two channels per op through
      // the nibble table (which holds q, or u - 2 in the symmetric mode)
      const float2 sm = e4m3x2_to_f2(sz[r]);
      const float2 s2 = make_float2(sm.x, sm.x), m2 = make_float2(sm.y, sm.y);
      float2 y2[4];
#pragma unroll
      for (int e = 0; e < 4; ++e)
        y2[e] = p.sym ? __fmul2_rn(s2, nlut[(code[r] >> (4 * e)) & 0xFu])
                      : __ffma2_rn(s2, nlut[(code[r] >> (4 * e)) & 0xFu], m2);
      auto add_row = [&](const uint4 w) {
        y2[0] = __fadd2_rn(y2[0], make_float2(__uint_as_float(w.x << 16), __uint_as_float(w.x & 0xFFFF0000u)));
        y2[1] = __fadd2_rn(y2[1], make_float2(__uint_as_float(w.y << 16), __uint_as_float(w.y & 0xFFFF0000u)));
        y2[2] = __fadd2_rn(y2[2], make_float2(__uint_as_float(w.z << 16), __uint_as_float(w.z & 0xFFFF0000u)));
        y2[3] = __fadd2_rn(y2[3], make_float2(__uint_as_float(w.w << 16), __uint_as_float(w.w & 0xFFFF0000u)));
      };
      if (TT > 0) {
#pragma unroll
        for (int t = TR - 1; t >= 0; --t) add_row(rows[r][t]);
      } else if (TT < 0) {
        const uint32_t tok = (uint32_t)(tok0 + r < p.Nk ? tok0 + r : p.Nk - 1);
        const uint8_t* asg = p.assign[which] + (int64_t)h * p.Nk;
        const __nv_bfloat16* tab = p.tab[which] + (int64_t)h * p.K * kD + c0;
        for (int t = T - 1; t >= 0; --t) {
          const int k = min((int)__ldg(asg + t * (int64_t)p.H * p.Nk + tok), p.K - 1);
          add_row(__ldg(reinterpret_cast<const uint4*>(tab + t * (int64_t)p.H * p.K * kD + (uint32_t)k * kD)));
        }
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) { y[r][2 * e] = y2[e].x; y[r][2 * e + 1] = y2[e].y; }
#pragma unroll
      for (int e = 0; e < 8; e += 2) {
        const uint32_t b = pack_bf16(y[r][e], y[r][e + 1]);
        y[r][e] = tok0 + r < p.Nk ? __uint_as_float(b << 16) : 0.0f;
        y[r][e + 1] = tok0 + r < p.Nk ? __uint_as_float(b & 0xFFFF0000u) : 0.0f;
      }
    }
  }
};

template <int TT>
__global__ void __launch_bounds__(kAtThreads, 1)
qvg_attention_fused(const AttnParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;                               // A of S: two query tiles x channels
  uint8_t* sK0 = sQ + kAtQTiles * kAtOpBytes;       // ring stage s: K at sK0 + 2s tiles, V after it
  float2* nlut = reinterpret_cast<float2*>(sK0 + 4 * kAtOpBytes);   // nibble -> two codes (q, or u - 2)
  AtBars* bars = reinterpret_cast<AtBars*>(nlut + 32);
  volatile int* abort_flag = &bars->abort_flag;
  auto stage_k = [&](int st) { return sK0 + (2 * st) * kAtOpBytes; };   // B of S
  auto stage_v = [&](int st) { return sK0 + (2 * st + 1) * kAtOpBytes; };

  const int h = blockIdx.y;
  // A cluster = pair x split CTAs.  Cluster rank = sr * pair + pr: the pair
  // (pr = 0, 1) holds two neighbouring blocks of 256 queries and shares the
  // reconstruction of every tile; split rank sr takes one range of the
  // cache's tiles.  Clusters x = unit * gsplit + gs take range gs of a
  // global split (merged through global memory by qvg_attention_merge).
  const int csize = p.pair * p.split;
  const int rank = (int)(blockIdx.x % (unsigned)csize);
  const int pr = rank % p.pair, sr = rank / p.pair;
  const unsigned ug = blockIdx.x / (unsigned)csize;
  const int gs = (int)(ug % (unsigned)p.gsplit);
  const int64_t q0 = ((int64_t)(ug / (unsigned)p.gsplit) * p.pair + pr) * (kAtQTiles * kAtTile);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_addr(&bars->s_done[i])));
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_addr(&bars->o_done[i])));
      // kv_full: one lane of every reconstruction warp of each CTA that writes the stage
      asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(&bars->kv_full[i])),
                   "r"(kAtReconThreads / 32 * p.pair));
      // kv_empty: one commit per query tile of each CTA that reads the stage's contents
      asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(&bars->kv_empty[i])), "r"(2 * p.pair));
    }
    bars->abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(
                     smem_addr(&bars->tmem_base)));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  if (threadIdx.x < 16) {
    const float off = p.sym ? 2.0f : 0.0f;
    nlut[threadIdx.x] = make_float2((float)(threadIdx.x & 3u) - off, (float)(threadIdx.x >> 2) - off);
  }
  // queries: rotary embedding at their positions, bf16, into the A layout
  // (all 512 threads: rows 4*rb .. 4*rb+3 of each tile, channels 8*cb ..)
  if (threadIdx.x < 512) {
    const int rb = threadIdx.x >> 4, cb = threadIdx.x & 15;
    for (int qt = 0; qt < kAtQTiles; ++qt) {
      for (int r = 0; r < 4; ++r) {
        const int qi = 4 * rb + r;
        const int64_t q = q0 + qt * kAtTile + qi;
        uint32_t w[4] = {0u, 0u, 0u, 0u};
        if (q < p.Nq) {
          const uint4 v = *reinterpret_cast<const uint4*>(p.Q + ((int64_t)h * p.Nq + q) * kD + 8 * cb);
          const uint32_t x[4] = {v.x, v.y, v.z, v.w};
          const int64_t pos = p.qpos[q];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float a = __uint_as_float(x[e] << 16), b = __uint_as_float(x[e] & 0xFFFF0000u);
            const float2 cs = rope_cs(p, pos, 4 * cb + e);
            w[e] = pack_bf16(__fsub_rn(__fmul_rn(a, cs.x), __fmul_rn(b, cs.y)),
                             __fadd_rn(__fmul_rn(a, cs.y), __fmul_rn(b, cs.x)));
          }
        }
        *reinterpret_cast<uint4*>(sQ + qt * kAtOpBytes + op_off(qi, 8 * cb)) = make_uint4(w[0], w[1], w[2], w[3]);
      }
    }
  }
  fence_before();
  __syncthreads();
  fence_after();
  // every CTA of the cluster has initialised its barriers before any remote
  // store or arrival
  if (csize > 1) cluster_sync();
  const uint32_t tmem = bars->tmem_base;
  // S of query tile t at column 128 t, O of query tile t at column 256 + 128 t
  const uint32_t tS = tmem, tO = tmem + 256;
  const int64_t ntot = (p.Nk + kAtTile - 1) / kAtTile;
  // range gs * split + sr of gsplit * split (one of the two is 1): tiles
  // j_begin .. j_begin + ntiles - 1, at least one
  const int parts = p.gsplit * p.split, part = gs * p.split + sr;
  const int j_begin = (int)(ntot * part / parts);
  const int ntiles = (int)(ntot * (part + 1) / parts) - j_begin;   // this CTA's tiles
  int s_issued = 0, o_issued = 0;                   // products committed (the issuing threads 0 and 128)
  float m_fin = 0.0f, l_fin = 0.0f;                 // the softmax thread's row maximum and sum at the end

  if (warp >= 8) {
    // ---------------------------------------------------------------- reconstruction warps
    // Registers move from the softmax warpgroups (48 each thread) to these
    // four (96): 256 x 48 + 512 x 96 = 768 x 80, the launch's allocation.
    asm volatile("setmaxnreg.inc.sync.aligned.u32 96;");
    // tile j goes to ring stage j mod 2 once the O products of tile j - 2
    // (the stage's last readers, in both CTAs of a pair) have completed.
    // Alone, the CTA reconstructs the whole tile (two passes of 64 keys);
    // paired, keys 64 pr .. 64 pr + 63 only, stored into both CTAs' stage.
    // Each warp arrives for itself once its lanes have stored their blocks,
    // so that the warps drift apart and their memory latencies overlap.
    const int r = threadIdx.x - kAtSoftmaxThreads;
    const int rb = r >> 4, cb = r & 15;             // K: two rows from 2*rb (4*rb alone), channels 8*cb ..
    const int rbv = r & 31, cbv = r >> 5;           // V: the same blocks, transposed
    const bool paired = p.pair > 1;
    const uint32_t own_base = smem_addr(smem);
    const uint32_t peer_base = paired ? cluster_addr(own_base, (uint32_t)(rank ^ 1)) : 0u;
    // Steps of 64 keys (two per tile alone, one paired).  With at most two
    // stages a thread's per-token bytes of the next step are loaded while it
    // works on this one (more stages' centroid rows leave no registers for it).
    constexpr bool kAhead = TT >= 0 && TT <= 2;
    const int nh = 2 / p.pair;
    const int nsteps = ntiles * nh;
    auto row_k = [&](int half) { return paired ? 64 * pr + 2 * rb : 4 * rb + 2 * half; };
    auto row_v = [&](int half) { return paired ? 64 * pr + 2 * rbv : 4 * rbv + 2 * half; };
    const int last = (int)p.Nk - 1;                   // the host checked that the tables cover it
    ReconBlock<TT, 2> bk, bv;
    if (kAhead && nsteps > 0) {
      bk.load_tokens(p, 0, h, j_begin * kAtTile + row_k(0), 8 * cb);
      bv.load_tokens(p, 1, h, j_begin * kAtTile + row_v(0), 8 * cbv);
    }
#pragma unroll 1
    for (int s = 0; s < nsteps; ++s) {
      const int j = nh == 1 ? s : s >> 1, half = s - j * nh;
      const int st = j & 1;
      if (half == 0) {
        const bool w = j < 2 || bar_wait_cluster(&bars->kv_empty[st], (uint32_t)(((j >> 1) - 1) & 1), abort_flag);
        if (__any_sync(0xffffffffu, !w || *abort_flag)) {
          *abort_flag = 1;
          break;
        }
        fence_after();
      }
      uint8_t* sK = stage_k(st);
      uint8_t* sV = stage_v(st);
      {
        float vk[2][8];
        const int r0 = row_k(half), tok0 = kAhead ? bk.tok0 : (j_begin + j) * kAtTile + r0;
        // V, transposed (channel 8*cbv + e holds keys rv, rv+1 in 4 contiguous
        // bytes), with the key and channel blocks swapped: the lanes of a store
        // phase write distinct key chunks of one channel row
        const int rv = row_v(half);
        if (!kAhead) {
          bk.load_tokens(p, 0, h, (j_begin + j) * kAtTile + r0, 8 * cb);
          bv.load_tokens(p, 1, h, (j_begin + j) * kAtTile + rv, 8 * cbv);
        }
        bk.load_rows(p, h);
        bv.load_rows(p, h);
        ReconBlock<TT, 2> nk, nv;
        if (kAhead && s + 1 < nsteps) {
          const int j1 = nh == 1 ? s + 1 : (s + 1) >> 1, half1 = s + 1 - j1 * nh;
          nk.load_tokens(p, 0, h, (j_begin + j1) * kAtTile + row_k(half1), 8 * cb);
          nv.load_tokens(p, 1, h, (j_begin + j1) * kAtTile + row_v(half1), 8 * cbv);
        }
        bk.finish(p, nlut, h, vk);
        // K rows: rotary embedding of the reconstructed values at their
        // positions (past the end: the last token's, result unused), then bf16
#pragma unroll
        for (int rr = 0; rr < 2; ++rr) {
          uint32_t w4[4];
          const float4* cs4 = reinterpret_cast<const float4*>(p.rope + (int64_t)min(tok0 + rr, last) * (kD / 2) + 4 * cb);
          const float4 c01 = __ldg(cs4), c23 = __ldg(cs4 + 1);
          const float2 csv[4] = {make_float2(c01.x, c01.y), make_float2(c01.z, c01.w), make_float2(c23.x, c23.y),
                                 make_float2(c23.z, c23.w)};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 cs = csv[e];
            const float a = vk[rr][2 * e], b = vk[rr][2 * e + 1];
            w4[e] = pack_bf16(__fsub_rn(__fmul_rn(a, cs.x), __fmul_rn(b, cs.y)),
                              __fadd_rn(__fmul_rn(a, cs.y), __fmul_rn(b, cs.x)));
          }
          const uint4 v4 = make_uint4(w4[0], w4[1], w4[2], w4[3]);
          uint8_t* dst = sK + op_off(r0 + rr, 8 * cb);
          *reinterpret_cast<uint4*>(dst) = v4;
          if (paired) st_cluster_v4(peer_base + (smem_addr(dst) - own_base), v4);
        }
        bv.finish(p, nlut, h, vk);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const uint32_t v2 = pack_bf16(vk[0][e], vk[1][e]);
          uint8_t* dst = sV + op_off(8 * cbv + e, rv);
          *reinterpret_cast<uint32_t*>(dst) = v2;
          if (paired) st_cluster_b32(peer_base + (smem_addr(dst) - own_base), v2);
        }
        if (kAhead) {
          bk.take_tokens(nk);
          bv.take_tokens(nv);
        }
      }
      if (half < nh - 1) continue;
      // visible to the tensor cores (of both CTAs when paired), then one
      // lane arrives for the warp (on both CTAs' barrier when paired)
      if (paired) asm volatile("fence.proxy.async.shared::cluster;" ::: "memory");
      else asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&bars->kv_full[st]);
        if (paired) mbar_arrive_remote(cluster_addr(smem_addr(&bars->kv_full[st]), (uint32_t)(rank ^ 1)));
      }
    }
    // Paired, the other CTA's commits arrive here too: the last use of each
    // stage must have completed before this CTA may leave (bounded; skipped
    // once a role has aborted).
    if (paired && r == 0 && !*abort_flag)
      for (int j = ntiles - 2 > 0 ? ntiles - 2 : 0; j < ntiles; ++j)
        if (!bar_wait_cluster(&bars->kv_empty[j & 1], (uint32_t)((j >> 1) & 1), abort_flag)) *abort_flag = 1;
  } else {
    // ---------------------------------------------------------------- softmax warps, two independent groups
    asm volatile("setmaxnreg.dec.sync.aligned.u32 48;");
    // Group g (warps 4g .. 4g+3) owns query tile g: row 32*(warp mod 4) + lane,
    // the warp's tensor-memory lane quarter.  Its first thread issues the
    // group's products: S_g = Q_g'K'^T when a stage is full, then, after the
    // group's softmax has written P_g over the first 64 columns of S_g (bf16,
    // two per column), O_g += P_g V with A read from tensor memory.  The two
    // groups run independently, so one group's softmax overlaps the other's
    // products.
    const int g = warp >> 2;
    const bool issuer = threadIdx.x == 128 * g;
    const int qi = 32 * (warp & 3) + lane;
    const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;
    const uint32_t tSt = tS + 128 * g, tOt = tO + 128 * g;
    float m_run = -3.0e38f, l_run = 0.0f;
    bool ok = true;
    for (int j = 0; j < ntiles; ++j) {
      const int st = j & 1;
      const int64_t k0 = (int64_t)(j_begin + j) * kAtTile;
      // 1. S_g once the stage is reconstructed and the previous O_g (which
      // read P_g from these columns) has completed
      if (issuer) {
        bool w = bar_wait_cluster(&bars->kv_full[st], (uint32_t)((j >> 1) & 1), abort_flag);
        if (w && j > 0) w = bar_wait_or_abort(&bars->o_done[g], (uint32_t)((j - 1) & 1), abort_flag);
        if (w) {
          fence_after();
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
          const uint32_t a0 = smem_addr(sQ + g * kAtOpBytes), b0 = smem_addr(stage_k(st));
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) mma(tSt, op_desc_k(a0, kk), op_desc_k(b0, kk), kk > 0 ? 1u : 0u);
          mma_commit(&bars->s_done[g]);
          ++s_issued;
        } else {
          *abort_flag = 1;
        }
      }
      // 2. the scores (the previous O_g is complete too: the issuer waited for it)
      bool w_ok = bar_wait_or_abort(&bars->s_done[g], (uint32_t)(j & 1), abort_flag);
      if (named_bar_or(1 + g, 128, !w_ok)) { ok = false; break; }
      fence_after();
      // 3. online softmax of the thread's query row; P_g into tensor memory
      {
        const int valid = (int)(p.Nk - k0 < kAtTile ? p.Nk - k0 : kAtTile);
        // pass 1: the largest raw score, 16 columns at a time (fp32 rounding is
        // monotonic, so sl times it is the largest scaled score); the keys past
        // the end of the cache take no part
        float mt = -3.0e38f;
        auto pass1 = [&](auto full) {
#pragma unroll 1
          for (int c = 0; c < 8; ++c) {
            uint32_t rg[16];
            tld16(tSt + lane_base + (uint32_t)(16 * c), rg);
#pragma unroll
            for (int e = 0; e < 16; ++e)
              if (decltype(full)::value || 16 * c + e < valid) mt = fmaxf(mt, __uint_as_float(rg[e]));
          }
        };
        if (valid == kAtTile) pass1(std::true_type{}); else pass1(std::false_type{});
        // The weights are taken against a reference maximum m_run, raised only
        // when the row's maximum exceeds it by more than 8: the weights stay
        // below 2^8 (exact in bf16 and fp32 alike), and O and l are rescaled
        // rarely.  O / l is the same for any reference.
        const float m_row = fmaxf(m_run, mt * p.sl);
        const float m_new = m_row > m_run + 8.0f ? m_row : m_run;
        const float alpha = exp2_approx(m_run - m_new);
        // pass 2: bf16 weights 2^(sl s - m), two columns per packed op, and
        // their sum (of the rounded weights, the ones the product uses)
        const float2 sl2 = make_float2(p.sl, p.sl), nm2 = make_float2(-m_new, -m_new);
        float2 sum2 = make_float2(0.0f, 0.0f);
        auto pass2 = [&](auto full) {
#pragma unroll 1
          for (int c = 0; c < 8; ++c) {
            uint32_t rg[16];
            tld16(tSt + lane_base + (uint32_t)(16 * c), rg);
            uint32_t w[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const float2 x = __ffma2_rn(make_float2(__uint_as_float(rg[2 * e]), __uint_as_float(rg[2 * e + 1])), sl2, nm2);
              float pa = exp2_approx(x.x), pb = exp2_approx(x.y);
              if (!decltype(full)::value) {
                if (16 * c + 2 * e >= valid) pa = 0.0f;
                if (16 * c + 2 * e + 1 >= valid) pb = 0.0f;
              }
              w[e] = pack_bf16(pa, pb);
              sum2 = __fadd2_rn(sum2, make_float2(__uint_as_float(w[e] << 16), __uint_as_float(w[e] & 0xFFFF0000u)));
            }
            // keys 16c .. 16c+15 -> columns 8c .. 8c+7, already read
            tst8(tSt + lane_base + (uint32_t)(8 * c), w);
          }
        };
        if (valid == kAtTile) pass2(std::true_type{}); else pass2(std::false_type{});
        const float sum = sum2.x + sum2.y;
        l_run = l_run * alpha + sum;
        m_run = m_new;
        if (j > 0 && __any_sync(0xffffffffu, alpha != 1.0f)) {   // rescale O_g
#pragma unroll 1
          for (int c = 0; c < 8; ++c) {
            uint32_t rg[16];
            tld16(tOt + lane_base + (uint32_t)(16 * c), rg);
#pragma unroll
            for (int e = 0; e < 16; e += 2) {
              const float2 v = __fmul2_rn(make_float2(__uint_as_float(rg[e]), __uint_as_float(rg[e + 1])),
                                          make_float2(alpha, alpha));
              rg[e] = __float_as_uint(v.x);
              rg[e + 1] = __float_as_uint(v.y);
            }
            tst16(tOt + lane_base + (uint32_t)(16 * c), rg);
          }
        }
        asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
      }
      fence_before();
      named_bar_or(1 + g, 128, false);                 // P_g written, O_g rescaled
      // 4. O_g += P_g V; the stage is free once both query tiles' products complete
      if (issuer) {
        fence_after();
        const uint32_t b0 = smem_addr(stage_v(st));
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ta(tOt, tSt + (uint32_t)(8 * kk), op_desc_k(b0, kk), (j > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&bars->o_done[g]);
        if (p.pair > 1) mma_commit_mc(&bars->kv_empty[st], (uint16_t)((1u << rank) | (1u << (rank ^ 1))));
        else mma_commit(&bars->kv_empty[st]);
        ++o_issued;
      }
    }
    // the last product, then O / l
    if (ok && ntiles > 0) {
      const bool w_ok = bar_wait_or_abort(&bars->o_done[g], (uint32_t)((ntiles - 1) & 1), abort_flag);
      ok = !named_bar_or(1 + g, 128, !w_ok);
      fence_after();
    }
    if (!ok) *abort_flag = 1;
    m_fin = m_run;
    l_fin = l_run;
    if (ok && ntiles > 0 && p.split == 1) {
      // O / l, or (a range of a global split) the unnormalised O with the
      // row's maximum and sum
      const int64_t q = q0 + g * kAtTile + qi;
      const bool partial = p.gsplit > 1;
      const float inv = partial ? 1.0f : 1.0f / l_run;
      float* orow = partial ? p.part_O + (((int64_t)gs * p.H + h) * p.Nq + q) * kD : p.O + ((int64_t)h * p.Nq + q) * kD;
      if (partial && q < p.Nq) p.part_ml[((int64_t)gs * p.H + h) * p.Nq + q] = make_float2(m_run, l_run);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t rg[32];
        tld32(tOt + lane_base + (uint32_t)(32 * c), rg);
        if (q < p.Nq) {
          float4* dst = reinterpret_cast<float4*>(orow + 32 * c);
#pragma unroll
          for (int e = 0; e < 8; ++e)
            dst[e] = make_float4(__uint_as_float(rg[4 * e]) * inv, __uint_as_float(rg[4 * e + 1]) * inv,
                                 __uint_as_float(rg[4 * e + 2]) * inv, __uint_as_float(rg[4 * e + 3]) * inv);
        }
      }
    }
  }
  fence_before();
  __syncthreads();
  if (*abort_flag && (threadIdx.x == 0 || threadIdx.x == 128)) {
    const int g = threadIdx.x >> 7;
    if (g == 0) atomicOr(p.status, 1u);
    // let the products this thread issued finish (bounded) before the tensor
    // memory is freed; a phase that already completed returns at once
    if (s_issued > 0) bar_wait(&bars->s_done[g], (uint32_t)((s_issued - 1) & 1));
    if (o_issued > 0) bar_wait(&bars->o_done[g], (uint32_t)((o_issued - 1) & 1));
  }
  __syncthreads();
  if (p.split > 1) {
    // The products are complete and the query and ring buffers free: leave
    // this CTA's unnormalised O rows there (row R = query q0 + R, channel
    // chunk c of 4 at chunk c ^ (R mod 8), so that a warp's stores hit
    // distinct banks) with the rows' maximum and sum after them.
    float* sX = reinterpret_cast<float*>(smem);
    float2* sML = reinterpret_cast<float2*>(smem + kAtQTiles * kAtTile * kD * sizeof(float));
    if (warp < 8) {
      const int R = threadIdx.x;
      const uint32_t tOt = tO + 128 * (warp >> 2), lane_base = (uint32_t)(32 * (warp & 3)) << 16;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t rg[32];
        tld32(tOt + lane_base + (uint32_t)(32 * c), rg);
#pragma unroll
        for (int e = 0; e < 8; ++e)
          *reinterpret_cast<float4*>(sX + R * kD + 4 * ((8 * c + e) ^ (R & 7))) =
              make_float4(__uint_as_float(rg[4 * e]), __uint_as_float(rg[4 * e + 1]),
                          __uint_as_float(rg[4 * e + 2]), __uint_as_float(rg[4 * e + 3]));
      }
      sML[R] = make_float2(m_fin, l_fin);
    }
    fence_before();
    cluster_sync();
    // Split rank sr merges rows [R0, R1) of its query block from the CTAs
    // that hold the block (cluster ranks m * pair + pr): O = sum_s 2^(m_s - M)
    // O_s / sum_s 2^(m_s - M) l_s, M = max_s m_s (a CTA with no tiles has
    // l = 0 and takes no part); a warp per row, a lane per chunk of four
    // channels.
    const int R0 = kAtQTiles * kAtTile * sr / p.split, R1 = kAtQTiles * kAtTile * (sr + 1) / p.split;
    for (int t = threadIdx.x; t < (R1 - R0) * 32; t += kAtThreads) {
      const int R = R0 + (t >> 5), c = t & 31;
      const uint32_t ml_a = smem_addr(sML + R), x_a = smem_addr(sX + R * kD + 4 * (c ^ (R & 7)));
      float M = -3.0e38f;
      for (int m = 0; m < p.split; ++m) {
        const float2 ml = ld_cluster_f2(cluster_addr(ml_a, (uint32_t)(m * p.pair + pr)));
        if (ml.y > 0.0f) M = fmaxf(M, ml.x);
      }
      float L = 0.0f;
      float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
      for (int m = 0; m < p.split; ++m) {
        const uint32_t src = (uint32_t)(m * p.pair + pr);
        const float2 ml = ld_cluster_f2(cluster_addr(ml_a, src));
        const float w = ml.y > 0.0f ? exp2_approx(ml.x - M) : 0.0f;
        if (w > 0.0f) {
          const float4 x = ld_cluster_f4(cluster_addr(x_a, src));
          acc.x += w * x.x; acc.y += w * x.y; acc.z += w * x.z; acc.w += w * x.w;
          L += w * ml.y;
        }
      }
      const int64_t q = q0 + R;
      if (q < p.Nq && !*abort_flag) {
        const float inv = 1.0f / L;
        *reinterpret_cast<float4*>(p.O + ((int64_t)h * p.Nq + q) * kD + 4 * c) =
            make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
      }
    }
  }
  // no CTA leaves while another still reads or writes its shared memory
  if (csize > 1) cluster_sync();
  if (warp == 0) {
    fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem));
  }
}

// The ranges of a global split merged, a warp per query row (a lane per four
// channels): O = sum_s 2^(m_s - M) O_s / sum_s 2^(m_s - M) l_s, M = max_s m_s,
// the rescaling of the cluster merge.
__global__ void __launch_bounds__(256)
qvg_attention_merge(const float* part_O, const float2* part_ml, float* O, int64_t rows, int S) {
  const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  float M = -3.0e38f;
  for (int s = 0; s < S; ++s) {
    const float2 ml = __ldg(part_ml + s * rows + row);
    if (ml.y > 0.0f) M = fmaxf(M, ml.x);
  }
  float L = 0.0f;
  float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
  for (int s = 0; s < S; ++s) {
    const float2 ml = __ldg(part_ml + s * rows + row);
    const float w = ml.y > 0.0f ? exp2_approx(ml.x - M) : 0.0f;
    if (w > 0.0f) {
      const float4 x = __ldg(reinterpret_cast<const float4*>(part_O + (s * rows + row) * kD) + lane);
      acc.x += w * x.x; acc.y += w * x.y; acc.z += w * x.z; acc.w += w * x.w;
      L += w * ml.y;
    }
  }
  const float inv = 1.0f / L;
  reinterpret_cast<float4*>(O + row * kD)[lane] = make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
}

// The (cos, sin) table of the rotary angles, formed in fp64 and rounded to
// fp32: rope[p][i] for the angle p theta_i, theta_i = base^(-2i/d).
__global__ void qvg_rope_tables_kernel(float2* rope, int64_t rows, double base) {
  const int i = threadIdx.x % (kD / 2);
  const int64_t row = (int64_t)blockIdx.x * (blockDim.x / (kD / 2)) + threadIdx.x / (kD / 2);
  if (row >= rows) return;
  const double theta = pow(base, -2.0 * i / (double)kD);
  double sn, cs;
  sincos((double)row * theta, &sn, &cs);
  rope[row * (kD / 2) + i] = make_float2(__double2float_rn(cs), __double2float_rn(sn));
}

}  // namespace

size_t attention_smem_bytes() {
  return 1024 + (size_t)(kAtQTiles + 4) * kAtOpBytes + 32 * sizeof(float2) + sizeof(AtBars);
}

cudaError_t launch_rope_tables(void* tables, int64_t max_pos, double base, cudaStream_t s) {
  float2* rope = reinterpret_cast<float2*>(static_cast<char*>(tables) + kRopeHeaderBytes);
  const int64_t rows = max_pos + 1;
  const int per = 256 / (kD / 2);
  qvg_rope_tables_kernel<<<(unsigned)((rows + per - 1) / per), 256, 0, s>>>(rope, rows, base);
  return cudaGetLastError();
}

template <int TT>
static cudaError_t launch_attention_t(const AttnParams& p, dim3 grid, size_t smem, cudaStream_t s) {
  cudaError_t e = ensure_dynamic_smem(reinterpret_cast<const void*>(qvg_attention_fused<TT>), smem);
  if (e != cudaSuccess) return e;
  if (p.split * p.pair == 1) {
    qvg_attention_fused<TT><<<grid, kAtThreads, smem, s>>>(p);
    return cudaGetLastError();
  }
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(kAtThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)(p.split * p.pair);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, qvg_attention_fused<TT>, p);
}

// Clusters of `split` attention CTAs that fit on the device at once (CTAs
// per SM times SMs for split = 1); 0 if none fits.  Cached per device,
// kernel instance and split.
template <int TT>
static int resident_clusters(int split) {
  static std::atomic<int> cache[kMaxDevices][kAtMaxSplit + 1];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 0;
  const int known = cache[dev][split].load(std::memory_order_relaxed);
  if (known > 0) return known - 1;
  const size_t smem = attention_smem_bytes();
  if (ensure_dynamic_smem(reinterpret_cast<const void*>(qvg_attention_fused<TT>), smem) != cudaSuccess) return 0;
  int n = 0;
  if (split == 1) {
    int per_sm = 0, sms = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, qvg_attention_fused<TT>, kAtThreads, smem) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return 0;
    n = per_sm * sms;
  } else {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)split, 1, 1);
    cfg.blockDim = dim3(kAtThreads);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)split;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaOccupancyMaxActiveClusters(&n, qvg_attention_fused<TT>, &cfg) != cudaSuccess) {
      (void)cudaGetLastError();
      n = 0;
    }
  }
  cache[dev][split].store(n + 1, std::memory_order_relaxed);
  return n;
}

// Bytes of the partial results of a global split into S ranges.
static size_t partial_bytes(int S, int H, int64_t Nq) {
  return (size_t)S * H * Nq * (kD * sizeof(float) + sizeof(float2));
}

// The launch shape.  pair = 2 when there are at least two blocks of 256
// queries (two CTAs share every tile's reconstruction).  The cache of a
// query block is cut into ranges either inside the cluster (split 1 .. 4,
// cluster size pair x split at most 8, merged through distributed shared
// memory) or, when the workspace holds the partial results, over clusters
// (gsplit 2 .. 16, merged by a second kernel).  The plan with the least
// estimated time wins: (waves of resident clusters) x (tiles per CTA + the
// fixed cost of a CTA, about two tiles), plus one tile for a merge kernel.
// A positive `forced` split is a cluster split, taken as it is.  Never more
// ranges than the cache has tiles.
struct SplitPlan { int pair, split, gsplit; };
template <int TT>
static SplitPlan choose_split(int64_t Nk, int64_t Nq, int H, int forced, size_t ws_bytes) {
  const int64_t ntot = (Nk + kAtTile - 1) / kAtTile;
  const int64_t qblocks = (Nq + kAtQTiles * kAtTile - 1) / (kAtQTiles * kAtTile);
  const int pair = qblocks >= 2 ? 2 : 1;
  const int cap = kAtMaxSplit / pair;
  const int smax = (int)(ntot < cap ? ntot : cap);
  if (forced > 0) return SplitPlan{pair, forced < smax ? forced : smax, 1};
  const int64_t units = (qblocks + pair - 1) / pair * H;
  SplitPlan best{pair, 1, 1};
  double best_cost = -1.0;
  for (int sp = 1; sp <= (smax < 4 ? smax : 4); ++sp) {
    const int n = resident_clusters<TT>(pair * sp);
    if (n <= 0) continue;
    const double cost = (double)((units + n - 1) / n) * (double)((ntot + sp - 1) / sp + 2);
    if (best_cost < 0.0 || cost < best_cost) { best = SplitPlan{pair, sp, 1}; best_cost = cost; }
  }
  const int n = resident_clusters<TT>(pair);
  const int gmax = (int)(ntot < kAtMaxGlobalSplit ? ntot : kAtMaxGlobalSplit);
  for (int gs = 2; n > 0 && gs <= gmax; ++gs) {
    if (partial_bytes(gs, H, Nq) > ws_bytes) break;
    const double cost = (double)((units * gs + n - 1) / n) * (double)((ntot + gs - 1) / gs + 2) + 1.0;
    if (best_cost < 0.0 || cost < best_cost) { best = SplitPlan{pair, 1, gs}; best_cost = cost; }
  }
  return best;
}

template <int TT>
static cudaError_t launch_attention_plan(AttnParams& p, int64_t Nq, size_t smem, int forced, size_t ws_bytes,
                                         cudaStream_t s) {
  const SplitPlan plan = choose_split<TT>(p.Nk, Nq, p.H, forced, ws_bytes);
  p.split = plan.split;
  p.pair = plan.pair;
  p.gsplit = plan.gsplit;
  // the partial results of a global split: O rows, then (maximum, sum) pairs
  if (plan.gsplit > 1) p.part_ml = reinterpret_cast<float2*>(p.part_O + (size_t)plan.gsplit * p.H * Nq * kD);
  const int64_t qblocks = (Nq + kAtQTiles * kAtTile - 1) / (kAtQTiles * kAtTile);
  const int64_t units = (qblocks + plan.pair - 1) / plan.pair;
  const dim3 grid((unsigned)(units * plan.gsplit * plan.pair * plan.split), (unsigned)p.H);
  cudaError_t e = launch_attention_t<TT>(p, grid, smem, s);
  if (e != cudaSuccess || plan.gsplit == 1) return e;
  const int64_t rows = (int64_t)p.H * Nq;
  qvg_attention_merge<<<(unsigned)((rows + 7) / 8), 256, 0, s>>>(p.part_O, p.part_ml, p.O, rows, plan.gsplit);
  return cudaGetLastError();
}

template <int TT>
static SplitPlan plan_for(int64_t Nk, int64_t Nq, int H, int forced, size_t ws_bytes) {
  return choose_split<TT>(Nk, Nq, H, forced, ws_bytes);
}
static SplitPlan plan_any(int T, int64_t Nk, int64_t Nq, int H, int forced, size_t ws_bytes) {
  switch (T) {
    case 0: return plan_for<0>(Nk, Nq, H, forced, ws_bytes);
    case 1: return plan_for<1>(Nk, Nq, H, forced, ws_bytes);
    case 2: return plan_for<2>(Nk, Nq, H, forced, ws_bytes);
    case 3: return plan_for<3>(Nk, Nq, H, forced, ws_bytes);
    case 4: return plan_for<4>(Nk, Nq, H, forced, ws_bytes);
    default: return plan_for<-1>(Nk, Nq, H, forced, ws_bytes);
  }
}

int attention_split(int T, int64_t Nk, int64_t Nq, int H, int forced, size_t ws_bytes) {
  const SplitPlan plan = plan_any(T, Nk, Nq, H, forced, ws_bytes);
  return plan.split * plan.gsplit;
}

size_t attention_workspace_bytes(int T, int64_t Nk, int64_t Nq, int H, int forced) {
  const SplitPlan plan = plan_any(T, Nk, Nq, H, forced, ~size_t(0));
  return plan.gsplit > 1 ? partial_bytes(plan.gsplit, H, Nq) : 0;
}

cudaError_t launch_attention(const AttentionArgs& a, cudaStream_t s) {
  AttnParams p{};
  for (int w = 0; w < 2; ++w) {
    const qvg_packed* pk = w == 0 ? a.k : a.v;
    p.codes[w] = pk->codes; p.scale[w] = pk->scale; p.zero[w] = pk->zero; p.assign[w] = pk->assign;
    p.tab[w] = static_cast<const __nv_bfloat16*>(pk->centroids);
  }
  p.Q = static_cast<const __nv_bfloat16*>(a.Q);
  p.qpos = a.qpos;
  p.rope = reinterpret_cast<const float2*>(static_cast<const char*>(a.tables) + kRopeHeaderBytes);
  p.O = a.O;
  p.status = reinterpret_cast<uint32_t*>(const_cast<void*>(a.tables));
  p.max_pos = a.max_pos;
  p.Nk = a.Nk; p.Nq = a.Nq; p.H = a.H; p.K = a.K; p.T = a.T; p.G = a.G; p.sym = a.sym;
  p.sl = 1.4426950408889634f / sqrtf((float)kD);
  const size_t ws = a.workspace != nullptr ? a.ws_bytes : 0;
  p.part_O = static_cast<float*>(a.workspace);
  const size_t smem = attention_smem_bytes();
  switch (a.T) {
    case 0: return launch_attention_plan<0>(p, a.Nq, smem, a.split, ws, s);
    case 1: return launch_attention_plan<1>(p, a.Nq, smem, a.split, ws, s);
    case 2: return launch_attention_plan<2>(p, a.Nq, smem, a.split, ws, s);
    case 3: return launch_attention_plan<3>(p, a.Nq, smem, a.split, ws, s);
    case 4: return launch_attention_plan<4>(p, a.Nq, smem, a.split, ws, s);
    default: return launch_attention_plan<-1>(p, a.Nq, smem, a.split, ws, s);
  }
}

}  // namespace qvg
