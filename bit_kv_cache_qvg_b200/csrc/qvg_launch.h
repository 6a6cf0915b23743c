// qvg_launch.h -- host-side launchers of the sm_100a kernels (internal to
// libqvg.so; the public surface is include/qvg.h).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "qvg.h"
#include "qvg_common.cuh"

namespace qvg {

// ---- launch helpers (qvg_api.cu)
// qvg_quantize with at most `max_lanes` waves of blocks in flight at once
// (1: every wave on the caller's stream, with no side stream and no events)
// and the first `warm_stages` stages started from init (-1: every stage when
// init is given, none otherwise).
qvg_status quantize_impl(const qvg_config* cfg, const void* X, qvg_dtype dtype, int64_t N, int32_t H,
                         int32_t d, const void* init, const qvg_packed* out, void* workspace,
                         size_t ws_bytes, qvg_stream_t stream, int max_lanes, int warm_stages);
// SM count of the current device (cached per device).
int device_sm_count();
// Host-side fault injection for tests: true when the comma-separated list in
// the environment variable QVG_FAULT_INJECT names `what` ("alloc", "stream",
// "timeout").  Read on every call; unset in normal use.
bool fault_injected(const char* what);
// The sticky status word of a workspace, cache or static reserve (its first
// four bytes): peek_sticky reads it without waiting (QVG_OK while work queued
// on `s` is still running or `s` is being captured); take_sticky waits for
// `s`, reads it and clears it.
qvg_status peek_sticky(const void* word, cudaStream_t s);
qvg_status take_sticky(void* word, cudaStream_t s);
// Raise a kernel's dynamic shared-memory limit to at least `bytes` (the
// attribute call is made once per kernel and size; later calls are cached).
cudaError_t ensure_dynamic_smem(const void* kernel, size_t bytes);

// ---- codec kernels (kernels_codec.cu)

// Fused reconstruction of a set of (chunk, head) blocks.
cudaError_t launch_dequant(const DequantParams& p, int dtype, cudaStream_t s);

// Residual pass over W units of N tokens:
//   r = round_S(R_in - C[pi])   (or r = R_in when C == nullptr)
// then either
//   quant == false: R_out = r (if R_out != nullptr) and rnorm2 = |r|^2 (fp32)
//   quant == true : 2-bit group quantisation of r into codes/scale/zero.
struct ResidualParams {
  const void* R_in;        // [W][N][d] storage dtype
  const void* C;           // [W][K][d] or nullptr
  const uint8_t* pi;       // [W][N]
  void* R_out;             // [W][N][d] or nullptr
  float* rnorm2;           // [W][N] or nullptr
  uint32_t* chmax;         // [W][d] or nullptr: atomic max of the bits of |value| per channel
                           // of the values read (no C) or written (with C); starts at zero
  uint32_t* chmin;         // [W][d], used with chmax: atomic max of 0x7FFFFFFF minus the bits of
                           // the smallest nonzero |value| per channel (0: none); starts at zero
  uint8_t* codes;          // [W][N][d/4]
  uint8_t* scale;          // [W][N][d/G]
  uint8_t* zero;           // [W][N][d/G] (unused when sym)
  int64_t N;
  int W;
  int K;
  int G;
  int sym;                 // 1: one E4M3 scale per group (symmetric signed INT2)
};
cudaError_t launch_residual(const ResidualParams& p, int dtype, bool quant, cudaStream_t s);

// *out += the sum over `rows` token rows of X of the E4M3 codes of the fp32
// ranges (max - min) of their groups of G channels (*out must start at zero).
cudaError_t launch_range_stat(const void* X, int64_t rows, int G, int dtype, unsigned long long* out,
                              cudaStream_t s);

// C[u] = rows of src[u] (first K rows of a stage input, or given tables);
// cn[u][k] = |c_k|^2 rounded to fp32 from an fp64 sum.
cudaError_t launch_init_centroids(const void* src, int64_t src_unit_stride, void* C,
                                  float* cn, int W, int K, int dtype, cudaStream_t s);

// ---- k-means kernels (kernels_kmeans.cu)

struct AssignParams {
  const void* R;               // [W][N][d]
  const float* rnorm2;         // [W][N]
  const void* C;               // [W][K][d]
  const float* cn;             // [W][K]
  uint8_t* pi;                 // [W][N]
  const uint32_t* list;        // [W][N] rows to (re)assign, or nullptr = every row
  const uint32_t* list_count;  // [W]
  int64_t N;
  int W;
  int K;
};
// Exact assignment: fp32 screening distances, exact fp64 distances for every
// centroid within the screening error bound, lowest index on exact ties.
cudaError_t launch_assign_exact(const AssignParams& p, int dtype, cudaStream_t s);

// Tensor-core assignment (kernel_assign_tc.cu): tcgen05 screening GEMM with a
// top-2 epilogue; tokens whose runner-up is within the error bound are listed
// for the exact pass (launch_assign_exact in list mode).  bf16 only.
struct AssignTcParams {
  const void* R;               // [W][N][d] bf16
  const float* rnorm2;         // [W][N]
  const void* C;               // [W][K][d] bf16
  const float* cn;             // [W][K]
  uint8_t* pi;                 // [W][N]
  uint2* list;                 // [W][N] listed tokens: {token, mask of candidate 8-centroid groups}
  uint32_t* list_count;        // [W], zero on entry
  uint32_t* status;            // workspace status word
  unsigned long long* flagged; // running total of listed tokens
  int64_t N;
  int W;
  int K;
  float gamma;
  int hook_withhold;           // test hook (QVG_FAULT_INJECT=timeout): tile the hooked CTA never loads, or -1
  uint64_t hook_wait_ns;       // test hook: wait limit of the hooked CTA, or 0 (hook off)
};
cudaError_t launch_assign_tc(const AssignTcParams& p, cudaStream_t s);
// Exact decision of the listed tokens: sequential fp64 squared distances to
// every centroid of the listed 8-centroid groups (all groups when the mask is
// empty), the least one wins, ties to the lowest index.
cudaError_t launch_assign_candidates(const void* R, const void* C, int K, int64_t N, int W,
                                     const uint2* list, const uint32_t* list_count, uint8_t* pi,
                                     cudaStream_t s);
size_t assign_tc_smem_bytes(int K);

struct UpdateParams {
  const void* R;          // [W][N][d] stage input
  const uint8_t* pi;      // [W][N] assignment of this iteration
  const uint8_t* pi_old;  // [W][N] assignment of the previous iteration, or nullptr (full sums)
  const uint32_t* chmax;  // [W][d] bits of the largest |value| of each channel of R
  const uint32_t* chmin;  // [W][d] 0x7FFFFFFF minus the bits of the smallest nonzero |value| (0: none)
  uint32_t* list;         // [W][2N] scratch: entries bucketed by centroid
  int* off;               // [W][K+1] scratch: bucket offsets
  int* cnt;               // [W][K]   scratch: member counts (first iteration) or their changes
  long long* S;           // [W][K][d] running member sums in fixed point (units of 2^L_c); channel c at (c % 8) * 16 + c / 8
  int* n;                 // [W][K]    member counts
  void* C;                // [W][K][d] centroids (updated in place)
  float* cn;              // [W][K]    squared centroid norms
  int64_t N;
  int W;
  int K;
  int log2n;              // smallest k with 2^k > N
  int stage_pi;           // (set by the bucket launcher) assignments staged in shared memory
};
// Exact fixed-point centroid sums: with pi_old == nullptr every token adds its
// row to its centroid; otherwise a token whose centroid changed adds its row
// to the new centroid and subtracts it from the old one.  Then every changed,
// non-empty centroid = round(S / n) in the storage dtype, and its |c|^2.
// Three launches: bucket the entries by centroid, sum them, recompute centroids.
cudaError_t launch_update_bucket(const UpdateParams& p, int dtype, cudaStream_t s);
cudaError_t launch_update_sum(const UpdateParams& p, int dtype, cudaStream_t s);
cudaError_t launch_update_centroids(const UpdateParams& p, int dtype, cudaStream_t s);

// ---- attention over the compressed cache (kernel_attention.cu)
// Rotary tables: a 256-byte header (its first 4 bytes are the status word
// of the attention calls that use the tables), then (cos, sin) in fp32 of
// p theta_i for every position p = 0 .. max_pos and pair i < d/2.
constexpr size_t kRopeHeaderBytes = 256;
constexpr size_t kRopeRowBytes = (kD / 2) * 2 * sizeof(float);
constexpr int64_t kRopeMaxPositions = int64_t(1) << 24;
cudaError_t launch_rope_tables(void* tables, int64_t max_pos, double base, cudaStream_t s);
struct AttentionArgs {
  const qvg_packed* k;         // K cache: H blocks of Nk tokens (bf16 tables)
  const qvg_packed* v;         // V cache, same configuration
  const void* Q;               // [H][Nq][d] bf16, before the rotary embedding
  const int64_t* qpos;         // [Nq]
  const void* tables;          // rotary tables (header + hi + lo)
  int64_t max_pos;             // largest position the tables cover
  float* O;                    // [H][Nq][d] fp32
  int64_t Nk, Nq;
  int H, K, T, G, sym;
  int split;                   // CTAs per cluster over the cache of a query block; 0 = chosen here
  void* workspace;             // partial results of a split over clusters (may be null)
  size_t ws_bytes;
};
cudaError_t launch_attention(const AttentionArgs& a, cudaStream_t s);
// The ranges the cache of a query block is cut into for these sizes and this
// workspace (forced > 0: a cluster split of that many CTAs, capped at the
// cache's tile count and the cluster limit).
int attention_split(int T, int64_t Nk, int64_t Nq, int H, int forced, size_t ws_bytes);
// The workspace the preferred plan needs (0: none).
size_t attention_workspace_bytes(int T, int64_t Nk, int64_t Nq, int H, int forced);
size_t attention_smem_bytes();

}  // namespace qvg
