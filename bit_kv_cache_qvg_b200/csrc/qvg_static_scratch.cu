// qvg_static_scratch.cu -- qvg_quantize_static: the compression call of
// qvg_quantize, run on a scratch area that the library reserves once per
// device in a static __device__ array, so that the call allocates nothing.
//
// Who needs it: a caller that must not touch the CUDA allocator while it
// runs, and has no workspace of its own to lend.  A cudaMalloc or cudaFree
// can synchronise the whole device, stalling every stream of the process.
// It can fail under memory pressure in the middle of a generation.  And a
// caching allocator elsewhere in the process may already hold the free
// memory that a raw allocation would need.  Such a caller (for example a
// per-chunk hook of a decoding loop) can call this entry with device
// buffers it already owns for the input and the outputs, and nothing else.
//
// The reserve is kStaticScratchBytes (32 MiB) of global memory.  It holds
// the k-means working set of as many blocks per wave as fit, and at least
// one: about 120,000 tokens per block at bf16, K = 256, T = 2.  A call whose
// single block needs more is rejected before any work is queued.
//
// Its first 16 bytes are the workspace status word and near-tie counter.  A
// __device__ array starts zeroed when the module loads, and no kernel needs
// those bytes to be zero (the status word is only ever set, the counter only
// ever added to), so a call queues no clearing of its own: a timeout that a
// bounded device-side wait records stays in the word until
// qvg_static_status reads and clears it.
#include <cuda_runtime.h>

#include <cstdint>

#include "qvg.h"
#include "qvg_launch.h"

namespace {

constexpr size_t kStaticScratchBytes = size_t(32) << 20;

// One reserve per device (a __device__ variable has one instance per device
// on which the library's device code is loaded).  256-byte alignment is the
// alignment qvg_quantize requires of a workspace.
__device__ __align__(256) unsigned char g_qvg_static_scratch[kStaticScratchBytes];

// Device address of the reserve on the current device.  It is looked up on
// every call (cheap once the module is loaded; the first lookup may load this
// file's device code), so that it stays right after a context teardown
// reloads the module at another address.
qvg_status scratch_on_current_device(void** out) {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_qvg_static_scratch) != cudaSuccess || p == nullptr) {
    cudaGetLastError();       // leave no error pending for a later launch check
    return QVG_ERR_CUDA;
  }
  *out = p;
  return QVG_OK;
}

}  // namespace

extern "C" QVG_API qvg_status qvg_quantize_static(const qvg_config* cfg, const void* X, qvg_dtype dtype,
                                                  int64_t N, int32_t H, int32_t d,
                                                  const void* init_centroids, const qvg_packed* out,
                                                  qvg_stream_t stream) {
  // One block's working set must fit in the reserve.  A zero size means the
  // arguments are invalid: qvg::quantize_impl then reports which, before it
  // queues anything.
  const size_t one_block = qvg_workspace_bytes(cfg, N, 1, d, dtype);
  if (one_block > kStaticScratchBytes) return QVG_ERR_WORKSPACE_TOO_SMALL;
  void* scratch = nullptr;
  const qvg_status st = scratch_on_current_device(&scratch);
  if (st != QVG_OK) return st;
  // The same checks and kernels as qvg_quantize, one wave at a time on the
  // caller's stream (no side stream, no events); a timeout recorded in the
  // reserve by earlier, completed work is returned before anything is queued.
  return qvg::quantize_impl(cfg, X, dtype, N, H, d, init_centroids, out, scratch, kStaticScratchBytes, stream, 1,
                           -1);
}

extern "C" QVG_API qvg_status qvg_static_status(qvg_stream_t stream) {
  void* scratch = nullptr;
  const qvg_status st = scratch_on_current_device(&scratch);
  if (st != QVG_OK) return st;
  return qvg::take_sticky(scratch, reinterpret_cast<cudaStream_t>(stream));
}
