// qvg_api.cu -- host side of libqvg.so: argument checks, workspace planning,
// the progressive-residual stage loop, and the streaming cache.  Every
// arithmetic step of the codec runs in the kernels; this file only
// schedules them (m.163.com article on Quant VideoGen, sections 三-五;
// gist.science/de, Technische Zusammenfassung 2A-2C).
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdio>
#include <mutex>
#include <string>
#include <vector>
#include <cstdlib>
#include <cstring>
#include <cstdint>

#include "qvg.h"
#include "qvg_launch.h"

using namespace qvg;

namespace qvg {

int device_sm_count() {
  static int cached[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) dev = 0;
  if (cached[dev] == 0) {
    int n = 148;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    cached[dev] = n;
  }
  return cached[dev];
}

bool fault_injected(const char* what) {
  const char* env = std::getenv("QVG_FAULT_INJECT");
  if (env == nullptr || *env == '\0') return false;
  const size_t n = std::strlen(what);
  for (const char* p = env; *p;) {
    const char* e = std::strchr(p, ',');
    const size_t len = e ? (size_t)(e - p) : std::strlen(p);
    if (len == n && std::strncmp(p, what, n) == 0) return true;
    if (e == nullptr) break;
    p = e + 1;
  }
  return false;
}

cudaError_t ensure_dynamic_smem(const void* kernel, size_t bytes) {
  if (bytes <= 48 * 1024) return cudaSuccess;
  // the attribute is per device: remember (kernel, device) pairs
  struct Done { const void* kernel; int dev; size_t bytes; };
  static std::mutex mu;
  static std::vector<Done> done;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> g(mu);
  for (auto& d : done)
    if (d.kernel == kernel && d.dev == dev && d.bytes >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e == cudaSuccess) done.push_back(Done{kernel, dev, bytes});
  return e;
}

// The sticky status word at `word` (device memory: the first 4 bytes of a
// workspace, of a cache's workspace or of the static reserve), read without
// waiting for the GPU: only when every operation queued on `s` has completed
// and `s` is not being captured into a graph.  While earlier work is still in
// flight its outcome is not known yet and the result is QVG_OK; a later call,
// or the status query of the object, reports it.
qvg_status peek_sticky(const void* word, cudaStream_t s) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(s, &cs) != cudaSuccess) { cudaGetLastError(); return QVG_OK; }
  if (cs != cudaStreamCaptureStatusNone) return QVG_OK;
  const cudaError_t q = cudaStreamQuery(s);
  if (q == cudaErrorNotReady) return QVG_OK;
  if (q != cudaSuccess) return QVG_ERR_CUDA;
  uint32_t w = 0;
  if (cudaMemcpyAsync(&w, word, sizeof(w), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return QVG_ERR_CUDA;
  return w == 0 ? QVG_OK : QVG_ERR_DEVICE_TIMEOUT;
}

// Read and clear a sticky status word after the work queued on `s` has
// completed (synchronises `s`).
qvg_status take_sticky(void* word, cudaStream_t s) {
  uint32_t w = 0;
  if (cudaMemcpyAsync(&w, word, sizeof(w), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess || cudaMemsetAsync(word, 0, sizeof(w), s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return QVG_ERR_CUDA;
  return w == 0 ? QVG_OK : QVG_ERR_DEVICE_TIMEOUT;
}

}  // namespace qvg

namespace {

constexpr size_t kAlign = 256;
inline size_t align_up(size_t x) { return (x + kAlign - 1) & ~(kAlign - 1); }

int esize(int dtype) { return dtype == kFP32 ? 4 : 2; }
bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Layout of the caller's workspace for a batch of W units.
struct Plan {
  int W = 0;
  int nR = 0;
  size_t off_R[2] = {0, 0};
  size_t off_rnorm = 0, off_cn = 0, off_list = 0, off_listcnt = 0;
  size_t off_chmax = 0, off_off = 0, off_cnt = 0, off_S = 0, off_n = 0, off_pi = 0;
  size_t off_status = 0, total = 0;
};

Plan make_plan(const qvg_config& c, int64_t N, int W, int dtype) {
  Plan p;
  p.W = W;
  p.nR = c.T >= 3 ? 2 : (c.T == 2 ? 1 : 0);
  const size_t esz = (size_t)esize(dtype);
  size_t o = 0;
  p.off_status = o;                       o = align_up(o + 16);
  for (int b = 0; b < p.nR; ++b) { p.off_R[b] = o; o = align_up(o + (size_t)W * N * kD * esz); }
  p.off_rnorm = o;                        o = align_up(o + (size_t)W * N * sizeof(float));
  p.off_cn = o;                           o = align_up(o + (size_t)W * kMaxK * sizeof(float));
  p.off_list = o;                         o = align_up(o + (size_t)W * N * 8);
  p.off_listcnt = o;                      o = align_up(o + (size_t)W * sizeof(uint32_t));
  p.off_chmax = o;                        o = align_up(o + 2 * (size_t)W * kD * sizeof(uint32_t));  // max, then min
  p.off_off = o;                          o = align_up(o + (size_t)W * (c.K + 1) * sizeof(int));
  p.off_cnt = o;                          o = align_up(o + (size_t)W * c.K * sizeof(int));
  p.off_S = o;                            o = align_up(o + (size_t)W * c.K * kD * sizeof(long long));
  p.off_n = o;                            o = align_up(o + (size_t)W * c.K * sizeof(int));
  p.off_pi = o;                           o = align_up(o + (size_t)W * N);
  p.total = o;
  return p;
}

int preferred_batch(const qvg_config& c, int64_t N, int H, int dtype) {
  if (const char* env = std::getenv("QVG_BATCH_UNITS")) {
    const int w = std::atoi(env);
    if (w > 0) return std::min(w, H);
  }
  // As many blocks per launch as a 2 GiB workspace holds, at most one per SM:
  // the tensor-core assignment runs one CTA per block, so a wave of exactly
  // one block per SM keeps every SM busy; other kernels split blocks further.
  const double budget = 2.0 * 1024.0 * 1024.0 * 1024.0;
  const double per_unit = (double)make_plan(c, N, 1, dtype).total;
  int w = (int)std::floor(budget / per_unit);
  return std::max(1, std::min(std::min(w, qvg::device_sm_count()), H));
}

// Waves of blocks are independent, so consecutive waves run on two streams
// ("lanes"), each with its own workspace: the latency-bound update kernels of
// one wave then overlap the other wave's tensor-core assignment.
// QVG_WAVE_LANES=1 keeps every wave on the caller's stream.
int wave_lanes(int H, int W) {
  if (H <= W) return 1;
  if (const char* env = std::getenv("QVG_WAVE_LANES")) {
    if (std::atoi(env) == 1) return 1;
  }
  return 2;
}

// The second lane's stream, one per device, created on first use.
cudaStream_t side_stream() {
  static std::mutex mu;
  static cudaStream_t streams[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) dev = 0;
  std::lock_guard<std::mutex> g(mu);
  if (streams[dev] == nullptr && cudaStreamCreateWithFlags(&streams[dev], cudaStreamNonBlocking) != cudaSuccess) {
    cudaGetLastError();
    streams[dev] = nullptr;
  }
  return streams[dev];
}

// Relative error bound assumed for the tensor-core sums (128 exact bf16 x bf16
// products plus three bf16 pieces of -|c|^2/2, accumulated in fp32 over nine
// MMA steps): 2^-16, about 7x a bound of two fp32 ulps per step.
constexpr float kTcGamma = 1.52587890625e-05f;

// QVG_ASSIGN_PATH=exact routes bf16 blocks through the CUDA-core exact
// assignment as well (diagnostics; the results are identical).
bool assign_path_tc() {
  const char* e = std::getenv("QVG_ASSIGN_PATH");
  return !(e != nullptr && std::strcmp(e, "exact") == 0);
}

bool g_supported(int G) { return G == 8 || G == 16 || G == 32 || G == 64 || G == 128; }

qvg_status check_config(const qvg_config* c, int64_t N, int32_t H, int32_t d, qvg_dtype dtype) {
  if (c == nullptr) return QVG_ERR_INVALID_ARG;
  if (dtype != QVG_BF16 && dtype != QVG_FP32) return QVG_ERR_INVALID_ARG;
  if (c->bits != 2 || c->K < 1 || c->K > 256 || c->T < 0) return QVG_ERR_INVALID_ARG;
  if (c->scale_mode != QVG_SCALE_ASYM && c->scale_mode != QVG_SCALE_SYM) return QVG_ERR_INVALID_ARG;
  if (c->group_size < 4 || c->group_size % 4 != 0 || d < 4 || d % c->group_size != 0)
    return QVG_ERR_INVALID_ARG;
  if (N < 0 || H < 1) return QVG_ERR_INVALID_ARG;
  if (N >= (int64_t(1) << 23)) return QVG_ERR_UNSUPPORTED;   // token indices are 23-bit in the update
  if (d != kD || !g_supported(c->group_size) || c->T > kMaxT) return QVG_ERR_UNSUPPORTED;
  return QVG_OK;
}

qvg_status cuda_status(cudaError_t e) { return e == cudaSuccess ? QVG_OK : QVG_ERR_CUDA; }



// ---------------------------------------------------------------- diagnostics
// Launch counts per kernel (always kept) and, when enabled, device time per
// kernel from CUDA events recorded on the launching stream around each launch.
enum Kind {
  K_DEQUANT, K_RESIDUAL, K_RESIDUAL_QUANT, K_ROWNORM, K_INIT, K_ASSIGN_EXACT, K_ASSIGN_TC,
  K_RECHECK, K_UPD_BUCKET, K_UPD_SUM, K_UPD_CENT, K_ATTN, K_ROPE, K_STAT, K_NKINDS
};
const char* const kKindNames[K_NKINDS] = {
  "qvg_dequant_fused", "qvg_residual", "qvg_residual_quant", "qvg_row_norms", "qvg_init_centroids",
  "qvg_assign_exact", "qvg_kmeans_assign", "qvg_assign_recheck", "qvg_update_bucket", "qvg_update_sum",
  "qvg_update_centroids", "qvg_attention_fused", "qvg_rope_tables", "qvg_range_stat"};

struct Profiler {
  std::mutex mu;
  std::atomic<bool> timing{false};
  std::atomic<long long> launches[K_NKINDS];
  std::vector<int> kinds;
  std::vector<cudaEvent_t> ev;     // pairs
  std::vector<cudaEvent_t> pool;
  double ms[K_NKINDS] = {};
  long long timed[K_NKINDS] = {};
  Profiler() { for (auto& l : launches) l = 0; }
};
Profiler& prof() {
  static Profiler p;
  return p;
}

cudaEvent_t pool_event(Profiler& p) {
  if (!p.pool.empty()) { cudaEvent_t e = p.pool.back(); p.pool.pop_back(); return e; }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}

template <class F>
cudaError_t plaunch(Kind k, cudaStream_t s, F&& f) {
  Profiler& p = prof();
  p.launches[k]++;
  if (!p.timing.load(std::memory_order_relaxed)) return f();
  cudaEvent_t a, b;
  {
    std::lock_guard<std::mutex> g(p.mu);
    a = pool_event(p);
    b = pool_event(p);
  }
  // Inside a stream capture the events must be external record nodes to be
  // timed when the graph replays.
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  cudaStreamIsCapturing(s, &cs);
  const unsigned flags = cs == cudaStreamCaptureStatusActive ? cudaEventRecordExternal : 0u;
  cudaEventRecordWithFlags(a, s, flags);
  const cudaError_t e = f();
  cudaEventRecordWithFlags(b, s, flags);
  std::lock_guard<std::mutex> g(p.mu);
  p.kinds.push_back((int)k);
  p.ev.push_back(a);
  p.ev.push_back(b);
  return e;
}

#define QVG_TRY(expr)                                    \
  do {                                                   \
    cudaError_t qvg_e_ = (expr);                         \
    if (qvg_e_ != cudaSuccess) return QVG_ERR_CUDA;      \
  } while (0)

}  // namespace

extern "C" {

const char* qvg_status_string(qvg_status s) {
  switch (s) {
    case QVG_OK: return "ok";
    case QVG_ERR_INVALID_ARG: return "invalid argument";
    case QVG_ERR_UNSUPPORTED: return "unsupported configuration";
    case QVG_ERR_NO_MEMORY: return "out of device memory";
    case QVG_ERR_CUDA: return "CUDA error";
    case QVG_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
    case QVG_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case QVG_ERR_CAPACITY: return "cache capacity exceeded";
  }
  return "unknown status";
}

const char* qvg_version(void) { return "qvg-b200 sm_100a"; }

size_t qvg_packed_bytes(const qvg_config* c, int64_t N, int32_t H, int32_t d, qvg_dtype dtype) {
  if (c == nullptr || c->bits != 2 || c->K < 1 || c->K > 256 || c->T < 0 || c->group_size < 4 ||
      c->group_size % 4 != 0 || d < 4 || d % c->group_size != 0 || N < 0 || H < 1 ||
      (dtype != QVG_BF16 && dtype != QVG_FP32) ||
      (c->scale_mode != QVG_SCALE_ASYM && c->scale_mode != QVG_SCALE_SYM))
    return 0;
  const size_t esz = (size_t)esize(dtype);
  const size_t codes = (size_t)H * N * d * c->bits / 8;
  const size_t scales = (c->scale_mode == QVG_SCALE_SYM ? 1 : 2) * (size_t)H * N * (d / c->group_size);
  const size_t assign = (size_t)c->T * H * N;
  const size_t cents = (size_t)c->T * H * c->K * d * esz;
  return codes + scales + assign + cents;
}

size_t qvg_workspace_bytes(const qvg_config* c, int64_t N, int32_t H, int32_t d, qvg_dtype dtype) {
  if (check_config(c, N, H, d, dtype) != QVG_OK || N < 1) return 0;
  const int W = preferred_batch(*c, N, H, dtype);
  return (size_t)wave_lanes(H, W) * make_plan(*c, N, W, dtype).total;
}

}  // extern "C"

namespace qvg {

qvg_status quantize_impl(const qvg_config* cfg, const void* X, qvg_dtype dtype, int64_t N, int32_t H,
                         int32_t d, const void* init, const qvg_packed* out, void* workspace,
                         size_t ws_bytes, qvg_stream_t stream_, int max_lanes, int warm_stages) {
  qvg_status st = check_config(cfg, N, H, d, dtype);
  if (st != QVG_OK) return st;
  const qvg_config c = *cfg;
  // stages t < warm_stages start from init (warm_iters iterations), the
  // others from the first K tokens of their input (iters iterations)
  if (warm_stages < 0) warm_stages = init != nullptr ? c.T : 0;
  if (warm_stages > c.T || (warm_stages > 0 && init == nullptr)) return QVG_ERR_INVALID_ARG;
  const bool warm = warm_stages > 0;
  const bool cold = warm_stages < c.T;
  const int iters = warm ? c.warm_iters : c.iters;   // validated below for the stages that use it
  if (N < 1 || X == nullptr || out == nullptr || workspace == nullptr) return QVG_ERR_INVALID_ARG;
  const bool sym = c.scale_mode == QVG_SCALE_SYM;
  if (out->codes == nullptr || out->scale == nullptr || (out->zero == nullptr && !sym)) return QVG_ERR_INVALID_ARG;
  if (!aligned(X, 16) || !aligned(init, 16) || !aligned(out->centroids, 16) || !aligned(out->codes, 2) ||
      !aligned(workspace, kAlign))
    return QVG_ERR_INVALID_ARG;
  if (c.T > 0) {
    if (out->assign == nullptr || out->centroids == nullptr) return QVG_ERR_INVALID_ARG;
    if ((warm && c.warm_iters < 1) || (cold && c.iters < 1) || iters < 1) return QVG_ERR_INVALID_ARG;
    if (cold && N < c.K) return QVG_ERR_INVALID_ARG;
  }
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream_);
  const int dt = (int)dtype;
  const size_t esz = (size_t)esize(dt);
  if (make_plan(c, N, 1, dt).total > ws_bytes) return QVG_ERR_WORKSPACE_TOO_SMALL;
  // a timeout recorded by earlier (completed) work on this workspace is
  // reported before anything is queued; qvg_workspace_status clears it
  st = peek_sticky(workspace, s);
  if (st != QVG_OK) return st;

  int W = preferred_batch(c, N, H, dt);
  int lanes = std::min(max_lanes, wave_lanes(H, W));
  Plan plan = make_plan(c, N, W, dt);
  while ((size_t)lanes * plan.total > ws_bytes && W > 1) {
    plan = make_plan(c, N, --W, dt);
    lanes = std::min(max_lanes, wave_lanes(H, W));
  }
  if ((size_t)lanes * plan.total > ws_bytes) lanes = 1;
  if (plan.total > ws_bytes) return QVG_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t s1 = lanes > 1 ? side_stream() : s;
  if (s1 == nullptr) { lanes = 1; s1 = s; }

  // the status word and the near-tie counter are shared by both lanes
  char* const ws0 = static_cast<char*>(workspace);
  uint32_t* status = reinterpret_cast<uint32_t*>(ws0 + plan.off_status);
  unsigned long long* flagged = reinterpret_cast<unsigned long long*>(ws0 + plan.off_status + 8);
  int log2n = 0;                      // smallest k with 2^k > N (fixed-point scale of the sums)
  while (log2n < 62 && (int64_t(1) << log2n) <= N) ++log2n;
  // bf16 blocks take the tensor-core assignment; fp32 blocks the exact CUDA-core one
  const bool use_tc = dt == kBF16 && assign_path_tc();
  const int ng = kD / c.group_size;
  // QVG_FAULT_INJECT=timeout: the tensor-core assignment's first CTA withholds
  // a tile load and waits 1 ms, so that its bounded waits run out (tests only)
  const bool hook_timeout = fault_injected("timeout");

  // one wave: blocks u0 .. u0+w-1 on stream s with workspace ws
  auto run_wave = [&](int u0, int w, cudaStream_t s, char* ws) -> qvg_status {
    float* rnorm = reinterpret_cast<float*>(ws + plan.off_rnorm);
    float* cn = reinterpret_cast<float*>(ws + plan.off_cn);
    uint2* list = reinterpret_cast<uint2*>(ws + plan.off_list);
    uint32_t* list_count = reinterpret_cast<uint32_t*>(ws + plan.off_listcnt);
    uint32_t* chmax = reinterpret_cast<uint32_t*>(ws + plan.off_chmax);
    uint32_t* chmin = chmax + (size_t)plan.W * kD;
    const char* Xu = static_cast<const char*>(X) + (size_t)u0 * N * kD * esz;
    ResidualParams rq{};
    rq.N = N; rq.W = w; rq.K = c.K; rq.G = c.group_size; rq.sym = sym ? 1 : 0;
    rq.codes = out->codes + (size_t)u0 * N * (kD / 4);
    rq.scale = out->scale + (size_t)u0 * N * ng;
    rq.zero = sym ? nullptr : out->zero + (size_t)u0 * N * ng;
    if (c.T == 0) {
      rq.R_in = Xu;
      QVG_TRY(plaunch(K_RESIDUAL_QUANT, s, [&] { return launch_residual(rq, dt, true, s); }));
      return QVG_OK;
    }
    const void* Rin = Xu;
    for (int t = 0; t < c.T; ++t) {
      char* Ct = static_cast<char*>(out->centroids) + ((size_t)t * H + u0) * c.K * kD * esz;
      uint8_t* pit = out->assign + ((size_t)t * H + u0) * N;
      if (t == 0) {   // squared row norms of X (assignment error bound), channel maxima (update scale)
        ResidualParams nq = rq;
        nq.R_in = Xu; nq.C = nullptr; nq.R_out = nullptr; nq.rnorm2 = rnorm; nq.chmax = chmax; nq.chmin = chmin;
        QVG_TRY(cudaMemsetAsync(chmax, 0, 2 * (size_t)plan.W * kD * sizeof(uint32_t), s));
        QVG_TRY(plaunch(K_ROWNORM, s, [&] { return launch_residual(nq, dt, false, s); }));
      }
      const bool stage_warm = t < warm_stages;
      const int it_t = stage_warm ? c.warm_iters : c.iters;
      if (stage_warm) {
        const char* src = static_cast<const char*>(init) + ((size_t)t * H + u0) * c.K * kD * esz;
        QVG_TRY(plaunch(K_INIT, s, [&] { return launch_init_centroids(src, (int64_t)c.K * kD, Ct, cn, w, c.K, dt, s); }));
      } else {
        QVG_TRY(plaunch(K_INIT, s, [&] { return launch_init_centroids(Rin, N * kD, Ct, cn, w, c.K, dt, s); }));
      }
      // The assignment of iteration `it` goes to pit or to the spare buffer, so
      // that the last iteration's lands in pit and the previous one is kept
      // for the incremental update.
      uint8_t* spare = reinterpret_cast<uint8_t*>(ws + plan.off_pi);
      for (int it = 0; it < it_t; ++it) {
        uint8_t* pi_new = ((it_t - 1 - it) % 2 == 0) ? pit : spare;
        uint8_t* pi_old = it == 0 ? nullptr : (pi_new == pit ? spare : pit);
        AssignParams ap{};
        ap.R = Rin; ap.rnorm2 = rnorm; ap.C = Ct; ap.cn = cn; ap.pi = pi_new;
        ap.list = nullptr; ap.list_count = nullptr; ap.N = N; ap.W = w; ap.K = c.K;
        if (use_tc) {
          // tensor-core screening; listed near-ties are decided exactly next
          QVG_TRY(cudaMemsetAsync(list_count, 0, (size_t)w * sizeof(uint32_t), s));
          AssignTcParams tp{};
          tp.R = Rin; tp.rnorm2 = rnorm; tp.C = Ct; tp.cn = cn; tp.pi = pi_new; tp.list = list;
          tp.list_count = list_count; tp.status = status; tp.flagged = flagged;
          tp.N = N; tp.W = w; tp.K = c.K; tp.gamma = kTcGamma;
          tp.hook_withhold = -1; tp.hook_wait_ns = 0;
          if (hook_timeout) { tp.hook_withhold = 0; tp.hook_wait_ns = 1000000ull; }   // 1 ms
          QVG_TRY(plaunch(K_ASSIGN_TC, s, [&] { return launch_assign_tc(tp, s); }));
          QVG_TRY(plaunch(K_RECHECK, s, [&] {
            return launch_assign_candidates(Rin, Ct, c.K, N, w, list, list_count, pi_new, s);
          }));
        } else {
          QVG_TRY(plaunch(K_ASSIGN_EXACT, s, [&] { return launch_assign_exact(ap, dt, s); }));
        }
        UpdateParams up{};
        up.R = Rin; up.pi = pi_new; up.pi_old = pi_old; up.chmax = chmax; up.chmin = chmin; up.C = Ct; up.cn = cn;
        up.N = N; up.W = w; up.K = c.K; up.log2n = log2n;
        up.list = reinterpret_cast<uint32_t*>(list);   // the near-tie list is consumed by now
        up.off = reinterpret_cast<int*>(ws + plan.off_off);
        up.cnt = reinterpret_cast<int*>(ws + plan.off_cnt);
        up.S = reinterpret_cast<long long*>(ws + plan.off_S);
        up.n = reinterpret_cast<int*>(ws + plan.off_n);
        QVG_TRY(plaunch(K_UPD_BUCKET, s, [&] { return launch_update_bucket(up, dt, s); }));
        QVG_TRY(plaunch(K_UPD_SUM, s, [&] { return launch_update_sum(up, dt, s); }));
        QVG_TRY(plaunch(K_UPD_CENT, s, [&] { return launch_update_centroids(up, dt, s); }));
      }
      ResidualParams rp = rq;
      rp.R_in = Rin; rp.C = Ct; rp.pi = pit;
      if (t + 1 < c.T) {
        void* Rout = ws + plan.off_R[t % 2];
        rp.R_out = Rout; rp.rnorm2 = rnorm; rp.chmax = chmax; rp.chmin = chmin;
        QVG_TRY(cudaMemsetAsync(chmax, 0, 2 * (size_t)plan.W * kD * sizeof(uint32_t), s));
        QVG_TRY(plaunch(K_RESIDUAL, s, [&] { return launch_residual(rp, dt, false, s); }));
        Rin = Rout;
      } else {
        QVG_TRY(plaunch(K_RESIDUAL_QUANT, s, [&] { return launch_residual(rp, dt, true, s); }));
      }
    }
    return QVG_OK;
  };

  if (lanes == 1) {
    for (int u0 = 0; u0 < H; u0 += W) {
      st = run_wave(u0, std::min(W, H - u0), s, ws0);
      if (st != QVG_OK) return st;
    }
    // QVG_FAULT_INJECT=stream: report the stream error a failed launch would
    return fault_injected("stream") ? QVG_ERR_CUDA : QVG_OK;
  }
  // Two lanes: the side stream joins after the caller's stream reaches this
  // call, and the caller's stream waits for the side stream at the end (also
  // on an error, so that a stream capture stays joined).
  cudaEvent_t fork = nullptr, join = nullptr;
  if (cudaEventCreateWithFlags(&fork, cudaEventDisableTiming) != cudaSuccess ||
      cudaEventCreateWithFlags(&join, cudaEventDisableTiming) != cudaSuccess) {
    cudaGetLastError();
    if (fork) cudaEventDestroy(fork);
    return QVG_ERR_CUDA;
  }
  st = QVG_OK;
  if (cudaEventRecord(fork, s) != cudaSuccess || cudaStreamWaitEvent(s1, fork, 0) != cudaSuccess) st = QVG_ERR_CUDA;
  for (int u0 = 0, wv = 0; st == QVG_OK && u0 < H; u0 += W, ++wv) {
    const int lane = wv & 1;
    st = run_wave(u0, std::min(W, H - u0), lane ? s1 : s, ws0 + (size_t)lane * plan.total);
  }
  if (cudaEventRecord(join, s1) != cudaSuccess || cudaStreamWaitEvent(s, join, 0) != cudaSuccess) st = QVG_ERR_CUDA;
  cudaEventDestroy(fork);
  cudaEventDestroy(join);
  if (st == QVG_OK && fault_injected("stream")) st = QVG_ERR_CUDA;
  return st;
}

}  // namespace qvg

extern "C" {

qvg_status qvg_quantize(const qvg_config* cfg, const void* X, qvg_dtype dtype, int64_t N,
                        int32_t H, int32_t d, const void* init, const qvg_packed* out,
                        void* workspace, size_t ws_bytes, qvg_stream_t stream_) {
  return qvg::quantize_impl(cfg, X, dtype, N, H, d, init, out, workspace, ws_bytes, stream_, 2, -1);
}

qvg_status qvg_dequantize(const qvg_config* cfg, const qvg_packed* packed, qvg_dtype dtype,
                          int64_t N, int32_t H, int32_t d, void* Y, qvg_stream_t stream_) {
  qvg_status st = check_config(cfg, N, H, d, dtype);
  if (st != QVG_OK) return st;
  if (packed == nullptr || Y == nullptr || packed->codes == nullptr || packed->scale == nullptr ||
      (packed->zero == nullptr && cfg->scale_mode != QVG_SCALE_SYM))
    return QVG_ERR_INVALID_ARG;
  if (cfg->T > 0 && (packed->assign == nullptr || packed->centroids == nullptr)) return QVG_ERR_INVALID_ARG;
  if (!aligned(Y, 16) || !aligned(packed->centroids, 16) || !aligned(packed->codes, 16)) return QVG_ERR_INVALID_ARG;
  if (N == 0) return QVG_OK;
  const int dt = (int)dtype;
  const size_t table = (size_t)cfg->K * kD * esize(dt);
  DequantParams p{};
  p.codes = packed->codes; p.scale = packed->scale; p.zero = packed->zero;
  p.assign = packed->assign; p.centroids = packed->centroids; p.Y = Y;
  p.chunk_off = nullptr; p.N = N; p.y_head_stride = N; p.n_chunks = 1; p.H = H;
  p.K = cfg->K; p.T = cfg->T; p.G = cfg->group_size; p.sym = cfg->scale_mode == QVG_SCALE_SYM;
  p.t_smem = std::min<int>(cfg->T, (int)((kDqTableSmemBytes) / table));
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream_);
  st = cuda_status(plaunch(K_DEQUANT, s, [&] { return launch_dequant(p, dt, s); }));
  if (st == QVG_OK && fault_injected("stream")) st = QVG_ERR_CUDA;
  return st;
}

size_t qvg_rope_tables_bytes(int32_t d, int64_t max_pos) {
  if (d != kD || max_pos < 0 || max_pos >= kRopeMaxPositions) return 0;
  return kRopeHeaderBytes + (size_t)(max_pos + 1) * kRopeRowBytes;
}

qvg_status qvg_rope_tables(double base, int32_t d, int64_t max_pos, void* tables, size_t bytes,
                           qvg_stream_t stream_) {
  const size_t need = qvg_rope_tables_bytes(d, max_pos);
  if (need == 0 || !(base > 1.0) || tables == nullptr || !aligned(tables, 16)) return QVG_ERR_INVALID_ARG;
  if (bytes < need) return QVG_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream_);
  QVG_TRY(cudaMemsetAsync(tables, 0, 16, s));
  return cuda_status(plaunch(K_ROPE, s, [&] { return launch_rope_tables(tables, max_pos, base, s); }));
}

// The split of qvg_attention_set_split (0 = the library's choice).
static std::atomic<int> g_attention_split{0};

int32_t qvg_attention_set_split(int32_t split) {
  if (split < 0 || split > 8) return -1;
  return g_attention_split.exchange(split);
}

int32_t qvg_attention_split(const qvg_config* cfg, int64_t Nk, int32_t H, int64_t Nq, size_t ws_bytes) {
  if (check_config(cfg, Nk, H, kD, QVG_BF16) != QVG_OK || Nk < 1 || Nq < 1) return -1;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) { (void)cudaGetLastError(); return -1; }
  return attention_split(cfg->T, Nk, Nq, H, g_attention_split.load(std::memory_order_relaxed), ws_bytes);
}

size_t qvg_attention_workspace_bytes(const qvg_config* cfg, int64_t Nk, int32_t H, int64_t Nq) {
  if (check_config(cfg, Nk, H, kD, QVG_BF16) != QVG_OK || Nk < 1 || Nq < 1) return 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) { (void)cudaGetLastError(); return 0; }
  return attention_workspace_bytes(cfg->T, Nk, Nq, H, g_attention_split.load(std::memory_order_relaxed));
}

qvg_status qvg_attention(const qvg_config* cfg, const qvg_packed* k, const qvg_packed* v, int64_t Nk, int32_t H,
                         int32_t d, const void* Q, const int64_t* q_pos, int64_t Nq, const void* tables,
                         size_t tables_bytes, float* O, void* workspace, size_t ws_bytes, qvg_stream_t stream_) {
  qvg_status st = check_config(cfg, Nk, H, d, QVG_BF16);
  if (st != QVG_OK) return st;
  const bool sym = cfg->scale_mode == QVG_SCALE_SYM;
  for (const qvg_packed* p : {k, v}) {
    if (p == nullptr || p->codes == nullptr || p->scale == nullptr || (p->zero == nullptr && !sym))
      return QVG_ERR_INVALID_ARG;
    if (cfg->T > 0 && (p->assign == nullptr || p->centroids == nullptr || !aligned(p->centroids, 16)))
      return QVG_ERR_INVALID_ARG;
    if (!aligned(p->codes, 2)) return QVG_ERR_INVALID_ARG;
  }
  if (Nk < 1 || Nq < 1 || Q == nullptr || q_pos == nullptr || tables == nullptr || O == nullptr ||
      !aligned(Q, 16) || !aligned(O, 16) || !aligned(tables, 16) || !aligned(workspace, 16) ||
      Nq >= (int64_t(1) << 31) * 128)
    return QVG_ERR_INVALID_ARG;
  if (tables_bytes < kRopeHeaderBytes + kRopeRowBytes) return QVG_ERR_INVALID_ARG;
  const int64_t max_pos = std::min<int64_t>((int64_t)((tables_bytes - kRopeHeaderBytes) / kRopeRowBytes),
                                            kRopeMaxPositions) - 1;
  if (Nk - 1 > max_pos) return QVG_ERR_INVALID_ARG;                // the cache's positions must be covered
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream_);
  st = peek_sticky(tables, s);
  if (st != QVG_OK) return st;
  AttentionArgs a{};
  a.k = k; a.v = v; a.Q = Q; a.qpos = q_pos; a.tables = tables; a.max_pos = max_pos; a.O = O;
  a.Nk = Nk; a.Nq = Nq; a.H = H; a.K = cfg->K; a.T = cfg->T; a.G = cfg->group_size; a.sym = sym ? 1 : 0;
  a.split = g_attention_split.load(std::memory_order_relaxed);
  a.workspace = workspace;
  a.ws_bytes = workspace != nullptr ? ws_bytes : 0;
  st = cuda_status(plaunch(K_ATTN, s, [&] { return launch_attention(a, s); }));
  if (st == QVG_OK && fault_injected("stream")) st = QVG_ERR_CUDA;
  return st;
}

int64_t qvg_workspace_flagged(void* workspace, size_t ws_bytes, qvg_stream_t stream_) {
  if (workspace == nullptr || ws_bytes < 16) return -1;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream_);
  unsigned long long n = 0;
  if (cudaMemcpyAsync(&n, static_cast<char*>(workspace) + 8, sizeof(n), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess || cudaMemsetAsync(static_cast<char*>(workspace) + 8, 0, 8, s) != cudaSuccess)
    return -1;
  return (int64_t)n;
}

qvg_status qvg_workspace_status(void* workspace, size_t ws_bytes, qvg_stream_t stream_) {
  if (workspace == nullptr || ws_bytes < 16) return QVG_ERR_INVALID_ARG;
  return take_sticky(workspace, reinterpret_cast<cudaStream_t>(stream_));
}


void qvg_profile_enable(int enable) { prof().timing = enable != 0; }

void qvg_profile_reset(void) {
  Profiler& p = prof();
  std::lock_guard<std::mutex> g(p.mu);
  for (auto& l : p.launches) l = 0;
  for (int k = 0; k < K_NKINDS; ++k) { p.ms[k] = 0.0; p.timed[k] = 0; }
  for (cudaEvent_t e : p.ev) p.pool.push_back(e);
  p.ev.clear();
  p.kinds.clear();
}

int64_t qvg_profile_launches(void) {
  Profiler& p = prof();
  long long n = 0;
  for (auto& l : p.launches) n += l.load();
  return n;
}

int qvg_profile_report(char* buf, size_t buf_bytes) {
  Profiler& p = prof();
  std::lock_guard<std::mutex> g(p.mu);
  if (!p.ev.empty()) {
    if (cudaDeviceSynchronize() != cudaSuccess) return -1;
    for (size_t i = 0; i < p.kinds.size(); ++i) {
      float t = 0.0f;
      if (cudaEventElapsedTime(&t, p.ev[2 * i], p.ev[2 * i + 1]) == cudaSuccess) {
        p.ms[p.kinds[i]] += t;
        p.timed[p.kinds[i]] += 1;
      }
    }
    for (cudaEvent_t e : p.ev) p.pool.push_back(e);
    p.ev.clear();
    p.kinds.clear();
  }
  std::string out = "{";
  bool first = true;
  for (int k = 0; k < K_NKINDS; ++k) {
    const long long n = p.launches[k].load();
    if (n == 0 && p.timed[k] == 0) continue;
    char item[256];
    std::snprintf(item, sizeof(item), "%s\"%s\": {\"launches\": %lld, \"timed\": %lld, \"ms\": %.6f}",
                  first ? "" : ", ", kKindNames[k], n, p.timed[k], p.ms[k]);
    out += item;
    first = false;
  }
  out += "}";
  if (buf == nullptr || buf_bytes < out.size() + 1) return (int)out.size() + 1;
  std::memcpy(buf, out.c_str(), out.size() + 1);
  return 0;
}

// ---------------------------------------------------------------- cache
struct qvg_cache {
  qvg_config cfg{};
  int dtype = 0, H = 0;
  int64_t max_tokens = 0;
  int64_t max_chunk_tokens = 0;
  int max_chunks = 0;
  uint8_t* codes = nullptr;
  uint8_t* scale = nullptr;
  uint8_t* zero = nullptr;
  uint8_t* assign = nullptr;
  char* tables = nullptr;
  int64_t* d_off = nullptr;     // device copy of the chunk offsets
  int64_t* h_off = nullptr;     // pinned host offsets [max_chunks + 1]
  int n_chunks = 0;
  void* ws = nullptr;
  size_t ws_bytes = 0;
  size_t bytes = 0;
  // adaptive caches (qvg_cache_create_adaptive): every chunk has its own
  // stage count and group size, chosen from the policy's ladder
  bool adaptive = false;
  qvg_adaptive_policy pol{};
  qvg_config level_cfg[4]{};
  int T_max = 0;
  ChunkDesc* d_desc = nullptr;              // device [max_chunks]
  ChunkDesc* h_desc = nullptr;              // pinned [max_chunks], the copies' sources
  std::vector<int32_t> level;               // per chunk
  std::vector<uint64_t> stat;               // per chunk
  unsigned long long* d_stat = nullptr;     // device counter of the range statistic
  unsigned long long* h_stat = nullptr;     // pinned
  int64_t next_scale_off = 0, next_assign_off = 0;
};

static void cache_free(qvg_cache* c) {
  if (c == nullptr) return;
  cudaFree(c->codes); cudaFree(c->scale); cudaFree(c->zero); cudaFree(c->assign);
  cudaFree(c->tables); cudaFree(c->d_off); cudaFree(c->ws); cudaFree(c->d_desc); cudaFree(c->d_stat);
  cudaFreeHost(c->h_off); cudaFreeHost(c->h_desc); cudaFreeHost(c->h_stat);
  delete c;
}

qvg_status qvg_cache_create(const qvg_config* cfg, qvg_dtype dtype, int32_t H, int32_t d,
                            int64_t max_tokens, int32_t max_chunks, int64_t max_chunk_tokens,
                            qvg_cache** out) {
  if (out == nullptr) return QVG_ERR_INVALID_ARG;
  *out = nullptr;
  qvg_status st = check_config(cfg, max_tokens, H, d, dtype);
  if (st != QVG_OK) return st;
  if (max_tokens < 1 || max_chunks < 1 || max_chunk_tokens < 0) return QVG_ERR_INVALID_ARG;
  if (max_chunk_tokens == 0 || max_chunk_tokens > max_tokens) max_chunk_tokens = max_tokens;
  if (cfg->T > 0 && (cfg->iters < 1 || cfg->warm_iters < 1)) return QVG_ERR_INVALID_ARG;
  if (cfg->T > 0 && max_chunk_tokens < cfg->K) return QVG_ERR_INVALID_ARG;   // chunk 0 needs K tokens
  // QVG_FAULT_INJECT=alloc: every device allocation of the cache fails
  if (fault_injected("alloc")) return QVG_ERR_NO_MEMORY;
  // the workspace of the largest chunk: any smaller chunk fits in it
  const size_t ws_bytes = qvg_workspace_bytes(cfg, max_chunk_tokens, H, d, dtype);
  if (ws_bytes == 0) return QVG_ERR_INVALID_ARG;
  qvg_cache* c = new qvg_cache();
  c->cfg = *cfg; c->dtype = (int)dtype; c->H = H; c->max_tokens = max_tokens; c->max_chunks = max_chunks;
  c->max_chunk_tokens = max_chunk_tokens;
  const size_t esz = (size_t)esize(c->dtype);
  const int ng = kD / cfg->group_size;
  const size_t n_codes = (size_t)H * max_tokens * (kD / 4);
  const size_t n_sc = (size_t)H * max_tokens * ng;
  const size_t n_zero = cfg->scale_mode == QVG_SCALE_SYM ? 16 : n_sc;   // no zero points when symmetric
  const size_t n_as = std::max<size_t>(1, (size_t)cfg->T * H * max_tokens);
  const size_t n_tab = std::max<size_t>(16, (size_t)max_chunks * cfg->T * H * cfg->K * kD * esz);
  bool ok = cudaMalloc(&c->codes, n_codes) == cudaSuccess && cudaMalloc(&c->scale, n_sc) == cudaSuccess &&
            cudaMalloc(&c->zero, n_zero) == cudaSuccess && cudaMalloc(&c->assign, n_as) == cudaSuccess &&
            cudaMalloc(&c->tables, n_tab) == cudaSuccess &&
            cudaMalloc(&c->d_off, sizeof(int64_t) * ((size_t)max_chunks + 1)) == cudaSuccess &&
            cudaMemset(c->d_off, 0, sizeof(int64_t) * ((size_t)max_chunks + 1)) == cudaSuccess &&
            cudaMallocHost(&c->h_off, sizeof(int64_t) * ((size_t)max_chunks + 1)) == cudaSuccess &&
            cudaMalloc(&c->ws, ws_bytes) == cudaSuccess && cudaMemset(c->ws, 0, 16) == cudaSuccess &&
            cudaDeviceSynchronize() == cudaSuccess;
  if (!ok) {
    cudaGetLastError();
    cache_free(c);
    return QVG_ERR_NO_MEMORY;
  }
  c->ws_bytes = ws_bytes;
  c->bytes = n_codes + n_sc + n_zero + n_as + n_tab + sizeof(int64_t) * ((size_t)max_chunks + 1);
  c->h_off[0] = 0;
  c->n_chunks = 0;
  *out = c;
  return QVG_OK;
}

static void chunk_view(const qvg_cache* c, int chunk, qvg_packed* v) {
  const int64_t o = c->h_off[chunk];
  const size_t esz = (size_t)esize(c->dtype);
  if (c->adaptive) {                        // this chunk's own layout
    const ChunkDesc& dsc = c->h_desc[chunk];
    v->codes = c->codes + (size_t)c->H * o * (kD / 4);
    v->scale = c->scale + dsc.scale_off;
    v->zero = c->cfg.scale_mode == QVG_SCALE_SYM ? nullptr : c->zero + dsc.scale_off;
    v->assign = c->assign + dsc.assign_off;
    v->centroids = c->tables + (size_t)dsc.table_off * esz;
    return;
  }
  const int ng = kD / c->cfg.group_size;
  v->codes = c->codes + (size_t)c->H * o * (kD / 4);
  v->scale = c->scale + (size_t)c->H * o * ng;
  v->zero = c->cfg.scale_mode == QVG_SCALE_SYM ? nullptr : c->zero + (size_t)c->H * o * ng;
  v->assign = c->assign + (size_t)c->cfg.T * c->H * o;
  v->centroids = c->tables + (size_t)chunk * c->cfg.T * c->H * c->cfg.K * kD * esz;
}

// The level of a chunk from its range statistic S over n_groups groups: the
// number of the policy's ascending thresholds (sixteenths of a code) that
// 16 S exceeds per group.
static int adaptive_level(const qvg_adaptive_policy& pol, uint64_t S, int64_t n_groups) {
  int lvl = 0;
  for (int j = 0; j + 1 < pol.levels; ++j)
    if ((double)S * 16.0 > (double)pol.thresholds[j] * (double)n_groups) lvl = j + 1;
  return lvl;
}

static qvg_status append_adaptive(qvg_cache* c, const void* X, int64_t n, cudaStream_t s) {
  const int chunk = c->n_chunks;
  // 1. the chunk's statistic (waits for the stream: the host picks the level)
  QVG_TRY(cudaMemsetAsync(c->d_stat, 0, sizeof(unsigned long long), s));
  QVG_TRY(plaunch(K_STAT, s, [&] {
    return launch_range_stat(X, (int64_t)c->H * n, c->pol.probe_group, c->dtype, c->d_stat, s);
  }));
  QVG_TRY(cudaMemcpyAsync(c->h_stat, c->d_stat, sizeof(unsigned long long), cudaMemcpyDeviceToHost, s));
  QVG_TRY(cudaStreamSynchronize(s));
  const uint64_t S = *c->h_stat;
  const int64_t n_groups = (int64_t)c->H * n * (kD / c->pol.probe_group);
  const int lvl = adaptive_level(c->pol, S, n_groups);
  const qvg_config& cc = c->level_cfg[lvl];
  // 2. centroid reuse: the previous chunk's tables for the stages both have
  int warm = 0;
  if (chunk > 0 && !(c->pol.refresh_every > 0 && chunk % c->pol.refresh_every == 0))
    warm = std::min(c->h_desc[chunk - 1].T, cc.T);
  if (cc.T > warm && n < cc.K) return QVG_ERR_INVALID_ARG;   // a cold stage needs K tokens
  // 3. this chunk's layout
  ChunkDesc& dsc = c->h_desc[chunk];
  dsc.o = c->h_off[chunk];
  dsc.n = n;
  dsc.scale_off = c->next_scale_off;
  dsc.assign_off = c->next_assign_off;
  dsc.table_off = (int64_t)chunk * c->T_max * c->H * cc.K * kD;
  dsc.T = cc.T;
  dsc.G = cc.group_size;
  qvg_packed v;
  chunk_view(c, chunk, &v);
  qvg_packed prev{};
  if (warm > 0) chunk_view(c, chunk - 1, &prev);
  qvg_status st = quantize_impl(&cc, X, (qvg_dtype)c->dtype, n, c->H, kD, warm > 0 ? prev.centroids : nullptr, &v,
                                c->ws, c->ws_bytes, reinterpret_cast<qvg_stream_t>(s), 2, warm);
  if (st != QVG_OK) return st;
  // 4. commit: offsets and the chunk's layout travel to the device in stream order
  c->h_off[chunk + 1] = c->h_off[chunk] + n;
  QVG_TRY(cudaMemcpyAsync(c->d_off + chunk + 1, &c->h_off[chunk + 1], sizeof(int64_t), cudaMemcpyHostToDevice, s));
  QVG_TRY(cudaMemcpyAsync(c->d_desc + chunk, &dsc, sizeof(ChunkDesc), cudaMemcpyHostToDevice, s));
  // scale rows of the next chunk start on a 16-byte boundary (a multiple of any row width)
  c->next_scale_off += ((int64_t)c->H * n * (kD / cc.group_size) + 15) & ~int64_t(15);
  c->next_assign_off += (int64_t)cc.T * c->H * n;
  c->level[chunk] = lvl;
  c->stat[chunk] = S;
  c->n_chunks = chunk + 1;
  return QVG_OK;
}

qvg_status qvg_append_chunk(qvg_cache* c, const void* X, int64_t n, qvg_stream_t stream_) {
  if (c == nullptr || X == nullptr || n < 1) return QVG_ERR_INVALID_ARG;
  const int chunk = c->n_chunks;
  if (chunk >= c->max_chunks || c->h_off[chunk] + n > c->max_tokens || n > c->max_chunk_tokens)
    return QVG_ERR_CAPACITY;
  if (c->adaptive) return append_adaptive(c, X, n, reinterpret_cast<cudaStream_t>(stream_));
  if (chunk == 0 && c->cfg.T > 0 && n < c->cfg.K) return QVG_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream_);
  // the workspace was sized at creation for the largest chunk: no allocation here
  qvg_packed v;
  chunk_view(c, chunk, &v);
  const void* init = nullptr;
  if (chunk > 0) {
    qvg_packed prev;
    chunk_view(c, chunk - 1, &prev);
    init = prev.centroids;
  }
  qvg_status st = qvg_quantize(&c->cfg, X, (qvg_dtype)c->dtype, n, c->H, kD, init, &v, c->ws,
                               c->ws_bytes, stream_);
  if (st != QVG_OK) return st;
  c->h_off[chunk + 1] = c->h_off[chunk] + n;
  // The new end offset travels to the device in stream order (pinned source,
  // written once and never changed afterwards).
  QVG_TRY(cudaMemcpyAsync(c->d_off + chunk + 1, &c->h_off[chunk + 1], sizeof(int64_t),
                          cudaMemcpyHostToDevice, s));
  c->n_chunks = chunk + 1;
  return QVG_OK;
}

qvg_status qvg_cache_dequantize(const qvg_cache* c, void* Y, qvg_stream_t stream_) {
  if (c == nullptr || Y == nullptr) return QVG_ERR_INVALID_ARG;
  const int n_chunks = c->n_chunks;
  if (n_chunks == 0) return QVG_OK;
  const size_t table = (size_t)c->cfg.K * kD * esize(c->dtype);
  DequantParams p{};
  p.codes = c->codes; p.scale = c->scale; p.zero = c->zero; p.assign = c->assign;
  p.centroids = c->tables; p.Y = Y; p.chunk_off = c->d_off; p.N = 0;
  p.y_head_stride = c->h_off[n_chunks]; p.n_chunks = n_chunks; p.H = c->H;
  p.K = c->cfg.K; p.T = c->cfg.T; p.G = c->cfg.group_size; p.sym = c->cfg.scale_mode == QVG_SCALE_SYM;
  p.t_smem = std::min<int>(c->cfg.T, (int)((kDqTableSmemBytes) / table));
  if (c->adaptive) {                 // per-chunk stage counts and group sizes
    p.desc = c->d_desc;
    p.T = c->T_max;
    p.t_smem = std::min<int>(c->T_max, (int)((kDqTableSmemBytes) / table));
  }
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream_);
  qvg_status st = cuda_status(plaunch(K_DEQUANT, s, [&] { return launch_dequant(p, c->dtype, s); }));
  if (st == QVG_OK && fault_injected("stream")) st = QVG_ERR_CUDA;
  return st;
}

int64_t qvg_cache_tokens(const qvg_cache* c) { return c ? c->h_off[c->n_chunks] : 0; }
int32_t qvg_cache_chunks(const qvg_cache* c) { return c ? c->n_chunks : 0; }

qvg_status qvg_cache_chunk_view(const qvg_cache* c, int32_t chunk, qvg_packed* view,
                                int64_t* first_token, int64_t* n_tokens) {
  if (c == nullptr || view == nullptr || chunk < 0 || chunk >= c->n_chunks)
    return QVG_ERR_INVALID_ARG;
  chunk_view(c, chunk, view);
  if (first_token) *first_token = c->h_off[chunk];
  if (n_tokens) *n_tokens = c->h_off[chunk + 1] - c->h_off[chunk];
  return QVG_OK;
}

size_t qvg_cache_device_bytes(const qvg_cache* c) { return c ? c->bytes + c->ws_bytes : 0; }

qvg_status qvg_cache_chunk_info(const qvg_cache* c, int32_t chunk, int32_t* level, int32_t* T, int32_t* G,
                                uint64_t* stat) {
  if (c == nullptr || chunk < 0 || chunk >= c->n_chunks) return QVG_ERR_INVALID_ARG;
  if (level) *level = c->adaptive ? c->level[chunk] : 0;
  if (T) *T = c->adaptive ? c->h_desc[chunk].T : c->cfg.T;
  if (G) *G = c->adaptive ? c->h_desc[chunk].G : c->cfg.group_size;
  if (stat) *stat = c->adaptive ? c->stat[chunk] : 0;
  return QVG_OK;
}

qvg_status qvg_cache_create_adaptive(const qvg_config* cfg, const qvg_adaptive_policy* pol, qvg_dtype dtype,
                                     int32_t H, int32_t d, int64_t max_tokens, int32_t max_chunks,
                                     int64_t max_chunk_tokens, qvg_cache** out) {
  if (out == nullptr || cfg == nullptr || pol == nullptr) return QVG_ERR_INVALID_ARG;
  *out = nullptr;
  if (pol->levels < 1 || pol->levels > 4 || pol->refresh_every < 0) return QVG_ERR_INVALID_ARG;
  if (!g_supported(pol->probe_group)) return QVG_ERR_INVALID_ARG;
  for (int j = 0; j + 2 < pol->levels; ++j)
    if (pol->thresholds[j] > pol->thresholds[j + 1]) return QVG_ERR_INVALID_ARG;
  if (max_tokens < 1 || max_chunks < 1 || max_chunk_tokens < 0) return QVG_ERR_INVALID_ARG;
  if (max_chunk_tokens == 0 || max_chunk_tokens > max_tokens) max_chunk_tokens = max_tokens;
  qvg_config lc[4];
  int T_max = 0, G_min = 128;
  size_t ws_bytes = 0;
  for (int l = 0; l < pol->levels; ++l) {
    lc[l] = *cfg;
    lc[l].T = pol->T[l];
    lc[l].group_size = pol->group_size[l];
    qvg_status st = check_config(&lc[l], max_tokens, H, d, dtype);
    if (st != QVG_OK) return st;
    if (lc[l].T > 0 && (lc[l].iters < 1 || lc[l].warm_iters < 1)) return QVG_ERR_INVALID_ARG;
    T_max = std::max(T_max, lc[l].T);
    G_min = std::min(G_min, lc[l].group_size);
    ws_bytes = std::max(ws_bytes, qvg_workspace_bytes(&lc[l], max_chunk_tokens, H, d, dtype));
  }
  if (ws_bytes == 0) return QVG_ERR_INVALID_ARG;
  if (fault_injected("alloc")) return QVG_ERR_NO_MEMORY;
  qvg_cache* c = new qvg_cache();
  c->cfg = lc[0]; c->dtype = (int)dtype; c->H = H; c->max_tokens = max_tokens; c->max_chunks = max_chunks;
  c->max_chunk_tokens = max_chunk_tokens;
  c->adaptive = true;
  c->pol = *pol;
  for (int l = 0; l < pol->levels; ++l) c->level_cfg[l] = lc[l];
  c->T_max = T_max;
  c->level.assign((size_t)max_chunks, 0);
  c->stat.assign((size_t)max_chunks, 0);
  const size_t esz = (size_t)esize(c->dtype);
  const size_t n_codes = (size_t)H * max_tokens * (kD / 4);
  const size_t n_sc = (size_t)H * max_tokens * (kD / G_min) + 16 * (size_t)max_chunks;
  const size_t n_zero = cfg->scale_mode == QVG_SCALE_SYM ? 16 : n_sc;
  const size_t n_as = std::max<size_t>(1, (size_t)T_max * H * max_tokens);
  const size_t n_tab = std::max<size_t>(16, (size_t)max_chunks * T_max * H * cfg->K * kD * esz);
  bool ok = cudaMalloc(&c->codes, n_codes) == cudaSuccess && cudaMalloc(&c->scale, n_sc) == cudaSuccess &&
            cudaMalloc(&c->zero, n_zero) == cudaSuccess && cudaMalloc(&c->assign, n_as) == cudaSuccess &&
            cudaMalloc(&c->tables, n_tab) == cudaSuccess &&
            cudaMalloc(&c->d_off, sizeof(int64_t) * ((size_t)max_chunks + 1)) == cudaSuccess &&
            cudaMemset(c->d_off, 0, sizeof(int64_t) * ((size_t)max_chunks + 1)) == cudaSuccess &&
            cudaMallocHost(&c->h_off, sizeof(int64_t) * ((size_t)max_chunks + 1)) == cudaSuccess &&
            cudaMalloc(&c->d_desc, sizeof(ChunkDesc) * (size_t)max_chunks) == cudaSuccess &&
            cudaMallocHost(&c->h_desc, sizeof(ChunkDesc) * (size_t)max_chunks) == cudaSuccess &&
            cudaMalloc(&c->d_stat, sizeof(unsigned long long)) == cudaSuccess &&
            cudaMallocHost(&c->h_stat, sizeof(unsigned long long)) == cudaSuccess &&
            cudaMalloc(&c->ws, ws_bytes) == cudaSuccess && cudaMemset(c->ws, 0, 16) == cudaSuccess &&
            cudaDeviceSynchronize() == cudaSuccess;
  if (!ok) {
    cudaGetLastError();
    cache_free(c);
    return QVG_ERR_NO_MEMORY;
  }
  c->ws_bytes = ws_bytes;
  c->bytes = n_codes + n_sc + n_zero + n_as + n_tab + sizeof(int64_t) * ((size_t)max_chunks + 1) +
             sizeof(ChunkDesc) * (size_t)max_chunks;
  c->h_off[0] = 0;
  *out = c;
  return QVG_OK;
}

qvg_status qvg_cache_status(qvg_cache* c, qvg_stream_t stream_) {
  if (c == nullptr || c->ws == nullptr) return QVG_ERR_INVALID_ARG;
  return take_sticky(c->ws, reinterpret_cast<cudaStream_t>(stream_));
}

void qvg_cache_destroy(qvg_cache* c) {
  if (c == nullptr) return;
  cudaDeviceSynchronize();
  cache_free(c);
}

}  // extern "C"
