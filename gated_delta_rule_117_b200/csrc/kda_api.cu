// C-ABI layer of libkda: argument validation, planning and dispatch.
// The interface and its contract are documented in include/kda.h.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#include <atomic>
#include <mutex>

#include "kda.h"
#include "kda_internal.cuh"
#include "kda_tmap.cuh"

namespace kda {

// Status word written by kernels whose bounded waits give up or whose
// device-side checks fail.  One per device (a __device__ variable is
// instantiated in every context that loads the module).
__device__ unsigned g_status_word;

namespace {
constexpr int kMaxDevices = 64;
// Address of g_status_word per device, valid for the context it was looked up
// in (a context re-created after cudaDeviceReset loads the module anew).
struct StatusCache {
  std::mutex mu;
  unsigned long long ctx[kMaxDevices] = {};
  unsigned *addr[kMaxDevices] = {};
} g_status_cache;
}  // namespace

unsigned *device_status_ptr() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  unsigned long long id = 0;
  bool have_id = current_context_id(&id);
  {
    std::lock_guard<std::mutex> lk(g_status_cache.mu);
    if (have_id && g_status_cache.addr[dev] && g_status_cache.ctx[dev] == id) return g_status_cache.addr[dev];
  }
  void *addr = nullptr;
  if (cudaGetSymbolAddress(&addr, g_status_word) != cudaSuccess || !addr) {
    (void)cudaGetLastError();  // leave no pending error for the caller's next runtime call
    return nullptr;
  }
  if (!have_id) have_id = current_context_id(&id);  // the lookup made the primary context current
  if (have_id) {
    std::lock_guard<std::mutex> lk(g_status_cache.mu);
    g_status_cache.ctx[dev] = id;
    g_status_cache.addr[dev] = (unsigned *)addr;
  }
  return (unsigned *)addr;
}

namespace {
// Failure-detection test settings; production calls never change them.
constexpr uint64_t kDefaultWaitNs = 2000000000ull;  // 2 s: far beyond any real wait
std::atomic<uint64_t> g_wait_ns{kDefaultWaitNs};
std::atomic<int> g_stall{0};
}  // namespace

uint64_t debug_wait_ns() { return g_wait_ns.load(std::memory_order_relaxed); }
int debug_stall() { return g_stall.load(std::memory_order_relaxed); }

}  // namespace kda

namespace {

bool supported_d(int d) { return d == 16 || d == 32 || d == 64 || d == 128; }

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

struct Range {
  uintptr_t lo, hi;  // [lo, hi)
};

Range range_of(const void *p, size_t bytes) {
  return Range{(uintptr_t)p, (uintptr_t)p + bytes};
}

bool overlap(Range a, Range b) { return a.lo < b.hi && b.lo < a.hi && a.lo != a.hi && b.lo != b.hi; }

// Device must be a Blackwell datacenter part (compute capability 10.x): the
// library is compiled for sm_100a only.
kda_status_t check_device() {
  int dev = 0, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return KDA_ERR_CUDA;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
    return KDA_ERR_CUDA;
  return major == 10 ? KDA_OK : KDA_ERR_UNSUPPORTED;
}

kda_status_t plan_prefill(int B, int H, int T, int dk, int dv, kda_dtype_t dtype, int chunk_size,
                          kda_plan_t *plan) {
  if (B < 0 || H < 0 || T < 0) return KDA_ERR_INVALID_ARG;
  if (dtype != KDA_DTYPE_F32 && dtype != KDA_DTYPE_BF16) return KDA_ERR_DTYPE;
  if (!supported_d(dk) || !supported_d(dv)) return KDA_ERR_SHAPE;
  if ((int64_t)B * H > (int64_t)INT32_MAX / 2) return KDA_ERR_SHAPE;
  if (chunk_size != 0 && chunk_size != 16 && chunk_size != 32) return KDA_ERR_SHAPE;
  const bool tc_ok = dtype == KDA_DTYPE_BF16 && dk == 128 && dv == 128;
  if (chunk_size == 32 && !tc_ok) return dtype == KDA_DTYPE_BF16 ? KDA_ERR_SHAPE : KDA_ERR_DTYPE;
  kda_plan_t p;
  const bool tc = chunk_size == 32 || (chunk_size == 0 && tc_ok);
  p.path = tc ? KDA_PATH_TC32 : KDA_PATH_SIMT16;
  p.chunk_size = tc ? 32 : 16;
  int seg_len = T;
  p.segments = 1;
  if (tc) kda::tc32_plan(B * H, T, &p.segments, &seg_len);
  p.segment_tokens = p.segments > 1 ? seg_len : T;
  p.launches = (B * H == 0) ? 0 : (p.segments > 1 ? 4 : 1);
  p.workspace = tc ? kda::tc32_workspace(B * H, T) : 0;
  *plan = p;
  return KDA_OK;
}

}  // namespace

extern "C" {

int kda_version(void) { return 100; }

const char *kda_status_string(kda_status_t s) {
  switch (s) {
    case KDA_OK: return "KDA_OK";
    case KDA_ERR_INVALID_ARG: return "KDA_ERR_INVALID_ARG: invalid argument";
    case KDA_ERR_SHAPE: return "KDA_ERR_SHAPE: unsupported shape";
    case KDA_ERR_DTYPE: return "KDA_ERR_DTYPE: unsupported dtype";
    case KDA_ERR_ALIGNMENT: return "KDA_ERR_ALIGNMENT: pointer misaligned";
    case KDA_ERR_ALIAS: return "KDA_ERR_ALIAS: output overlaps an input";
    case KDA_ERR_WORKSPACE: return "KDA_ERR_WORKSPACE: workspace missing or too small";
    case KDA_ERR_CUDA: return "KDA_ERR_CUDA: CUDA runtime error";
    case KDA_ERR_TIMEOUT: return "KDA_ERR_TIMEOUT: a bounded device wait gave up";
    case KDA_ERR_UNSUPPORTED: return "KDA_ERR_UNSUPPORTED: device or path not supported";
    case KDA_ERR_DEVICE: return "KDA_ERR_DEVICE: device-side check failed";
  }
  return "KDA_ERR_UNKNOWN";
}

kda_status_t kda_chunk_fwd_plan(int B, int H, int T, int dk, int dv, kda_dtype_t dtype,
                                int chunk_size, kda_plan_t *plan) {
  if (!plan) return KDA_ERR_INVALID_ARG;
  return plan_prefill(B, H, T, dk, dv, dtype, chunk_size, plan);
}

size_t kda_chunk_fwd_workspace_size(int B, int H, int T, int dk, int dv, kda_dtype_t dtype,
                                    int chunk_size) {
  kda_plan_t p;
  if (plan_prefill(B, H, T, dk, dv, dtype, chunk_size, &p) != KDA_OK) return (size_t)-1;
  return p.workspace;
}

}  // extern "C"

namespace {

// Optional parts of a prefill call: state checkpoints, the fused Eq. 5 gate
// (g then holds the logits z), the fused Eq. 6 output edge (o then receives y).
struct Extras {
  float *ckpt = nullptr;
  int ckpt_interval = 0;
  const float *A_log = nullptr;
  float g_min = 0.f;
  const void *gate = nullptr;
  const float *rms_w = nullptr;
  float eps = 0.f;
};

// kda_chunk_fwd and its variants.
kda_status_t chunk_fwd(const void *q, const void *k, const void *v, const void *g, const void *beta,
                       const float *h0, void *o, float *h_T, const Extras &x, int B, int H, int T, int dk, int dv,
                       kda_dtype_t dtype, int chunk_size, float scale, void *workspace, size_t workspace_bytes,
                       kda_stream_t stream) {
  float *const ckpt = x.ckpt;
  const int ckpt_interval = x.ckpt_interval;
  const float *const A_log = x.A_log;
  const float g_min = x.g_min;
  kda_plan_t plan;
  kda_status_t st = plan_prefill(B, H, T, dk, dv, dtype, chunk_size, &plan);
  if (st != KDA_OK) return st;
  if (!isfinite(scale)) return KDA_ERR_INVALID_ARG;
  const int n_ckpt = ckpt_interval > 0 ? T / ckpt_interval : 0;
  if (B * H == 0) return KDA_OK;
  if (T > 0 && (!q || !k || !v || !g || !beta || !o)) return KDA_ERR_INVALID_ARG;
  if (n_ckpt > 0 && !ckpt) return KDA_ERR_INVALID_ARG;
  if (A_log && ((uintptr_t)A_log & 3u) != 0) return KDA_ERR_ALIGNMENT;
  const size_t e = dtype == KDA_DTYPE_BF16 ? 2 : 4;
  const void *ptrs[] = {q, k, v, g, h0, o, h_T, workspace, n_ckpt > 0 ? ckpt : nullptr};
  for (const void *p : ptrs)
    if (p && !aligned16(p)) return KDA_ERR_ALIGNMENT;
  if (beta && ((uintptr_t)beta % e) != 0) return KDA_ERR_ALIGNMENT;
  if (plan.workspace > 0 && (!workspace || workspace_bytes < plan.workspace)) return KDA_ERR_WORKSPACE;

  const size_t n = (size_t)B * H;
  const Range rq = range_of(q, n * T * dk * e), rk = range_of(k, n * T * dk * e),
              rv = range_of(v, n * T * dv * e), rg = range_of(g, n * T * dk * e),
              rb = range_of(beta, n * T * e), rh0 = range_of(h0, h0 ? n * dk * dv * 4 : 0),
              ro = range_of(o, n * T * dv * e), rhT = range_of(h_T, h_T ? n * dk * dv * 4 : 0),
              rw = range_of(workspace, plan.workspace),
              rc = range_of(ckpt, n_ckpt > 0 ? n * n_ckpt * dk * dv * 4 : 0);
  const Range ins[] = {rq, rk, rv, rg, rb, rh0};
  for (const Range &r : ins)
    if (overlap(ro, r)) return KDA_ERR_ALIAS;
  for (int i = 0; i < 5; ++i)
    if (overlap(rhT, ins[i])) return KDA_ERR_ALIAS;
  if (h_T && h0 && overlap(rhT, rh0) && (const void *)h_T != (const void *)h0) return KDA_ERR_ALIAS;
  if (overlap(rhT, ro)) return KDA_ERR_ALIAS;
  for (const Range &r : ins)
    if (overlap(rw, r) || overlap(rc, r)) return KDA_ERR_ALIAS;
  if (overlap(rw, ro) || overlap(rw, rhT)) return KDA_ERR_ALIAS;
  if (overlap(rc, ro) || overlap(rc, rhT) || overlap(rc, rw)) return KDA_ERR_ALIAS;
  const Range ra = range_of(A_log, A_log ? (size_t)H * dk * 4 : 0);
  if (overlap(ra, ro) || overlap(ra, rhT) || overlap(ra, rw) || overlap(ra, rc)) return KDA_ERR_ALIAS;
  if (x.gate) {  // the output edge's inputs are read while y (in o) is written
    if (!aligned16(x.gate) || !aligned16(x.rms_w)) return KDA_ERR_ALIGNMENT;
    const Range rg2 = range_of(x.gate, n * T * dv * e), rw2 = range_of(x.rms_w, (size_t)H * dv * 4);
    if (overlap(rg2, ro) || overlap(rw2, ro) || overlap(rg2, rhT) || overlap(rw2, rhT) || overlap(rg2, rw) ||
        overlap(rw2, rw))
      return KDA_ERR_ALIAS;
  }

  st = check_device();
  if (st != KDA_OK) return st;

  kda::ChunkArgs a;
  a.q = q; a.k = k; a.v = v; a.g = g; a.beta = beta; a.h0 = h0; a.o = o; a.hT = h_T;
  a.B = B; a.H = H; a.T = T; a.dk = dk; a.dv = dv;
  a.bf16 = dtype == KDA_DTYPE_BF16;
  a.scale = scale > 0.f ? scale : 1.0f / sqrtf((float)dk);
  a.status = kda::device_status_ptr();
  a.workspace = workspace;
  a.segments = plan.segments;
  a.ckpt = n_ckpt > 0 ? ckpt : nullptr;
  a.ckpt_interval = ckpt_interval;
  a.n_ckpt = n_ckpt;
  a.A_log = A_log;
  a.g_min = g_min;
  a.wait_ns = kda::debug_wait_ns();
  a.stall = kda::debug_stall();
  a.gate = x.gate;
  a.rms_w = x.rms_w;
  a.eps = x.eps;
  if (!a.status) return KDA_ERR_CUDA;
  if (T == 0 && !h_T) return KDA_OK;
  // T == 0 is a pure state copy (h_T = h0, or zeros): the CUDA-core kernel does
  // that with no token to load, while the tensor-core path would need tensor
  // maps over empty (possibly null) tensors
  const bool tc = plan.path == KDA_PATH_TC32 && T > 0;
  // the CUDA-core kernel has no fused output edge: it writes o into y's buffer
  // and the edge kernel then turns it into y in place
  if (!tc) a.gate = nullptr;
  cudaError_t ce = tc ? kda::launch_chunk_tc32(a, (cudaStream_t)stream) : kda::launch_chunk_simt16(a, (cudaStream_t)stream);
  if (ce == cudaSuccess && !tc && x.gate && T > 0) {
    kda::OutGateArgs og;
    og.o = o; og.gate = x.gate; og.w = x.rms_w; og.y = o;
    og.B = B; og.H = H; og.T = T; og.dv = dv;
    og.bf16 = dtype == KDA_DTYPE_BF16;
    og.eps = x.eps;
    ce = kda::launch_out_gate(og, (cudaStream_t)stream);
  }
  return ce == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

}  // namespace

extern "C" {

kda_status_t kda_chunk_fwd(const void *q, const void *k, const void *v, const void *g,
                           const void *beta, const float *h0, void *o, float *h_T, int B, int H,
                           int T, int dk, int dv, kda_dtype_t dtype, int chunk_size, float scale,
                           void *workspace, size_t workspace_bytes, kda_stream_t stream) {
  return chunk_fwd(q, k, v, g, beta, h0, o, h_T, Extras(), B, H, T, dk, dv, dtype, chunk_size, scale, workspace,
                   workspace_bytes, stream);
}

kda_status_t kda_chunk_fwd_ckpt(const void *q, const void *k, const void *v, const void *g,
                                const void *beta, const float *h0, void *o, float *h_T, float *ckpt,
                                int ckpt_interval, int B, int H, int T, int dk, int dv,
                                kda_dtype_t dtype, int chunk_size, float scale, void *workspace,
                                size_t workspace_bytes, kda_stream_t stream) {
  if (ckpt_interval <= 0 || ckpt_interval % 64 != 0) return KDA_ERR_INVALID_ARG;
  Extras x;
  x.ckpt = ckpt;
  x.ckpt_interval = ckpt_interval;
  return chunk_fwd(q, k, v, g, beta, h0, o, h_T, x, B, H, T, dk, dv, dtype, chunk_size, scale, workspace,
                   workspace_bytes, stream);
}

kda_status_t kda_chunk_fwd_gated(const void *q, const void *k, const void *v, const void *z,
                                 const float *A_log, float g_min, const void *beta, const float *h0,
                                 void *o, float *h_T, int B, int H, int T, int dk, int dv,
                                 kda_dtype_t dtype, int chunk_size, float scale, void *workspace,
                                 size_t workspace_bytes, kda_stream_t stream) {
  if (!(g_min >= -5.f && g_min < 0.f)) return KDA_ERR_INVALID_ARG;  // also rejects NaN
  if (B > 0 && H > 0 && T > 0 && !A_log) return KDA_ERR_INVALID_ARG;
  Extras x;
  x.A_log = A_log;
  x.g_min = g_min;
  return chunk_fwd(q, k, v, z, beta, h0, o, h_T, x, B, H, T, dk, dv, dtype, chunk_size, scale, workspace,
                   workspace_bytes, stream);
}

kda_status_t kda_chunk_fwd_outgate(const void *q, const void *k, const void *v, const void *g, const void *beta,
                                   const float *h0, const void *gate, const float *rms_weight, float eps, void *y,
                                   float *h_T, int B, int H, int T, int dk, int dv, kda_dtype_t dtype,
                                   int chunk_size, float scale, void *workspace, size_t workspace_bytes,
                                   kda_stream_t stream) {
  if (!(eps >= 0.f) || !isfinite(eps)) return KDA_ERR_INVALID_ARG;
  if (B > 0 && H > 0 && T > 0 && (!gate || !rms_weight)) return KDA_ERR_INVALID_ARG;
  Extras x;
  x.gate = (B > 0 && H > 0 && T > 0) ? gate : nullptr;
  x.rms_w = rms_weight;
  x.eps = eps;
  return chunk_fwd(q, k, v, g, beta, h0, y, h_T, x, B, H, T, dk, dv, dtype, chunk_size, scale, workspace,
                   workspace_bytes, stream);
}

kda_status_t kda_chunk_transition(const void *k, const void *v, const void *g, const void *beta, float *St,
                                  float *M, int B, int H, int T, int dk, int dv, kda_dtype_t dtype,
                                  kda_stream_t stream) {
  if (B < 0 || H < 0 || T < 0) return KDA_ERR_INVALID_ARG;
  if (dtype != KDA_DTYPE_F32 && dtype != KDA_DTYPE_BF16) return KDA_ERR_DTYPE;
  if (!supported_d(dk) || !supported_d(dv)) return KDA_ERR_SHAPE;
  if ((int64_t)B * H > (int64_t)INT32_MAX / 2) return KDA_ERR_SHAPE;
  // the transition-only kernel is the tensor-core one
  if (dtype != KDA_DTYPE_BF16) return KDA_ERR_DTYPE;
  if (dk != 128 || dv != 128) return KDA_ERR_SHAPE;
  const size_t n = (size_t)B * H;
  if (n == 0) return KDA_OK;
  if (!St || !M || (T > 0 && (!k || !v || !g || !beta))) return KDA_ERR_INVALID_ARG;
  const void *ptrs[] = {T > 0 ? k : nullptr, T > 0 ? v : nullptr, T > 0 ? g : nullptr, St, M};
  for (const void *p : ptrs)
    if (p && !aligned16(p)) return KDA_ERR_ALIGNMENT;
  if (T > 0 && ((uintptr_t)beta & 1u) != 0) return KDA_ERR_ALIGNMENT;
  const size_t e = 2;
  const Range rk = range_of(k, n * T * dk * e), rv = range_of(v, n * T * dv * e), rg = range_of(g, n * T * dk * e),
              rb = range_of(beta, n * T * e), rs = range_of(St, n * dk * dv * 4), rm = range_of(M, n * dk * dk * 4);
  const Range ins[] = {rk, rv, rg, rb};
  for (const Range &r : ins)
    if (overlap(rs, r) || overlap(rm, r)) return KDA_ERR_ALIAS;
  if (overlap(rs, rm)) return KDA_ERR_ALIAS;
  kda_status_t st = check_device();
  if (st != KDA_OK) return st;
  kda::ChunkArgs a;
  memset(&a, 0, sizeof(a));
  a.k = k; a.v = v; a.g = g; a.beta = beta;
  a.B = B; a.H = H; a.T = T; a.dk = dk; a.dv = dv;
  a.bf16 = 1;
  a.scale = 1.f;
  a.status = kda::device_status_ptr();
  a.segments = 1;
  a.wait_ns = kda::debug_wait_ns();
  a.stall = kda::debug_stall();
  if (!a.status) return KDA_ERR_CUDA;
  return kda::launch_chunk_tc32_transition(a, St, M, (cudaStream_t)stream) == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

kda_status_t kda_output_gate(const void *o, const void *gate, const float *rms_weight, float eps, void *y,
                             int B, int H, int T, int dv, kda_dtype_t dtype, kda_stream_t stream) {
  if (B < 0 || H < 0 || T < 0) return KDA_ERR_INVALID_ARG;
  if (dtype != KDA_DTYPE_F32 && dtype != KDA_DTYPE_BF16) return KDA_ERR_DTYPE;
  if (!supported_d(dv)) return KDA_ERR_SHAPE;
  if ((int64_t)B * H > (int64_t)INT32_MAX / 2) return KDA_ERR_SHAPE;
  if (!(eps >= 0.f) || !isfinite(eps)) return KDA_ERR_INVALID_ARG;
  const size_t rows = (size_t)B * H * T;
  if (rows == 0) return KDA_OK;
  if (!o || !gate || !rms_weight || !y) return KDA_ERR_INVALID_ARG;
  const void *ptrs[] = {o, gate, rms_weight, y};
  for (const void *p : ptrs)
    if (!aligned16(p)) return KDA_ERR_ALIGNMENT;
  const size_t e = dtype == KDA_DTYPE_BF16 ? 2 : 4;
  const Range ro = range_of(o, rows * dv * e), rg = range_of(gate, rows * dv * e),
              rw = range_of(rms_weight, (size_t)H * dv * 4), ry = range_of(y, rows * dv * e);
  if (overlap(ry, rg) || overlap(ry, rw)) return KDA_ERR_ALIAS;
  if (overlap(ry, ro) && y != o) return KDA_ERR_ALIAS;
  kda_status_t st = check_device();
  if (st != KDA_OK) return st;
  kda::OutGateArgs a;
  a.o = o; a.gate = gate; a.w = rms_weight; a.y = y;
  a.B = B; a.H = H; a.T = T; a.dv = dv;
  a.bf16 = dtype == KDA_DTYPE_BF16;
  a.eps = eps;
  return kda::launch_out_gate(a, (cudaStream_t)stream) == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

kda_status_t kda_kcp_compose(const float *M, const float *St, const float *h0, float *S_in, int R, int B,
                             int H, int dk, int dv, kda_stream_t stream) {
  if (R < 0 || B < 0 || H < 0) return KDA_ERR_INVALID_ARG;
  if (!supported_d(dk) || !supported_d(dv)) return KDA_ERR_SHAPE;
  if ((int64_t)B * H > (int64_t)INT32_MAX / 2) return KDA_ERR_SHAPE;
  const size_t n = (size_t)B * H;
  if (n == 0) return KDA_OK;
  if (!S_in || (R > 0 && (!M || !St))) return KDA_ERR_INVALID_ARG;
  const void *ptrs[] = {R > 0 ? M : nullptr, R > 0 ? St : nullptr, h0, S_in};
  for (const void *p : ptrs)
    if (p && !aligned16(p)) return KDA_ERR_ALIGNMENT;
  const Range rs = range_of(S_in, n * dk * dv * 4), rm = range_of(M, R > 0 ? (size_t)R * n * dk * dk * 4 : 0),
              rt = range_of(St, R > 0 ? (size_t)R * n * dk * dv * 4 : 0), rh = range_of(h0, h0 ? n * dk * dv * 4 : 0);
  if (overlap(rs, rm) || overlap(rs, rt) || overlap(rs, rh)) return KDA_ERR_ALIAS;
  kda_status_t st = check_device();
  if (st != KDA_OK) return st;
  return kda::launch_kcp_compose(M, St, h0, S_in, R, (int)n, dk, dv, (cudaStream_t)stream) == cudaSuccess
             ? KDA_OK
             : KDA_ERR_CUDA;
}

namespace {
kda_status_t spec_replay(const void *q, const void *k, const void *v, const void *g, const void *beta, float *S,
                         void *o, const int *n_replay, int B, int H, int W, int dk, int dv, kda_dtype_t dtype,
                         float scale, const float *A_log, float g_min, const void *gate, const float *rms_w, float eps,
                         kda_stream_t stream);
}  // namespace

kda_status_t kda_spec_replay_verify_fused(const void *q, const void *k, const void *v, const void *z,
                                          const float *A_log, float g_min, const void *beta, float *S,
                                          const void *gate, const float *rms_weight, float eps, void *y,
                                          const int *n_replay, int B, int H, int W, int dk, int dv,
                                          kda_dtype_t dtype, float scale, kda_stream_t stream) {
  if (B < 0 || H < 0 || W < 0) return KDA_ERR_INVALID_ARG;
  if (dtype != KDA_DTYPE_F32 && dtype != KDA_DTYPE_BF16) return KDA_ERR_DTYPE;
  if (dk != 128 || dv != 128) return KDA_ERR_SHAPE;
  if (!(g_min >= -5.f && g_min < 0.f)) return KDA_ERR_INVALID_ARG;  // also rejects NaN
  if (!(eps >= 0.f) || !isfinite(eps)) return KDA_ERR_INVALID_ARG;
  if (B * H == 0 || W == 0) return KDA_OK;
  if (!A_log || !gate || !rms_weight) return KDA_ERR_INVALID_ARG;
  if (((uintptr_t)A_log & 3u) || ((uintptr_t)rms_weight & 3u)) return KDA_ERR_ALIGNMENT;
  const size_t e = dtype == KDA_DTYPE_BF16 ? 2 : 4;
  if ((uintptr_t)gate % e) return KDA_ERR_ALIGNMENT;
  const size_t n = (size_t)B * H;
  const Range ry = range_of(y, n * W * dv * e), rg = range_of(gate, n * W * dv * e),
              ra = range_of(A_log, (size_t)H * dk * 4), rw = range_of(rms_weight, (size_t)H * dv * 4),
              rS = range_of(S, n * dk * dv * 4);
  if (overlap(ry, rg) || overlap(ry, ra) || overlap(ry, rw) || overlap(rS, rg) || overlap(rS, ra) || overlap(rS, rw))
    return KDA_ERR_ALIAS;
  return spec_replay(q, k, v, z, beta, S, y, n_replay, B, H, W, dk, dv, dtype, scale, A_log, g_min, gate, rms_weight,
                     eps, stream);
}

kda_status_t kda_spec_replay_verify(const void *q, const void *k, const void *v, const void *g,
                                    const void *beta, float *S, void *o, const int *n_replay, int B,
                                    int H, int W, int dk, int dv, kda_dtype_t dtype, float scale,
                                    kda_stream_t stream) {
  return spec_replay(q, k, v, g, beta, S, o, n_replay, B, H, W, dk, dv, dtype, scale, nullptr, 0.f, nullptr, nullptr,
                     0.f, stream);
}

}  // extern "C"

namespace {
kda_status_t spec_replay(const void *q, const void *k, const void *v, const void *g, const void *beta, float *S,
                         void *o, const int *n_replay, int B, int H, int W, int dk, int dv, kda_dtype_t dtype,
                         float scale, const float *A_log, float g_min, const void *gate, const float *rms_w, float eps,
                         kda_stream_t stream) {
  if (B < 0 || H < 0 || W < 0) return KDA_ERR_INVALID_ARG;
  if (dtype != KDA_DTYPE_F32 && dtype != KDA_DTYPE_BF16) return KDA_ERR_DTYPE;
  if (!supported_d(dk) || !supported_d(dv)) return KDA_ERR_SHAPE;
  if ((int64_t)B * H > (int64_t)INT32_MAX / 2) return KDA_ERR_SHAPE;
  if (!isfinite(scale)) return KDA_ERR_INVALID_ARG;
  if (B * H == 0 || W == 0) return KDA_OK;
  if (!q || !k || !v || !g || !beta || !S || !o || !n_replay) return KDA_ERR_INVALID_ARG;
  const size_t e = dtype == KDA_DTYPE_BF16 ? 2 : 4;
  if (!aligned16(S) || ((uintptr_t)n_replay & 3u) != 0) return KDA_ERR_ALIGNMENT;
  const void *ptrs[] = {q, k, v, g, beta, o};
  for (const void *p : ptrs)
    if (((uintptr_t)p % e) != 0) return KDA_ERR_ALIGNMENT;
  const size_t n = (size_t)B * H;
  const Range rq = range_of(q, n * W * dk * e), rk = range_of(k, n * W * dk * e), rv = range_of(v, n * W * dv * e),
              rg = range_of(g, n * W * dk * e), rb = range_of(beta, n * W * e), rn = range_of(n_replay, (size_t)B * 4),
              rS = range_of(S, n * dk * dv * 4), ro = range_of(o, n * W * dv * e);
  const Range ins[] = {rq, rk, rv, rg, rb, rn};
  for (const Range &r : ins)
    if (overlap(ro, r) || overlap(rS, r)) return KDA_ERR_ALIAS;
  if (overlap(ro, rS)) return KDA_ERR_ALIAS;
  kda_status_t st = check_device();
  if (st != KDA_OK) return st;
  kda::SpecArgs a;
  a.q = q; a.k = k; a.v = v; a.g = g; a.beta = beta; a.S = S; a.o = o; a.n_replay = n_replay;
  a.B = B; a.H = H; a.W = W; a.dk = dk; a.dv = dv;
  a.bf16 = dtype == KDA_DTYPE_BF16;
  a.scale = scale > 0.f ? scale : 1.0f / sqrtf((float)dk);
  a.A_log = A_log;
  a.g_min = g_min;
  a.gate = gate;
  a.rms_w = rms_w;
  a.eps = eps;
  return kda::launch_spec_replay_verify(a, (cudaStream_t)stream) == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}
}  // namespace

extern "C" {

kda_status_t kda_recurrent_step(const void *q, const void *k, const void *v, const void *g,
                                const void *beta, float *S, void *o, int B, int H, int dk, int dv,
                                kda_dtype_t dtype, float scale, kda_stream_t stream) {
  if (B < 0 || H < 0) return KDA_ERR_INVALID_ARG;
  if (dtype != KDA_DTYPE_F32 && dtype != KDA_DTYPE_BF16) return KDA_ERR_DTYPE;
  if (!supported_d(dk) || !supported_d(dv)) return KDA_ERR_SHAPE;
  if ((int64_t)B * H > (int64_t)INT32_MAX / 2) return KDA_ERR_SHAPE;
  if (!isfinite(scale)) return KDA_ERR_INVALID_ARG;
  if (B * H == 0) return KDA_OK;
  if (!q || !k || !v || !g || !beta || !S || !o) return KDA_ERR_INVALID_ARG;
  const size_t e = dtype == KDA_DTYPE_BF16 ? 2 : 4;
  if (!aligned16(S)) return KDA_ERR_ALIGNMENT;
  const void *ptrs[] = {q, k, v, g, beta, o};
  for (const void *p : ptrs)
    if (((uintptr_t)p % e) != 0) return KDA_ERR_ALIGNMENT;
  const size_t n = (size_t)B * H;
  const Range rq = range_of(q, n * dk * e), rk = range_of(k, n * dk * e), rv = range_of(v, n * dv * e),
              rg = range_of(g, n * dk * e), rb = range_of(beta, n * e),
              rS = range_of(S, n * dk * dv * 4), ro = range_of(o, n * dv * e);
  const Range ins[] = {rq, rk, rv, rg, rb};
  for (const Range &r : ins)
    if (overlap(ro, r) || overlap(rS, r)) return KDA_ERR_ALIAS;
  if (overlap(ro, rS)) return KDA_ERR_ALIAS;
  kda_status_t st = check_device();
  if (st != KDA_OK) return st;
  kda::DecodeArgs a;
  a.q = q; a.k = k; a.v = v; a.g = g; a.beta = beta; a.S = S; a.o = o;
  a.B = B; a.H = H; a.dk = dk; a.dv = dv;
  a.bf16 = dtype == KDA_DTYPE_BF16;
  a.scale = scale > 0.f ? scale : 1.0f / sqrtf((float)dk);
  const cudaError_t ce = kda::launch_recurrent_step(a, (cudaStream_t)stream);
  return ce == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

kda_status_t kda_debug_set_wait_limit(unsigned long long ns) {
  kda::g_wait_ns.store(ns == 0 ? kda::kDefaultWaitNs : (uint64_t)ns, std::memory_order_relaxed);
  return KDA_OK;
}

kda_status_t kda_debug_inject_stall(int on) {
  kda::g_stall.store(on ? 1 : 0, std::memory_order_relaxed);
  return KDA_OK;
}

kda_status_t kda_get_device_status(kda_stream_t stream) {
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return KDA_ERR_CUDA;
  unsigned *p = kda::device_status_ptr();
  if (!p) return KDA_ERR_CUDA;
  unsigned w = 0;
  if (cudaMemcpy(&w, p, sizeof(w), cudaMemcpyDeviceToHost) != cudaSuccess) return KDA_ERR_CUDA;
  if (w != kda::kDevOk) {
    const unsigned zero = 0;
    if (cudaMemcpy(p, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess) return KDA_ERR_CUDA;
  }
  if (w == kda::kDevTimeout) return KDA_ERR_TIMEOUT;
  if (w != kda::kDevOk) return KDA_ERR_DEVICE;
  return KDA_OK;
}

}  // extern "C"
