// extern "C" entry points of libs2attn.so: argument checks, workspace carving, kernel
// selection and launch, device status, and optional per-kernel event timing.
#include <math.h>
#include <stdint.h>

#include <mutex>
#include <vector>

#include <cudaTypedefs.h>

#include "../../include/s2attn.h"
#include "common.cuh"
#include "kernels.h"
#include "tc_kernels.h"

namespace s2 {
namespace {

// ----------------------------------------------------------------------------- profiling

enum KernelId {
  kRopeTable = 0,
  kRopePi,
  kFwdTc,
  kFwdSimt,
  kBwdRowsum,
  kBwdDkdvTc,
  kBwdDqTc,
  kBwdDqSimt,
  kBwdDkdvSimt,
  kNumKernels
};

const char* const kKernelNames[kNumKernels] = {
    "rope_table", "rope_pi", "fwd_tc", "fwd_simt", "bwd_rowsum", "bwd_dkdv_tc", "bwd_dq_tc",
    "bwd_dq_simt", "bwd_dkdv_simt"};

struct Record {
  int id;
  cudaEvent_t start, stop;
};

constexpr size_t kMaxRecords = 8192;

struct Profiler {
  std::mutex mu;
  bool on = false;
  int dropped = 0;
  std::vector<Record> pending;
  std::vector<cudaEvent_t> pool;
  int launches[kNumKernels] = {};
  double total_ms[kNumKernels] = {};

  cudaEvent_t get_event() {
    if (!pool.empty()) {
      cudaEvent_t e = pool.back();
      pool.pop_back();
      return e;
    }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    return e;
  }

  // Folds finished records into the totals; returns the first CUDA error seen.
  cudaError_t drain() {
    cudaError_t first = cudaSuccess;
    for (auto& r : pending) {
      float ms = 0.f;
      cudaError_t e = cudaEventSynchronize(r.stop);
      if (e == cudaSuccess) e = cudaEventElapsedTime(&ms, r.start, r.stop);
      if (e == cudaSuccess) {
        launches[r.id] += 1;
        total_ms[r.id] += ms;
      } else if (first == cudaSuccess) {
        first = e;
      }
      pool.push_back(r.start);
      pool.push_back(r.stop);
    }
    pending.clear();
    return first;
  }
};

Profiler& profiler() {
  static Profiler* p = new Profiler();  // never destroyed: events may outlive static teardown
  return *p;
}

// Launches `fn` on `st`; when profiling is on, brackets it with events on the same stream.
template <typename F>
cudaError_t timed_launch(int id, cudaStream_t st, F fn) {
  Profiler& pr = profiler();
  cudaEvent_t a = nullptr, b = nullptr;
  {
    std::lock_guard<std::mutex> lk(pr.mu);
    if (pr.on) {
      if (pr.pending.size() < kMaxRecords) {
        a = pr.get_event();
        b = pr.get_event();
        if (!a || !b) {
          if (a) pr.pool.push_back(a);
          if (b) pr.pool.push_back(b);
          a = b = nullptr;
          pr.dropped++;
        }
      } else {
        pr.dropped++;
      }
    }
  }
  if (a && cudaEventRecord(a, st) != cudaSuccess) return cudaGetLastError();
  cudaError_t e = fn();
  if (e != cudaSuccess) return e;
  if (a) {
    if (cudaEventRecord(b, st) != cudaSuccess) return cudaGetLastError();
    std::lock_guard<std::mutex> lk(pr.mu);
    pr.pending.push_back(Record{id, a, b});
  }
  return cudaSuccess;
}

// ----------------------------------------------------------------------------- arguments

constexpr size_t kAlign = 256;

inline size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

struct WsLayout {
  size_t qr, kr, cs, dsum, rowterms, status, total;
};

bool shape_ok(int B, int N, int Hq, int Hkv, int G) {
  if (B <= 0 || N <= 0 || Hq <= 0 || Hkv <= 0 || G <= 0) return false;
  if (G > N || N % G != 0 || G % 2 != 0) return false;
  if (Hq % 2 != 0 || Hkv % 2 != 0 || Hq % Hkv != 0) return false;
  // every index the kernels form per tensor must fit in 64 bits and rows in 32 bits
  if ((long long)B * N * Hq > (1LL << 31) - 1) return false;
  return true;
}

bool headdim_ok(int d) { return d >= 32 && d <= 256 && d % 32 == 0; }

bool dtype_ok(int dt) { return dt == S2_BF16 || dt == S2_FP32; }

WsLayout ws_layout(int B, int N, int Hq, int Hkv, int d, int dt) {
  // The status word sits at offset 0 so that s2attn_device_status() finds it without the
  // shape; the tensors follow, each on a 256-byte boundary.
  const size_t es = dt == S2_BF16 ? 2 : 4;
  WsLayout w;
  w.status = 0;
  size_t off = kAlign;
  w.qr = off;
  off = align_up(off + (size_t)B * Hq * N * d * es);
  w.kr = off;
  off = align_up(off + (size_t)B * Hkv * N * d * es);
  w.cs = off;
  off = align_up(off + (size_t)N * (d / 2) * sizeof(float2));
  w.dsum = off;
  off = align_up(off + (size_t)B * Hq * N * sizeof(float));
  w.rowterms = off;
  off = align_up(off + (size_t)B * Hq * N * 16 * 2);
  w.total = off;
  return w;
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

// tcgen05 kernels: bf16, d == 128, and G/2 a whole number of 128-row tiles (no tile
// straddles the wrap of the shifted heads).
bool tc_path(int d, int G, int dt) { return dt == S2_BF16 && d == 128 && G % 256 == 0; }

// RoPE+PI stage, then the forward kernel of the selected family.
cudaError_t enqueue_forward(const Params& p, int dt, cudaStream_t s) {
  const bool bf16 = dt == S2_BF16;
  cudaError_t e = timed_launch(kRopeTable, s, [&] { return launch_rope_table(p, s); });
  if (e == cudaSuccess) e = timed_launch(kRopePi, s, [&] { return launch_rope_pi(p, bf16, s); });
  if (e != cudaSuccess) return e;
  if (tc_path(p.d, p.G, dt)) return timed_launch(kFwdTc, s, [&] { return launch_tc_fwd(p, s); });
  return timed_launch(kFwdSimt, s, [&] { return launch_simt_fwd(p, bf16, s); });
}

// mode = S2_CAUSAL or 0, ORed with one S2_SHIFT_* pattern; nothing else.
bool mode_ok(int mode) {
  const int shift = mode & ~S2_CAUSAL;
  return shift == S2_SHIFT_HALF || shift == S2_SHIFT_ALTERNATE || shift == S2_SHIFT_NONE;
}

int shift_pattern(int mode) {
  const int shift = mode & ~S2_CAUSAL;
  return shift == S2_SHIFT_ALTERNATE ? kShiftAlternate
         : shift == S2_SHIFT_NONE    ? kShiftNone
                                     : kShiftHalf;
}

s2_status common_checks(int B, int N, int Hq, int Hkv, int d, int G, int mode, float s,
                        float base, int dt, void* ws, size_t ws_bytes) {
  if (!dtype_ok(dt)) return S2_ERR_DTYPE;
  if (!shape_ok(B, N, Hq, Hkv, G)) return S2_ERR_SHAPE;
  if (!headdim_ok(d)) return S2_ERR_HEADDIM;
  if (!(isfinite(s) && s > 0.f) || !(isfinite(base) && base > 0.f) || !mode_ok(mode))
    return S2_ERR_ARG;
  if (!ws) return S2_ERR_WORKSPACE;
  if (!aligned16(ws)) return S2_ERR_ALIGN;
  if (ws_bytes < ws_layout(B, N, Hq, Hkv, d, dt).total) return S2_ERR_WORKSPACE;
  return S2_OK;
}

Params make_params(int B, int N, int Hq, int Hkv, int d, int G, int mode, float s, float base,
                   int dt, void* ws) {
  Params p{};
  p.B = B; p.N = N; p.Hq = Hq; p.Hkv = Hkv; p.d = d; p.G = G;
  p.causal = mode & S2_CAUSAL;
  p.shift = shift_pattern(mode);
  p.pi_scale = s;
  p.rope_base = base;
  p.scale = (float)(1.0 / sqrt((double)d));
  p.scale_log2 = (float)(1.4426950408889634 / sqrt((double)d));
  WsLayout w = ws_layout(B, N, Hq, Hkv, d, dt);
  char* c = static_cast<char*>(ws);
  p.qr = c + w.qr;
  p.kr = c + w.kr;
  p.cs = reinterpret_cast<float2*>(c + w.cs);
  p.Dsum = reinterpret_cast<float*>(c + w.dsum);
  p.rowterms = c + w.rowterms;
  p.status = reinterpret_cast<unsigned*>(c + w.status);
  p.wait_limit_ns = kWaitLimitNs;
  p.inject = kInjectNone;
  return p;
}

s2_status to_status(cudaError_t e) { return e == cudaSuccess ? S2_OK : S2_ERR_CUDA; }

// FNV-1a (64-bit) over the arguments that determine the rotation a call leaves in (or
// expects from) the workspace. Set after the q and k pointers are.
void set_fingerprint(Params& p, int mode, int dtype) {
  uint64_t h = 1469598103934665603ull;
  auto mix = [&h](const void* x, size_t n) {
    const unsigned char* c = static_cast<const unsigned char*>(x);
    for (size_t i = 0; i < n; i++) h = (h ^ c[i]) * 1099511628211ull;
  };
  const int ints[8] = {p.B, p.N, p.Hq, p.Hkv, p.d, p.G, mode, dtype};
  mix(ints, sizeof(ints));
  mix(&p.pi_scale, sizeof(float));
  mix(&p.rope_base, sizeof(float));
  mix(&p.q, sizeof(void*));
  mix(&p.k, sizeof(void*));
  p.fingerprint = h;
}

}  // namespace
}  // namespace s2

using namespace s2;

extern "C" {

size_t s2attn_workspace_bytes(int B, int N, int H_q, int H_kv, int d, int dtype) {
  if (!dtype_ok(dtype) || !headdim_ok(d)) return 0;
  if (B <= 0 || N <= 0 || H_q <= 0 || H_kv <= 0 || H_q % 2 || H_kv % 2 || H_q % H_kv) return 0;
  return ws_layout(B, N, H_q, H_kv, d, dtype).total;
}

int s2attn_kernel_path(int B, int N, int H_q, int H_kv, int d, int G, int mode, int dtype) {
  if (!dtype_ok(dtype) || !shape_ok(B, N, H_q, H_kv, G) || !headdim_ok(d) || !mode_ok(mode))
    return -1;
  return tc_path(d, G, dtype) ? 1 : 0;
}

s2_status s2attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                     int N, int H_q, int H_kv, int d, int G, int mode, float pi_scale,
                     float rope_base, int dtype, void* workspace, size_t ws_bytes,
                     void* cuda_stream) {
  if (!q || !k || !v || !o || !lse) return S2_ERR_NULL;
  s2_status st = common_checks(B, N, H_q, H_kv, d, G, mode, pi_scale, rope_base, dtype,
                               workspace, ws_bytes);
  if (st != S2_OK) return st;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
    return S2_ERR_ALIGN;
  Params p = make_params(B, N, H_q, H_kv, d, G, mode, pi_scale, rope_base, dtype, workspace);
  p.q = q; p.k = k; p.v = v; p.o = o; p.lse = lse;
  set_fingerprint(p, mode, dtype);
  return to_status(enqueue_forward(p, dtype, static_cast<cudaStream_t>(cuda_stream)));
}

namespace s2 {
namespace {

// Shared body of the two backward entry points. rotate = false reuses the rotated q~, k~
// and the (cos, sin) table that the forward left in the workspace.
s2_status backward_impl(const void* q, const void* k, const void* v, const void* o,
                        const float* lse, const void* dout, void* dq, void* dk, void* dv, int B,
                        int N, int H_q, int H_kv, int d, int G, int mode, float pi_scale,
                        float rope_base, int dtype, void* workspace, size_t ws_bytes,
                        void* cuda_stream, bool rotate, int inject = kInjectNone) {
  if (!q || !k || !v || !o || !lse || !dout || !dq || !dk || !dv) return S2_ERR_NULL;
  s2_status st = common_checks(B, N, H_q, H_kv, d, G, mode, pi_scale, rope_base, dtype,
                               workspace, ws_bytes);
  if (st != S2_OK) return st;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse) ||
      !aligned16(dout) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
    return S2_ERR_ALIGN;
  Params p = make_params(B, N, H_q, H_kv, d, G, mode, pi_scale, rope_base, dtype, workspace);
  p.q = q; p.k = k; p.v = v; p.o = const_cast<void*>(o); p.lse = const_cast<float*>(lse);
  p.dout = dout; p.dq = dq; p.dk = dk; p.dv = dv;
  set_fingerprint(p, mode, dtype);
  p.check_fingerprint = !rotate;
  if (inject != kInjectNone) {
    p.inject = inject;
    p.wait_limit_ns = kSelftestWaitLimitNs;
  }
  const bool bf16 = dtype == S2_BF16;
  cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
  cudaError_t e = cudaSuccess;
  if (rotate) {
    e = timed_launch(kRopeTable, s, [&] { return launch_rope_table(p, s); });
    if (e == cudaSuccess) e = timed_launch(kRopePi, s, [&] { return launch_rope_pi(p, bf16, s); });
  }
  if (e == cudaSuccess)
    e = timed_launch(kBwdRowsum, s, [&] { return launch_bwd_rowsum(p, bf16, s); });
  if (e != cudaSuccess) return to_status(e);
  if (tc_path(d, G, dtype)) {
    e = timed_launch(kBwdDkdvTc, s, [&] { return launch_tc_bwd_dkdv(p, s); });
    if (e == cudaSuccess) e = timed_launch(kBwdDqTc, s, [&] { return launch_tc_bwd_dq(p, s); });
  } else {
    e = timed_launch(kBwdDkdvSimt, s, [&] { return launch_simt_dkdv(p, bf16, s); });
    if (e == cudaSuccess)
      e = timed_launch(kBwdDqSimt, s, [&] { return launch_simt_dq(p, bf16, s); });
  }
  return to_status(e);
}

}  // namespace
}  // namespace s2

s2_status s2attn_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
                     const void* dout, void* dq, void* dk, void* dv, int B, int N, int H_q,
                     int H_kv, int d, int G, int mode, float pi_scale, float rope_base,
                     int dtype, void* workspace, size_t ws_bytes, void* cuda_stream) {
  return backward_impl(q, k, v, o, lse, dout, dq, dk, dv, B, N, H_q, H_kv, d, G, mode,
                       pi_scale, rope_base, dtype, workspace, ws_bytes, cuda_stream, true);
}

s2_status s2attn_bwd_after_fwd(const void* q, const void* k, const void* v, const void* o,
                               const float* lse, const void* dout, void* dq, void* dk, void* dv,
                               int B, int N, int H_q, int H_kv, int d, int G, int mode,
                               float pi_scale, float rope_base, int dtype, void* workspace,
                               size_t ws_bytes, void* cuda_stream) {
  return backward_impl(q, k, v, o, lse, dout, dq, dk, dv, B, N, H_q, H_kv, d, G, mode,
                       pi_scale, rope_base, dtype, workspace, ws_bytes, cuda_stream, false);
}

s2_status s2attn_device_status(void* workspace, size_t ws_bytes, void* cuda_stream) {
  if (!workspace) return S2_ERR_NULL;
  if (ws_bytes < kAlign) return S2_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
  unsigned word = 0;
  if (cudaMemcpyAsync(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return S2_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return S2_ERR_CUDA;
  if (word != 0) {
    if (cudaMemsetAsync(workspace, 0, sizeof(word), s) != cudaSuccess) return S2_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return S2_ERR_CUDA;
    return (word & kStatusStale) ? S2_ERR_STALE_WORKSPACE : S2_ERR_DEVICE_TIMEOUT;
  }
  return S2_OK;
}

s2_status s2attn_selftest_wait_timeout(void* workspace, size_t ws_bytes, void* cuda_stream) {
  if (!workspace) return S2_ERR_NULL;
  if (ws_bytes < kAlign) return S2_ERR_WORKSPACE;
  if (!aligned16(workspace)) return S2_ERR_ALIGN;
  return to_status(launch_wait_timeout_selftest(static_cast<unsigned*>(workspace),
                                                kSelftestWaitLimitNs,
                                                static_cast<cudaStream_t>(cuda_stream)));
}

s2_status s2attn_selftest_inject(int site, const void* q, const void* k, const void* v, void* o,
                                 float* lse, const void* dout, void* dq, void* dk, void* dv, int B,
                                 int N, int H_q, int H_kv, int d, int G, int mode,
                                 float pi_scale, float rope_base, int dtype, void* workspace,
                                 size_t ws_bytes, void* cuda_stream) {
  if (site != S2_INJECT_FWD && site != S2_INJECT_DKDV) return S2_ERR_ARG;
  if (s2attn_kernel_path(B, N, H_q, H_kv, d, G, mode, dtype) != 1) return S2_ERR_ARG;
  if (site == S2_INJECT_DKDV)
    return backward_impl(q, k, v, o, lse, dout, dq, dk, dv, B, N, H_q, H_kv, d, G, mode,
                         pi_scale, rope_base, dtype, workspace, ws_bytes, cuda_stream, true,
                         kInjectDkdv);
  if (!q || !k || !v || !o || !lse) return S2_ERR_NULL;
  s2_status st = common_checks(B, N, H_q, H_kv, d, G, mode, pi_scale, rope_base, dtype,
                               workspace, ws_bytes);
  if (st != S2_OK) return st;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
    return S2_ERR_ALIGN;
  Params p = make_params(B, N, H_q, H_kv, d, G, mode, pi_scale, rope_base, dtype, workspace);
  p.q = q; p.k = k; p.v = v; p.o = o; p.lse = lse;
  set_fingerprint(p, mode, dtype);
  p.inject = kInjectFwd;
  p.wait_limit_ns = kSelftestWaitLimitNs;
  return to_status(enqueue_forward(p, dtype, static_cast<cudaStream_t>(cuda_stream)));
}

s2_status s2attn_selftest_exp2(const float* x, float* y, int n, void* cuda_stream) {
  if (!x || !y) return S2_ERR_NULL;
  if (n <= 0) return S2_ERR_ARG;
  return to_status(launch_exp2_poly_selftest(x, y, n, static_cast<cudaStream_t>(cuda_stream)));
}

const char* s2attn_status_string(int status) {
  switch (status) {
    case S2_OK: return "ok";
    case S2_ERR_NULL: return "a required pointer is NULL";
    case S2_ERR_SHAPE: return "invalid shape (B,N,H_q,H_kv,G > 0; G <= N; N % G == 0; G, H_q, "
                              "H_kv even; H_q % H_kv == 0)";
    case S2_ERR_DTYPE: return "unknown dtype";
    case S2_ERR_HEADDIM: return "head dim d must be a multiple of 32 in [32, 256]";
    case S2_ERR_ALIGN: return "a pointer is not 16-byte aligned";
    case S2_ERR_WORKSPACE: return "workspace missing or smaller than s2attn_workspace_bytes()";
    case S2_ERR_CUDA: return "a CUDA call failed";
    case S2_ERR_DEVICE_TIMEOUT: return "a bounded device-side wait expired";
    case S2_ERR_ARG: return "invalid argument (pi_scale, rope_base finite and > 0; mode = "
                             "S2_CAUSAL or 0 | one S2_SHIFT_* pattern)";
    case S2_ERR_STALE_WORKSPACE: return "s2attn_bwd_after_fwd: the workspace's rotation "
                                        "belongs to another forward (other q, k or arguments)";
    default: return "unknown status";
  }
}

s2_status s2attn_profile_enable(int on) {
  Profiler& pr = profiler();
  std::lock_guard<std::mutex> lk(pr.mu);
  cudaError_t e = pr.drain();
  if (on) {
    for (int i = 0; i < kNumKernels; i++) {
      pr.launches[i] = 0;
      pr.total_ms[i] = 0.0;
    }
    pr.dropped = 0;
  }
  pr.on = on != 0;
  return to_status(e);
}

int s2attn_profile_num_kernels(void) { return kNumKernels; }

s2_status s2attn_profile_query(int kernel_id, const char** name, int* launches,
                               double* total_ms) {
  if (kernel_id < 0 || kernel_id >= kNumKernels) return S2_ERR_ARG;
  Profiler& pr = profiler();
  std::lock_guard<std::mutex> lk(pr.mu);
  cudaError_t e = pr.drain();
  if (name) *name = kKernelNames[kernel_id];
  if (launches) *launches = pr.launches[kernel_id];
  if (total_ms) *total_ms = pr.total_ms[kernel_id];
  return to_status(e);
}

int s2attn_profile_dropped(void) {
  Profiler& pr = profiler();
  std::lock_guard<std::mutex> lk(pr.mu);
  return pr.dropped;
}

}  // extern "C"

// ----------------------------------------------------------------------------- no-allocation forward
//
// Some callers must not allocate device memory for a call: a plugin whose host application
// owns every device allocation, a latency-critical loop that cannot afford cudaMalloc's
// implicit device synchronisation, or a plain C caller with no allocator at hand. For them
// s2attn_fwd_noalloc runs the same kernels as s2attn_fwd, with the workspace replaced by a
// fixed array compiled into this library (allocated by the driver when the library's
// device code is loaded, held by every device that loads it until the process exits).
namespace s2 {
namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[S2ATTN_NOALLOC_SCRATCH_BYTES];

// The current CUDA context (cuCtxGetCurrent, reached through the runtime's driver
// entry-point query so that the library does not link libcuda directly), or null.
CUcontext current_context() {
  static PFN_cuCtxGetCurrent_v4000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &f, 4000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(f);
  });
  CUcontext ctx = nullptr;
  if (!fn || fn(&ctx) != CUDA_SUCCESS) return nullptr;
  return ctx;
}

// Device address of g_noalloc_scratch on the current device. In host code the array's
// name is only a host-side stand-in, so the address is looked up with the device current,
// once per device, and cached together with the context it belongs to: after a device
// reset the device has a new context, the library's device code is loaded again and the
// array may sit elsewhere, so a changed context makes the lookup run again.
cudaError_t noalloc_scratch_address(void** out) {
  static std::mutex mu;
  struct Entry {
    CUcontext ctx;
    void* addr;
  };
  static std::vector<Entry> cache;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lk(mu);
  if ((int)cache.size() <= dev) cache.resize(dev + 1, Entry{nullptr, nullptr});
  Entry& c = cache[dev];
  // A thread that has not yet used the runtime has no current context (null): the lookup
  // below then binds the device's context to it.
  CUcontext ctx = current_context();
  if (!c.addr || !ctx || c.ctx != ctx) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    c.addr = p;
    c.ctx = current_context();
  }
  *out = c.addr;
  return cudaSuccess;
}

}  // namespace
}  // namespace s2

extern "C" s2_status s2attn_fwd_noalloc(const void* q, const void* k, const void* v, void* o,
                                        float* lse, int B, int N, int H_q, int H_kv, int d, int G,
                                        int mode, float pi_scale, float rope_base, int dtype,
                                        void* cuda_stream) {
  if (!q || !k || !v || !o || !lse) return S2_ERR_NULL;
  if (!dtype_ok(dtype)) return S2_ERR_DTYPE;
  if (!shape_ok(B, N, H_q, H_kv, G)) return S2_ERR_SHAPE;
  if (!headdim_ok(d)) return S2_ERR_HEADDIM;
  if (!(isfinite(pi_scale) && pi_scale > 0.f) || !(isfinite(rope_base) && rope_base > 0.f) ||
      !mode_ok(mode))
    return S2_ERR_ARG;
  if (ws_layout(B, N, H_q, H_kv, d, dtype).total > (size_t)S2ATTN_NOALLOC_SCRATCH_BYTES)
    return S2_ERR_WORKSPACE;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
    return S2_ERR_ALIGN;
  void* scratch = nullptr;
  if (noalloc_scratch_address(&scratch) != cudaSuccess) return S2_ERR_CUDA;
  // The status word at the start of the scratch is reset by the first kernel of the call;
  // everything else the kernels read from the scratch is written earlier in the same call.
  Params p = make_params(B, N, H_q, H_kv, d, G, mode, pi_scale, rope_base, dtype, scratch);
  p.q = q; p.k = k; p.v = v; p.o = o; p.lse = lse;
  set_fingerprint(p, mode, dtype);
  return to_status(enqueue_forward(p, dtype, static_cast<cudaStream_t>(cuda_stream)));
}

extern "C" s2_status s2attn_noalloc_device_status(void* cuda_stream) {
  void* scratch = nullptr;
  if (noalloc_scratch_address(&scratch) != cudaSuccess) return S2_ERR_CUDA;
  // The word sits at offset 0 of the scratch, exactly where a workspace keeps it.
  return s2attn_device_status(scratch, S2ATTN_NOALLOC_SCRATCH_BYTES, cuda_stream);
}
