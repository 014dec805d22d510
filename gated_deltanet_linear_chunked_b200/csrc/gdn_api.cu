// gdn_api.cu -- the C ABI (include/gdn.h): host-side validation and dispatch.
//
// Every entry point validates its arguments on the host before enqueueing
// anything, then launches onto the caller's stream and returns without
// synchronising.  Nothing here throws, aborts or prints.
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <new>

#include "gdn_internal.h"

namespace gdn {
namespace {

// Device error word set by kernels whose bounded waits expire.
__device__ unsigned int g_error_word;

constexpr long long kDefaultWaitLimit = 1LL << 26;
std::atomic<long long> g_wait_limit{kDefaultWaitLimit};

std::atomic<unsigned long long> g_launches{0};

constexpr int kMaxDevices = 64;
std::mutex g_err_mu;
unsigned int* g_err_ptr[kMaxDevices] = {};

// Device address of the error word on the current device.
cudaError_t error_word(unsigned int** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_err_mu);
  if (!g_err_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_error_word);
    if (e != cudaSuccess) return e;
    g_err_ptr[dev] = static_cast<unsigned int*>(p);
  }
  *out = g_err_ptr[dev];
  return cudaSuccess;
}

bool debug_sync() {
  const char* s = std::getenv("GDN_DEBUG_SYNC");
  return s && s[0] && std::strcmp(s, "0") != 0;
}

struct Range {
  uintptr_t lo, hi;  // [lo, hi)
};

Range range_of(const void* p, size_t bytes) {
  const uintptr_t lo = reinterpret_cast<uintptr_t>(p);
  return {lo, lo + bytes};
}

bool overlaps(Range a, Range b) {
  if (a.lo == a.hi || b.lo == b.hi) return false;
  return a.lo < b.hi && b.lo < a.hi;
}

bool aligned16(const void* p) {
  return (reinterpret_cast<uintptr_t>(p) & 15u) == 0;
}

bool supported_dim(int d) { return d >= 16 && d <= 128 && d % 16 == 0; }

// A pointer the current device can use as ordinary device memory.
gdn_status check_device_pointer(const void* p, int dev) {
  cudaPointerAttributes attr;
  const cudaError_t e = cudaPointerGetAttributes(&attr, p);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return GDN_ERR_CUDA;
  }
  if (attr.type == cudaMemoryTypeManaged) return GDN_OK;
  if (attr.type != cudaMemoryTypeDevice) return GDN_ERR_INVALID_ARG;
  if (attr.device != dev) return GDN_ERR_INVALID_ARG;
  return GDN_OK;
}

gdn_status finish(cudaStream_t s, cudaError_t launch_err, unsigned int* err) {
  if (launch_err != cudaSuccess) return GDN_ERR_CUDA;
  if (!debug_sync()) return GDN_OK;
  if (cudaStreamSynchronize(s) != cudaSuccess) return GDN_ERR_CUDA;
  if (err) {
    unsigned int word = 0;
    if (cudaMemcpy(&word, err, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess)
      return GDN_ERR_CUDA;
    if (word != kErrNone) {
      const unsigned int zero = 0;
      cudaMemcpy(err, &zero, sizeof(zero), cudaMemcpyHostToDevice);
      return GDN_ERR_TIMEOUT;
    }
  }
  return GDN_OK;
}

gdn_status scan(const void* q, const void* k, const void* v, const float* g,
                const float* beta, const float* state_in, float* state_out,
                void* out, int B, int T, int H, int Dk, int Dv, gdn_dtype dtype,
                int chunk, void* stream, bool bidir) {
  // ---- pure host checks (no CUDA call)
  if (dtype != GDN_F32 && dtype != GDN_BF16) return GDN_ERR_INVALID_ARG;
  if (B < 0 || T < 0 || H < 0 || Dk < 0 || Dv < 0) return GDN_ERR_INVALID_ARG;
  if (!supported_dim(Dk) || !supported_dim(Dv)) return GDN_ERR_UNSUPPORTED;
  if (chunk != 0 && chunk != 16 && chunk != 32 && chunk != 64)
    return GDN_ERR_INVALID_ARG;
  if (chunk == 0) chunk = 64;
  if (B == 0 || H == 0) return GDN_OK;

  const size_t es = dtype == GDN_BF16 ? 2 : 4;
  const size_t rows = (size_t)B * T * H;
  const size_t state_bytes = (size_t)B * H * Dk * Dv * sizeof(float);
  const Range rq = range_of(q, rows * Dk * es), rk = range_of(k, rows * Dk * es);
  const Range rv = range_of(v, rows * Dv * es), ro = range_of(out, rows * Dv * es);
  const Range rg = range_of(g, rows * 4), rb = range_of(beta, rows * 4);
  const Range rsi = range_of(state_in, state_in ? state_bytes : 0);
  const Range rso = range_of(state_out, state_out ? state_bytes : 0);

  if (T > 0 && (!q || !k || !v || !g || !beta || !out)) return GDN_ERR_INVALID_ARG;
  const void* ptrs[] = {q, k, v, g, beta, state_in, state_out, out};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return GDN_ERR_INVALID_ARG;
  if (T > 0) {
    for (Range r : {rq, rk, rv, rg, rb, rsi, rso})
      if (overlaps(ro, r)) return GDN_ERR_ALIAS;
    for (Range r : {rq, rk, rv, rg, rb})
      if (overlaps(rso, r)) return GDN_ERR_ALIAS;
  }
  if (state_in && state_out && state_in != state_out && overlaps(rsi, rso))
    return GDN_ERR_ALIAS;

  // ---- device checks
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return GDN_ERR_CUDA;
  }
  for (const void* p : ptrs) {
    if (!p) continue;
    if (T == 0 && p != state_in && p != state_out) continue;
    const gdn_status st = check_device_pointer(p, dev);
    if (st != GDN_OK) return st;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaGetLastError();  // start from a clean launch-error state

  if (T == 0) {
    if (!state_out) return GDN_OK;
    cudaError_t e = cudaSuccess;
    if (!state_in) e = cudaMemsetAsync(state_out, 0, state_bytes, s);
    else if (state_in != state_out)
      e = cudaMemcpyAsync(state_out, state_in, state_bytes, cudaMemcpyDeviceToDevice, s);
    return finish(s, e, nullptr);
  }

  unsigned int* err = nullptr;
  if (error_word(&err) != cudaSuccess) return GDN_ERR_CUDA;

  ScanArgs a;
  a.q = q; a.k = k; a.v = v; a.g = g; a.beta = beta;
  a.state_in = state_in; a.state_out = state_out; a.out = out;
  a.B = B; a.T = T; a.H = H; a.Dk = Dk; a.Dv = Dv;
  a.dtype = dtype; a.chunk = chunk; a.bidir = bidir; a.stream = s;
  a.err = err; a.wait_limit = g_wait_limit.load();

  cudaError_t e;
  if (dtype == GDN_F32) {
    e = launch_scan_serial(a);
  } else {
    // bf16: chunked tensor-core path with stream-ordered scratch
    void* ws = nullptr;
    const size_t bytes = chunk_tc_workspace_bytes(B, T, H, Dk, Dv, bidir);
    e = cudaMallocAsync(&ws, bytes, s);
    if (e == cudaSuccess) {
      e = launch_chunk_tc(a, ws);
      const cudaError_t f = cudaFreeAsync(ws, s);
      if (e == cudaSuccess) e = f;
    }
  }
  return finish(s, e, err);
}

}  // namespace

void count_launches(unsigned n) { g_launches.fetch_add(n); }

cudaError_t current_error_word(unsigned int** out) { return error_word(out); }
long long current_wait_limit() { return g_wait_limit.load(); }

// ------------------------------------------------------------- profiling
namespace {
struct Profile {
  std::mutex mu;
  bool armed = false;
  int capacity = 0, used = 0;
  cudaEvent_t* ev = nullptr;  // 2 per launch
  int* ids = nullptr;
};
Profile g_prof;
}  // namespace

ProfileScope::ProfileScope(cudaStream_t s, int kernel_id) : stream_(s), slot_(-1) {
  std::lock_guard<std::mutex> lock(g_prof.mu);
  if (!g_prof.armed || g_prof.used >= g_prof.capacity) return;
  slot_ = g_prof.used++;
  g_prof.ids[slot_] = kernel_id;
  cudaEventRecord(g_prof.ev[2 * slot_], stream_);
}

ProfileScope::~ProfileScope() {
  if (slot_ < 0) return;
  cudaEventRecord(g_prof.ev[2 * slot_ + 1], stream_);
}

}  // namespace gdn

extern "C" {

gdn_status gdn_chunk_fwd(const void* q, const void* k, const void* v,
                         const float* g, const float* beta,
                         const float* state_in, float* state_out, void* out,
                         int B, int T, int H, int Dk, int Dv, gdn_dtype dtype,
                         int chunk, void* stream) {
  return gdn::scan(q, k, v, g, beta, state_in, state_out, out, B, T, H, Dk, Dv,
                   dtype, chunk, stream, false);
}

gdn_status gdn_chunk_bidir(const void* q, const void* k, const void* v,
                           const float* g, const float* beta,
                           const float* state_in, float* state_out, void* out,
                           int B, int T, int H, int Dk, int Dv,
                           gdn_dtype dtype, int chunk, void* stream) {
  return gdn::scan(q, k, v, g, beta, state_in, state_out, out, B, T, H, Dk, Dv,
                   dtype, chunk, stream, true);
}

gdn_status gdn_state_reset(float* state, int B, int H, int Dk, int Dv,
                           void* stream) {
  if (B < 0 || H < 0 || Dk < 0 || Dv < 0) return GDN_ERR_INVALID_ARG;
  const size_t bytes = (size_t)B * H * Dk * Dv * sizeof(float);
  if (bytes == 0) return GDN_OK;
  if (!state || !gdn::aligned16(state)) return GDN_ERR_INVALID_ARG;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return GDN_ERR_CUDA;
  }
  const gdn_status st = gdn::check_device_pointer(state, dev);
  if (st != GDN_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return gdn::finish(s, cudaMemsetAsync(state, 0, bytes, s), nullptr);
}

gdn_status gdn_device_error(void* stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return GDN_ERR_CUDA;
  unsigned int* err = nullptr;
  if (gdn::error_word(&err) != cudaSuccess) return GDN_ERR_CUDA;
  unsigned int word = 0;
  if (cudaMemcpy(&word, err, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess)
    return GDN_ERR_CUDA;
  if (word == gdn::kErrNone) return GDN_OK;
  const unsigned int zero = 0;
  if (cudaMemcpy(err, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess)
    return GDN_ERR_CUDA;
  return GDN_ERR_TIMEOUT;
}

long long gdn_set_wait_limit(long long polls) {
  if (polls <= 0) polls = gdn::kDefaultWaitLimit;
  return gdn::g_wait_limit.exchange(polls);
}

const char* gdn_status_string(gdn_status status) {
  switch (status) {
    case GDN_OK: return "GDN_OK";
    case GDN_ERR_INVALID_ARG: return "GDN_ERR_INVALID_ARG";
    case GDN_ERR_UNSUPPORTED: return "GDN_ERR_UNSUPPORTED";
    case GDN_ERR_ALIAS: return "GDN_ERR_ALIAS";
    case GDN_ERR_CUDA: return "GDN_ERR_CUDA";
    case GDN_ERR_TIMEOUT: return "GDN_ERR_TIMEOUT";
    case GDN_ERR_SCRATCH_LIMIT: return "GDN_ERR_SCRATCH_LIMIT";
  }
  return "GDN_ERR_UNKNOWN";
}

int gdn_version(void) { return 100; }

unsigned long long gdn_launch_count(void) { return gdn::g_launches.load(); }

gdn_status gdn_profile_begin(int max_launches) {
  using gdn::g_prof;
  if (max_launches < 1) return GDN_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lock(g_prof.mu);
  if (g_prof.armed) return GDN_ERR_INVALID_ARG;
  g_prof.ev = new (std::nothrow) cudaEvent_t[2 * (size_t)max_launches];
  g_prof.ids = new (std::nothrow) int[max_launches];
  if (!g_prof.ev || !g_prof.ids) {
    delete[] g_prof.ev; delete[] g_prof.ids;
    g_prof.ev = nullptr; g_prof.ids = nullptr;
    return GDN_ERR_INVALID_ARG;
  }
  for (int i = 0; i < 2 * max_launches; ++i) {
    if (cudaEventCreate(&g_prof.ev[i]) != cudaSuccess) {
      for (int j = 0; j < i; ++j) cudaEventDestroy(g_prof.ev[j]);
      delete[] g_prof.ev; delete[] g_prof.ids;
      g_prof.ev = nullptr; g_prof.ids = nullptr;
      cudaGetLastError();
      return GDN_ERR_CUDA;
    }
  }
  g_prof.capacity = max_launches;
  g_prof.used = 0;
  g_prof.armed = true;
  return GDN_OK;
}

gdn_status gdn_profile_end(float* ms, int* n, int nids) {
  using gdn::g_prof;
  std::lock_guard<std::mutex> lock(g_prof.mu);
  if (!g_prof.armed) return GDN_ERR_INVALID_ARG;
  for (int i = 0; i < nids; ++i) {
    if (ms) ms[i] = 0.f;
    if (n) n[i] = 0;
  }
  gdn_status st = GDN_OK;
  for (int i = 0; i < g_prof.used; ++i) {
    float t = 0.f;
    if (cudaEventSynchronize(g_prof.ev[2 * i + 1]) != cudaSuccess ||
        cudaEventElapsedTime(&t, g_prof.ev[2 * i], g_prof.ev[2 * i + 1]) != cudaSuccess) {
      st = GDN_ERR_CUDA;
      cudaGetLastError();
      continue;
    }
    const int id = g_prof.ids[i];
    if (id >= 0 && id < nids) {
      if (ms) ms[id] += t;
      if (n) n[id] += 1;
    }
  }
  for (int i = 0; i < 2 * g_prof.capacity; ++i) cudaEventDestroy(g_prof.ev[i]);
  delete[] g_prof.ev; delete[] g_prof.ids;
  g_prof.ev = nullptr; g_prof.ids = nullptr;
  g_prof.capacity = g_prof.used = 0;
  g_prof.armed = false;
  return st;
}

const char* gdn_kernel_name(int id) {
  switch (id) {
    case gdn::kKernSerial: return "gdn_scan_serial_kernel";
    case gdn::kKernPrep: return "gdn_prep_kernel";
    case gdn::kKernRecur: return "gdn_recur_kernel";
    case gdn::kKernOutput: return "gdn_output_kernel";
  }
  return "unknown";
}

}  // extern "C"
