// gdn_api.cu -- the C ABI (include/gdn.h): host-side validation and dispatch.
//
// Every entry point validates its arguments on the host before it enqueues
// anything -- first every check that needs no CUDA call, then that each
// pointer is device memory of the current device -- then launches onto the
// caller's stream and returns without synchronising.  Nothing here throws,
// aborts or prints.
//
// Per-stream context.  The chunked path needs scratch between its kernels,
// and every bounded wait needs a word to report an expiry in.  Both are kept
// per (device, stream): the first call on a stream allocates them
// (cudaMalloc), later calls reuse them, and a larger problem replaces the
// scratch with a larger one.  Calls on one stream are ordered, so they can
// share the scratch; calls on different streams never share anything.  A
// replaced scratch buffer is not freed (a captured CUDA graph may still name
// it) until gdn_workspace_release.  A call made while its stream is being
// captured, on a stream with no context yet or with too small a scratch,
// cannot allocate outside the graph: it falls back to a stream-ordered
// allocation (captured as graph memory nodes) and to the device-wide error
// word.
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <functional>
#include <mutex>
#include <new>
#include <thread>
#include <vector>

#include "gdn_internal.h"

namespace gdn {
namespace {

// Device-wide error word: used by calls without a per-stream context (the
// allocation-free entry point, and calls captured before their stream had a
// context).
__device__ unsigned int g_error_word;

constexpr long long kDefaultWaitLimit = 1LL << 26;
std::atomic<long long> g_wait_limit{kDefaultWaitLimit};

std::atomic<unsigned long long> g_launches{0};
std::atomic<int> g_time_segments{0};

constexpr int kMaxDevices = 64;
std::mutex g_err_mu;
unsigned int* g_err_ptr[kMaxDevices] = {};

// Device address of the device-wide error word on the current device.
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

// Reads and clears one error word; GDN_ERR_TIMEOUT if it was set.
gdn_status take_error(unsigned int* err) {
  unsigned int word = 0;
  if (cudaMemcpy(&word, err, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess) {
    cudaGetLastError();
    return GDN_ERR_CUDA;
  }
  if (word == kErrNone) return GDN_OK;
  const unsigned int zero = 0;
  if (cudaMemcpy(err, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess) {
    cudaGetLastError();
    return GDN_ERR_CUDA;
  }
  return GDN_ERR_TIMEOUT;
}

// ------------------------------------------------------ per-stream contexts
struct StreamCtx {
  int dev;
  cudaStream_t stream;
  size_t thread;        // owning host thread for the per-thread default stream, else 0
  unsigned int* err;    // error word of this stream's calls
  void* ws;             // chunked-path scratch
  size_t ws_bytes;
};

std::mutex g_ctx_mu;
std::vector<StreamCtx*> g_ctx;
struct Retired {
  int dev;
  void* p;
};
std::vector<Retired> g_retired;  // scratch buffers replaced by larger ones

size_t thread_key(cudaStream_t s) {
  if (s != cudaStreamPerThread) return 0;
  return std::hash<std::thread::id>()(std::this_thread::get_id()) | 1u;
}

bool capturing(cudaStream_t s) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  const cudaError_t e = cudaStreamIsCapturing(s, &cs);
  if (e != cudaSuccess) {  // e.g. the legacy stream while another stream captures
    cudaGetLastError();
    return true;
  }
  return cs != cudaStreamCaptureStatusNone;
}

// The error word and scratch of (dev, s), the context created or its scratch
// grown to at least `bytes` as needed.  Both are copied out under the lock.
// Sets them to nullptr (and returns GDN_OK) when the stream is being captured
// and its context cannot serve the call as it is.
gdn_status stream_context(int dev, cudaStream_t s, size_t bytes, unsigned int** err,
                          void** ws) {
  *err = nullptr;
  *ws = nullptr;
  const size_t tk = thread_key(s);
  std::lock_guard<std::mutex> lock(g_ctx_mu);
  StreamCtx* c = nullptr;
  for (StreamCtx* x : g_ctx)
    if (x->dev == dev && x->stream == s && x->thread == tk) c = x;
  if (!(c && c->ws_bytes >= bytes)) {
    if (capturing(s)) return GDN_OK;
    if (!c) {
      void* p = nullptr;
      if (cudaMalloc(&p, 256) != cudaSuccess) {
        cudaGetLastError();
        return GDN_ERR_CUDA;
      }
      if (cudaMemsetAsync(p, 0, 256, s) != cudaSuccess) {
        cudaGetLastError();
        cudaFree(p);
        return GDN_ERR_CUDA;
      }
      c = new (std::nothrow) StreamCtx{dev, s, tk, static_cast<unsigned int*>(p), nullptr, 0};
      if (!c) {
        cudaFree(p);
        return GDN_ERR_CUDA;
      }
      g_ctx.push_back(c);
    }
    if (bytes > c->ws_bytes) {
      const size_t grain = size_t(2) << 20;
      const size_t nb = (bytes + grain - 1) / grain * grain;
      void* p = nullptr;
      if (cudaMalloc(&p, nb) != cudaSuccess) {
        cudaGetLastError();
        return GDN_ERR_CUDA;
      }
      if (c->ws) g_retired.push_back({dev, c->ws});
      c->ws = p;
      c->ws_bytes = nb;
    }
  }
  *err = c->err;
  *ws = c->ws;
  return GDN_OK;
}

gdn_status scan(const void* q, const void* k, const void* v, const void* g,
                const void* beta, const float* state_in, float* state_out,
                void* out, int B, int T, int H, int Dk, int Dv, gdn_dtype dtype,
                int chunk, void* stream, bool bidir, bool gate_logits) {
  ScanArgs a;
  int dev = 0;
  gdn_status st = prepare_scan(q, k, v, g, beta, state_in, state_out, out, B, T, H, Dk, Dv,
                               dtype, chunk, stream, bidir, gate_logits, &a, &dev);
  if (st != GDN_OK) return st;
  if (a.B == 0 || a.H == 0) return GDN_OK;
  if (a.T == 0) return trivial_state_copy(a);

  const size_t bytes =
      dtype == GDN_BF16 ? chunk_tc_workspace_bytes(B, T, H, Dk, Dv, bidir) : 0;
  void* ws = nullptr;
  st = stream_context(dev, a.stream, bytes, &a.err, &ws);
  if (st != GDN_OK) return st;
  if (!a.err && error_word(&a.err) != cudaSuccess) {
    cudaGetLastError();
    return GDN_ERR_CUDA;
  }
  a.wait_limit = g_wait_limit.load();

  cudaError_t e;
  if (dtype == GDN_F32) {
    e = launch_scan_serial(a);
  } else if (ws) {
    e = launch_chunk_tc(a, ws);
  } else {
    // under capture without a large enough cached scratch: stream-ordered
    // allocation, captured as graph memory nodes
    e = cudaMallocAsync(&ws, bytes, a.stream);
    if (e == cudaSuccess) {
      e = launch_chunk_tc(a, ws);
      const cudaError_t f = cudaFreeAsync(ws, a.stream);
      if (e == cudaSuccess) e = f;
    }
  }
  return finish(a.stream, e, a.err);
}

}  // namespace

gdn_status check_scan_host(const void* q, const void* k, const void* v, const void* g,
                           const void* beta, const float* state_in, float* state_out,
                           void* out, int B, int T, int H, int Dk, int Dv, gdn_dtype dtype,
                           int chunk, void* stream, bool bidir, bool gate_logits, ScanArgs* a) {
  if (dtype != GDN_F32 && dtype != GDN_BF16) return GDN_ERR_INVALID_ARG;
  if (B < 0 || T < 0 || H < 0 || Dk < 0 || Dv < 0) return GDN_ERR_INVALID_ARG;
  if (!supported_dim(Dk) || !supported_dim(Dv)) return GDN_ERR_UNSUPPORTED;
  if (chunk != 0 && chunk != 16 && chunk != 32 && chunk != 64)
    return GDN_ERR_INVALID_ARG;
  if (chunk == 0) chunk = 64;

  a->q = q; a->k = k; a->v = v; a->g = g; a->beta = beta;
  a->state_in = state_in; a->state_out = state_out; a->out = out;
  a->B = B; a->T = T; a->H = H; a->Dk = Dk; a->Dv = Dv;
  a->dtype = dtype; a->chunk = chunk; a->bidir = bidir; a->gate_logits = gate_logits;
  a->stream = static_cast<cudaStream_t>(stream);
  a->err = nullptr;
  a->wait_limit = 0;
  if (B == 0 || H == 0) return GDN_OK;

  const size_t es = dtype == GDN_BF16 ? 2 : 4;
  const size_t rows = (size_t)B * T * H;
  const size_t state_bytes = (size_t)B * H * Dk * Dv * sizeof(float);
  const Range rq = range_of(q, rows * Dk * es), rk = range_of(k, rows * Dk * es);
  const Range rv = range_of(v, rows * Dv * es), ro = range_of(out, rows * Dv * es);
  const size_t gs = gate_logits ? es : 4;  // logits come in the I/O dtype
  const Range rg = range_of(g, rows * gs), rb = range_of(beta, rows * gs);
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
  return GDN_OK;
}

gdn_status check_scan_device(const ScanArgs& a, int* dev_out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return GDN_ERR_CUDA;
  }
  const void* ptrs[] = {a.q, a.k, a.v, a.g, a.beta, a.state_in, a.state_out, a.out};
  for (const void* p : ptrs) {
    if (!p) continue;
    if (a.T == 0 && p != a.state_in && p != a.state_out) continue;
    const gdn_status st = check_device_pointer(p, dev);
    if (st != GDN_OK) return st;
  }
  cudaGetLastError();  // start from a clean launch-error state
  *dev_out = dev;
  return GDN_OK;
}

gdn_status prepare_scan(const void* q, const void* k, const void* v, const void* g,
                        const void* beta, const float* state_in, float* state_out,
                        void* out, int B, int T, int H, int Dk, int Dv, gdn_dtype dtype,
                        int chunk, void* stream, bool bidir, bool gate_logits, ScanArgs* a,
                        int* dev_out) {
  *dev_out = 0;
  const gdn_status st = check_scan_host(q, k, v, g, beta, state_in, state_out, out, B, T, H, Dk,
                                        Dv, dtype, chunk, stream, bidir, gate_logits, a);
  if (st != GDN_OK || B == 0 || H == 0) return st;
  return check_scan_device(*a, dev_out);
}

gdn_status trivial_state_copy(const ScanArgs& a) {
  if (!a.state_out) return GDN_OK;
  const size_t state_bytes = (size_t)a.B * a.H * a.Dk * a.Dv * sizeof(float);
  cudaError_t e = cudaSuccess;
  if (!a.state_in)
    e = cudaMemsetAsync(a.state_out, 0, state_bytes, a.stream);
  else if (a.state_in != a.state_out)
    e = cudaMemcpyAsync(a.state_out, a.state_in, state_bytes, cudaMemcpyDeviceToDevice, a.stream);
  return finish(a.stream, e, nullptr);
}

gdn_status finish(cudaStream_t s, cudaError_t launch_err, unsigned int* err) {
  if (launch_err != cudaSuccess) {
    cudaGetLastError();
    return GDN_ERR_CUDA;
  }
  if (!debug_sync()) return GDN_OK;
  if (cudaStreamSynchronize(s) != cudaSuccess) {
    cudaGetLastError();
    return GDN_ERR_CUDA;
  }
  return err ? take_error(err) : GDN_OK;
}

void count_launches(unsigned n) { g_launches.fetch_add(n); }

gdn_status stream_scratch(int dev, cudaStream_t s, size_t bytes, unsigned int** err, void** ws) {
  return stream_context(dev, s, bytes, err, ws);
}

namespace {
gdn_status backward(const void* q, const void* k, const void* v, const float* g,
                    const float* beta, const float* state_in, const void* d_out,
                    const float* d_state_out, void* dq, void* dk, void* dv, float* dg,
                    float* dbeta, float* d_state_in, int B, int T, int H, int Dk, int Dv,
                    gdn_dtype dtype, void* stream, bool bidir) {
  // the forward's host checks on the forward's arguments (out := d_out, which
  // is only read here; state_out := d_state_in, written), then the gradients'
  // host checks, then the device checks of both: a bad argument is reported
  // before any CUDA call
  ScanArgs a;
  int dev = 0;
  gdn_status st = check_scan_host(q, k, v, g, beta, state_in, d_state_in,
                                  const_cast<void*>(d_out), B, T, H, Dk, Dv, dtype, 0, stream,
                                  bidir, false, &a);
  if (st != GDN_OK) return st;
  if (B == 0 || H == 0) return GDN_OK;
  const size_t es = dtype == GDN_BF16 ? 2 : 4;
  const size_t rows = (size_t)B * T * H;
  const size_t sbytes = (size_t)B * H * Dk * Dv * 4;
  if (T > 0 && (!dq || !dk || !dv || !dg || !dbeta)) return GDN_ERR_INVALID_ARG;
  const void* outs[] = {dq, dk, dv, dg, dbeta, d_out, d_state_out};
  for (const void* p : outs)
    if (p && !aligned16(p)) return GDN_ERR_INVALID_ARG;
  // the gradients written must not overlap anything else of the call
  const Range w[] = {range_of(dq, rows * Dk * es), range_of(dk, rows * Dk * es),
                     range_of(dv, rows * Dv * es), range_of(dg, rows * 4),
                     range_of(dbeta, rows * 4), range_of(d_state_in, d_state_in ? sbytes : 0)};
  const Range r[] = {range_of(q, rows * Dk * es), range_of(k, rows * Dk * es),
                     range_of(v, rows * Dv * es), range_of(g, rows * 4), range_of(beta, rows * 4),
                     range_of(state_in, state_in ? sbytes : 0), range_of(d_out, rows * Dv * es),
                     range_of(d_state_out, d_state_out ? sbytes : 0)};
  if (T > 0) {
    for (int i = 0; i < 6; ++i) {
      for (const Range& x : r)
        if (overlaps(w[i], x)) return GDN_ERR_ALIAS;
      for (int j = i + 1; j < 6; ++j)
        if (overlaps(w[i], w[j])) return GDN_ERR_ALIAS;
    }
  }
  st = check_scan_device(a, &dev);
  if (st != GDN_OK) return st;
  for (const void* p : outs) {
    if (!p || (T == 0 && p != d_state_out)) continue;
    st = check_device_pointer(p, dev);
    if (st != GDN_OK) return st;
  }
  cudaStream_t s = a.stream;
  if (T == 0) {  // state_out = state_in: d_state_in = d_state_out (or zero)
    if (!d_state_in) return GDN_OK;
    cudaError_t e = d_state_out
                        ? cudaMemcpyAsync(d_state_in, d_state_out, sbytes, cudaMemcpyDeviceToDevice, s)
                        : cudaMemsetAsync(d_state_in, 0, sbytes, s);
    return finish(s, e, nullptr);
  }
  unsigned int* err = nullptr;
  void* ws = nullptr;
  const size_t bytes = bwd_workspace_bytes(B, T, H, Dk, Dv, dtype, bidir);
  st = stream_context(dev, s, bytes, &err, &ws);
  if (st != GDN_OK) return st;
  if (!err && error_word(&err) != cudaSuccess) {
    cudaGetLastError();
    return GDN_ERR_CUDA;
  }
  BwdCall c;
  c.q = q; c.k = k; c.v = v; c.g = g; c.beta = beta; c.state_in = state_in;
  c.d_out = d_out; c.d_state_out = d_state_out;
  c.dq = dq; c.dk = dk; c.dv = dv; c.dg = dg; c.dbeta = dbeta; c.d_state_in = d_state_in;
  c.B = B; c.T = T; c.H = H; c.Dk = Dk; c.Dv = Dv; c.dtype = dtype; c.bidir = bidir; c.stream = s;
  c.err = err;
  c.wait_limit = g_wait_limit.load();
  cudaError_t e;
  if (ws) {
    e = launch_backward(c, ws);
  } else {  // under capture without a large enough cached scratch
    e = cudaMallocAsync(&ws, bytes, s);
    if (e == cudaSuccess) {
      e = launch_backward(c, ws);
      const cudaError_t f = cudaFreeAsync(ws, s);
      if (e == cudaSuccess) e = f;
    }
  }
  return finish(s, e, err);
}
gdn_status sink_window(const void* q, const void* k, const void* v, void* k_cache,
                       void* v_cache, void* out, int B, int Tc, int H, int D, int n_sink,
                       int window, int chunk, gdn_dtype dtype, void* stream) {
  // ---- pure host checks
  if (dtype != GDN_F32 && dtype != GDN_BF16) return GDN_ERR_INVALID_ARG;
  if (B < 0 || Tc < 0 || H < 0 || D < 0) return GDN_ERR_INVALID_ARG;
  if (n_sink < 0 || window < 1 || n_sink + window > kSwaMaxSeg || chunk < 0)
    return GDN_ERR_INVALID_ARG;
  if (dtype != GDN_BF16 || !supported_dim(D)) return GDN_ERR_UNSUPPORTED;
  if ((long long)B * H > 65535) return GDN_ERR_UNSUPPORTED;
  if (B == 0 || H == 0 || Tc == 0) return GDN_OK;
  const void* ptrs[] = {q, k, v, k_cache, v_cache, out};
  for (const void* p : ptrs)
    if (!p || !aligned16(p)) return GDN_ERR_INVALID_ARG;
  const size_t chunk_bytes = (size_t)B * Tc * H * D * 2;
  const int nslot = n_sink + window;
  const size_t cache_bytes = chunk_bytes * nslot;
  const Range rq = range_of(q, chunk_bytes), rk = range_of(k, chunk_bytes);
  const Range rv = range_of(v, chunk_bytes), ro = range_of(out, chunk_bytes);
  const Range rkc = range_of(k_cache, cache_bytes), rvc = range_of(v_cache, cache_bytes);
  for (Range r : {rq, rk, rv, rkc, rvc})
    if (overlaps(ro, r)) return GDN_ERR_ALIAS;
  if (overlaps(rkc, rvc) || overlaps(rkc, rq) || overlaps(rvc, rq)) return GDN_ERR_ALIAS;
  // k (v) may be exactly this chunk's slot of its own cache: with B > 1 a
  // slot is strided over the batch, so only B == 1 makes it one block
  const int slot = sink_window_slot(chunk, n_sink, window);
  const uint8_t* kslot = static_cast<const uint8_t*>(k_cache) + (size_t)slot * Tc * H * D * 2;
  const uint8_t* vslot = static_cast<const uint8_t*>(v_cache) + (size_t)slot * Tc * H * D * 2;
  if (overlaps(rk, rkc) && !(B == 1 && k == kslot)) return GDN_ERR_ALIAS;
  if (overlaps(rv, rvc) && !(B == 1 && v == vslot)) return GDN_ERR_ALIAS;
  if (overlaps(rk, rvc) || overlaps(rv, rkc)) return GDN_ERR_ALIAS;

  // ---- device checks
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return GDN_ERR_CUDA;
  }
  for (const void* p : ptrs) {
    const gdn_status st = check_device_pointer(p, dev);
    if (st != GDN_OK) return st;
  }
  cudaGetLastError();
  SwaCall c;
  c.q = q; c.k = k; c.v = v; c.k_cache = k_cache; c.v_cache = v_cache; c.out = out;
  c.B = B; c.Tc = Tc; c.H = H; c.D = D; c.n_sink = n_sink; c.window = window; c.chunk = chunk;
  c.stream = static_cast<cudaStream_t>(stream);
  void* ws = nullptr;
  gdn_status st = stream_context(dev, c.stream, 0, &c.err, &ws);
  if (st != GDN_OK) return st;
  if (!c.err && error_word(&c.err) != cudaSuccess) {
    cudaGetLastError();
    return GDN_ERR_CUDA;
  }
  c.limit = g_wait_limit.load();
  return finish(c.stream, launch_sink_window(c), c.err);
}

}  // namespace

cudaError_t current_error_word(unsigned int** out) { return error_word(out); }
long long current_wait_limit() { return g_wait_limit.load(); }
int current_time_segments() { return g_time_segments.load(); }

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
                   dtype, chunk, stream, false, false);
}

gdn_status gdn_chunk_bidir(const void* q, const void* k, const void* v,
                           const float* g, const float* beta,
                           const float* state_in, float* state_out, void* out,
                           int B, int T, int H, int Dk, int Dv,
                           gdn_dtype dtype, int chunk, void* stream) {
  return gdn::scan(q, k, v, g, beta, state_in, state_out, out, B, T, H, Dk, Dv,
                   dtype, chunk, stream, true, false);
}

gdn_status gdn_chunk_fwd_logits(const void* q, const void* k, const void* v,
                                const void* g_logit, const void* beta_logit,
                                const float* state_in, float* state_out, void* out, int B,
                                int T, int H, int Dk, int Dv, gdn_dtype dtype, int chunk,
                                void* stream) {
  return gdn::scan(q, k, v, g_logit, beta_logit, state_in, state_out, out, B, T, H, Dk, Dv,
                   dtype, chunk, stream, false, true);
}

gdn_status gdn_chunk_bidir_logits(const void* q, const void* k, const void* v,
                                  const void* g_logit, const void* beta_logit,
                                  const float* state_in, float* state_out, void* out, int B,
                                  int T, int H, int Dk, int Dv, gdn_dtype dtype, int chunk,
                                  void* stream) {
  return gdn::scan(q, k, v, g_logit, beta_logit, state_in, state_out, out, B, T, H, Dk, Dv,
                   dtype, chunk, stream, true, true);
}

gdn_status gdn_chunk_fwd_backward(const void* q, const void* k, const void* v,
                                  const float* g, const float* beta, const float* state_in,
                                  const void* d_out, const float* d_state_out, void* dq,
                                  void* dk, void* dv, float* dg, float* dbeta,
                                  float* d_state_in, int B, int T, int H, int Dk, int Dv,
                                  gdn_dtype dtype, void* stream) {
  return gdn::backward(q, k, v, g, beta, state_in, d_out, d_state_out, dq, dk, dv, dg, dbeta,
                       d_state_in, B, T, H, Dk, Dv, dtype, stream, false);
}

gdn_status gdn_chunk_bidir_backward(const void* q, const void* k, const void* v,
                                    const float* g, const float* beta, const float* state_in,
                                    const void* d_out, const float* d_state_out, void* dq,
                                    void* dk, void* dv, float* dg, float* dbeta,
                                    float* d_state_in, int B, int T, int H, int Dk, int Dv,
                                    gdn_dtype dtype, void* stream) {
  return gdn::backward(q, k, v, g, beta, state_in, d_out, d_state_out, dq, dk, dv, dg, dbeta,
                       d_state_in, B, T, H, Dk, Dv, dtype, stream, true);
}

gdn_status gdn_sink_window_attention(const void* q, const void* k, const void* v, void* k_cache,
                                     void* v_cache, void* out, int B, int Tc, int H, int D,
                                     int n_sink, int window, int chunk_index, gdn_dtype dtype,
                                     void* stream) {
  return gdn::sink_window(q, k, v, k_cache, v_cache, out, B, Tc, H, D, n_sink, window,
                          chunk_index, dtype, stream);
}

int gdn_sink_window_slot(int chunk_index, int n_sink, int window) {
  if (chunk_index < 0 || n_sink < 0 || window < 1) return -1;
  return gdn::sink_window_slot(chunk_index, n_sink, window);
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
  if (cudaStreamSynchronize(s) != cudaSuccess) {
    cudaGetLastError();
    return GDN_ERR_CUDA;
  }
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return GDN_ERR_CUDA;
  }
  unsigned int* own = nullptr;
  {
    const size_t tk = gdn::thread_key(s);
    std::lock_guard<std::mutex> lock(gdn::g_ctx_mu);
    for (const gdn::StreamCtx* c : gdn::g_ctx)
      if (c->dev == dev && c->stream == s && c->thread == tk) own = c->err;
  }
  unsigned int* shared = nullptr;
  if (gdn::error_word(&shared) != cudaSuccess) {
    cudaGetLastError();
    return GDN_ERR_CUDA;
  }
  const gdn_status a = own ? gdn::take_error(own) : GDN_OK;
  const gdn_status b = gdn::take_error(shared);
  if (a == GDN_ERR_CUDA || b == GDN_ERR_CUDA) return GDN_ERR_CUDA;
  return (a == GDN_ERR_TIMEOUT || b == GDN_ERR_TIMEOUT) ? GDN_ERR_TIMEOUT : GDN_OK;
}

gdn_status gdn_workspace_release(void) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return GDN_ERR_CUDA;
  }
  if (cudaDeviceSynchronize() != cudaSuccess) {
    cudaGetLastError();
    return GDN_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lock(gdn::g_ctx_mu);
  gdn_status st = GDN_OK;
  std::vector<gdn::StreamCtx*> keep;
  for (gdn::StreamCtx* c : gdn::g_ctx) {
    if (c->dev != dev) {
      keep.push_back(c);
      continue;
    }
    if (c->ws && cudaFree(c->ws) != cudaSuccess) st = GDN_ERR_CUDA;
    if (c->err && cudaFree(c->err) != cudaSuccess) st = GDN_ERR_CUDA;
    delete c;
  }
  gdn::g_ctx.swap(keep);
  std::vector<gdn::Retired> left;
  for (const gdn::Retired& r : gdn::g_retired) {
    if (r.dev != dev) {
      left.push_back(r);
      continue;
    }
    if (cudaFree(r.p) != cudaSuccess) st = GDN_ERR_CUDA;
  }
  gdn::g_retired.swap(left);
  if (st != GDN_OK) cudaGetLastError();
  return st;
}

int gdn_set_time_segments(int segments) {
  if (segments < 0) segments = 0;
  return gdn::g_time_segments.exchange(segments);
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

int gdn_version(void) { return 200; }

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
    case gdn::kKernSegPrefix: return "gdn_segment_prefix_kernel";
    case gdn::kKernBwdScan: return "gdn_bwd_scan_kernel";
    case gdn::kKernBwdReduce: return "gdn_bwd_reduce_kernel";
    case gdn::kKernSinkWindow: return "gdn_sink_window_kernel";
    case gdn::kKernBwdChunk: return "gdn_bwd_pre_kernel";
    case gdn::kKernBwdChain: return "gdn_bwd_chain_kernel";
    case gdn::kKernBwdGrad: return "gdn_bwd_grad_kernel";
  }
  return "unknown";
}

}  // extern "C"
