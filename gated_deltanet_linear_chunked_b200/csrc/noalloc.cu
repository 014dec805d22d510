// noalloc.cu -- gdn_chunk_fwd_noalloc: the bf16 tensor-core causal scan with
// its scratch in one fixed device array instead of a stream-ordered
// allocation, for callers that cannot allocate device memory (a server whose
// HBM is already handed out to its caches, or a process without the CUDA
// memory-pool API).  The kernels and their launch sequence are those of
// gdn_chunk_fwd; only where the scratch lives differs.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "gdn_internal.h"

namespace gdn {
namespace {

constexpr size_t kScratchBytes = GDN_NOALLOC_SCRATCH_BYTES;

// The scratch: every device that loads this library holds it until exit.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Host-side name of a __device__ array is only a stand-in: the device address
// is looked up once per device, with that device current.
cudaError_t scratch_address(int dev, void** out) {
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

struct Span {
  uintptr_t lo, hi;
};
Span span(const void* p, size_t bytes) {
  const uintptr_t lo = reinterpret_cast<uintptr_t>(p);
  return {lo, lo + bytes};
}
bool overlap(Span a, Span b) {
  if (a.lo == a.hi || b.lo == b.hi) return false;
  return a.lo < b.hi && b.lo < a.hi;
}
bool is_aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool dim_ok(int d) { return d >= 16 && d <= 128 && d % 16 == 0; }

gdn_status device_pointer_ok(const void* p, int dev) {
  cudaPointerAttributes attr;
  if (cudaPointerGetAttributes(&attr, p) != cudaSuccess) {
    cudaGetLastError();
    return GDN_ERR_CUDA;
  }
  if (attr.type == cudaMemoryTypeManaged) return GDN_OK;
  if (attr.type != cudaMemoryTypeDevice || attr.device != dev) return GDN_ERR_INVALID_ARG;
  return GDN_OK;
}

}  // namespace
}  // namespace gdn

extern "C" gdn_status gdn_chunk_fwd_noalloc(const void* q, const void* k, const void* v,
                                            const float* g, const float* beta,
                                            const float* state_in, float* state_out,
                                            void* out, int B, int T, int H, int Dk, int Dv,
                                            gdn_dtype dtype, int chunk, void* stream) {
  using namespace gdn;
  // ---- host checks, as gdn_chunk_fwd
  if (dtype != GDN_F32 && dtype != GDN_BF16) return GDN_ERR_INVALID_ARG;
  if (B < 0 || T < 0 || H < 0 || Dk < 0 || Dv < 0) return GDN_ERR_INVALID_ARG;
  if (!dim_ok(Dk) || !dim_ok(Dv)) return GDN_ERR_UNSUPPORTED;
  if (chunk != 0 && chunk != 16 && chunk != 32 && chunk != 64) return GDN_ERR_INVALID_ARG;
  if (dtype != GDN_BF16) return GDN_ERR_UNSUPPORTED;  // the scratch-using path is bf16
  if (chunk == 0) chunk = 64;
  if (B == 0 || H == 0) return GDN_OK;
  if (T > 0 && chunk_tc_workspace_bytes(B, T, H, Dk, Dv, false) > kScratchBytes)
    return GDN_ERR_SCRATCH_LIMIT;

  const size_t rows = (size_t)B * T * H;
  const size_t state_bytes = (size_t)B * H * Dk * Dv * sizeof(float);
  const Span sq = span(q, rows * Dk * 2), sk = span(k, rows * Dk * 2);
  const Span sv = span(v, rows * Dv * 2), so = span(out, rows * Dv * 2);
  const Span sg = span(g, rows * 4), sb = span(beta, rows * 4);
  const Span ssi = span(state_in, state_in ? state_bytes : 0);
  const Span sso = span(state_out, state_out ? state_bytes : 0);
  if (T > 0 && (!q || !k || !v || !g || !beta || !out)) return GDN_ERR_INVALID_ARG;
  const void* ptrs[] = {q, k, v, g, beta, state_in, state_out, out};
  for (const void* p : ptrs)
    if (p && !is_aligned16(p)) return GDN_ERR_INVALID_ARG;
  if (T > 0) {
    for (Span r : {sq, sk, sv, sg, sb, ssi, sso})
      if (overlap(so, r)) return GDN_ERR_ALIAS;
    for (Span r : {sq, sk, sv, sg, sb})
      if (overlap(sso, r)) return GDN_ERR_ALIAS;
  }
  if (state_in && state_out && state_in != state_out && overlap(ssi, sso)) return GDN_ERR_ALIAS;

  // ---- device checks
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return GDN_ERR_CUDA;
  }
  for (const void* p : ptrs) {
    if (!p) continue;
    if (T == 0 && p != state_in && p != state_out) continue;
    const gdn_status st = device_pointer_ok(p, dev);
    if (st != GDN_OK) return st;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaGetLastError();
  if (T == 0) {
    if (!state_out) return GDN_OK;
    cudaError_t e = cudaSuccess;
    if (!state_in) e = cudaMemsetAsync(state_out, 0, state_bytes, s);
    else if (state_in != state_out)
      e = cudaMemcpyAsync(state_out, state_in, state_bytes, cudaMemcpyDeviceToDevice, s);
    return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
  }

  void* scratch = nullptr;
  if (scratch_address(dev, &scratch) != cudaSuccess) {
    cudaGetLastError();
    return GDN_ERR_CUDA;
  }
  unsigned int* err = nullptr;
  if (current_error_word(&err) != cudaSuccess) return GDN_ERR_CUDA;

  ScanArgs a;
  a.q = q; a.k = k; a.v = v; a.g = g; a.beta = beta;
  a.state_in = state_in; a.state_out = state_out; a.out = out;
  a.B = B; a.T = T; a.H = H; a.Dk = Dk; a.Dv = Dv;
  a.dtype = dtype; a.chunk = chunk; a.bidir = false; a.stream = s;
  a.err = err; a.wait_limit = current_wait_limit();
  return launch_chunk_tc(a, scratch) == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}
