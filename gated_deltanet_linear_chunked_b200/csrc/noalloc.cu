// noalloc.cu -- gdn_chunk_fwd_noalloc: the bf16 tensor-core causal scan with
// its scratch in one fixed device array instead of an allocation, for callers
// that cannot allocate device memory (a server whose HBM is already handed
// out to its caches, or a process without the CUDA memory-pool API).  The
// kernels, their launch sequence, the argument checks and the error handling
// are those of gdn_chunk_fwd; only where the scratch lives differs.
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

// In host code the array's name is only a stand-in: its device address is
// looked up once per device, with that device current.
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

}  // namespace
}  // namespace gdn

extern "C" gdn_status gdn_chunk_fwd_noalloc(const void* q, const void* k, const void* v,
                                            const float* g, const float* beta,
                                            const float* state_in, float* state_out,
                                            void* out, int B, int T, int H, int Dk, int Dv,
                                            gdn_dtype dtype, int chunk, void* stream) {
  using namespace gdn;
  ScanArgs a;
  int dev = 0;
  gdn_status st = check_scan_host(q, k, v, g, beta, state_in, state_out, out, B, T, H, Dk, Dv,
                                  dtype, chunk, stream, false, false, &a);
  if (st != GDN_OK) return st;
  if (dtype != GDN_BF16) return GDN_ERR_UNSUPPORTED;  // the scratch-using path is bf16
  if (a.B == 0 || a.H == 0) return GDN_OK;
  st = check_scan_device(a, &dev);
  if (st != GDN_OK) return st;
  if (a.T == 0) return trivial_state_copy(a);
  if (chunk_tc_workspace_bytes(B, T, H, Dk, Dv, false) > kScratchBytes)
    return GDN_ERR_SCRATCH_LIMIT;

  void* scratch = nullptr;
  if (scratch_address(dev, &scratch) != cudaSuccess || current_error_word(&a.err) != cudaSuccess) {
    cudaGetLastError();
    return GDN_ERR_CUDA;
  }
  a.wait_limit = current_wait_limit();
  return finish(a.stream, launch_chunk_tc(a, scratch), a.err);
}
