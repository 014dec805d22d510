// Internal interface between the C-ABI front end (gdn_api.cu) and the kernel
// translation units.  Not installed; callers use include/gdn.h.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "gdn.h"

namespace gdn {

// One scan call, after validation.  Pointers are device pointers.
struct ScanArgs {
  const void* q;
  const void* k;
  const void* v;
  const void* g;           // fp32 g, or the decay logits (dtype) when gate_logits
  const void* beta;        // fp32 beta, or the write-strength logits (dtype)
  const float* state_in;   // nullptr => zero state
  float* state_out;        // nullptr => not written
  void* out;
  int B, T, H, Dk, Dv;
  gdn_dtype dtype;
  int chunk;               // sub-chunk length (already defaulted)
  bool bidir;
  bool gate_logits;        // g and beta hold the gate layer's logits
  cudaStream_t stream;
  unsigned int* err;       // device error word (bounded waits report here)
  long long wait_limit;    // polls before a bounded wait gives up
  bool skip_output = false;  // chunked path: stages A and B only (workspace filled, out untouched)
  void* t_out = nullptr;     // chunked path: stage A also writes each chunk's (I + A)^-1, bf16
                             // in scan order as core matrices [8 column slabs][64 rows][8],
                             // one 8 KB block per (dir, b*h, chunk)
};

// Kernel ids for the profiling hook.
enum KernelId : int {
  kKernSerial = 0,
  kKernPrep = 1,
  kKernRecur = 2,
  kKernOutput = 3,
  kKernSegPrefix = 4,
  kKernBwdScan = 5,
  kKernBwdReduce = 6,
  kKernSinkWindow = 7,
  kKernBwdChunk = 8,   // the chunked backward's pre pass
  kKernBwdChain = 9,
  kKernBwdGrad = 10,
  kNumKernelIds = 11,
};

// While profiling is armed, records CUDA events around one launch.
class ProfileScope {
 public:
  ProfileScope(cudaStream_t s, int kernel_id);
  ~ProfileScope();
 private:
  cudaStream_t stream_;
  int slot_;
};

// Every check gdn.h lists for a scan call: check_scan_host, then
// check_scan_device.  On GDN_OK `a` holds the validated call (chunk defaulted;
// err and wait_limit not yet set) and `*dev` the current device.  B == 0 or
// H == 0 returns GDN_OK with a->B or a->H zero: the caller has nothing to do.
gdn_status prepare_scan(const void* q, const void* k, const void* v, const void* g,
                        const void* beta, const float* state_in, float* state_out,
                        void* out, int B, int T, int H, int Dk, int Dv, gdn_dtype dtype,
                        int chunk, void* stream, bool bidir, bool gate_logits, ScanArgs* a,
                        int* dev);

// The two halves of prepare_scan.  check_scan_host makes no CUDA call: dtype,
// sizes, head dims, chunk, null pointers, 16-byte alignment and overlaps; on
// GDN_OK it fills `a` (and stops there when B or H is zero).
// check_scan_device checks that each pointer of a host-checked call is device
// memory of the current device (with T == 0 only the states, the only buffers
// touched); on GDN_OK `*dev` is that device.  Entry points with checks of
// their own run all host checks before the device ones.
gdn_status check_scan_host(const void* q, const void* k, const void* v, const void* g,
                           const void* beta, const float* state_in, float* state_out,
                           void* out, int B, int T, int H, int Dk, int Dv, gdn_dtype dtype,
                           int chunk, void* stream, bool bidir, bool gate_logits, ScanArgs* a);
gdn_status check_scan_device(const ScanArgs& a, int* dev);

// T == 0: state_out = state_in (or zero); out untouched.
gdn_status trivial_state_copy(const ScanArgs& a);

// Maps a launch result to a status.  With GDN_DEBUG_SYNC set in the
// environment it also synchronises the stream and reads (and clears) the
// error word `err`, returning GDN_ERR_TIMEOUT if a bounded wait expired.
gdn_status finish(cudaStream_t s, cudaError_t launch_err, unsigned int* err);

// Device address of the device-wide error word on the current device (used by
// calls that have no per-stream context), and the poll limit handed to
// bounded waits.
cudaError_t current_error_word(unsigned int** out);
long long current_wait_limit();

// The time-segment setting of gdn_set_time_segments (0: automatic).
int current_time_segments();

// Adds n to the process-wide count of kernels the library has enqueued.
void count_launches(unsigned n);

// Token-serial SIMT scan (fp32 arithmetic, fp32 or bf16 I/O).
cudaError_t launch_scan_serial(const ScanArgs& a);

// Chunked tcgen05 path (bf16 I/O): stage A prep, stage B recurrence, stage C
// output.  `workspace` must hold chunk_tc_workspace_bytes(...) bytes.
size_t chunk_tc_workspace_bytes(int B, int T, int H, int Dk, int Dv, bool bidir);
cudaError_t launch_chunk_tc(const ScanArgs& a, void* workspace);
// Layout of one (direction, b*h, chunk) block of the chunked path's
// workspace (block index ((dir * B*H) + bh) * nC + chunk; rows in time order):
//   W, K~ [Dk/8][64][8] bf16, decay (fp32 e^{gamma_C}), g [64] fp32,
//   U~, U [Dv/8][64][8] bf16, S (chunk-start state) [Dv/8][Dk][8] bf16.
struct WsLayout {
  size_t block_bytes;
  uint32_t off_w, off_kt, off_decay, off_g, off_ut, off_u, off_s;
};
WsLayout chunk_tc_ws_layout(int Dk, int Dv);

// One backward call, after validation (device pointers).
struct BwdCall {
  const void *q, *k, *v;
  const float *g, *beta, *state_in;   // state_in may be nullptr (zero state)
  const void* d_out;                  // [B,T,H,Dv] dtype
  const float* d_state_out;           // may be nullptr (no gradient on state_out)
  void *dq, *dk, *dv;                 // dtype
  float *dg, *dbeta, *d_state_in;     // d_state_in may be nullptr
  int B, T, H, Dk, Dv;
  gdn_dtype dtype;
  bool bidir;
  cudaStream_t stream;
  unsigned int* err;     // error word of the forward stages' bounded waits
  long long wait_limit;
};
size_t bwd_workspace_bytes(int B, int T, int H, int Dk, int Dv, gdn_dtype dtype, bool bidir);
cudaError_t launch_backward(const BwdCall& c, void* workspace);
// bf16 I/O: the chunked backward (forward stages A and B, then a pre pass,
// the reverse chain over the chunks and a chunk-parallel gradient pass);
// returns the partials' addresses in the workspace for the reduction (dvb
// holds the gradient of diag(beta) V's rows, not dv).
bool bwd_chunked_fits(int Dk, int Dv);  // its shared-memory layout fits (Dk, Dv <= 112)
size_t bwd_chunked_workspace_bytes(int B, int T, int H, int Dk, int Dv, bool bidir);
cudaError_t launch_backward_chunked(const BwdCall& c, void* workspace, float** pq, float** pk,
                                    float** pab, float** dvb);

// A [nb, T, H, D] bf16 tensor viewed as 5-D (8 features, T, D/8 feature
// slabs, H, nb) so that one box (8 x box_rows tokens x D/8 slabs x 1 x 1)
// lands in shared memory in the [slab][token][8] core-matrix layout.
bool make_tile_map(CUtensorMap* m, const void* base, int nb, int T, int H, int D, int box_rows);

// Streaming multiprocessors of the current device (cached per device).
int num_sms();

// One sink + sliding-window attention call, after validation.
constexpr int kSwaMaxSeg = 16;  // n_sink + window at most
struct SwaCall {
  const void *q, *k, *v;       // [B, Tc, H, D] bf16: this chunk
  void *k_cache, *v_cache;     // [B, n_sink + window, Tc, H, D] bf16
  void* out;                   // [B, Tc, H, D] bf16
  int B, Tc, H, D, n_sink, window, chunk;
  cudaStream_t stream;
  unsigned int* err;
  long long limit;
};
// Cache slot of stream chunk `chunk`: sink chunks keep their own slots, the
// rest share `window` ring slots.
int sink_window_slot(int chunk, int n_sink, int window);
cudaError_t launch_sink_window(const SwaCall& c);

// The per-(device, stream) scratch of at least `bytes` (nullptr under stream
// capture when it cannot be provided); GDN_OK or GDN_ERR_CUDA.
gdn_status stream_scratch(int dev, cudaStream_t s, size_t bytes, unsigned int** err, void** ws);

// Device error word values.
enum : unsigned int {
  kErrNone = 0,
  kErrTimeout = 1,
};

}  // namespace gdn
