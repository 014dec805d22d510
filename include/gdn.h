/*
 * gdn.h -- C ABI of libgdn.so: the chunked Gated DeltaNet (GDN) scan of the
 * GDN blocks of SANA-Streaming's hybrid diffusion Transformer, on sm_100a.
 *
 * The operation.  Per batch row b and head h the scan carries a state
 * S (Dk x Dv, fp32) through the gated delta rule
 *
 *     q^_t = q_t / sqrt(max(|q_t|^2, 1e-12)),   k^_t likewise
 *     S_t  = a_t (I - beta_t k^_t k^_t^T) S_{t-1} + beta_t k^_t v_t^T,
 *     o_t  = S_t^T q^_t,                        a_t = exp(g_t), g_t <= 0.
 *
 * The pages describe GDN only in words: a fixed-size memory updated
 * recursively from the previous state ("[논문리뷰] SANA-Streaming: Real-time
 * Streaming Video Editing with Hybrid Diffusion Transformer", 1. Key Terms &
 * Definitions).  Streaming runs a forward scan that starts from the previous
 * chunk's cache, and the streaming model adds a backward scan inside the chunk
 * ("SANA-Streaming：基于混合扩散Transformer的实时流式视频编辑系统",
 * 方法步骤详情, second and fourth steps; the fourth names the fused kernel's
 * three stages: frame summaries, recurrent scan, state application).
 *
 * Layouts (row-major, contiguous, element strides implied by the sizes):
 *   q, k       [B, T, H, Dk]   dtype (GDN_F32: float, GDN_BF16: bf16)
 *   v, out     [B, T, H, Dv]   dtype
 *   g, beta    [B, T, H]       float   (g <= 0 is the log of the decay a_t;
 *                                       beta in [0, 1])
 *   state      [B, H, Dk, Dv]  float
 *
 * Ownership.  The caller owns every buffer; all pointers are device (or
 * managed) pointers.  The library keeps no pointer to a caller's buffer after
 * a call returns.  It keeps, per (device, stream), one small context: the
 * scratch the bf16 path passes between its kernels and an error word.  The
 * first call on a stream allocates it (cudaMalloc), a larger problem grows
 * it, and gdn_workspace_release frees it.  Calls on one stream share their
 * context (they are ordered); calls on different streams share nothing.  A
 * call made while its stream is being captured into a CUDA graph cannot
 * allocate outside the graph: if the stream has no context yet, or too small
 * a scratch, the call allocates stream-ordered (cudaMallocAsync /
 * cudaFreeAsync, captured as graph memory nodes) and reports through the
 * device-wide error word.  Make one call on a stream before capturing on it
 * to keep memory nodes out of the graph.  Contexts are found by the stream's
 * handle, and cudaStreamDestroy returns before the stream's work is done: let
 * a stream's calls finish before destroying it, since a stream created
 * afterwards may get the same handle, and with it the same scratch.
 *
 * Execution.  Work is enqueued on `stream` (a cudaStream_t; NULL is the
 * legacy default stream) and the call returns without synchronising;
 * results are stream-ordered.  No call throws, aborts or prints.  Calls may
 * come from several host threads at once.
 *
 * Errors.  Arguments are validated on the host before anything is enqueued;
 * on any error nothing is launched and a status is returned.  The checks that
 * need no CUDA call (sizes, dims, dtype, chunk, null pointers, alignment,
 * overlaps) all run before those that do (that each pointer is device memory
 * of the current device), so a bad argument is reported as such even when no
 * device is usable:
 *   GDN_ERR_INVALID_ARG  null pointer where data is needed, negative size,
 *                        pointer not 16-byte aligned, host (pageable or
 *                        pinned) pointer, unknown dtype, bad chunk value
 *   GDN_ERR_UNSUPPORTED  Dk or Dv not a multiple of 16 in [16, 128]
 *   GDN_ERR_ALIAS        out overlaps an input or the state; state_out
 *                        overlaps an input or partially overlaps state_in
 *   GDN_ERR_CUDA         a CUDA runtime call or a launch failed
 *   GDN_ERR_TIMEOUT      a kernel's bounded wait expired (reported by
 *                        gdn_device_error for the stream it ran on, or by
 *                        the calls themselves when the environment sets
 *                        GDN_DEBUG_SYNC=1: every scan entry point then
 *                        synchronises its stream before it returns)
 *   GDN_ERR_SCRATCH_LIMIT  (gdn_chunk_fwd_noalloc only) the problem needs more
 *                        scratch than its fixed device array holds
 */
#ifndef GDN_H_
#define GDN_H_

#if defined(__GNUC__)
#define GDN_API __attribute__((visibility("default")))
#else
#define GDN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  GDN_OK = 0,
  GDN_ERR_INVALID_ARG = 1,
  GDN_ERR_UNSUPPORTED = 2,
  GDN_ERR_ALIAS = 3,
  GDN_ERR_CUDA = 4,
  GDN_ERR_TIMEOUT = 5,
  GDN_ERR_SCRATCH_LIMIT = 6
} gdn_status;

typedef enum { GDN_F32 = 0, GDN_BF16 = 1 } gdn_dtype;

/*
 * Causal (forward) scan of one streaming chunk with a carried state.
 *
 * state_in   previous chunk's final state, or NULL for a zero state.
 * state_out  receives the final state; may equal state_in (in place);
 *            may be NULL when the caller does not need it.
 * out        receives o_t for every token, in `dtype`.
 * chunk      sub-chunk length hint: 0 (default), 16, 32 or 64; any other
 *            value is GDN_ERR_INVALID_ARG.  The chunked form equals the
 *            recurrence for every sub-chunk length, so the hint can change
 *            rounding only, never the result's definition.  The bf16
 *            tensor-core path tiles time with 64 tokens whatever the hint;
 *            the fp32 path scans token by token.
 * T == 0     is allowed: state_out = state_in (or zero), out is untouched.
 * B == 0 or H == 0 is allowed and does nothing.
 */
GDN_API gdn_status gdn_chunk_fwd(const void* q, const void* k, const void* v,
                         const float* g, const float* beta,
                         const float* state_in, float* state_out, void* out,
                         int B, int T, int H, int Dk, int Dv, gdn_dtype dtype,
                         int chunk, void* stream);

/*
 * Bidirectional scan of one chunk: out = (forward scan from state_in) +
 * (the same recurrence over the time-reversed chunk from a zero state, each
 * token keeping its own g_t and beta_t), summed per token.  state_out is the
 * forward scan's final state.  Arguments as for gdn_chunk_fwd.
 */
GDN_API gdn_status gdn_chunk_bidir(const void* q, const void* k, const void* v,
                           const float* g, const float* beta,
                           const float* state_in, float* state_out, void* out,
                           int B, int T, int H, int Dk, int Dv,
                           gdn_dtype dtype, int chunk, void* stream);

/*
 * The same two scans with the fused GDN prologue for the gates: instead of g
 * and beta the caller passes the gate layer's two logits per (token, head),
 * g_logit and beta_logit [B, T, H] in `dtype` (bf16 for the tensor-core path,
 * which is how the gate layer runs under mixed precision), and the library
 * forms
 *     g_t = -softplus(g_logit_t) = -log(1 + e^{g_logit_t})     (so g_t <= 0)
 *     beta_t = sigmoid(beta_logit_t)                           (in (0, 1))
 * inside its kernels.  The pages name the gate layer and keep it in BF16
 * ("SANA-Streaming：基于混合扩散Transformer的实时流式视频编辑系统", 实验结果)
 * but do not write its activations; these are the plainest maps onto the
 * scan's ranges.  q and k are L2-normalised inside the library as for every
 * call.  Arguments, layouts and errors are otherwise those of gdn_chunk_fwd /
 * gdn_chunk_bidir.
 */
GDN_API gdn_status gdn_chunk_fwd_logits(const void* q, const void* k, const void* v,
                                        const void* g_logit, const void* beta_logit,
                                        const float* state_in, float* state_out, void* out,
                                        int B, int T, int H, int Dk, int Dv, gdn_dtype dtype,
                                        int chunk, void* stream);
GDN_API gdn_status gdn_chunk_bidir_logits(const void* q, const void* k, const void* v,
                                          const void* g_logit, const void* beta_logit,
                                          const float* state_in, float* state_out, void* out,
                                          int B, int T, int H, int Dk, int Dv,
                                          gdn_dtype dtype, int chunk, void* stream);

/*
 * Gradients of the two scans (the pages train the bidirectional GDN:
 * "SANA-Streaming：基于混合扩散Transformer的实时流式视频编辑系统", 方法步骤详情,
 * second step).  Given the forward call's inputs and the gradients of a loss
 * with respect to its results -- d_out [B, T, H, Dv] (dtype) and, optionally,
 * d_state_out [B, H, Dk, Dv] (fp32; NULL: the final state is unused) -- they
 * write the gradients with respect to the inputs:
 *   dq, dk [B, T, H, Dk] and dv [B, T, H, Dv] in dtype; dg, dbeta [B, T, H]
 *   fp32; d_state_in [B, H, Dk, Dv] fp32 (may be NULL; zero-state calls pass
 *   state_in = NULL and get the gradient of a zero start state).
 * bf16 I/O with Dk, Dv <= 112 runs the chunked reverse mode on tensor cores
 * (the forward's stages A and B, then a pre pass, the reverse walk over the
 * chunks and a chunk-parallel gradient pass; bf16 operands, fp32
 * accumulation, within 2e-2 of the definition); fp32 I/O and wider heads
 * walk the recurrence in fp32 on CUDA cores (token-serial, with checkpoints
 * every 64 tokens, within 1e-4).  Scratch comes from the stream's context.
 * g and beta are taken as given (no gate-logit form).
 * The gradient outputs may not overlap each other or any input.  Errors as
 * for gdn_chunk_fwd.
 */
GDN_API gdn_status gdn_chunk_fwd_backward(const void* q, const void* k, const void* v,
                                          const float* g, const float* beta,
                                          const float* state_in, const void* d_out,
                                          const float* d_state_out, void* dq, void* dk, void* dv,
                                          float* dg, float* dbeta, float* d_state_in, int B,
                                          int T, int H, int Dk, int Dv, gdn_dtype dtype,
                                          void* stream);
GDN_API gdn_status gdn_chunk_bidir_backward(const void* q, const void* k, const void* v,
                                            const float* g, const float* beta,
                                            const float* state_in, const void* d_out,
                                            const float* d_state_out, void* dq, void* dk,
                                            void* dv, float* dg, float* dbeta, float* d_state_in,
                                            int B, int T, int H, int Dk, int Dv, gdn_dtype dtype,
                                            void* stream);

/*
 * gdn_chunk_fwd for callers that cannot allocate device memory (no
 * counterpart on the pages).  Some callers cannot let a library allocate: a
 * streaming server that has already handed all remaining HBM to its caches
 * (an allocation in the middle of a stream can fail or stall on the memory
 * pool), or a process whose CUDA memory-pool API is unavailable or turned
 * off.  This entry point runs the same bf16 tensor-core kernels as
 * gdn_chunk_fwd but takes their scratch from one fixed array of
 * GDN_NOALLOC_SCRATCH_BYTES (96 MiB) that the library declares in device
 * memory; every GPU that loads the library holds that array until the process
 * exits.  It calls no cudaMalloc, cudaMallocAsync, cudaFree or other
 * allocating routine.
 *
 * Arguments and layouts are those of gdn_chunk_fwd, with dtype GDN_BF16
 * only (other dtypes: GDN_ERR_UNSUPPORTED).  A problem whose scratch exceeds
 * the array returns GDN_ERR_SCRATCH_LIMIT and launches nothing.  The scratch
 * is about 81 KB per 64-token chunk of one head at Dk = Dv = 112, so about
 * 1200 chunk-heads (B * H * ceil(T / 64)) fit: the 2640-token x 20-head
 * streaming chunk (840) does, two of them in one call (1680) do not.
 *
 * The first call on a device looks up the array's device address
 * (cudaGetSymbolAddress, once per device, with that device current); make
 * that first call before any stream capture.  All calls share the one array
 * and it keeps the last call's contents (every scratch byte a call reads was
 * written earlier in the same call, so nothing needs clearing); calls whose
 * work overlaps on the GPU -- two streams, or two host threads -- race on it,
 * so order them on one stream.  Argument checks and statuses are those of
 * gdn_chunk_fwd.  A bounded wait that expires is reported through the
 * device-wide error word (gdn_device_error on any stream of the device), or
 * by the call itself when GDN_DEBUG_SYNC=1.
 */
#define GDN_NOALLOC_SCRATCH_BYTES (96ull << 20)
GDN_API gdn_status gdn_chunk_fwd_noalloc(const void* q, const void* k, const void* v,
                                         const float* g, const float* beta,
                                         const float* state_in, float* state_out,
                                         void* out, int B, int T, int H, int Dk, int Dv,
                                         gdn_dtype dtype, int chunk, void* stream);

/*
 * Zero a state [B, H, Dk, Dv] (streaming restart: the state is the only thing
 * a stream keeps, "SANA-Streaming：基于混合扩散Transformer的实时流式视频编辑系统",
 * 前置知识, 流式生成).  Any positive Dk, Dv are accepted here.
 */
GDN_API gdn_status gdn_state_reset(float* state, int B, int H, int Dk, int Dv,
                           void* stream);

/*
 * Synchronise `stream`, then read and clear the error words that kernels set
 * when a bounded wait expires: the stream's own word (calls made on this
 * stream) and the current device's device-wide word (calls of
 * gdn_chunk_fwd_noalloc and calls captured before the stream had a
 * context).  Returns GDN_OK, GDN_ERR_TIMEOUT or GDN_ERR_CUDA.  A timeout of
 * a call on another stream is not reported here.
 */
GDN_API gdn_status gdn_device_error(void* stream);

/*
 * Free every per-stream context (scratch and error word) the library holds
 * on the current device, after synchronising the device.  Call it only when
 * no captured CUDA graph that contains this library's launches will be
 * replayed again: such a graph names the freed scratch.  Later calls create
 * new contexts.  Returns GDN_OK or GDN_ERR_CUDA.
 */
GDN_API gdn_status gdn_workspace_release(void);

/*
 * Test hook: the number of polls a kernel's bounded wait makes before it
 * gives up (0 restores the default).  Affects launches enqueued after the
 * call, on every device and stream: it is one process-wide setting, meant
 * for fault-injection tests, not for production tuning.  Returns the
 * previous value.
 */
GDN_API long long gdn_set_wait_limit(long long polls);

/*
 * The softmax blocks' attention: sink + sliding window over a streaming KV
 * cache.  The hybrid DiT places softmax attention blocks among the GDN blocks
 * at even intervals; each keeps a persistent sink and a sliding window, so
 * its memory is fixed by the window while it still sees fine correspondences
 * across chunk boundaries ("SANA-Streaming：基于混合扩散Transformer的实时流式
 * 视频编辑系统", 核心方法; softmax attention is the dot-product, softmax-
 * normalised token interaction of the same page's 线性注意力 vs Softmax注意力).
 * The pages give neither size nor unit; here both count whole chunks.  A
 * query of stream chunk c (chunk_index, from 0) attends to every token of
 * chunk m iff m <= c and (m < n_sink or m > c - window):
 *
 *     out = softmax(q K^T / sqrt(D)) V      per (b, h), fp32 softmax and
 *                                           accumulation, bf16 P and out
 *
 * over those keys, its own chunk's in both directions.  During the same call
 * the chunk's k and v are written into the cache slot
 * gdn_sink_window_slot(c, n_sink, window); the chunks read come from their
 * slots, so a stream is a sequence of calls with c = 0, 1, 2, ... on one
 * cache (chunks that left the window are overwritten, sink chunks never).
 *
 *   q, k, v, out   [B, Tc, H, D]                      bf16 (this chunk)
 *   k_cache,       [B, n_sink + window, Tc, H, D]     bf16, caller-owned;
 *   v_cache         a slot holds one chunk
 *
 * Requirements: dtype GDN_BF16 (else GDN_ERR_UNSUPPORTED); D a multiple of
 * 16 in [16, 128] (else GDN_ERR_UNSUPPORTED); n_sink >= 0, window >= 1,
 * n_sink + window <= 16, chunk_index >= 0 (else GDN_ERR_INVALID_ARG);
 * B * H <= 65535 (else GDN_ERR_UNSUPPORTED); all six pointers device memory,
 * 16-byte aligned.  out must not overlap anything; the two caches must not
 * overlap each other, q or out; k (v) may overlap k_cache (v_cache) only by
 * being exactly this chunk's slot in it (the projection wrote there).
 * Otherwise GDN_ERR_ALIAS.  Tc, B or H zero: nothing to do, GDN_OK.  Errors
 * and the per-stream error word as for the scan.
 */
GDN_API gdn_status gdn_sink_window_attention(const void* q, const void* k, const void* v,
                                             void* k_cache, void* v_cache, void* out, int B,
                                             int Tc, int H, int D, int n_sink, int window,
                                             int chunk_index, gdn_dtype dtype, void* stream);

/*
 * Cache slot that holds stream chunk `chunk_index` (host-only arithmetic):
 * chunk_index itself for a sink chunk (chunk_index < n_sink), else
 * n_sink + (chunk_index - n_sink) mod window.  -1 for invalid arguments.
 */
GDN_API int gdn_sink_window_slot(int chunk_index, int n_sink, int window);

/*
 * Time segments of the bf16 path's recurrence.  The stage that walks the
 * chunks is a dependent chain of ceil(T / 64) steps per (head, 16 state
 * columns).  When a call has too few such chains to fill the GPU and many
 * chunks, the library splits time into G segments: each segment's affine
 * map (S_out = P S_in + R) is formed in parallel, an exclusive prefix over
 * the segments gives every segment its start state, and the segments are
 * walked again in parallel from there -- a serial depth of about
 * 2 ceil(T / 64) / G + G chunk steps for three times the chain's work.  The
 * stream's carry is a forward scan that starts from the previous chunk's
 * cache ("SANA-Streaming：基于混合扩散Transformer的实时流式视频编辑系统",
 * 方法步骤详情), so the prefix runs over the same affine maps in time order.
 * 0 (the default) lets the library choose G; 1 never segments; G >= 2 forces
 * G segments (at most ceil(T / 64) / 2).  One process-wide setting, read
 * when a call is made; meant for tests and benchmarks.  Returns the previous
 * value.
 */
GDN_API int gdn_set_time_segments(int segments);

/*
 * Instrumentation (no counterpart on the pages): the number of kernels this
 * process has enqueued through the library so far, on all devices and
 * streams (launches captured into a CUDA graph count once, at capture).
 */
GDN_API unsigned long long gdn_launch_count(void);

/*
 * Instrumentation (no counterpart on the pages): per-kernel device times.
 * gdn_profile_begin arms CUDA-event timing of every kernel the library
 * launches from then on (on the launching stream, up to `max_launches`
 * launches, current device); gdn_profile_end synchronises the recorded
 * events, disarms, and writes for each kernel id i < nids the total
 * milliseconds ms[i] and launch count n[i].  Kernel ids: 0 token-serial scan,
 * 1 stage A (prep), 2 stage B (recurrence, every pass), 3 stage C (output),
 * 4 the time-segment prefix, 5 the token-serial backward, 6 the backward
 * reduction, 7 the sink + window attention, 8 / 9 / 10 the chunked
 * backward's pre, chain and gradient passes; names from gdn_kernel_name.  Not thread-safe against concurrent calls on other
 * threads; meant for benchmarks.
 */
GDN_API gdn_status gdn_profile_begin(int max_launches);
GDN_API gdn_status gdn_profile_end(float* ms, int* n, int nids);
GDN_API const char* gdn_kernel_name(int id);

/* Static, human-readable name of a status; never NULL. */
GDN_API const char* gdn_status_string(gdn_status status);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
GDN_API int gdn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GDN_H_ */
