// scan_serial.cu -- token-serial GDN scan on CUDA cores, fp32 arithmetic.
//
// This is the library's fp32 path (and its reference-precision path): the
// gated delta rule applied one token at a time,
//
//   u_t = beta_t (v_t - a_t S^T k^_t),   S <- a_t S + k^_t u_t^T,
//   o_t = S_new^T q^_t = a_t S^T q^_t + (k^_t . q^_t) u_t,
//
// which is S_t = a_t (I - beta_t k^ k^^T) S_{t-1} + beta_t k^ v_t^T rearranged
// so that both reductions over Dk read the old state and run together.  The
// Gated DeltaNet keeps a fixed-size state updated recursively ("[논문리뷰]
// SANA-Streaming: Real-time Streaming Video Editing with Hybrid Diffusion
// Transformer", 1. Key Terms & Definitions); streaming starts the forward scan
// from the previous chunk's cache and the bidirectional mode adds a backward
// scan inside the chunk ("SANA-Streaming：基于混合扩散Transformer的实时流式视频
// 编辑系统", 方法步骤详情).
//
// Parallelism: columns of S evolve independently (column j of S and of o
// depend only on column j of v and of S_in), so one CTA owns a 16-column
// slice of one (b, h) state and walks the whole sequence.  4 warps x 4
// columns; lane l holds rows l, l+32, l+64, l+96 of its 4 columns (16 fp32
// registers).  Tokens are staged 32 at a time in shared memory, where their
// q/k norms and k^.q^ are computed in parallel before the serial walk.
#include <cuda_bf16.h>

#include "gates.cuh"
#include "gdn_internal.h"

namespace gdn {
namespace {

constexpr int kCols = 16;
constexpr int kWarps = 4;
constexpr int kColsPerWarp = kCols / kWarps;
constexpr int kThreads = 32 * kWarps;
constexpr int kMaxD = 128;
constexpr int kRows = kMaxD / 32;
constexpr int kTB = 32;

__device__ __forceinline__ float ld_in(const float* p) { return __ldg(p); }
__device__ __forceinline__ float ld_in(const __nv_bfloat16* p) {
  return __bfloat162float(*p);
}
__device__ __forceinline__ void st_out(float* p, float x) { *p = x; }
__device__ __forceinline__ void st_out(__nv_bfloat16* p, float x) {
  *p = __float2bfloat16_rn(x);
}
__device__ __forceinline__ float ld_out(const float* p) { return *p; }
__device__ __forceinline__ float ld_out(const __nv_bfloat16* p) {
  return __bfloat162float(*p);
}

struct SerialSmem {
  float k[kTB][kMaxD];
  float q[kTB][kMaxD];
  float v[kTB][kCols];
  float o[kTB][kCols];
  float a[kTB], beta[kTB], rk[kTB], rq[kTB], kq[kTB];
};

// One direction of the scan over the CTA's column slice.
//   reverse = false: positions p = 0..T-1 are tokens t = p, S starts at S_in,
//                    results go to `first` (fp32 scratch or out itself).
//   reverse = true:  tokens t = T-1-p, S starts at 0, results are added to
//                    `first` and written to out.
template <typename IO>
__device__ void scan_direction(SerialSmem& sm, float (&S)[kRows][kColsPerWarp],
                               const IO* __restrict__ q, const IO* __restrict__ k,
                               const IO* __restrict__ v,
                               const void* __restrict__ g,
                               const void* __restrict__ beta, int logits, IO* out,
                               float* acc, int b, int h, int j0, int T, int H,
                               int Dk, int Dv, bool reverse) {
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  for (int p0 = 0; p0 < T; p0 += kTB) {
    const int n = min(kTB, T - p0);
    // ---- stage n tokens
    for (int idx = tid; idx < n * Dk; idx += kThreads) {
      const int tok = idx / Dk, i = idx - tok * Dk;
      const int t = reverse ? T - 1 - (p0 + tok) : p0 + tok;
      const size_t row = ((size_t)b * T + t) * H + h;
      sm.k[tok][i] = ld_in(k + row * Dk + i);
      sm.q[tok][i] = ld_in(q + row * Dk + i);
    }
    for (int idx = tid; idx < n * kCols; idx += kThreads) {
      const int tok = idx / kCols, c = idx - tok * kCols;
      const int t = reverse ? T - 1 - (p0 + tok) : p0 + tok;
      const size_t row = ((size_t)b * T + t) * H + h;
      sm.v[tok][c] = ld_in(v + row * Dv + j0 + c);
    }
    if (tid < n) {
      const int t = reverse ? T - 1 - (p0 + tid) : p0 + tid;
      const size_t row = ((size_t)b * T + t) * H + h;
      if (logits) {  // the fused prologue: gates from the gate layer's logits
        sm.a[tid] = expf(gate_g_from_logit(ld_in(static_cast<const IO*>(g) + row)));
        sm.beta[tid] = gate_beta_from_logit(ld_in(static_cast<const IO*>(beta) + row));
      } else {
        sm.a[tid] = expf(__ldg(static_cast<const float*>(g) + row));
        sm.beta[tid] = __ldg(static_cast<const float*>(beta) + row);
      }
    }
    __syncthreads();
    // ---- per-token norms and k^.q^ (one warp per token)
    for (int tok = warp; tok < n; tok += kWarps) {
      float kk = 0.f, qq = 0.f, kq = 0.f;
      for (int i = lane; i < Dk; i += 32) {
        const float ki = sm.k[tok][i], qi = sm.q[tok][i];
        kk = fmaf(ki, ki, kk);
        qq = fmaf(qi, qi, qq);
        kq = fmaf(ki, qi, kq);
      }
#pragma unroll
      for (int off = 16; off; off >>= 1) {
        kk += __shfl_xor_sync(0xffffffffu, kk, off);
        qq += __shfl_xor_sync(0xffffffffu, qq, off);
        kq += __shfl_xor_sync(0xffffffffu, kq, off);
      }
      if (lane == 0) {
        const float rk = 1.0f / sqrtf(fmaxf(kk, 1e-12f));
        const float rq = 1.0f / sqrtf(fmaxf(qq, 1e-12f));
        sm.rk[tok] = rk;
        sm.rq[tok] = rq;
        sm.kq[tok] = kq * rk * rq;
      }
    }
    __syncthreads();
    // ---- serial walk over the staged tokens
    for (int tok = 0; tok < n; ++tok) {
      const float a = sm.a[tok], bt = sm.beta[tok];
      const float rk = sm.rk[tok], rq = sm.rq[tok], kq = sm.kq[tok];
      float kr[kRows];
      float red[2 * kColsPerWarp];
#pragma unroll
      for (int c = 0; c < 2 * kColsPerWarp; ++c) red[c] = 0.f;
#pragma unroll
      for (int r = 0; r < kRows; ++r) {
        const int i = lane + 32 * r;
        const bool ok = i < Dk;
        kr[r] = ok ? sm.k[tok][i] * rk : 0.f;
        const float qr = ok ? sm.q[tok][i] * rq : 0.f;
#pragma unroll
        for (int c = 0; c < kColsPerWarp; ++c) {
          red[c] = fmaf(kr[r], S[r][c], red[c]);
          red[kColsPerWarp + c] = fmaf(qr, S[r][c], red[kColsPerWarp + c]);
        }
      }
#pragma unroll
      for (int off = 16; off; off >>= 1)
#pragma unroll
        for (int c = 0; c < 2 * kColsPerWarp; ++c)
          red[c] += __shfl_xor_sync(0xffffffffu, red[c], off);
      float o_mine = 0.f;
#pragma unroll
      for (int c = 0; c < kColsPerWarp; ++c) {
        const float u = bt * (sm.v[tok][warp * kColsPerWarp + c] - a * red[c]);
#pragma unroll
        for (int r = 0; r < kRows; ++r) S[r][c] = fmaf(a, S[r][c], kr[r] * u);
        const float o = fmaf(a, red[kColsPerWarp + c], u * kq);
        if (lane == c) o_mine = o;
      }
      if (lane < kColsPerWarp) sm.o[tok][warp * kColsPerWarp + lane] = o_mine;
    }
    __syncthreads();
    // ---- write the staged outputs
    for (int idx = tid; idx < n * kCols; idx += kThreads) {
      const int tok = idx / kCols, c = idx - tok * kCols;
      const int t = reverse ? T - 1 - (p0 + tok) : p0 + tok;
      const size_t off = (((size_t)b * T + t) * H + h) * Dv + j0 + c;
      const float o = sm.o[tok][c];
      if (!reverse) {
        if (acc) acc[off] = o;
        else st_out(out + off, o);
      } else {
        const float prev = acc ? acc[off] : ld_out(out + off);
        st_out(out + off, prev + o);
      }
    }
    __syncthreads();
  }
}

template <typename IO>
__global__ void __launch_bounds__(kThreads)
gdn_scan_serial_kernel(const IO* __restrict__ q, const IO* __restrict__ k,
                       const IO* __restrict__ v, const void* __restrict__ g,
                       const void* __restrict__ beta, int logits,
                       const float* state_in, float* state_out, IO* out,
                       float* acc, int T, int H, int Dk, int Dv, int bidir) {
  __shared__ SerialSmem sm;
  const int j0 = blockIdx.x * kCols;
  const int h = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int jw = j0 + warp * kColsPerWarp;
  const size_t sbase = ((size_t)b * H + h) * (size_t)Dk * Dv;

  float S[kRows][kColsPerWarp];
#pragma unroll
  for (int r = 0; r < kRows; ++r) {
    const int i = lane + 32 * r;
    float4 s4 = make_float4(0.f, 0.f, 0.f, 0.f);
    if (state_in && i < Dk)
      s4 = *reinterpret_cast<const float4*>(state_in + sbase + (size_t)i * Dv + jw);
    S[r][0] = s4.x; S[r][1] = s4.y; S[r][2] = s4.z; S[r][3] = s4.w;
  }
  // Every thread has read its part of state_in before anyone writes
  // state_out (they may alias; slices are disjoint across CTAs).
  __syncthreads();

  scan_direction<IO>(sm, S, q, k, v, g, beta, logits, out, bidir ? acc : nullptr, b, h,
                     j0, T, H, Dk, Dv, false);

  if (state_out) {
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
      const int i = lane + 32 * r;
      if (i < Dk)
        *reinterpret_cast<float4*>(state_out + sbase + (size_t)i * Dv + jw) =
            make_float4(S[r][0], S[r][1], S[r][2], S[r][3]);
    }
  }
  if (!bidir) return;
#pragma unroll
  for (int r = 0; r < kRows; ++r)
#pragma unroll
    for (int c = 0; c < kColsPerWarp; ++c) S[r][c] = 0.f;
  scan_direction<IO>(sm, S, q, k, v, g, beta, logits, out, acc, b, h, j0, T, H, Dk, Dv,
                     true);
}

}  // namespace

cudaError_t launch_scan_serial(const ScanArgs& a) {
  const dim3 grid(a.Dv / kCols, a.H, a.B);
  float* acc = nullptr;
  cudaError_t e = cudaSuccess;
  // With bf16 outputs the bidirectional sum is formed in fp32 scratch so the
  // forward half is not rounded twice; with fp32 outputs `out` holds it.
  if (a.bidir && a.dtype == GDN_BF16) {
    const size_t bytes = (size_t)a.B * a.T * a.H * a.Dv * sizeof(float);
    e = cudaMallocAsync(reinterpret_cast<void**>(&acc), bytes, a.stream);
    if (e != cudaSuccess) return e;
  }
  ProfileScope ps(a.stream, kKernSerial);
  if (a.dtype == GDN_F32) {
    gdn_scan_serial_kernel<float><<<grid, kThreads, 0, a.stream>>>(
        static_cast<const float*>(a.q), static_cast<const float*>(a.k),
        static_cast<const float*>(a.v), a.g, a.beta, a.gate_logits ? 1 : 0, a.state_in, a.state_out,
        static_cast<float*>(a.out), nullptr, a.T, a.H, a.Dk, a.Dv, a.bidir);
  } else {
    gdn_scan_serial_kernel<__nv_bfloat16><<<grid, kThreads, 0, a.stream>>>(
        static_cast<const __nv_bfloat16*>(a.q),
        static_cast<const __nv_bfloat16*>(a.k),
        static_cast<const __nv_bfloat16*>(a.v), a.g, a.beta, a.gate_logits ? 1 : 0, a.state_in,
        a.state_out, static_cast<__nv_bfloat16*>(a.out), acc, a.T, a.H, a.Dk,
        a.Dv, a.bidir);
  }
  e = cudaGetLastError();
  if (e == cudaSuccess) count_launches(1);
  if (acc) {
    const cudaError_t f = cudaFreeAsync(acc, a.stream);
    if (e == cudaSuccess) e = f;
  }
  return e;
}

}  // namespace gdn
