// backward.cu -- gradients of the GDN scan (fp32 arithmetic, fp32 or bf16 I/O).
//
// The pages train the bidirectional GDN ("SANA-Streaming：基于混合扩散
// Transformer的实时流式视频编辑系统", 方法步骤详情, second step: bidirectional
// short training); this is the reverse mode of the scan the forward entry
// points compute.  Per token, in scan order, with x = k^^T S_{t-1} and
// u = beta (v - a x):
//
//   S_t = a S_{t-1} + k^ u^T,   o_t = S_t^T q^
//
// so, walking the tokens backwards with dS = dL/dS_t (fp32, in registers):
//
//   dS    += q^ do^T                  dq^  += S_t do
//   du     = dS^T k^                  dv    = beta du
//   dx     = -a beta du               dk^  += dS u + S_{t-1} dx
//   da     = <dS, S_{t-1}> - beta du.x      dbeta = du.(v - a x)
//   dS_{t-1} = a dS + k^ dx^T          dg = a da
//
// and through the normalisation x^ = x / |x| (|x|^2 clamped at 1e-12):
// dx = (dx^ - x^ (x^.dx^)) / |x|, or dx^ / 1e-6 when clamped.  The
// bidirectional mode adds the same recurrence over the time-reversed chunk
// from a zero state; the two directions' gradients add.
//
// Parallelism as in the forward fp32 path: columns of S (and of dS) evolve
// independently, so one CTA owns 16 columns of one (b, h, direction) and
// walks the sequence; dq^, dk^, da and dbeta sum over all columns, so every
// CTA writes its own partial sums and a second kernel adds them.  The states
// S_t the backward walk needs come from checkpoints: a forward walk stores S
// at the start of every 64-token block, and each block is recomputed (its 64
// states kept in this CTA's global scratch, L2-resident) right before it is
// walked backwards.
#include <cuda_bf16.h>

#include "gdn_internal.h"

namespace gdn {
namespace {

constexpr int kBCols = 16;            // state columns per CTA
constexpr int kBWarps = 4;            // 4 columns per warp
constexpr int kBCpw = kBCols / kBWarps;
constexpr int kBThreads = 32 * kBWarps;
constexpr int kBRows = 4;             // rows per lane (Dk <= 128)
constexpr int kBGroup = 16;           // tokens staged together
constexpr int kBBlock = 64;           // tokens between checkpoints
constexpr int kBState = kBThreads * kBRows * kBCpw;  // floats of one state slice (lane-major)

__device__ __forceinline__ float ld_io(const float* p) { return __ldg(p); }
__device__ __forceinline__ float ld_io(const __nv_bfloat16* p) { return __bfloat162float(*p); }

struct BwdSmem {
  float q[kBGroup][128], k[kBGroup][128];  // q^, k^ of the staged tokens
  float v[kBGroup][kBCols], dout[kBGroup][kBCols];
  float a[kBGroup], beta[kBGroup];
  float rq[kBGroup], rk[kBGroup];          // 1 / |q|, 1 / |k| (clamped)
  float x[kBBlock][kBCols], u[kBBlock][kBCols];  // forward intermediates of the block
  float part[kBGroup][kBWarps][2 * 128 + 2];     // per warp: dq^, dk^, da, dbeta
};

struct BwdArgs {
  const void *q, *k, *v;
  const float *g, *beta, *state_in, *d_out_f;
  const void* d_out;          // [B,T,H,Dv] dtype
  const float* d_state_out;   // [B,H,Dk,Dv] or nullptr
  float* d_state_in;          // [B,H,Dk,Dv] or nullptr
  float* ckpt;                // [dir][bh][slice][nblk + 1][kBState]
  float* stbuf;               // [dir][bh][slice][kBBlock][kBState]
  float* pq;                  // [dir][slice][B T H][Dk]   partial dq^
  float* pk;                  // [dir][slice][B T H][Dk]   partial dk^
  float* pab;                 // [dir][slice][B T H][2]    partial da, dbeta
  float* dvb;                 // [dir][B T H][Dv]          dv of each direction
  int B, T, H, Dk, Dv, nslice, nblk;
};

// Stage tokens p0 .. p0 + n - 1 (scan order) of direction `rev`: q^, k^,
// this CTA's 16 columns of v and d_out, a = e^g, beta.
template <typename IO>
__device__ void stage_tokens(BwdSmem& sm, const BwdArgs& A, int b, int h, int j0, int p0, int n,
                             bool rev) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const IO* q = static_cast<const IO*>(A.q);
  const IO* k = static_cast<const IO*>(A.k);
  const IO* v = static_cast<const IO*>(A.v);
  const IO* dout = static_cast<const IO*>(A.d_out);
  for (int e = tid; e < n * A.Dk; e += kBThreads) {
    const int tok = e / A.Dk, i = e - tok * A.Dk;
    const int t = rev ? A.T - 1 - (p0 + tok) : p0 + tok;
    const size_t row = ((size_t)b * A.T + t) * A.H + h;
    sm.q[tok][i] = ld_io(q + row * A.Dk + i);
    sm.k[tok][i] = ld_io(k + row * A.Dk + i);
  }
  for (int e = tid; e < n * kBCols; e += kBThreads) {
    const int tok = e / kBCols, c = e - tok * kBCols;
    const int t = rev ? A.T - 1 - (p0 + tok) : p0 + tok;
    const size_t row = ((size_t)b * A.T + t) * A.H + h;
    sm.v[tok][c] = ld_io(v + row * A.Dv + j0 + c);
    sm.dout[tok][c] = ld_io(dout + row * A.Dv + j0 + c);
  }
  if (tid < n) {
    const int t = rev ? A.T - 1 - (p0 + tid) : p0 + tid;
    const size_t row = ((size_t)b * A.T + t) * A.H + h;
    sm.a[tid] = expf(__ldg(A.g + row));
    sm.beta[tid] = __ldg(A.beta + row);
  }
  __syncthreads();
  for (int tok = warp; tok < n; tok += kBWarps) {  // norms, one warp per token
    float qq = 0.f, kk = 0.f;
    for (int i = lane; i < A.Dk; i += 32) {
      qq = fmaf(sm.q[tok][i], sm.q[tok][i], qq);
      kk = fmaf(sm.k[tok][i], sm.k[tok][i], kk);
    }
#pragma unroll
    for (int off = 16; off; off >>= 1) {
      qq += __shfl_xor_sync(0xffffffffu, qq, off);
      kk += __shfl_xor_sync(0xffffffffu, kk, off);
    }
    const float rq = 1.0f / sqrtf(fmaxf(qq, 1e-12f)), rk = 1.0f / sqrtf(fmaxf(kk, 1e-12f));
    for (int i = lane; i < A.Dk; i += 32) {
      sm.q[tok][i] *= rq;
      sm.k[tok][i] *= rk;
    }
    if (lane == 0) {
      sm.rq[tok] = rq;
      sm.rk[tok] = rk;
    }
  }
  __syncthreads();
}

// This thread's 16 floats of a lane-major state slice.
__device__ __forceinline__ void st_state(float* base, const float (&S)[kBRows][kBCpw]) {
  float4* p = reinterpret_cast<float4*>(base + threadIdx.x * (kBRows * kBCpw));
#pragma unroll
  for (int r = 0; r < kBRows; ++r) p[r] = make_float4(S[r][0], S[r][1], S[r][2], S[r][3]);
}
__device__ __forceinline__ void ld_state(const float* base, float (&S)[kBRows][kBCpw]) {
  const float4* p = reinterpret_cast<const float4*>(base + threadIdx.x * (kBRows * kBCpw));
#pragma unroll
  for (int r = 0; r < kBRows; ++r) {
    const float4 x = p[r];
    S[r][0] = x.x; S[r][1] = x.y; S[r][2] = x.z; S[r][3] = x.w;
  }
}

// One forward token (staged token `tok`): S <- a S + k^ u^T; returns x, u of
// this warp's columns through xo, uo (identical in every lane).
__device__ __forceinline__ void fwd_token(const BwdSmem& sm, int tok, int Dk, float (&S)[kBRows][kBCpw],
                                          float (&xo)[kBCpw], float (&uo)[kBCpw]) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const float a = sm.a[tok], bt = sm.beta[tok];
  float kr[kBRows];
#pragma unroll
  for (int c = 0; c < kBCpw; ++c) xo[c] = 0.f;
#pragma unroll
  for (int r = 0; r < kBRows; ++r) {
    const int i = lane + 32 * r;
    kr[r] = i < Dk ? sm.k[tok][i] : 0.f;
#pragma unroll
    for (int c = 0; c < kBCpw; ++c) xo[c] = fmaf(kr[r], S[r][c], xo[c]);
  }
#pragma unroll
  for (int off = 16; off; off >>= 1)
#pragma unroll
    for (int c = 0; c < kBCpw; ++c) xo[c] += __shfl_xor_sync(0xffffffffu, xo[c], off);
#pragma unroll
  for (int c = 0; c < kBCpw; ++c) {
    uo[c] = bt * (sm.v[tok][warp * kBCpw + c] - a * xo[c]);
#pragma unroll
    for (int r = 0; r < kBRows; ++r) S[r][c] = fmaf(a, S[r][c], kr[r] * uo[c]);
  }
}

template <typename IO>
__global__ void __launch_bounds__(kBThreads)
gdn_bwd_scan_kernel(BwdArgs A) {
  extern __shared__ __align__(16) uint8_t bwd_raw[];
  BwdSmem& sm = *reinterpret_cast<BwdSmem*>(bwd_raw);
  const int slice = blockIdx.x, bh = blockIdx.y, dir = blockIdx.z;
  const int b = bh / A.H, h = bh - b * A.H, j0 = kBCols * slice;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int Dk = A.Dk, Dv = A.Dv, T = A.T;
  const bool rev = dir == 1;
  const size_t cta = ((size_t)dir * (A.B * A.H) + bh) * A.nslice + slice;
  float* ckpt = A.ckpt + cta * (size_t)(A.nblk + 1) * kBState;
  float* stbuf = A.stbuf + cta * (size_t)kBBlock * kBState;
  const int jw = j0 + kBCpw * warp;  // this warp's first column
  const size_t sbase = (size_t)bh * Dk * Dv;

  // ---- forward walk: checkpoints at the start of every block
  float S[kBRows][kBCpw];
#pragma unroll
  for (int r = 0; r < kBRows; ++r) {
    const int i = lane + 32 * r;
#pragma unroll
    for (int c = 0; c < kBCpw; ++c)
      S[r][c] = (!rev && A.state_in && i < Dk) ? A.state_in[sbase + (size_t)i * Dv + jw + c] : 0.f;
  }
  for (int p0 = 0; p0 < T; p0 += kBGroup) {
    const int n = min(kBGroup, T - p0);
    stage_tokens<IO>(sm, A, b, h, j0, p0, n, rev);
    for (int tok = 0; tok < n; ++tok) {
      if ((p0 + tok) % kBBlock == 0) st_state(ckpt + (size_t)((p0 + tok) / kBBlock) * kBState, S);
      float x[kBCpw], u[kBCpw];
      fwd_token(sm, tok, Dk, S, x, u);
    }
    __syncthreads();
  }

  // ---- backward walk, block by block from the end
  float dS[kBRows][kBCpw];
#pragma unroll
  for (int r = 0; r < kBRows; ++r) {
    const int i = lane + 32 * r;
#pragma unroll
    for (int c = 0; c < kBCpw; ++c)
      dS[r][c] = (!rev && A.d_state_out && i < Dk) ? A.d_state_out[sbase + (size_t)i * Dv + jw + c] : 0.f;
  }
  const size_t rows_bth = (size_t)A.B * T * A.H;
  float* pq = A.pq + ((size_t)dir * A.nslice + slice) * rows_bth * Dk;
  float* pk = A.pk + ((size_t)dir * A.nslice + slice) * rows_bth * Dk;
  float* pab = A.pab + ((size_t)dir * A.nslice + slice) * rows_bth * 2;
  float* dvb = A.dvb + (size_t)dir * rows_bth * Dv;
  for (int blk = A.nblk - 1; blk >= 0; --blk) {
    const int pb0 = blk * kBBlock, nb = min(kBBlock, T - pb0);
    // recompute the block: its post-update states and x, u
    ld_state(ckpt + (size_t)blk * kBState, S);
    for (int g0 = 0; g0 < nb; g0 += kBGroup) {
      const int n = min(kBGroup, nb - g0);
      stage_tokens<IO>(sm, A, b, h, j0, pb0 + g0, n, rev);
      for (int tok = 0; tok < n; ++tok) {
        float x[kBCpw], u[kBCpw];
        fwd_token(sm, tok, Dk, S, x, u);
        st_state(stbuf + (size_t)(g0 + tok) * kBState, S);
        if (lane < kBCpw) {
          sm.x[g0 + tok][warp * kBCpw + lane] = x[lane];
          sm.u[g0 + tok][warp * kBCpw + lane] = u[lane];
        }
      }
      __syncthreads();
    }
    // walk it backwards, a group of tokens at a time
    for (int g1 = nb; g1 > 0; g1 -= kBGroup) {
      const int n = min(kBGroup, g1), g0 = g1 - n;
      stage_tokens<IO>(sm, A, b, h, j0, pb0 + g0, n, rev);
      float St[kBRows][kBCpw], Sp[kBRows][kBCpw];  // S_t, S_{t-1}
      ld_state(stbuf + (size_t)(g0 + n - 1) * kBState, St);
      for (int tok = n - 1; tok >= 0; --tok) {
        const int lt = g0 + tok;  // token within the block
        if (lt > 0) ld_state(stbuf + (size_t)(lt - 1) * kBState, Sp);
        else ld_state(ckpt + (size_t)blk * kBState, Sp);
        const float a = sm.a[tok], bt = sm.beta[tok];
        float doc[kBCpw], xc[kBCpw], uc[kBCpw], vc[kBCpw];
#pragma unroll
        for (int c = 0; c < kBCpw; ++c) {
          doc[c] = sm.dout[tok][warp * kBCpw + c];
          xc[c] = sm.x[lt][warp * kBCpw + c];
          uc[c] = sm.u[lt][warp * kBCpw + c];
          vc[c] = sm.v[tok][warp * kBCpw + c];
        }
        float kr[kBRows], qr[kBRows];
#pragma unroll
        for (int r = 0; r < kBRows; ++r) {
          const int i = lane + 32 * r;
          kr[r] = i < Dk ? sm.k[tok][i] : 0.f;
          qr[r] = i < Dk ? sm.q[tok][i] : 0.f;
        }
        // dS += q^ do^T;  dq^ (this warp's columns) = S_t do
        float pqr[kBRows], du[kBCpw];
#pragma unroll
        for (int c = 0; c < kBCpw; ++c) du[c] = 0.f;
#pragma unroll
        for (int r = 0; r < kBRows; ++r) {
          pqr[r] = 0.f;
#pragma unroll
          for (int c = 0; c < kBCpw; ++c) {
            dS[r][c] = fmaf(qr[r], doc[c], dS[r][c]);
            pqr[r] = fmaf(St[r][c], doc[c], pqr[r]);
            du[c] = fmaf(kr[r], dS[r][c], du[c]);
          }
        }
#pragma unroll
        for (int off = 16; off; off >>= 1)
#pragma unroll
          for (int c = 0; c < kBCpw; ++c) du[c] += __shfl_xor_sync(0xffffffffu, du[c], off);
        float dx[kBCpw];
        float pa = 0.f, pbeta = 0.f;
#pragma unroll
        for (int c = 0; c < kBCpw; ++c) {
          dx[c] = -a * bt * du[c];
          pbeta = fmaf(du[c], vc[c] - a * xc[c], pbeta);
          pa = fmaf(-bt * du[c], xc[c], pa);
        }
        // dk^ = dS u + S_{t-1} dx;  <dS, S_{t-1}>;  then dS_{t-1} = a dS + k^ dx^T
        float pkr[kBRows], ds = 0.f;
#pragma unroll
        for (int r = 0; r < kBRows; ++r) {
          pkr[r] = 0.f;
#pragma unroll
          for (int c = 0; c < kBCpw; ++c) {
            pkr[r] = fmaf(dS[r][c], uc[c], fmaf(Sp[r][c], dx[c], pkr[r]));
            ds = fmaf(dS[r][c], Sp[r][c], ds);
            dS[r][c] = fmaf(a, dS[r][c], kr[r] * dx[c]);
          }
        }
#pragma unroll
        for (int off = 16; off; off >>= 1) ds += __shfl_xor_sync(0xffffffffu, ds, off);
        // this warp's partials of the token
        float* pw = sm.part[tok][warp];
#pragma unroll
        for (int r = 0; r < kBRows; ++r) {
          const int i = lane + 32 * r;
          if (i < Dk) {
            pw[i] = pqr[r];
            pw[128 + i] = pkr[r];
          }
        }
        if (lane == 0) {
          pw[256] = ds + pa;  // da over this warp's columns
          pw[257] = pbeta;
        }
        const int t = rev ? T - 1 - (pb0 + lt) : pb0 + lt;
        const size_t row = ((size_t)b * T + t) * A.H + h;
        if (lane < kBCpw) dvb[row * Dv + jw + lane] = bt * du[lane];
#pragma unroll
        for (int r = 0; r < kBRows; ++r)
#pragma unroll
          for (int c = 0; c < kBCpw; ++c) St[r][c] = Sp[r][c];
      }
      __syncthreads();
      // this CTA's partials of the group: sum over the warps
      for (int e = tid; e < n * (2 * Dk + 2); e += kBThreads) {
        const int tok = e / (2 * Dk + 2), f = e - tok * (2 * Dk + 2);
        const int fi = f < 2 * Dk ? (f < Dk ? f : 128 + f - Dk) : 256 + f - 2 * Dk;
        float acc = 0.f;
#pragma unroll
        for (int w = 0; w < kBWarps; ++w) acc += sm.part[tok][w][fi];
        const int t = rev ? T - 1 - (pb0 + g0 + tok) : pb0 + g0 + tok;
        const size_t row = ((size_t)b * T + t) * A.H + h;
        if (f < Dk) pq[row * Dk + f] = acc;
        else if (f < 2 * Dk) pk[row * Dk + f - Dk] = acc;
        else pab[row * 2 + f - 2 * Dk] = acc;
      }
      __syncthreads();
    }
  }
  if (!rev && A.d_state_in) {
#pragma unroll
    for (int r = 0; r < kBRows; ++r) {
      const int i = lane + 32 * r;
      if (i < Dk)
#pragma unroll
        for (int c = 0; c < kBCpw; ++c) A.d_state_in[sbase + (size_t)i * Dv + jw + c] = dS[r][c];
    }
  }
}

// Sum the partials of every slice and direction for one (b, t, h) row, apply
// the normalisation's Jacobian, and write dq, dk, dv, dg, dbeta.
// pab[..][0] holds dL/da (token-serial path: dg = e^g da) or dL/dg itself
// (chunked path, `chunked`).  dvb holds dv itself, or (chunked path) the
// gradient of the rows of X_u = diag(beta) V: then dv = beta dX_u and beta
// gains v . dX_u.  One warp per (b, t, h) row, four rows per
// block; lane l holds elements 4 l .. 4 l + 3 (D <= 128), read 16 bytes at a
// time from the fp32 partials.
constexpr int kRedRows = 4;

__device__ __forceinline__ void ld4_io(const float* p, float (&x)[4]) {
  const float4 v = *reinterpret_cast<const float4*>(p);
  x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
}
__device__ __forceinline__ void ld4_io(const __nv_bfloat16* p, float (&x)[4]) {
  const uint2 v = *reinterpret_cast<const uint2*>(p);
  x[0] = __uint_as_float(v.x << 16); x[1] = __uint_as_float(v.x & 0xFFFF0000u);
  x[2] = __uint_as_float(v.y << 16); x[3] = __uint_as_float(v.y & 0xFFFF0000u);
}
__device__ __forceinline__ void st4_io(float* p, const float (&x)[4]) {
  *reinterpret_cast<float4*>(p) = make_float4(x[0], x[1], x[2], x[3]);
}
__device__ __forceinline__ void st4_io(__nv_bfloat16* p, const float (&x)[4]) {
  const __nv_bfloat162 a = __floats2bfloat162_rn(x[0], x[1]), b = __floats2bfloat162_rn(x[2], x[3]);
  *reinterpret_cast<uint2*>(p) = make_uint2(*reinterpret_cast<const uint32_t*>(&a),
                                            *reinterpret_cast<const uint32_t*>(&b));
}

template <typename IO>
__global__ void __launch_bounds__(32 * kRedRows)
gdn_bwd_reduce_kernel(BwdArgs A, int ndir, void* dq_, void* dk_, void* dv_, float* dg, float* dbeta,
                      int chunked) {
  const size_t rows_bth = (size_t)A.B * A.T * A.H;
  const size_t row = (size_t)blockIdx.x * kRedRows + (threadIdx.x >> 5);
  if (row >= rows_bth) return;  // whole warps
  const int lane = threadIdx.x & 31, Dk = A.Dk, Dv = A.Dv, c = 4 * lane;
  const IO* q = static_cast<const IO*>(A.q);
  const IO* k = static_cast<const IO*>(A.k);
  IO* dq = static_cast<IO*>(dq_);
  IO* dk = static_cast<IO*>(dk_);
  IO* dv = static_cast<IO*>(dv_);
  // Every load of the row first (two directions at most; with one slice per
  // direction -- the chunked path -- nothing waits on another load), then the
  // arithmetic and the stores.
  float gq[4] = {0.f, 0.f, 0.f, 0.f}, gk[4] = {0.f, 0.f, 0.f, 0.f};
  float qi[4] = {0.f, 0.f, 0.f, 0.f}, ki[4] = {0.f, 0.f, 0.f, 0.f}, vi[4] = {0.f, 0.f, 0.f, 0.f};
  float pqv[2][4] = {}, pkv[2][4] = {}, dvv[2][4] = {};
  const bool one_slice = A.nslice == 1;
  if (c < Dk) {
    ld4_io(q + row * Dk + c, qi);
    ld4_io(k + row * Dk + c, ki);
    if (one_slice) {
#pragma unroll
      for (int d = 0; d < 2; ++d)
        if (d < ndir) {
          const size_t base = (size_t)d * rows_bth + row;
          ld4_io(A.pq + base * Dk + c, pqv[d]);
          ld4_io(A.pk + base * Dk + c, pkv[d]);
        }
    }
  }
  if (c < Dv) {
#pragma unroll
    for (int d = 0; d < 2; ++d)
      if (d < ndir) ld4_io(A.dvb + ((size_t)d * rows_bth + row) * Dv + c, dvv[d]);
    if (chunked) ld4_io(static_cast<const IO*>(A.v) + row * Dv + c, vi);
  }
  const float bt = chunked ? __ldg(A.beta + row) : 0.f;
  float2 pab2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};  // (da, dbeta) per direction
  if (one_slice && lane == 0) {
#pragma unroll
    for (int d = 0; d < 2; ++d)
      if (d < ndir) pab2[d] = *reinterpret_cast<const float2*>(A.pab + ((size_t)d * rows_bth + row) * 2);
  }
  if (c < Dk) {
    if (one_slice) {
#pragma unroll
      for (int d = 0; d < 2; ++d)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          gq[e] += pqv[d][e];
          gk[e] += pkv[d][e];
        }
    } else {
      for (int d = 0; d < ndir; ++d)
        for (int s = 0; s < A.nslice; ++s) {
          const size_t base = ((size_t)d * A.nslice + s) * rows_bth + row;
          float x[4], y[4];
          ld4_io(A.pq + base * Dk + c, x);
          ld4_io(A.pk + base * Dk + c, y);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            gq[e] += x[e];
            gk[e] += y[e];
          }
        }
    }
  }
  // |q|^2, |k|^2, q . dq^, k . dk^ over the row
  float t4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    t4[0] = fmaf(qi[e], qi[e], t4[0]);
    t4[1] = fmaf(ki[e], ki[e], t4[1]);
    t4[2] = fmaf(qi[e], gq[e], t4[2]);
    t4[3] = fmaf(ki[e], gk[e], t4[3]);
  }
#pragma unroll
  for (int off = 16; off; off >>= 1)
#pragma unroll
    for (int e = 0; e < 4; ++e) t4[e] += __shfl_xor_sync(0xffffffffu, t4[e], off);
  if (c < Dk) {
    // x^ = x r with r = 1 / max(|x|, 1e-6): dx = r (dx^ - x^ (x^ . dx^)) when
    // |x|^2 > 1e-12, else r dx^ (the clamp makes r constant)
    const float rq = 1.0f / sqrtf(fmaxf(t4[0], 1e-12f)), rk = 1.0f / sqrtf(fmaxf(t4[1], 1e-12f));
    float oq[4], ok[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      oq[e] = t4[0] > 1e-12f ? rq * (gq[e] - qi[e] * rq * rq * t4[2]) : rq * gq[e];
      ok[e] = t4[1] > 1e-12f ? rk * (gk[e] - ki[e] * rk * rk * t4[3]) : rk * gk[e];
    }
    st4_io(dq + row * Dk + c, oq);
    st4_io(dk + row * Dk + c, ok);
  }
  float vdx = 0.f;  // v . dX_u (chunked path)
  if (c < Dv) {
    float sv[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) sv[e] = dvv[0][e] + dvv[1][e];
    if (chunked) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        vdx = fmaf(vi[e], sv[e], vdx);
        sv[e] *= bt;
      }
    }
    st4_io(dv + row * Dv + c, sv);
  }
  if (chunked)
#pragma unroll
    for (int off = 16; off; off >>= 1) vdx += __shfl_xor_sync(0xffffffffu, vdx, off);
  if (lane == 0) {
    float da = pab2[0].x + pab2[1].x, db = pab2[0].y + pab2[1].y;
    if (!one_slice)
      for (int d = 0; d < ndir; ++d)
        for (int s = 0; s < A.nslice; ++s) {
          const size_t base = ((size_t)d * A.nslice + s) * rows_bth;
          da += A.pab[(base + row) * 2];
          db += A.pab[(base + row) * 2 + 1];
        }
    dg[row] = chunked ? da : expf(__ldg(A.g + row)) * da;
    dbeta[row] = db + vdx;
  }
}

}  // namespace

size_t bwd_workspace_bytes(int B, int T, int H, int Dk, int Dv, gdn_dtype dtype, bool bidir) {
  if (dtype == GDN_BF16 && bwd_chunked_fits(Dk, Dv)) return bwd_chunked_workspace_bytes(B, T, H, Dk, Dv, bidir);
  const size_t ndir = bidir ? 2 : 1, nslice = Dv / kBCols, nblk = (T + kBBlock - 1) / kBBlock;
  const size_t rows = (size_t)B * T * H, ctas = ndir * B * H * nslice;
  // the (da, dbeta) partials are rounded up to 4 floats so that dv's start
  // stays 16-byte aligned for the reduction's vector loads
  return sizeof(float) * (ctas * (nblk + 1) * kBState + ctas * kBBlock * kBState +
                          2 * ndir * nslice * rows * Dk + ((ndir * nslice * rows * 2 + 3) & ~size_t(3)) +
                          ndir * rows * Dv);
}

cudaError_t launch_backward(const BwdCall& c, void* workspace) {
  if (c.dtype == GDN_BF16 && bwd_chunked_fits(c.Dk, c.Dv)) {
    BwdArgs A = {};
    A.q = c.q; A.k = c.k; A.v = c.v; A.g = c.g; A.beta = c.beta;
    A.B = c.B; A.T = c.T; A.H = c.H; A.Dk = c.Dk; A.Dv = c.Dv; A.nslice = 1;
    cudaError_t e = launch_backward_chunked(c, workspace, &A.pq, &A.pk, &A.pab, &A.dvb);
    if (e != cudaSuccess) return e;
    const size_t rows = (size_t)c.B * c.T * c.H;
    {
      ProfileScope ps(c.stream, kKernBwdReduce);
      gdn_bwd_reduce_kernel<__nv_bfloat16><<<(unsigned)((rows + kRedRows - 1) / kRedRows), 32 * kRedRows, 0, c.stream>>>(
          A, c.bidir ? 2 : 1, c.dq, c.dk, c.dv, c.dg, c.dbeta, 1);
    }
    e = cudaGetLastError();
    if (e == cudaSuccess) count_launches(1);
    return e;
  }
  const int ndir = c.bidir ? 2 : 1, nslice = c.Dv / kBCols, nblk = (c.T + kBBlock - 1) / kBBlock;
  const size_t rows = (size_t)c.B * c.T * c.H, ctas = (size_t)ndir * c.B * c.H * nslice;
  BwdArgs A;
  A.q = c.q; A.k = c.k; A.v = c.v; A.g = c.g; A.beta = c.beta; A.state_in = c.state_in;
  A.d_out_f = nullptr; A.d_out = c.d_out; A.d_state_out = c.d_state_out; A.d_state_in = c.d_state_in;
  A.B = c.B; A.T = c.T; A.H = c.H; A.Dk = c.Dk; A.Dv = c.Dv; A.nslice = nslice; A.nblk = nblk;
  float* w = static_cast<float*>(workspace);
  A.ckpt = w;
  w += ctas * (nblk + 1) * kBState;
  A.stbuf = w;
  w += ctas * kBBlock * kBState;
  A.pq = w;
  w += (size_t)ndir * nslice * rows * c.Dk;
  A.pk = w;
  w += (size_t)ndir * nslice * rows * c.Dk;
  A.pab = w;
  w += ((size_t)ndir * nslice * rows * 2 + 3) & ~size_t(3);
  A.dvb = w;
  const int smem = (int)sizeof(BwdSmem);
  cudaError_t e;
  const dim3 grid(nslice, c.B * c.H, ndir);
  if (c.dtype == GDN_F32) {
    e = cudaFuncSetAttribute(gdn_bwd_scan_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    {
      ProfileScope ps(c.stream, kKernBwdScan);
      gdn_bwd_scan_kernel<float><<<grid, kBThreads, smem, c.stream>>>(A);
    }
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    ProfileScope ps(c.stream, kKernBwdReduce);
    gdn_bwd_reduce_kernel<float><<<(unsigned)((rows + kRedRows - 1) / kRedRows), 32 * kRedRows, 0, c.stream>>>(A, ndir, c.dq, c.dk, c.dv, c.dg,
                                                                       c.dbeta, 0);
  } else {
    e = cudaFuncSetAttribute(gdn_bwd_scan_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             smem);
    if (e != cudaSuccess) return e;
    {
      ProfileScope ps(c.stream, kKernBwdScan);
      gdn_bwd_scan_kernel<__nv_bfloat16><<<grid, kBThreads, smem, c.stream>>>(A);
    }
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    ProfileScope ps(c.stream, kKernBwdReduce);
    gdn_bwd_reduce_kernel<__nv_bfloat16><<<(unsigned)((rows + kRedRows - 1) / kRedRows), 32 * kRedRows, 0, c.stream>>>(A, ndir, c.dq, c.dk, c.dv,
                                                                               c.dg, c.dbeta, 0);
  }
  e = cudaGetLastError();
  if (e == cudaSuccess) count_launches(2);
  return e;
}

}  // namespace gdn
