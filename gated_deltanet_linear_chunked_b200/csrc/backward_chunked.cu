// backward_chunked.cu -- gradients of the GDN scan for bf16 I/O, in the
// chunked (WY / UT) form on tensor cores.
//
// The pages train the bidirectional GDN ("SANA-Streaming：基于混合扩散
// Transformer的实时流式视频编辑系统", 方法步骤详情, second step); this is the
// reverse mode of the chunked forward the bf16 path computes.  Per 64-token
// chunk, in scan order, entered with state S0 (Dk x Dv) and left with S_e:
//
//   A_pi = beta_p e^{g_p - g_i} k^_p . k^_i (i < p),  T = (I + A)^-1
//   X_w = diag(beta e^gam) K^,  X_u = diag(beta) V,  W = T X_w,  U~ = T X_u
//   U = U~ - W S0,  P = M o (Q^ K^T) with M_pi = e^{gam_p - gam_i} (i <= p)
//   O = diag(e^gam) Q^ S0 + P U,  S_e = e^{gam_C} S0 + K~^T U,  K~ = diag(e^{gam_C - gam}) K^
//
// (gam: cumulative log decay in the chunk, gam_C its last value).  Walking the
// chunks backwards with dS_e = dL/dS_e (fp32):
//
//   dU  = P^T dO + K~ dS_e                   dK~ = U dS_e^T
//   dS0 = e^{gam_C} dS_e + Q^^T diag(e^gam) dO - W^T dU      (next chunk's dS_e)
//   dP  = dO U^T,  dQK = M o dP:   dq^ = dQK K^ + diag(e^gam) dO S0^T,  dk^ += dQK^T Q^
//   dW  = -dU S0^T,  dU~ = dU:     [dX_w | dX_u] solves (I + A)^T X = [dW | dU~]
//   dA  = -(dX_w W^T + dX_u U~^T)  on i < p   (= -T^T dT T^T, as T X_w = W, T X_u = U~)
//   dG  = dA o (beta_p e^{gam_p - gam_i}),    dk^ += (dG + dG^T) K^
//   dk^ += diag(beta e^gam) dX_w + diag(e^{gam_C - gam}) dK~,   dv = diag(beta) dX_u
//
// and beta and gam collect the matching row sums (each exponent gam_p - gam_i
// sends +c to row p and -c to row i); dg_p is the suffix sum of dgam over the
// chunk in scan order plus dgam_C.  The forward's stages A and B provide W,
// K~, U~, U and S0 of every chunk (their workspace); this kernel, one CTA per
// (b, h, direction), walks the chunks in reverse, recomputes Q^ K^T, K^ K^T
// and the gates, and runs every product above on tf32 mma.sync (fp32
// accumulate).  dq^ and dk^ (before the normalisation's Jacobian), dv, dg and
// dbeta of each direction go to per-direction partials that the reduction
// kernel of backward.cu sums.
#include <cuda_bf16.h>

#include "gdn_internal.h"

namespace gdn {
namespace {

constexpr int kBcThreads = 256;
constexpr int kBcWarps = kBcThreads / 32;
constexpr int kLd64 = 68;   // fp32 row stride of the 64 x 64 tiles
constexpr int kLdE = 72;    // bf16 row stride of the 64 x 64 E tile
constexpr int kMaxBlocks = 4;  // 16 x 16 output blocks per warp of a 64 x Dk product, Dk <= 112

// Shared memory of one CTA, laid out by (Dk, Dv) (byte offsets; all 16-byte
// aligned).  bf16 tiles have row strides Dk + 8 or Dv + 8, fp32 ones Dk + 4,
// Dv + 4 or 68.  Rows are scan positions.
struct BcLayout {
  int lbk, lbv, ldk, ldv;  // strides: bf16 Dk / Dv tiles, fp32 Dk / Dv tiles
  uint32_t q, k, dout, w, ktut, u, s0, P, A, E, dU, dW, small, total;
  __host__ __device__ BcLayout(int Dk, int Dv) {
    lbk = Dk + 8;
    lbv = Dv + 8;
    ldk = Dk + 4;
    ldv = Dv + 4;
    const int lbmax = lbk > lbv ? lbk : lbv;
    uint32_t o = 0;
    q = o;    o += 64 * lbk * 2;    // q^
    k = o;    o += 64 * lbk * 2;    // k^
    dout = o; o += 64 * lbv * 2;    // dO
    w = o;    o += 64 * lbk * 2;    // W
    ktut = o; o += 64 * lbmax * 2;  // K~, then U~
    u = o;    o += 64 * lbv * 2;    // U
    s0 = o;   o += Dk * lbv * 2;    // S0 [Dk][Dv]
    P = o;    o += 64 * kLd64 * 4;  // P, then dQK, then dG
    A = o;    o += 64 * kLd64 * 4;  // A
    E = o;    o += 64 * kLdE * 2;   // e^{gam_p - gam_i} K^ K^T (i < p), bf16
    dU = o;   o += 64 * ldv * 4;    // dU, then dX_u
    dW = o;                          // dS_e (bf16 [Dk][Dv]), then dq^, then dW, then dX_w
    {
      const uint32_t a = 64u * ldk * 4, b = (uint32_t)Dk * lbv * 2;
      o += a > b ? a : b;
    }
    small = o; o += 8 * 64 * 4 + 64;
    total = o;
  }
};

struct BcSmall {
  float g[64], beta[64], gam[64], eg[64], dgam[64], dbeta[64], cK[64];
  int row[64];  // (b, t, h) row of scan position p, -1 past T
  float red[kBcWarps];
};

struct BcArgs {
  const __nv_bfloat16 *q, *k, *v, *dout;
  const float *g, *beta;
  const float* d_state_out;  // dL/dS of the forward scan's final state, or null
  float* d_state_in;         // dL/dS0 of the forward scan, or null
  const uint8_t* ws;         // the forward's workspace
  WsLayout wl;
  float* dS;                 // [dir][bh][Dk][Dv] running dS_e
  float *pq, *pk, *pab, *dvb;  // [dir][rows][Dk], [dir][rows][Dk], [dir][rows][2], [dir][rows][Dv]
  int B, T, H, Dk, Dv, nC, NBH;
};

// tf32 operands are fp32 bit patterns whose low 13 mantissa bits the tensor
// core ignores: bf16-sourced values are exact, fp32 intermediates are
// truncated (relative error below 2^-10).
__device__ __forceinline__ uint32_t tf32(float x) { return __float_as_uint(x); }
__device__ __forceinline__ float bf(const __nv_bfloat16& x) { return __bfloat162float(x); }
__device__ __forceinline__ void cp16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                   static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
               "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// The 16 x 8 tile product D = sum_k A(m0 + i, k) B(k, n0 + j), k < K, on
// tf32 mma.sync.m16n8k8 (fp32 accumulate).
// Two neighbouring 16 x 8 tiles (columns n0 and n0 + 8) at once: the A
// fragment is shared and the two accumulator chains are independent.
template <class FA, class FB>
__device__ __forceinline__ void tile_mma(int m0, int n0, int K, FA A, FB B, float (&d)[2][4]) {
  const int lane = threadIdx.x & 31, gq = lane >> 2, tq = lane & 3;
#pragma unroll
  for (int h = 0; h < 2; ++h) d[h][0] = d[h][1] = d[h][2] = d[h][3] = 0.f;
#pragma unroll 2
  for (int k0 = 0; k0 < K; k0 += 8) {
    const uint32_t a0 = tf32(A(m0 + gq, k0 + tq)), a1 = tf32(A(m0 + gq + 8, k0 + tq));
    const uint32_t a2 = tf32(A(m0 + gq, k0 + tq + 4)), a3 = tf32(A(m0 + gq + 8, k0 + tq + 4));
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint32_t b0 = tf32(B(k0 + tq, n0 + 8 * h + gq)), b1 = tf32(B(k0 + tq + 4, n0 + 8 * h + gq));
      asm volatile(
          "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 "
          "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
          : "+f"(d[h][0]), "+f"(d[h][1]), "+f"(d[h][2]), "+f"(d[h][3])
          : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
    }
  }
}
// Element e (0..3) of a thread's accumulator tile: row and column offsets.
__device__ __forceinline__ int tile_row(int e) { return ((threadIdx.x & 31) >> 2) + (e >= 2 ? 8 : 0); }
__device__ __forceinline__ int tile_col(int e) { return 2 * (threadIdx.x & 3) + (e & 1); }

// Out (M x N) = A B: warps take the 16 x 8 output tiles in turn and hand
// each element to epi(m, n, value).  M % 16 == N % 8 == K % 8 == 0.
template <class FA, class FB, class FE>
__device__ __forceinline__ void gemm(int M, int N, int K, FA A, FB B, FE epi) {
  const int warp = threadIdx.x >> 5;
  const int tn = N >> 4, nt = (M >> 4) * tn;  // 16 x 16 blocks
  for (int t = warp; t < nt; t += kBcWarps) {
    const int m0 = (t / tn) << 4, n0 = (t % tn) << 4;
    float d[2][4];
    tile_mma(m0, n0, K, A, B, d);
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
      for (int e = 0; e < 4; ++e) epi(m0 + tile_row(e), n0 + 8 * h + tile_col(e), d[h][e]);
  }
}
// Row and column sums of a per-element contribution c(m, n, value) over each
// output tile, reduced across the tile's lanes with shuffles and added to
// rsum[m] (+) and csum[n] (-) with one shared atomic per row / column; epi
// runs on every element as in gemm.
template <class FA, class FB, class FC, class FE>
__device__ __forceinline__ void gemm_rc(int M, int N, int K, FA A, FB B, FC contrib, FE epi,
                                        float* rsum, float* csum) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tn = N >> 4, nt = (M >> 4) * tn;  // 16 x 16 blocks
  for (int t = warp; t < nt; t += kBcWarps) {
    const int m0 = (t / tn) << 4, nb = (t % tn) << 4;
    float dd[2][4];
    tile_mma(m0, nb, K, A, B, dd);
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
    const int n0 = nb + 8 * hh;
    float d[4], c[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      d[e] = dd[hh][e];
      c[e] = contrib(m0 + tile_row(e), n0 + tile_col(e), d[e]);
      epi(m0 + tile_row(e), n0 + tile_col(e), d[e]);
    }
    float r0 = c[0] + c[1], r1 = c[2] + c[3];  // rows gq, gq + 8: sum over the 4 lanes of a row
    r0 += __shfl_xor_sync(0xffffffffu, r0, 1);
    r1 += __shfl_xor_sync(0xffffffffu, r1, 1);
    r0 += __shfl_xor_sync(0xffffffffu, r0, 2);
    r1 += __shfl_xor_sync(0xffffffffu, r1, 2);
    if (rsum && (lane & 3) == 0) {
      atomicAdd(&rsum[m0 + tile_row(0)], r0);
      atomicAdd(&rsum[m0 + tile_row(2)], r1);
    }
    if (csum) {
      float c0 = c[0] + c[2], c1 = c[1] + c[3];  // columns 2 tq, 2 tq + 1: sum over the 8 rows
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) {
        c0 += __shfl_xor_sync(0xffffffffu, c0, off);
        c1 += __shfl_xor_sync(0xffffffffu, c1, off);
      }
      if (lane < 4) {
        atomicAdd(&csum[n0 + tile_col(0)], -c0);
        atomicAdd(&csum[n0 + tile_col(1)], -c1);
      }
    }
    }
  }
}

// The same for a 64 x N product accumulated in registers: block i of warp w
// is output block w + 8 i, acc[i][h][e] += epi(m, n, value).
template <class FA, class FB, class FE>
__device__ __forceinline__ void gemm_acc(int N, int K, FA A, FB B, float (&acc)[kMaxBlocks][2][4], FE epi) {
  const int warp = threadIdx.x >> 5;
  const int tn = N >> 4, nt = 4 * tn;  // 16 x 16 blocks of a 64-row product
#pragma unroll
  for (int i = 0; i < kMaxBlocks; ++i) {
    const int t = warp + kBcWarps * i;
    if (t < nt) {
      const int m0 = (t / tn) << 4, n0 = (t % tn) << 4;
      float d[2][4];
      tile_mma(m0, n0, K, A, B, d);
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int e = 0; e < 4; ++e)
          acc[i][h][e] += epi(m0 + tile_row(e), n0 + 8 * h + tile_col(e), d[h][e]);
    }
  }
}

// x_p = r_p - sum_{t > p} A[t][p] x_t for p = 63 .. 0: (I + A)^T x = r for
// one column held in registers.  Each sum takes the newest x_t (t = p + 1)
// last, so row p's accumulation overlaps rows p + 1, p + 2, ...
__device__ __forceinline__ void solve_upper(const float* A, float (&x)[64]) {
#pragma unroll
  for (int p = 62; p >= 0; --p) {
    float s = x[p];
#pragma unroll
    for (int t = 63; t > p; --t) s = fmaf(-A[t * kLd64 + p], x[t], s);
    x[p] = s;
  }
}

__global__ void __launch_bounds__(kBcThreads, 1) gdn_bwd_chunk_kernel(BcArgs a) {
  extern __shared__ __align__(16) uint8_t bc_raw[];
  const int Dk = a.Dk, Dv = a.Dv;
  const BcLayout L(Dk, Dv);
  __nv_bfloat16* sQ = reinterpret_cast<__nv_bfloat16*>(bc_raw + L.q);
  __nv_bfloat16* sK = reinterpret_cast<__nv_bfloat16*>(bc_raw + L.k);
  __nv_bfloat16* sO = reinterpret_cast<__nv_bfloat16*>(bc_raw + L.dout);
  __nv_bfloat16* sW = reinterpret_cast<__nv_bfloat16*>(bc_raw + L.w);
  __nv_bfloat16* sKU = reinterpret_cast<__nv_bfloat16*>(bc_raw + L.ktut);
  __nv_bfloat16* sU = reinterpret_cast<__nv_bfloat16*>(bc_raw + L.u);
  __nv_bfloat16* sS0 = reinterpret_cast<__nv_bfloat16*>(bc_raw + L.s0);
  float* sP = reinterpret_cast<float*>(bc_raw + L.P);
  float* sA = reinterpret_cast<float*>(bc_raw + L.A);
  __nv_bfloat16* sE = reinterpret_cast<__nv_bfloat16*>(bc_raw + L.E);
  float* sdU = reinterpret_cast<float*>(bc_raw + L.dU);
  float* sdW = reinterpret_cast<float*>(bc_raw + L.dW);
  __nv_bfloat16* sdS = reinterpret_cast<__nv_bfloat16*>(bc_raw + L.dW);  // steps 2-3 only
  BcSmall& sm = *reinterpret_cast<BcSmall*>(bc_raw + L.small);
  const int lbk = L.lbk, lbv = L.lbv, ldk = L.ldk, ldv = L.ldv;

  const int bh = blockIdx.x, dir = blockIdx.y;
  const int b = bh / a.H, h = bh - b * a.H;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const size_t rows_bth = (size_t)a.B * a.T * a.H;
  float* dS = a.dS + ((size_t)dir * a.NBH + bh) * Dk * Dv;
  float* pq = a.pq + (size_t)dir * rows_bth * Dk;
  float* pk = a.pk + (size_t)dir * rows_bth * Dk;
  float* pab = a.pab + (size_t)dir * rows_bth * 2;
  float* dvb = a.dvb + (size_t)dir * rows_bth * Dv;

  // dS_e of the last chunk walked first: the final state's gradient (forward
  // scan) or zero (the reverse scan's final state is not an output)
  for (int e = tid; e < Dk * Dv; e += kBcThreads)
    dS[e] = (dir == 0 && a.d_state_out) ? a.d_state_out[(size_t)bh * Dk * Dv + e] : 0.f;
  __syncthreads();

  for (int step = 0; step < a.nC; ++step) {
    // chunks in reverse scan order: time chunk j; scan position p is time
    // row p (forward) or 63 - p (reverse) of the tile
    const int j = dir == 0 ? a.nC - 1 - step : step;
    const int t0 = 64 * j;
    const uint8_t* blk = a.ws + (((size_t)dir * a.NBH + bh) * a.nC + j) * a.wl.block_bytes;

    // ---- stage the chunk
    if (tid < 64) {
      const int p = tid, t = t0 + (dir == 0 ? p : 63 - p);
      const bool valid = t < a.T;
      const size_t r = ((size_t)b * a.T + t) * a.H + h;
      sm.row[p] = valid ? (int)r : -1;
      sm.g[p] = valid ? __ldg(a.g + r) : 0.f;
      sm.beta[p] = valid ? __ldg(a.beta + r) : 0.f;
      sm.dgam[p] = 0.f;
      sm.dbeta[p] = 0.f;
      sm.cK[p] = 0.f;
    }
    __syncthreads();
    {
      // q, k, dO rows (zero past T); W, K~, U tiles and S0 from the workspace
      const int ck = Dk / 8, cv = Dv / 8;
      for (int e = tid; e < 64 * (2 * ck + cv); e += kBcThreads) {
        const int p = e / (2 * ck + cv), c = e - p * (2 * ck + cv), r = sm.row[p];
        __nv_bfloat16* dst;
        const __nv_bfloat16* src;
        if (c < ck) {
          dst = sQ + p * lbk + 8 * c;
          src = a.q + (size_t)r * Dk + 8 * c;
        } else if (c < 2 * ck) {
          dst = sK + p * lbk + 8 * (c - ck);
          src = a.k + (size_t)r * Dk + 8 * (c - ck);
        } else {
          dst = sO + p * lbv + 8 * (c - 2 * ck);
          src = a.dout + (size_t)r * Dv + 8 * (c - 2 * ck);
        }
        if (r >= 0) cp16(dst, src);
        else *reinterpret_cast<uint4*>(dst) = make_uint4(0, 0, 0, 0);
      }
      // [slab][time row][8] -> [scan row][8 slab ..]
      for (int e = tid; e < 64 * (2 * ck + cv); e += kBcThreads) {
        const int sl = e >> 6, t = e & 63, p = dir == 0 ? t : 63 - t;
        if (sl < ck) {
          cp16(sW + p * lbk + 8 * sl, blk + a.wl.off_w + 16 * (sl * 64 + t));
        } else if (sl < 2 * ck) {
          cp16(sKU + p * lbk + 8 * (sl - ck), blk + a.wl.off_kt + 16 * ((sl - ck) * 64 + t));
        } else {
          cp16(sU + p * lbv + 8 * (sl - 2 * ck), blk + a.wl.off_u + 16 * ((sl - 2 * ck) * 64 + t));
        }
      }
      for (int e = tid; e < cv * Dk; e += kBcThreads) {  // S0: [Dv/8][Dk][8] -> [Dk][Dv]
        const int sl = e / Dk, d = e - sl * Dk;
        cp16(sS0 + d * lbv + 8 * sl, blk + a.wl.off_s + 16 * (sl * Dk + d));
      }
      // dS_e rounded to bf16 for the two products that read it
      for (int e = tid; e < Dk * Dv / 4; e += kBcThreads) {
        const int d = (4 * e) / Dv, c = 4 * e - d * Dv;
        const float4 x = *reinterpret_cast<const float4*>(dS + 4 * e);
        __nv_bfloat162* o = reinterpret_cast<__nv_bfloat162*>(sdS + d * lbv + c);
        o[0] = __floats2bfloat162_rn(x.x, x.y);
        o[1] = __floats2bfloat162_rn(x.z, x.w);
      }
      cp_wait_all();
    }
    if (warp == 0) {  // gam = inclusive prefix sum of g in scan order
      const float a0 = sm.g[2 * lane], a1 = sm.g[2 * lane + 1];
      float incl = a0 + a1;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += y;
      }
      const float excl = incl - (a0 + a1);
      sm.gam[2 * lane] = excl + a0;
      sm.gam[2 * lane + 1] = incl;
      sm.eg[2 * lane] = expf(excl + a0);
      sm.eg[2 * lane + 1] = expf(incl);
    }
    __syncthreads();
    for (int p = warp; p < 64; p += kBcWarps) {  // q^ = q / |q|, k^ likewise, in place
      float qq = 0.f, kk = 0.f;
      for (int d = lane; d < Dk; d += 32) {
        const float qv = bf(sQ[p * lbk + d]), kv = bf(sK[p * lbk + d]);
        qq = fmaf(qv, qv, qq);
        kk = fmaf(kv, kv, kk);
      }
#pragma unroll
      for (int off = 16; off; off >>= 1) {
        qq += __shfl_xor_sync(0xffffffffu, qq, off);
        kk += __shfl_xor_sync(0xffffffffu, kk, off);
      }
      const float rq = 1.f / sqrtf(fmaxf(qq, 1e-12f)), rk = 1.f / sqrtf(fmaxf(kk, 1e-12f));
      for (int d = lane; d < Dk; d += 32) {
        sQ[p * lbk + d] = __float2bfloat16_rn(bf(sQ[p * lbk + d]) * rq);
        sK[p * lbk + d] = __float2bfloat16_rn(bf(sK[p * lbk + d]) * rk);
      }
    }
    __syncthreads();
    const float gamC = sm.gam[63], eC = expf(gamC);
    auto Qh = [&](int p, int d) { return bf(sQ[p * lbk + d]); };
    auto Kh = [&](int p, int d) { return bf(sK[p * lbk + d]); };
    auto dO = [&](int p, int c) { return bf(sO[p * lbv + c]); };

    // ---- 1. P = M o (Q^ K^T); A = beta_p E, E = e^{gam_p - gam_i} K^ K^T (i < p)
    gemm(64, 64, Dk, Qh, [&](int kk, int n) { return Kh(n, kk); },
         [&](int m, int n, float v) { sP[m * kLd64 + n] = n <= m ? expf(sm.gam[m] - sm.gam[n]) * v : 0.f; });
    gemm(64, 64, Dk, Kh, [&](int kk, int n) { return Kh(n, kk); }, [&](int m, int n, float v) {
      const float e = n < m ? expf(sm.gam[m] - sm.gam[n]) * v : 0.f;
      sE[m * kLdE + n] = __float2bfloat16_rn(e);
      sA[m * kLd64 + n] = sm.beta[m] * e;
    });
    __syncthreads();

    // ---- 2. dU = P^T dO + K~ dS_e
    gemm(64, Dv, 64 + Dk,
         [&](int m, int kk) { return kk < 64 ? sP[kk * kLd64 + m] : bf(sKU[m * lbk + kk - 64]); },
         [&](int kk, int n) { return kk < 64 ? dO(kk, n) : bf(sdS[(kk - 64) * lbv + n]); },
         [&](int m, int n, float v) { sdU[m * ldv + n] = v; });
    // ---- 3. dK~ = U dS_e^T: dk^ starts as e^{gam_C - gam} dK~; c_i = K~_i . dK~_i
    float dk[kMaxBlocks][2][4];
#pragma unroll
    for (int i = 0; i < kMaxBlocks; ++i)
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) dk[i][hh][0] = dk[i][hh][1] = dk[i][hh][2] = dk[i][hh][3] = 0.f;
    gemm_acc(Dk, Dv, [&](int m, int kk) { return bf(sU[m * lbv + kk]); },
             [&](int kk, int n) { return bf(sdS[n * lbv + kk]); }, dk,
             [&](int m, int, float v) { return expf(gamC - sm.gam[m]) * v; });
    {  // c_m = K~_m . dK~_m = k^_m . dk^_m so far (K~ = e^{gam_C - gam} K^), per block row
      const int tn = Dk >> 4, nt = 4 * tn;
#pragma unroll
      for (int i = 0; i < kMaxBlocks; ++i) {
        const int t = warp + kBcWarps * i;
        if (t < nt) {
          const int m0 = (t / tn) << 4, n0 = (t % tn) << 4;
          float r0 = 0.f, r1 = 0.f;
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            r0 += Kh(m0 + tile_row(0), n0 + 8 * hh + tile_col(0)) * dk[i][hh][0] +
                  Kh(m0 + tile_row(1), n0 + 8 * hh + tile_col(1)) * dk[i][hh][1];
            r1 += Kh(m0 + tile_row(2), n0 + 8 * hh + tile_col(2)) * dk[i][hh][2] +
                  Kh(m0 + tile_row(3), n0 + 8 * hh + tile_col(3)) * dk[i][hh][3];
          }
          r0 += __shfl_xor_sync(0xffffffffu, r0, 1);
          r1 += __shfl_xor_sync(0xffffffffu, r1, 1);
          r0 += __shfl_xor_sync(0xffffffffu, r0, 2);
          r1 += __shfl_xor_sync(0xffffffffu, r1, 2);
          if ((lane & 3) == 0) {
            atomicAdd(&sm.cK[m0 + tile_row(0)], r0);
            atomicAdd(&sm.cK[m0 + tile_row(2)], r1);
          }
        }
      }
    }
    {  // <dS_e, S0> -> dgam_C
      float dot = 0.f;
      for (int e = tid; e < Dk * Dv / 4; e += kBcThreads) {
        const int d = (4 * e) / Dv, c = 4 * e - d * Dv;
        const float4 x = *reinterpret_cast<const float4*>(dS + 4 * e);
        const __nv_bfloat16* s0 = sS0 + d * lbv + c;
        dot = fmaf(x.x, bf(s0[0]), fmaf(x.y, bf(s0[1]), fmaf(x.z, bf(s0[2]), fmaf(x.w, bf(s0[3]), dot))));
      }
#pragma unroll
      for (int off = 16; off; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
      if (lane == 0) sm.red[warp] = dot;
    }
    __syncthreads();  // every read of dS_e and of K~ is done
    float dgamC = 0.f;
#pragma unroll
    for (int w = 0; w < kBcWarps; ++w) dgamC += sm.red[w];
    dgamC *= eC;
    {  // U~ into K~'s buffer (read in step 12)
      const int cv = Dv / 8;
      for (int e = tid; e < 64 * cv; e += kBcThreads) {
        const int sl = e >> 6, t = e & 63, p = dir == 0 ? t : 63 - t;
        cp16(sKU + p * lbv + 8 * sl, blk + a.wl.off_ut + 16 * (sl * 64 + t));
      }
    }

    // ---- 4. dS0 = e^{gam_C} dS_e + Q^^T diag(e^gam) dO - W^T dU  (in place, fp32)
    gemm(Dk, Dv, 128,
         [&](int m, int kk) { return kk < 64 ? Qh(kk, m) * sm.eg[kk] : -bf(sW[(kk - 64) * lbk + m]); },
         [&](int kk, int n) { return kk < 64 ? dO(kk, n) : sdU[(kk - 64) * ldv + n]; },
         [&](int m, int n, float v) { dS[m * Dv + n] = fmaf(eC, dS[m * Dv + n], v); });
    // ---- 5. dP = dO U^T -> dQK = M o dP; gam gets dP o P
    gemm_rc(64, 64, Dv, dO, [&](int kk, int n) { return bf(sU[n * lbv + kk]); },
            [&](int m, int n, float v) { return n <= m ? v * sP[m * kLd64 + n] : 0.f; },
            [&](int m, int n, float v) {
              sP[m * kLd64 + n] = n <= m ? expf(sm.gam[m] - sm.gam[n]) * v : 0.f;
            },
            sm.dgam, sm.dgam);
    // ---- 6. Z = diag(e^gam) dO S0^T: dq^ = Z, gam_p gets q^_p . Z_p
    gemm_rc(64, Dk, Dv, [&](int m, int kk) { return sm.eg[m] * dO(m, kk); },
            [&](int kk, int n) { return bf(sS0[n * lbv + kk]); },
            [&](int m, int n, float v) { return Qh(m, n) * v; },
            [&](int m, int n, float v) { sdW[m * ldk + n] = v; }, sm.dgam, nullptr);
    __syncthreads();
    // ---- 7. dq^ += dQK K^ (same tile owners as step 6)
    gemm(64, Dk, 64, [&](int m, int kk) { return sP[m * kLd64 + kk]; }, Kh,
         [&](int m, int n, float v) { sdW[m * ldk + n] += v; });
    // ---- 8. dk^ += dQK^T Q^
    gemm_acc(Dk, 64, [&](int m, int kk) { return sP[kk * kLd64 + m]; }, Qh, dk,
             [&](int, int, float v) { return v; });
    __syncthreads();
    for (int e = tid; e < 64 * Dk; e += kBcThreads) {  // dq^ out
      const int p = e / Dk, d = e - p * Dk;
      if (sm.row[p] >= 0) pq[(size_t)sm.row[p] * Dk + d] = sdW[p * ldk + d];
    }
    __syncthreads();
    // ---- 9. dW = -dU S0^T
    gemm(64, Dk, Dv, [&](int m, int kk) { return sdU[m * ldv + kk]; },
         [&](int kk, int n) { return bf(sS0[n * lbv + kk]); },
         [&](int m, int n, float v) { sdW[m * ldk + n] = -v; });
    __syncthreads();
    // ---- 10. [dX_w | dX_u] solves (I + A)^T X = [dW | dU], a column per thread
    for (int c = tid; c < Dk + Dv; c += kBcThreads) {
      float* col = c < Dk ? sdW + c : sdU + (c - Dk);
      const int ld = c < Dk ? ldk : ldv;
      float x[64];
#pragma unroll
      for (int p = 0; p < 64; ++p) x[p] = col[p * ld];
      solve_upper(sA, x);
#pragma unroll
      for (int p = 0; p < 64; ++p) col[p * ld] = x[p];
    }
    cp_wait_all();  // U~
    __syncthreads();
    // ---- 11. dk^ += diag(beta e^gam) dX_w;  dv = diag(beta) dX_u;  beta and gam
    //          from the rows of X_w = diag(beta e^gam) K^ and X_u = diag(beta) V
    {
      const int tn = Dk >> 4, nt = 4 * tn;
#pragma unroll
      for (int i = 0; i < kMaxBlocks; ++i) {
        const int t = warp + kBcWarps * i;
        if (t < nt) {
          const int m0 = (t / tn) << 4, n0 = (t % tn) << 4;
#pragma unroll
          for (int hh = 0; hh < 2; ++hh)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int m = m0 + tile_row(e), n = n0 + 8 * hh + tile_col(e);
              dk[i][hh][e] = fmaf(sm.beta[m] * sm.eg[m], sdW[m * ldk + n], dk[i][hh][e]);
            }
        }
      }
    }
    for (int p = warp; p < 64; p += kBcWarps) {
      const int r = sm.row[p];
      float sw = 0.f, su = 0.f;
      for (int d = lane; d < Dk; d += 32) sw = fmaf(Kh(p, d), sdW[p * ldk + d], sw);
      if (r >= 0) {
        for (int c = lane; c < Dv; c += 32) {
          const float xu = sdU[p * ldv + c];
          dvb[(size_t)r * Dv + c] = sm.beta[p] * xu;
          su = fmaf(bf(a.v[(size_t)r * Dv + c]), xu, su);
        }
      }
#pragma unroll
      for (int off = 16; off; off >>= 1) {
        sw += __shfl_xor_sync(0xffffffffu, sw, off);
        su += __shfl_xor_sync(0xffffffffu, su, off);
      }
      if (lane == 0) {  // step 12's epilogues may already be adding to these rows
        atomicAdd(&sm.dbeta[p], sm.eg[p] * sw + su);
        atomicAdd(&sm.dgam[p], sm.beta[p] * sm.eg[p] * sw);
      }
    }
    // ---- 12. dA = -(dX_w W^T + dX_u U~^T) on i < p -> dG; gam and beta from A
    // (dA o E) into sP first: its row sums feed beta, then it becomes dG
    gemm_rc(64, 64, Dk + Dv,
            [&](int m, int kk) { return kk < Dk ? sdW[m * ldk + kk] : sdU[m * ldv + kk - Dk]; },
            [&](int kk, int n) { return kk < Dk ? bf(sW[n * lbk + kk]) : bf(sKU[n * lbv + kk - Dk]); },
            [&](int m, int n, float v) { return n < m ? -v * sA[m * kLd64 + n] : 0.f; },
            [&](int m, int n, float v) { sP[m * kLd64 + n] = n < m ? -v : 0.f; }, sm.dgam, sm.dgam);
    __syncthreads();
    for (int p = warp; p < 64; p += kBcWarps) {  // dbeta_p += sum_i dA_pi E_pi; dG = dA beta_p e^{..}
      float sb = 0.f;
      for (int i = lane; i < p; i += 32) {
        const float dA = sP[p * kLd64 + i];
        sb = fmaf(dA, bf(sE[p * kLdE + i]), sb);
        sP[p * kLd64 + i] = dA * sm.beta[p] * expf(sm.gam[p] - sm.gam[i]);
      }
#pragma unroll
      for (int off = 16; off; off >>= 1) sb += __shfl_xor_sync(0xffffffffu, sb, off);
      if (lane == 0) atomicAdd(&sm.dbeta[p], sb);
    }
    __syncthreads();
    // ---- 13. dk^ += (dG + dG^T) K^
    gemm_acc(Dk, 64, [&](int m, int kk) { return sP[m * kLd64 + kk] + sP[kk * kLd64 + m]; }, Kh, dk,
             [&](int, int, float v) { return v; });
    // ---- 14. outputs: dk^, dbeta, dg = suffix sum of dgam + dgam_C
    {
      const int tn = Dk >> 4, nt = 4 * tn;
#pragma unroll
      for (int i = 0; i < kMaxBlocks; ++i) {
        const int t = warp + kBcWarps * i;
        if (t < nt) {
          const int m0 = (t / tn) << 4, n0 = (t % tn) << 4;
#pragma unroll
          for (int hh = 0; hh < 2; ++hh)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int m = m0 + tile_row(e), n = n0 + 8 * hh + tile_col(e);
              if (sm.row[m] >= 0) pk[(size_t)sm.row[m] * Dk + n] = dk[i][hh][e];
            }
        }
      }
    }
    __syncthreads();  // every addition to dgam and dbeta is done
    if (warp == 0) {
      // K~ = diag(e^{gam_C - gam}) K^: row p's exponent gives -c_p to gam_p
      // and +c_p to gam_C
      float cs = sm.cK[2 * lane] + sm.cK[2 * lane + 1];
#pragma unroll
      for (int off = 16; off; off >>= 1) cs += __shfl_xor_sync(0xffffffffu, cs, off);
      const float dC = dgamC + cs;
      const float d0 = sm.dgam[2 * lane] - sm.cK[2 * lane];
      const float d1 = sm.dgam[2 * lane + 1] - sm.cK[2 * lane + 1];
      // suffix sums over scan positions 2 lane, 2 lane + 1 .. 63
      float incl = d0 + d1;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const float y = __shfl_down_sync(0xffffffffu, incl, off);
        if (lane + off < 32) incl += y;
      }
      const float g0 = incl + dC, g1 = incl - d0 + dC;
      const int r0 = sm.row[2 * lane], r1 = sm.row[2 * lane + 1];
      if (r0 >= 0) {
        pab[(size_t)r0 * 2] = g0;
        pab[(size_t)r0 * 2 + 1] = sm.dbeta[2 * lane];
      }
      if (r1 >= 0) {
        pab[(size_t)r1 * 2] = g1;
        pab[(size_t)r1 * 2 + 1] = sm.dbeta[2 * lane + 1];
      }
    }
    __syncthreads();
  }
  if (dir == 0 && a.d_state_in)
    for (int e = tid; e < Dk * Dv; e += kBcThreads) a.d_state_in[(size_t)bh * Dk * Dv + e] = dS[e];
}

}  // namespace

bool bwd_chunked_fits(int Dk, int Dv) {
  return Dk <= 112 && Dv <= 112 && BcLayout(Dk, Dv).total <= 227u * 1024u;
}

size_t bwd_chunked_workspace_bytes(int B, int T, int H, int Dk, int Dv, bool bidir) {
  const size_t ndir = bidir ? 2 : 1, rows = (size_t)B * T * H, NBH = (size_t)B * H;
  const size_t fwd = (chunk_tc_workspace_bytes(B, T, H, Dk, Dv, bidir) + 255) & ~size_t(255);
  return fwd + sizeof(float) * ndir * (NBH * Dk * Dv + rows * (2 * Dk + 2 + Dv));
}

cudaError_t launch_backward_chunked(const BwdCall& c, void* workspace, float** pq, float** pk,
                                    float** pab, float** dvb) {
  const int ndir = c.bidir ? 2 : 1;
  const size_t rows = (size_t)c.B * c.T * c.H, NBH = (size_t)c.B * c.H;
  uint8_t* base = static_cast<uint8_t*>(workspace);
  const size_t fwd = (chunk_tc_workspace_bytes(c.B, c.T, c.H, c.Dk, c.Dv, c.bidir) + 255) & ~size_t(255);
  // the forward's stages A and B fill the workspace (W, K~, U~, U, S per chunk)
  ScanArgs f;
  f.q = c.q; f.k = c.k; f.v = c.v; f.g = c.g; f.beta = c.beta;
  f.state_in = c.state_in; f.state_out = nullptr; f.out = nullptr;
  f.B = c.B; f.T = c.T; f.H = c.H; f.Dk = c.Dk; f.Dv = c.Dv;
  f.dtype = GDN_BF16; f.chunk = 64; f.bidir = c.bidir; f.gate_logits = false;
  f.stream = c.stream; f.err = c.err; f.wait_limit = c.wait_limit; f.skip_output = true;
  cudaError_t e = launch_chunk_tc(f, base);
  if (e != cudaSuccess) return e;

  BcArgs a;
  a.q = static_cast<const __nv_bfloat16*>(c.q);
  a.k = static_cast<const __nv_bfloat16*>(c.k);
  a.v = static_cast<const __nv_bfloat16*>(c.v);
  a.dout = static_cast<const __nv_bfloat16*>(c.d_out);
  a.g = c.g; a.beta = c.beta;
  a.d_state_out = c.d_state_out; a.d_state_in = c.d_state_in;
  a.ws = base;
  a.wl = chunk_tc_ws_layout(c.Dk, c.Dv);
  float* w = reinterpret_cast<float*>(base + fwd);
  a.dS = w;
  w += ndir * NBH * c.Dk * c.Dv;
  a.pq = w;
  w += ndir * rows * c.Dk;
  a.pk = w;
  w += ndir * rows * c.Dk;
  a.pab = w;
  w += ndir * rows * 2;
  a.dvb = w;
  a.B = c.B; a.T = c.T; a.H = c.H; a.Dk = c.Dk; a.Dv = c.Dv;
  a.nC = (c.T + 63) / 64;
  a.NBH = (int)NBH;
  *pq = a.pq; *pk = a.pk; *pab = a.pab; *dvb = a.dvb;
  const int smem = (int)BcLayout(c.Dk, c.Dv).total;
  e = cudaFuncSetAttribute(gdn_bwd_chunk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  {
    ProfileScope ps(c.stream, kKernBwdChunk);
    gdn_bwd_chunk_kernel<<<dim3((unsigned)NBH, ndir), kBcThreads, smem, c.stream>>>(a);
  }
  e = cudaGetLastError();
  if (e == cudaSuccess) count_launches(1);
  return e;
}

}  // namespace gdn
