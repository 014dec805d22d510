// backward_chunked.cu -- gradients of the GDN scan for bf16 I/O, in the
// chunked (WY / UT) form on tensor cores.
//
// The pages train the bidirectional GDN ("SANA-Streaming：基于混合扩散
// Transformer的实时流式视频编辑系统", 方法步骤详情, second step); this is the
// reverse mode of the chunked forward the bf16 path computes.  Per 64-token
// chunk, in scan order, entered with state S0 (Dk x Dv) and left with S_e:
//
//   A_pi = beta_p e^{gam_p - gam_i} k^_p . k^_i (i < p),  T = (I + A)^-1
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
// K~, U~, U and S0 of every chunk (their workspace).  Only dU and dS0 depend
// on the chunks after this one, so three kernels share the work:
//   gdn_bwd_pre_kernel    every chunk at once: X = P^T dO, Y = Q^^T diag(e^gam) dO
//                         (stored transposed, bf16)
//   gdn_bwd_chain_kernel  per (16 columns of dS, b*h, direction), the chunks in
//                         reverse: dU = X + K~ dS_e, dS0 = e^{gam_C} dS_e + Y - W^T dU
//                         (the columns of dS evolve independently; the state in
//                         fp32 accumulators), each chunk's dU and dS_e stored (bf16)
//   gdn_bwd_grad_kernel   every chunk at once: the other products, from that
//                         chunk's dU and dS_e
// all on bf16 mma.sync.m16n8k16 (fp32 accumulate) fed by ldmatrix or by
// fragments held in registers.  dq^ and dk^ (before the normalisation's
// Jacobian), dX_u, dg and dbeta of each direction go to per-direction
// partials that the reduction kernel of backward.cu sums (forming dv =
// diag(beta) dX_u and beta's share v . dX_u there).
#include <cuda_bf16.h>

#include <algorithm>

#include "gdn_internal.h"
#include "sm100.cuh"

namespace gdn {
namespace {

using namespace sm100;

constexpr int kBcThreads = 256;
constexpr long long kDrainPolls = 1LL << 40;  // drains are bounded by the 2 s timer
constexpr int kLdE = 72;    // bf16 row stride of the 64 x 64 E tile
// The gradient pass runs 16 warps: every phase has many independent 16 x 16
// tiles, and with one CTA per SM the extra warps hide their latencies.
constexpr int kGrThreads = 512;
constexpr int kGrWarps = kGrThreads / 32;
constexpr int kMaxBlocks = 2;  // 16 x 16 output blocks per warp of a 64 x Dk product, Dk <= 128

struct BcSmall {
  float g[64], beta[64], gam[64], eg[64], dgam[64], dbeta[64], cK[64];
  int row[64];  // (b, t, h) row of scan position p, -1 past T
  uint64_t full[5];  // the gradient pass's staged tile groups have landed
};

struct BcArgs {
  const __nv_bfloat16 *q, *k, *v, *dout;
  const float *g, *beta;
  const float* d_state_out;  // dL/dS of the forward scan's final state, or null
  float* d_state_in;         // dL/dS0 of the forward scan, or null
  const uint8_t* ws;         // the forward's workspace
  WsLayout wl;
  // per (direction, b*h, time chunk), rows in scan order:
  // (all bf16, transposed so that a slice of 16 columns is contiguous):
  __nv_bfloat16* XT;         // (P^T dO)^T, Dv x 64 in fragment order [Dv/16][4][32 lanes][8]
  __nv_bfloat16* YT;         // (Q^^T diag(e^gam) dO)^T, Dv x Dk, [Dv/16][Dk/16][32][8]
  __nv_bfloat16* dUT;        // dU^T, Dv x 64, core-matrix [64/8][Dv][8]
  __nv_bfloat16* dSeT;       // dS_e^T, Dv x Dk, [Dk/8][Dv][8] (dS_e: gradient of the chunk's end state)
  const __nv_bfloat16* tinv; // (I + A)^-1 from the forward's stage A, [64/8][64][8] (scan order)
  float* dot;                // <dS_e, S0> (bf16 operands): zeroed by the pre pass, summed by the chain
  float *pq, *pk, *pab, *dvb;  // [dir][rows][Dk], [dir][rows][Dk], [dir][rows][2], [dir][rows][Dv] (dX_u)
  int B, T, H, Dk, Dv, nC, NBH;
  unsigned* err;             // device error word (the chain's bounded waits)
  long long limit;           // polls before a bounded wait gives up
  __device__ size_t blk(int dir, int bh, int j) const { return ((size_t)dir * NBH + bh) * nC + j; }
};

__device__ __forceinline__ float bf(const __nv_bfloat16& x) { return __bfloat162float(x); }

// Element e (0..3) of a thread's accumulator tile: row and column offsets.
__device__ __forceinline__ int tile_row(int e) { return ((threadIdx.x & 31) >> 2) + (e >= 2 ? 8 : 0); }
__device__ __forceinline__ int tile_col(int e) { return 2 * (threadIdx.x & 3) + (e & 1); }

// A bf16 matrix in shared memory.  Element (r, c) sits at byte
//   base + (c / 8) slab + row(r) rs + 2 (c % 8),  row(r) = r, or rrev - r
// for a tile whose rows are stored in reverse.  Row-major with row stride ld
// elements: slab = 16, rs = 2 ld.  The core-matrix layout [c/8][rows][8]
// (each 8-column slab a run of 16-byte rows, as the workspace and TMA tiles
// store them): slab = 16 rows, rs = 16.  As the A operand (m x k): element
// (m, k) = (m, k), or (k, m) when read transposed; as the B operand (k x n):
// element (k, n) = (k, n), or (n, k) when read transposed.
struct BMat {
  uint32_t base;
  int slab, rs;
  int rrev;  // 0: rows in order
};
__device__ __forceinline__ BMat row_major(const void* p, int ld) { return {smem_u32(p), 16, 2 * ld, 0}; }
__device__ __forceinline__ BMat core_mat(const void* p, int rows, bool rev) {
  return {smem_u32(p), 16 * rows, 16, rev ? rows - 1 : 0};
}
__device__ __forceinline__ uint32_t bm_at(const BMat& M, int r, int c8) {
  return M.base + c8 * M.slab + (M.rrev ? M.rrev - r : r) * M.rs;
}
// Element index (in bf16 units) of (r, c) in a core-matrix tile of `rows`
// rows, rows stored reversed when rev.
__device__ __forceinline__ int cidx(int r, int c, int rows, bool rev) {
  return ((c >> 3) * rows + (rev ? rows - 1 - r : r)) * 8 + (c & 7);
}

// 16 x 16 output block (m0, n0) += A B over k < K (K % 16 == 0): per k16
// step one ldmatrix.x4 of each operand and two MMAs; odd steps go to a
// second accumulator, which halves the dependent MMA chains.
template <bool TA, bool TB>
__device__ __forceinline__ void blk16(int m0, int n0, int K, const BMat& A, const BMat& B,
                                      float (&d)[2][4]) {
  const int l = threadIdx.x & 31;
  uint32_t pa, pb;
  int da, db;  // address steps per k16
  if (TA) {
    pa = bm_at(A, (l & 7) + 8 * (l >> 4), (m0 >> 3) + ((l >> 3) & 1));
    da = A.rrev ? -16 * A.rs : 16 * A.rs;
  } else {
    pa = bm_at(A, m0 + (l & 15), l >> 4);
    da = 2 * A.slab;
  }
  if (TB) {
    pb = bm_at(B, n0 + (l & 7) + 8 * (l >> 4), (l >> 3) & 1);
    db = 2 * B.slab;
  } else {
    pb = bm_at(B, (l & 7) + 8 * ((l >> 3) & 1), (n0 >> 3) + (l >> 4));
    db = B.rrev ? -16 * B.rs : 16 * B.rs;
  }
  auto step = [&](float (&acc)[2][4]) {
    uint32_t a[4], bb[4];
    if (TA) ldmatrix_x4_trans(pa, a);
    else ldmatrix_x4(pa, a);
    if (TB) ldmatrix_x4(pb, bb);
    else ldmatrix_x4_trans(pb, bb);
    mma_16816(acc[0], a, bb[0], bb[1]);
    mma_16816(acc[1], a, bb[2], bb[3]);
    pa += da;
    pb += db;
  };
  float e[2][4] = {};
  int k0 = 0;
#pragma unroll 1
  for (; k0 + 32 <= K; k0 += 32) {
    step(d);
    step(e);
  }
  if (k0 < K) step(d);
#pragma unroll
  for (int h = 0; h < 2; ++h)
#pragma unroll
    for (int i = 0; i < 4; ++i) d[h][i] += e[h][i];
}
// Two 16 x 16 output blocks, d0 = block (m0[0], n0[0]) of A0 B0 over k < K0
// and d1 = block (m0[1], n0[1]) of A1 B1 over k < K1 (added to d0, d1), their
// k-steps interleaved: independent chains hide each other's latency.
template <bool TA0, bool TB0, bool TA1, bool TB1>
__device__ __forceinline__ void blk16x2(const int (&m0)[2], const int (&n0)[2], const BMat& A0,
                                        const BMat& B0, int K0, const BMat& A1, const BMat& B1, int K1,
                                        float (&d0)[2][4], float (&d1)[2][4]) {
  const int l = threadIdx.x & 31;
  auto a_at = [&](bool ta, const BMat& A, int m) {
    return ta ? bm_at(A, (l & 7) + 8 * (l >> 4), (m >> 3) + ((l >> 3) & 1)) : bm_at(A, m + (l & 15), l >> 4);
  };
  auto b_at = [&](bool tb, const BMat& B, int n) {
    return tb ? bm_at(B, n + (l & 7) + 8 * (l >> 4), (l >> 3) & 1)
              : bm_at(B, (l & 7) + 8 * ((l >> 3) & 1), (n >> 3) + (l >> 4));
  };
  auto a_step = [](bool ta, const BMat& A) { return ta ? (A.rrev ? -16 * A.rs : 16 * A.rs) : 2 * A.slab; };
  auto b_step = [](bool tb, const BMat& B) { return tb ? 2 * B.slab : (B.rrev ? -16 * B.rs : 16 * B.rs); };
  uint32_t pa0 = a_at(TA0, A0, m0[0]), pb0 = b_at(TB0, B0, n0[0]);
  uint32_t pa1 = a_at(TA1, A1, m0[1]), pb1 = b_at(TB1, B1, n0[1]);
  const int da0 = a_step(TA0, A0), db0 = b_step(TB0, B0), da1 = a_step(TA1, A1), db1 = b_step(TB1, B1);
  const int K = K0 > K1 ? K0 : K1;
#pragma unroll 1
  for (int k0 = 0; k0 < K; k0 += 16) {
    uint32_t a[2][4], bb[2][4];
    if (k0 < K0) {
      if (TA0) ldmatrix_x4_trans(pa0, a[0]);
      else ldmatrix_x4(pa0, a[0]);
      if (TB0) ldmatrix_x4(pb0, bb[0]);
      else ldmatrix_x4_trans(pb0, bb[0]);
      pa0 += da0;
      pb0 += db0;
    }
    if (k0 < K1) {
      if (TA1) ldmatrix_x4_trans(pa1, a[1]);
      else ldmatrix_x4(pa1, a[1]);
      if (TB1) ldmatrix_x4(pb1, bb[1]);
      else ldmatrix_x4_trans(pb1, bb[1]);
      pa1 += da1;
      pb1 += db1;
    }
    if (k0 < K0) {
      mma_16816(d0[0], a[0], bb[0][0], bb[0][1]);
      mma_16816(d0[1], a[0], bb[0][2], bb[0][3]);
    }
    if (k0 < K1) {
      mma_16816(d1[0], a[1], bb[1][0], bb[1][1]);
      mma_16816(d1[1], a[1], bb[1][2], bb[1][3]);
    }
  }
}
__device__ __forceinline__ void zero2(float (&d)[2][4]) {
#pragma unroll
  for (int h = 0; h < 2; ++h) d[h][0] = d[h][1] = d[h][2] = d[h][3] = 0.f;
}

// Out (M x N) = A1 B1 (+ A2 B2): warps take 16 x 16 blocks in turn; epi(m, n,
// value) per element; with rsum / csum, the row / column sums of contrib(m,
// n, value) over each block are added to rsum[m] (+) and csum[n] (-).
// rsum and csum belong to the calling warp alone (plain read-modify-writes:
// shared-memory float atomics cost more than the products here).
template <bool TA1, bool TB1, bool TA2, bool TB2, class FC, class FE>
__device__ __forceinline__ void gemm2(int M, int N, const BMat& A1, const BMat& B1, int K1, const BMat& A2,
                                      const BMat& B2, int K2,
                                      FC contrib, FE epi, float* rsum, float* csum) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  const int tn = N >> 4, nt = (M >> 4) * tn;
  auto finish = [&](int m0, int nb, float (&dd)[2][4]) {
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const int n0 = nb + 8 * hh;
      float c[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        c[e] = rsum || csum ? contrib(m0 + tile_row(e), n0 + tile_col(e), dd[hh][e]) : 0.f;
        epi(m0 + tile_row(e), n0 + tile_col(e), dd[hh][e]);
      }
      if (rsum) {
        float r0 = c[0] + c[1], r1 = c[2] + c[3];
        r0 += __shfl_xor_sync(0xffffffffu, r0, 1);
        r1 += __shfl_xor_sync(0xffffffffu, r1, 1);
        r0 += __shfl_xor_sync(0xffffffffu, r0, 2);
        r1 += __shfl_xor_sync(0xffffffffu, r1, 2);
        if ((lane & 3) == 0) {
          rsum[m0 + tile_row(0)] += r0;
          rsum[m0 + tile_row(2)] += r1;
        }
      }
      if (csum) {
        float c0 = c[0] + c[2], c1 = c[1] + c[3];
#pragma unroll
        for (int off = 4; off < 32; off <<= 1) {
          c0 += __shfl_xor_sync(0xffffffffu, c0, off);
          c1 += __shfl_xor_sync(0xffffffffu, c1, off);
        }
        if (lane < 4) {
          csum[n0 + tile_col(0)] -= c0;
          csum[n0 + tile_col(1)] -= c1;
        }
      }
    }
  };
  for (int t = warp; t < nt; t += 2 * nw) {
    const int m0[2] = {(t / tn) << 4, ((t + nw) / tn) << 4};
    const int nb[2] = {(t % tn) << 4, ((t + nw) % tn) << 4};
    if (t + nw < nt) {  // two blocks, interleaved
      float d0[2][4], d1[2][4];
      zero2(d0);
      zero2(d1);
      blk16x2<TA1, TB1, TA1, TB1>(m0, nb, A1, B1, K1, A1, B1, K1, d0, d1);
      if (K2) blk16x2<TA2, TB2, TA2, TB2>(m0, nb, A2, B2, K2, A2, B2, K2, d0, d1);
      finish(m0[0], nb[0], d0);
      finish(m0[1], nb[1], d1);
    } else {
      float dd[2][4];
      zero2(dd);
      if (K2) {  // the two operand pairs of the one block as two chains
        float d2[2][4];
        zero2(d2);
        const int mm[2] = {m0[0], m0[0]}, nn[2] = {nb[0], nb[0]};
        blk16x2<TA1, TB1, TA2, TB2>(mm, nn, A1, B1, K1, A2, B2, K2, dd, d2);
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int e = 0; e < 4; ++e) dd[h][e] += d2[h][e];
      } else {
        blk16<TA1, TB1>(m0[0], nb[0], K1, A1, B1, dd);
      }
      finish(m0[0], nb[0], dd);
    }
  }
}
// Out (M x N) = A B, stored to global memory as bf16 in mma fragment order:
// 16 x 16 block (bm, bn) at dst + ((bm (N / 16) + bn) 32 + lane) 8, a lane's
// eight values being its accumulator pairs (rows gq, gq + 8 of columns
// 2 tq, 2 tq + 1, then the same of columns 8 + 2 tq, 9 + 2 tq) -- what a warp
// using the block as its accumulator start, or as an A fragment, loads with
// one 16-byte access per lane.
template <bool TA, bool TB>
__device__ __forceinline__ void gemm_store_frag(int M, int N, const BMat& A, const BMat& B, int K,
                                                __nv_bfloat16* dst) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  const int tn = N >> 4, nt = (M >> 4) * tn;
  auto put = [&](int t, const float (&dd)[2][4]) {
    *reinterpret_cast<uint4*>(dst + ((size_t)t * 32 + lane) * 8) =
        make_uint4(pack_bf16x2(dd[0][0], dd[0][1]), pack_bf16x2(dd[0][2], dd[0][3]),
                   pack_bf16x2(dd[1][0], dd[1][1]), pack_bf16x2(dd[1][2], dd[1][3]));
  };
  for (int t = warp; t < nt; t += 2 * nw) {
    const int m0[2] = {(t / tn) << 4, ((t + nw) / tn) << 4}, nb[2] = {(t % tn) << 4, ((t + nw) % tn) << 4};
    float d0[2][4], d1[2][4];
    zero2(d0);
    zero2(d1);
    if (t + nw < nt) {  // two blocks, interleaved
      blk16x2<TA, TB, TA, TB>(m0, nb, A, B, K, A, B, K, d0, d1);
      put(t, d0);
      put(t + nw, d1);
    } else {
      blk16<TA, TB>(m0[0], nb[0], K, A, B, d0);
      put(t, d0);
    }
  }
}

// gam (inclusive prefix sum of the gates in scan order) and e^gam from sm.g;
// one warp.
__device__ void gate_prefix(BcSmall& sm) {
  const int lane = threadIdx.x & 31;
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
// q^ = q / |q| and k^ = k / |k| in place, row by row, for two core-matrix
// [Dk/8][64][8] tiles (rows of zeros stay zero); with sQs, also e^gam times
// the rounded q^ there (eg by scan row; memory row r is scan row 63 - r when
// rev).  Warp w takes rows 8 (w % 8) .. + 7 of q and k (with 16 warps, of
// q for w < 8 and of k for the rest); lane l reads the 4-byte word l % 4 of
// row l / 4 in every 8-column slab, so a warp's read of a slab is 128
// contiguous bytes (a row's slabs are 1 KB apart: lanes spread along a row
// would all hit the same four banks).  8 or 16 warps.  No barrier.
__device__ void normalize_rows_core(const BcArgs& a, __nv_bfloat16* sQ, __nv_bfloat16* sK,
                                    __nv_bfloat16* sQs = nullptr, const float* eg = nullptr,
                                    bool rev = false) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  const int ns = a.Dk / 8;
  const int r = 8 * (warp & 7) + (lane >> 2);
  const int at0 = r * 4 + (lane & 3);  // word index in slab 0; + 256 words a slab
  const int t0 = nw >= 16 ? (warp >> 3) : 0, tstep = nw >= 16 ? 2 : 1;
  for (int ts = t0; ts < 2; ts += tstep) {
    const bool is_q = ts == 0;
    uint32_t* x2 = reinterpret_cast<uint32_t*>(is_q ? sQ : sK);
    float ss = 0.f;
    for (int sl = 0; sl < ns; ++sl) {
      float x0, x1;
      unpack_bf16x2(x2[at0 + 256 * sl], x0, x1);
      ss = fmaf(x0, x0, fmaf(x1, x1, ss));
    }
    ss += __shfl_xor_sync(0xffffffffu, ss, 1);
    ss += __shfl_xor_sync(0xffffffffu, ss, 2);
    const float rn = 1.f / sqrtf(fmaxf(ss, 1e-12f));
    const float e = (sQs && is_q) ? eg[rev ? 63 - r : r] : 0.f;
    for (int sl = 0; sl < ns; ++sl) {
      float x0, x1;
      unpack_bf16x2(x2[at0 + 256 * sl], x0, x1);
      const uint32_t xn = pack_bf16x2(x0 * rn, x1 * rn);
      x2[at0 + 256 * sl] = xn;
      if (sQs && is_q) {  // e^gam times the rounded q^
        unpack_bf16x2(xn, x0, x1);
        reinterpret_cast<uint32_t*>(sQs)[at0 + 256 * sl] = pack_bf16x2(x0 * e, x1 * e);
      }
    }
  }
}

// Tile t of the chunk-parallel passes: chunk j fastest, then b*h, then direction.
struct GrTile {
  int j, bh, dir, b, h;
  size_t bi;  // block index in the per-chunk buffers
};
__device__ __forceinline__ GrTile gr_tile(const BcArgs& a, int t) {
  GrTile c;
  c.j = t % a.nC;
  const int rest = t / a.nC;
  c.bh = rest % a.NBH;
  c.dir = rest / a.NBH;
  c.b = c.bh / a.H;
  c.h = c.bh - c.b * a.H;
  c.bi = a.blk(c.dir, c.bh, c.j);
  return c;
}

// ---------------------------------------------------------------- pre pass
// Every chunk at once: X = P^T dO and Y = Q^^T diag(e^gam) dO, which do not
// depend on the later chunks, stored transposed (X^T = dO^T P, Y^T = dO^T
// diag(e^gam) Q^) in bf16.  Shared memory: q^, k^, dO, diag(e^gam) Q^, P (bf16).
struct PreLayout {
  uint32_t q, k, dout, qs, P, small, total;
  __host__ __device__ PreLayout(int Dk, int Dv) {
    uint32_t o = 0;  // q, k, dO: TMA tiles, core-matrix [D/8][64][8] in time order
    q = o;    o += 64 * Dk * 2;
    k = o;    o += 64 * Dk * 2;
    dout = o; o += 64 * Dv * 2;
    qs = o;   o += 64 * Dk * 2;     // diag(e^gam) Q^ (bf16, the same layout)
    P = o;    o += 64 * kLdE * 2;   // M o (Q^ K^^T) (bf16, row-major, scan order)
    small = o; o += sizeof(BcSmall);
    total = (o + 15) & ~15u;
  }
};

__global__ void __launch_bounds__(kBcThreads)
gdn_bwd_pre_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_o, BcArgs a) {
  extern __shared__ __align__(128) uint8_t bp_raw[];
  using bf16 = __nv_bfloat16;
  const int Dk = a.Dk, Dv = a.Dv;
  const PreLayout L(Dk, Dv);
  bf16* sQ = reinterpret_cast<bf16*>(bp_raw + L.q);
  bf16* sK = reinterpret_cast<bf16*>(bp_raw + L.k);
  bf16* sO = reinterpret_cast<bf16*>(bp_raw + L.dout);
  bf16* sQs = reinterpret_cast<bf16*>(bp_raw + L.qs);
  bf16* sP = reinterpret_cast<bf16*>(bp_raw + L.P);
  BcSmall& sm = *reinterpret_cast<BcSmall*>(bp_raw + L.small);
  const int j = blockIdx.x, bh = blockIdx.y, dir = blockIdx.z;
  const int b = bh / a.H, h = bh - b * a.H;
  const int tid = threadIdx.x;
  const GrTile c = gr_tile(a, j + a.nC * (bh + a.NBH * dir));
  // the gates by 64 threads; q, k, dO by TMA (one thread, one mbarrier)
  if (tid < 64) {
    const int t = 64 * j + (dir == 0 ? tid : 63 - tid);
    const bool valid = t < a.T;
    const size_t r = ((size_t)b * a.T + t) * a.H + h;
    sm.g[tid] = valid ? __ldg(a.g + r) : 0.f;
  }
  if (tid == 0) {
    mbar_init(&sm.full[0], 1);
    fence_mbar_init();
    mbar_arrive_expect_tx(&sm.full[0], 64 * (2 * Dk + Dv) * 2);
    tma_load_tile(sQ, &tm_q, &sm.full[0], 64 * c.j, c.h, c.b);
    tma_load_tile(sK, &tm_k, &sm.full[0], 64 * c.j, c.h, c.b);
    tma_load_tile(sO, &tm_o, &sm.full[0], 64 * c.j, c.h, c.b);
  }
  __syncthreads();
  if ((tid >> 5) == 0) gate_prefix(sm);
  if (!__syncthreads_and(mbar_wait(&sm.full[0], 0, a.limit))) {
    if (tid == 0) atomicOr(a.err, kErrTimeout);
    mbar_wait(&sm.full[0], 0, kDrainPolls);  // nothing may land after the CTA leaves
    return;
  }
  const bool rev = dir != 0;  // the tiles' time rows run against the scan
  normalize_rows_core(a, sQ, sK, sQs, sm.eg, rev);
  __syncthreads();
  auto none = [](int, int, float) { return 0.f; };
  const BMat Q = core_mat(sQ, 64, rev), K = core_mat(sK, 64, rev), O = core_mat(sO, 64, rev);
  const BMat Qs = core_mat(sQs, 64, rev), Pm = row_major(sP, kLdE);
  gemm2<false, true, false, true>(64, 64, Q, K, Dk, Q, K, 0, none, [&](int m, int n, float v) {
    sP[m * kLdE + n] = __float2bfloat16_rn(n <= m ? expf(sm.gam[m] - sm.gam[n]) * v : 0.f);
  }, nullptr, nullptr);
  __syncthreads();
  const size_t blk = a.blk(dir, bh, j);
  if (tid == 0) a.dot[blk] = 0.f;  // the chain pass adds into it
  gemm_store_frag<true, false>(Dv, 64, O, Pm, 64, a.XT + blk * Dv * 64);
  gemm_store_frag<true, false>(Dv, Dk, O, Qs, 64, a.YT + blk * Dv * Dk);
}

// -------------------------------------------------------------- chain pass
// One CTA per (kChSlices slices of 16 columns of dS, b*h, direction): four
// warps per slice and one producer warp, the chunks in reverse scan order.
// A slice runs on the transposed gradient state dS^T (16 x Dk) held in
// mma.sync accumulators.  An accumulator block of dS^T, packed to bf16, is
// the A fragment of the same block, so the slice's warps trade their blocks
// through shared memory in fragment order and nothing is transposed:
//   dU^T  = X^T + dS_e^T K~^T                  (16 x 64, K = Dk; warp w: tokens 16w ..)
//   dS0^T = e^{gam_C} dS_e^T + Y^T - dU^T W    (16 x Dk, K = 64; warp w: k16 blocks w, w + 4)
// B fragments come from the staged W and K~ tiles by ldmatrix (the
// workspace's [slab][time row][8] layout; a lane's row address picks the
// scan-order token).  W, K~ and e^{gam_C} arrive by one bulk copy per chunk
// and the slices' X^T, Y^T and S0 columns by one each, into kChStages stages
// that the producer refills as the slices release them.  Each step writes
// the chunk's dS_e^T and dU^T (bf16) for the gradient pass and adds the
// slice's part of <dS_e, S0> to the chunk's sum.
// One slice per CTA: slices sharing a stage would wait for one another, and
// the step is bound by its dependent MMAs and exchanges, not by the loads.
constexpr int kChSlices = 1;
constexpr int kChStages = 2;
constexpr int kChThreads = 32 * (4 * kChSlices + 1);

struct ChainBarsBwd {
  uint64_t full[kChStages], empty[kChStages];
  int fail[kChSlices];  // a bounded wait of the slice's warps expired
};
static_assert(sizeof(ChainBarsBwd) <= 128, "the chain's barriers fit their slot");

struct ChainSmem {
  uint32_t xs, xu, stage0, stage, xt, yt, s0, total;
  __host__ __device__ explicit ChainSmem(int Dk) {
    xs = 128;                                   // dS_e^T A fragments: [slice][Dk/16][32 lanes][16 B]
    xu = xs + kChSlices * (Dk / 16) * 512;      // dU^T A fragments: [slice][4][32 lanes][16 B]
    stage0 = (xu + kChSlices * 2048 + 127) & ~127u;
    xt = (Dk * 256 + 16 + 127) & ~127u;         // after W, K~ and e^{gam_C}
    yt = xt + kChSlices * 16 * 64 * 2;
    s0 = yt + kChSlices * 16 * Dk * 2;          // the slices' columns of S0: [2 slice][Dk][8]
    stage = (s0 + kChSlices * 16 * Dk * 2 + 127) & ~127u;
    total = stage0 + kChStages * stage;
  }
};

// The producer (one thread): chunk step s into stage s % kChStages once
// every active slice has released the stage's previous chunk.
__device__ void bwd_chain_loads(const BcArgs& a, uint8_t* smem, const ChainSmem& L, int active,
                                int s0, int bh, int dir) {
  ChainBarsBwd& bars = *reinterpret_cast<ChainBarsBwd*>(smem);
  const int Dk = a.Dk, Dv = a.Dv, nC = a.nC;
  const uint32_t wk_bytes = Dk * 256 + 16;
  const uint32_t xt_bytes = active * 16 * 64 * 2, yt_bytes = active * 16 * Dk * 2;
  const uint32_t s0_bytes = active * 16 * Dk * 2;
  int issued = 0;
  bool ok = true;
  for (; issued < nC; ++issued) {
    const int st = issued % kChStages;
    if (issued >= kChStages &&
        !mbar_wait(&bars.empty[st], ((issued / kChStages) - 1) & 1, a.limit)) {
      ok = false;
      break;
    }
    const size_t blk = a.blk(dir, bh, dir == 0 ? nC - 1 - issued : issued);
    uint8_t* dst = smem + L.stage0 + st * L.stage;
    mbar_arrive_expect_tx(&bars.full[st], wk_bytes + xt_bytes + yt_bytes + s0_bytes);
    bulk_load(dst, a.ws + blk * a.wl.block_bytes + a.wl.off_w, wk_bytes, &bars.full[st]);
    bulk_load(dst + L.s0, a.ws + blk * a.wl.block_bytes + a.wl.off_s + (size_t)s0 * 2 * Dk * 16, s0_bytes,
              &bars.full[st]);
    bulk_load(dst + L.xt, a.XT + (blk * Dv + 16 * s0) * 64, xt_bytes, &bars.full[st]);
    bulk_load(dst + L.yt, a.YT + (blk * Dv + 16 * s0) * Dk, yt_bytes, &bars.full[st]);
  }
  if (!ok) atomicOr(a.err, kErrTimeout);
  // nothing may still be landing in shared memory when the CTA leaves
  for (int st = 0; st < kChStages && st < issued; ++st) {
    const int last = st + ((issued - 1 - st) / kChStages) * kChStages;
    mbar_wait(&bars.full[st], (last / kChStages) & 1, kDrainPolls);
  }
}

template <int NKB>
__global__ void __launch_bounds__(kChThreads, 2) gdn_bwd_chain_kernel(BcArgs a) {
  extern __shared__ __align__(128) uint8_t bch_raw[];
  ChainBarsBwd& bars = *reinterpret_cast<ChainBarsBwd*>(bch_raw);
  constexpr int Dk = 16 * NKB;
  constexpr int KPW = (NKB + 3) / 4;  // k16 blocks of dS^T per warp
  const int Dv = a.Dv;
  const ChainSmem L(Dk);
  const int bh = blockIdx.y, dir = blockIdx.z, s0 = blockIdx.x * kChSlices;
  const int active = min(kChSlices, Dv / 16 - s0);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kChStages; ++i) {
      mbar_init(&bars.full[i], 1);
      mbar_init(&bars.empty[i], 4 * active);
    }
    for (int i = 0; i < kChSlices; ++i) bars.fail[i] = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (warp == 4 * kChSlices) {
    if (lane == 0) bwd_chain_loads(a, bch_raw, L, active, s0, bh, dir);
    return;
  }
  const int g = warp >> 2, q = warp & 3;
  if (g >= active) return;
  const int c0 = 16 * (s0 + g), gq = lane >> 2, tq = lane & 3;
  const uint32_t xs_u = smem_u32(bch_raw + L.xs + g * NKB * 512) + lane * 16;
  const uint32_t xu_u = smem_u32(bch_raw + L.xu + g * 2048) + lane * 16;
  volatile int* fail = &bars.fail[g];
  // the lane's ldmatrix row addresses in a W / K~ tile (time rows; scan row
  // p is time row p, or 63 - p in the reverse direction)
  const int mi = lane >> 3, r8 = lane & 7;
  auto trow = [&](int p) { return dir == 0 ? p : 63 - p; };
  const uint32_t k_off = (mi & 1) * 1024 + trow(16 * q + 8 * (mi >> 1) + r8) * 16;
  uint32_t w_off[4];
#pragma unroll
  for (int kt = 0; kt < 4; ++kt) w_off[kt] = (mi >> 1) * 1024 + trow(16 * kt + 8 * (mi & 1) + r8) * 16;

  // dS^T blocks kb = q + 4 i: S[i][h][e] is (column gq + 8 (e >> 1), row d =
  // 16 kb + 8 h + 2 tq + (e & 1)) of dS
  float S[KPW][2][4];
#pragma unroll
  for (int i = 0; i < KPW; ++i)
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int kb = q + 4 * i, col = gq + 8 * (e >> 1), d = 16 * kb + 8 * h + 2 * tq + (e & 1);
        S[i][h][e] = (kb < NKB && dir == 0 && a.d_state_out)
                         ? a.d_state_out[((size_t)bh * Dk + d) * Dv + c0 + col]
                         : 0.f;
      }
  int st = 0;
  uint32_t ph = 0;
  bool ok = true;
  // <dS_e, S0> of the previous chunk: this lane's part, reduced over the warp
  // and added to its block's sum one step later, off the chain's critical path
  float dot_pend = 0.f;
  size_t blk_pend = 0;
  auto flush_dot = [&]() {
#pragma unroll
    for (int off = 16; off; off >>= 1) dot_pend += __shfl_xor_sync(0xffffffffu, dot_pend, off);
    if (lane == 0) atomicAdd(a.dot + blk_pend, dot_pend);
  };
  for (int s = 0; s < a.nC; ++s) {
    const size_t blk = a.blk(dir, bh, dir == 0 ? a.nC - 1 - s : s);
    // dS_e^T (the state entering this chunk) to the slice's warps, in
    // fragment order, and to the gradient pass
    // (dS_e^T of the block: core-matrix [Dk/8][Dv][8], rows c, columns d)
    uint32_t* dse = reinterpret_cast<uint32_t*>(a.dSeT + blk * Dv * Dk);
    uint32_t fse[KPW][4];  // this warp's dS_e^T blocks in bf16 (kept for <dS_e, S0>)
#pragma unroll
    for (int i = 0; i < KPW; ++i) {
      const int kb = q + 4 * i;
      if (kb < NKB) {
        uint32_t (&f)[4] = fse[i];
        f[0] = pack_bf16x2(S[i][0][0], S[i][0][1]);
        f[1] = pack_bf16x2(S[i][0][2], S[i][0][3]);
        f[2] = pack_bf16x2(S[i][1][0], S[i][1][1]);
        f[3] = pack_bf16x2(S[i][1][2], S[i][1][3]);
        st_shared_v4(xs_u + kb * 512, f);
        const int c = c0 + gq, d = 16 * kb + 2 * tq;
        dse[(((d >> 3) * Dv + c) * 8 + (d & 7)) >> 1] = f[0];
        dse[(((d >> 3) * Dv + c + 8) * 8 + (d & 7)) >> 1] = f[1];
        dse[((((d + 8) >> 3) * Dv + c) * 8 + (d & 7)) >> 1] = f[2];
        dse[((((d + 8) >> 3) * Dv + c + 8) * 8 + (d & 7)) >> 1] = f[3];
      }
    }
    const bool okw = __all_sync(0xffffffffu, mbar_wait(&bars.full[st], ph, a.limit));
    uint8_t* sb = bch_raw + L.stage0 + st * L.stage;
    float u[2][4];
    if (okw) {
      // X^T starts dU^T, and e^{gam_C} dS_e^T + Y^T starts dS0^T (both
      // stored in fragment order: one 16-byte load per block)
      const uint32_t xt = smem_u32(sb + L.xt) + g * 2048 + lane * 16;
      const uint32_t yt = smem_u32(sb + L.yt) + g * NKB * 512 + lane * 16;
      const float decay = *reinterpret_cast<const float*>(sb + Dk * 256);
      uint32_t xf[4];
      ld_shared_v4(xt + q * 512, xf);
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int rr = 0; rr < 2; ++rr) unpack_bf16x2(xf[2 * h + rr], u[h][2 * rr], u[h][2 * rr + 1]);
#pragma unroll
      for (int i = 0; i < KPW; ++i) {
        const int kb = q + 4 * i;
        if (kb < NKB) {
          uint32_t yf[4];
          ld_shared_v4(yt + kb * 512, yf);
#pragma unroll
          for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int rr = 0; rr < 2; ++rr) {
              float y0, y1;
              unpack_bf16x2(yf[2 * h + rr], y0, y1);
              S[i][h][2 * rr] = fmaf(decay, S[i][h][2 * rr], y0);
              S[i][h][2 * rr + 1] = fmaf(decay, S[i][h][2 * rr + 1], y1);
            }
        }
      }
    } else if (lane == 0) {
      *fail = 1;
    }
    named_barrier(1 + g, 128);
    if (*fail) {
      ok = false;
      break;
    }
    const uint32_t sw = smem_u32(sb), sk = sw + Dk * 128;
    // ---- dU^T (+)= dS_e^T K~^T over tokens 16 q .. 16 q + 15 (the odd
    //      k16 blocks in a second accumulator: shorter dependent chains)
    {
      uint32_t af[NKB][4], bk[NKB][4];
#pragma unroll
      for (int kb = 0; kb < NKB; ++kb) {
        ld_shared_v4(xs_u + kb * 512, af[kb]);
        ldmatrix_x4(sk + 2 * kb * 1024 + k_off, bk[kb]);
      }
      float u2[2][4] = {};
#pragma unroll
      for (int kb = 0; kb < NKB; ++kb) {
        float (&acc)[2][4] = (kb & 1) ? u2 : u;
        mma_16816(acc[0], af[kb], bk[kb][0], bk[kb][1]);
        mma_16816(acc[1], af[kb], bk[kb][2], bk[kb][3]);
      }
      if (s > 0) flush_dot();  // while the MMAs above run
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int e = 0; e < 4; ++e) u[h][e] += u2[h][e];
    }
    {
      const uint32_t f[4] = {pack_bf16x2(u[0][0], u[0][1]), pack_bf16x2(u[0][2], u[0][3]),
                             pack_bf16x2(u[1][0], u[1][1]), pack_bf16x2(u[1][2], u[1][3])};
      st_shared_v4(xu_u + q * 512, f);
      // dU^T of the block: core-matrix [64/8][Dv][8] (rows c, columns p)
      uint32_t* du = reinterpret_cast<uint32_t*>(a.dUT + blk * Dv * 64);
      const int c = c0 + gq, p = 16 * q + 2 * tq;
      du[(((p >> 3) * Dv + c) * 8 + (p & 7)) >> 1] = f[0];
      du[(((p >> 3) * Dv + c + 8) * 8 + (p & 7)) >> 1] = f[1];
      du[((((p + 8) >> 3) * Dv + c) * 8 + (p & 7)) >> 1] = f[2];
      du[((((p + 8) >> 3) * Dv + c + 8) * 8 + (p & 7)) >> 1] = f[3];
    }
    named_barrier(1 + g, 128);
    // ---- dS0^T (+)= -dU^T W over this warp's blocks
    {
      uint32_t ua[4][4];
#pragma unroll
      for (int kt = 0; kt < 4; ++kt) {
        ld_shared_v4(xu_u + kt * 512, ua[kt]);
#pragma unroll
        for (int e = 0; e < 4; ++e) ua[kt][e] ^= 0x80008000u;  // -dU^T
      }
#pragma unroll
      for (int i = 0; i < KPW; ++i) {
        const int kb = q + 4 * i;
        if (kb < NKB) {
          uint32_t bw[4][4];
#pragma unroll
          for (int kt = 0; kt < 4; ++kt) ldmatrix_x4_trans(sw + 2 * kb * 1024 + w_off[kt], bw[kt]);
          float s2[2][4] = {};  // token blocks 2, 3 (shorter dependent chains)
#pragma unroll
          for (int kt = 0; kt < 4; ++kt) {
            float (&acc)[2][4] = kt < 2 ? S[i] : s2;
            mma_16816(acc[0], ua[kt], bw[kt][0], bw[kt][1]);
            mma_16816(acc[1], ua[kt], bw[kt][2], bw[kt][3]);
          }
#pragma unroll
          for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int e = 0; e < 4; ++e) S[i][h][e] += s2[h][e];
        }
      }
    }
    {  // this lane's part of <dS_e, S0> (bf16 operands, as the gradient pass's
       // products use them), while the MMAs above run: fse[i][2 h + rr] holds
       // columns gq + 8 rr, rows d, d + 1 (d = 16 kb + 8 h + 2 tq); the staged
       // slice of S0 is [2][Dk][8] (rows d)
      const __nv_bfloat16* s0s = reinterpret_cast<const __nv_bfloat16*>(sb + L.s0) + g * 16 * Dk;
      float dot = 0.f;
#pragma unroll
      for (int i = 0; i < KPW; ++i) {
        const int kb = q + 4 * i;
        if (kb < NKB) {
#pragma unroll
          for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int rr = 0; rr < 2; ++rr) {
              const int d = 16 * kb + 8 * h + 2 * tq;
              float x0, x1;
              unpack_bf16x2(fse[i][2 * h + rr], x0, x1);
              dot = fmaf(x0, bf(s0s[(rr * Dk + d) * 8 + gq]), dot);
              dot = fmaf(x1, bf(s0s[(rr * Dk + d + 1) * 8 + gq]), dot);
            }
        }
      }
      dot_pend = dot;
      blk_pend = blk;
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&bars.empty[st]);  // this warp's reads of the stage are done
    if (++st == kChStages) {
      st = 0;
      ph ^= 1;
    }
  }
  if (!ok) {
    if (lane == 0) atomicOr(a.err, kErrTimeout);
    return;
  }
  flush_dot();  // the last chunk's
  if (dir == 0 && a.d_state_in) {
#pragma unroll
    for (int i = 0; i < KPW; ++i)
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int kb = q + 4 * i, col = gq + 8 * (e >> 1), d = 16 * kb + 8 * h + 2 * tq + (e & 1);
          if (kb < NKB) a.d_state_in[((size_t)bh * Dk + d) * Dv + c0 + col] = S[i][h][e];
        }
  }
}

using ChainKernel = void (*)(BcArgs);
ChainKernel chain_kernel_for(int nkb) {
  switch (nkb) {
    case 1: return gdn_bwd_chain_kernel<1>;
    case 2: return gdn_bwd_chain_kernel<2>;
    case 3: return gdn_bwd_chain_kernel<3>;
    case 4: return gdn_bwd_chain_kernel<4>;
    case 5: return gdn_bwd_chain_kernel<5>;
    case 6: return gdn_bwd_chain_kernel<6>;
    default: return gdn_bwd_chain_kernel<7>;
  }
}

// ----------------------------------------------------------- gradient pass
// Every chunk (persistent CTAs, one per SM, walking the (chunk, b*h,
// direction) tiles), from the chunk's dU and dS_e: every product but the
// chain's.  All product operands are bf16 tiles in shared memory -- the
// staged ones in their sources' core-matrix layouts, brought by one thread
// a chunk ahead -- fed to mma.sync.m16n8k16 by ldmatrix (the .trans form
// where a tile is read transposed); dq^ and dk^ accumulate in registers;
// the triangular solve is the product with the forward's own
// T = (I + A)^-1, which its stage A leaves in the workspace.
struct GradLayout {
  int lbk, lbv;
  uint32_t q, k, dout, w, ut, u, s0, dse, P, Tb, E, dU, dW, xw, xu, part, small, total;
  __host__ __device__ GradLayout(int Dk, int Dv) {
    lbk = Dk + 8;
    lbv = Dv + 8;
    uint32_t o = 0;
    // core-matrix tiles [cols/8][rows][8], as their sources store them
    q = o;    o += 64 * Dk * 2;     // q^ (time rows)
    k = o;    o += 2 * 64 * Dk * 2; // k^ (time rows), two buffers: this chunk's and the next's
    dout = o; o += 64 * Dv * 2;     // dO (time rows)
    w = o;    o += 64 * Dk * 2;     // W  (time rows)
    ut = o;   o += 64 * Dv * 2;     // U~ (time rows)
    u = o;    o += 64 * Dv * 2;     // U  (time rows)
    s0 = o;   o += Dk * Dv * 2;     // S0: rows d, columns c; then dX_u (64 x Dv)
    dse = o;  o += Dv * Dk * 2;     // dS_e^T: rows c, columns d; then dX_w (64 x Dk)
    Tb = o;   o += 64 * 64 * 2;     // T = (I + A)^-1 (scan rows)
    dU = o;   o += 64 * Dv * 2;     // dU^T: rows c, columns p
    // row-major tiles the pass writes itself
    P = o;    o += 64 * kLdE * 2;   // P, then dQK, then dA / dG (bf16)
    E = o;    o += 64 * kLdE * 2;   // e^{gam_p - gam_i} K^ K^T (i < p), bf16
    dW = o;   o += 64 * lbk * 2;    // dW (bf16)
    // dX_w (64 x Dk) and dX_u (64 x Dv), core-matrix, in the dS_e^T and S0
    // tiles where they fit (Dv >= 64, Dk >= 64), else tiles of their own
    if (Dv >= 64) xw = dse; else { xw = o; o += 64 * Dk * 2; }
    if (Dk >= 64) xu = s0; else { xu = o; o += 64 * Dv * 2; }
    part = o; o += 3 * kGrWarps * 64 * 4;  // per-warp partial row sums of dgam, dbeta, c
    small = o; o += sizeof(BcSmall);
    total = (o + 15) & ~15u;
  }
};

// A 64 x N product accumulated in registers: block i of warp w is output
// block w + 8 i; acc[i][h][e] += scale(m) * value.
template <bool TA, bool TB, class FS>
__device__ __forceinline__ void gemm_acc2(int N, int K, const BMat& A, const BMat& B, float (&acc)[kMaxBlocks][2][4],
                                          FS scale) {
  static_assert(kMaxBlocks == 2, "two register blocks per warp");
  const int warp = threadIdx.x >> 5;
  const int tn = N >> 4, nt = 4 * tn;
  const int t1 = warp + kGrWarps;
  const int m0[2] = {(warp / tn) << 4, (t1 / tn) << 4}, n0[2] = {(warp % tn) << 4, (t1 % tn) << 4};
  float d[2][2][4];
  zero2(d[0]);
  zero2(d[1]);
  if (t1 < nt) blk16x2<TA, TB, TA, TB>(m0, n0, A, B, K, A, B, K, d[0], d[1]);
  else if (warp < nt) blk16<TA, TB>(m0[0], n0[0], K, A, B, d[0]);
#pragma unroll
  for (int i = 0; i < 2; ++i)
    if (warp + kGrWarps * i < nt)
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[i][h][e] += scale(m0[i] + tile_row(e)) * d[i][h][e];
}
// The register blocks' elements: f(i, h, e, m, n) for every one this thread holds.
template <class F>
__device__ __forceinline__ void for_acc(int N, F f) {
  const int warp = threadIdx.x >> 5;
  const int tn = N >> 4, nt = 4 * tn;
#pragma unroll
  for (int i = 0; i < kMaxBlocks; ++i) {
    const int t = warp + kGrWarps * i;
    if (t < nt) {
      const int m0 = (t / tn) << 4, n0 = (t % tn) << 4;
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int e = 0; e < 4; ++e) f(i, h, e, m0 + tile_row(e), n0 + 8 * h + tile_col(e));
    }
  }
}
// Row sums of f(i, h, e, m, n) over the register blocks, added to dst[m]
// (dst belongs to the calling warp alone).
template <class F>
__device__ __forceinline__ void acc_row_sums(int N, float* dst, F f) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tn = N >> 4, nt = 4 * tn;
#pragma unroll
  for (int i = 0; i < kMaxBlocks; ++i) {
    const int t = warp + kGrWarps * i;
    if (t < nt) {
      const int m0 = (t / tn) << 4, n0 = (t % tn) << 4;
      float r0 = 0.f, r1 = 0.f;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        r0 += f(i, h, 0, m0 + tile_row(0), n0 + 8 * h + tile_col(0)) +
              f(i, h, 1, m0 + tile_row(1), n0 + 8 * h + tile_col(1));
        r1 += f(i, h, 2, m0 + tile_row(2), n0 + 8 * h + tile_col(2)) +
              f(i, h, 3, m0 + tile_row(3), n0 + 8 * h + tile_col(3));
      }
      r0 += __shfl_xor_sync(0xffffffffu, r0, 1);
      r1 += __shfl_xor_sync(0xffffffffu, r1, 1);
      r0 += __shfl_xor_sync(0xffffffffu, r0, 2);
      r1 += __shfl_xor_sync(0xffffffffu, r1, 2);
      if ((lane & 3) == 0) {
        dst[m0 + tile_row(0)] += r0;
        dst[m0 + tile_row(2)] += r1;
      }
    }
  }
}

// The register blocks to fp32 rows of global memory: dst[rows[m] ld + n] for
// rows[m] >= 0, a thread's two neighbouring columns per 8-byte store.
__device__ __forceinline__ void store_acc(int N, const float (&acc)[kMaxBlocks][2][4], float* dst,
                                          int ld, const int* rows) {
  const int warp = threadIdx.x >> 5;
  const int tn = N >> 4, nt = 4 * tn;
#pragma unroll
  for (int i = 0; i < kMaxBlocks; ++i) {
    const int t = warp + kGrWarps * i;
    if (t < nt) {
      const int m0 = (t / tn) << 4, n0 = (t % tn) << 4;
      const int r0 = rows[m0 + tile_row(0)], r1 = rows[m0 + tile_row(2)];
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int n = n0 + 8 * hh + tile_col(0);
        if (r0 >= 0) *reinterpret_cast<float2*>(dst + (size_t)r0 * ld + n) = make_float2(acc[i][hh][0], acc[i][hh][1]);
        if (r1 >= 0) *reinterpret_cast<float2*>(dst + (size_t)r1 * ld + n) = make_float2(acc[i][hh][2], acc[i][hh][3]);
      }
    }
  }
}

// Persistent: CTA x walks tiles x, x + gridDim.x, ...; each group of the
// next tile's inputs is fetched by one thread as soon as this tile has done
// with the buffers it lands in, so the next tile starts with its data on chip.
__global__ void __launch_bounds__(kGrThreads, 1)
gdn_bwd_grad_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_o, BcArgs a, int ntiles) {
  extern __shared__ __align__(128) uint8_t bg_raw[];
  const int Dk = a.Dk, Dv = a.Dv;
  const GradLayout L(Dk, Dv);
  using bf16 = __nv_bfloat16;
  bf16* sQ = reinterpret_cast<bf16*>(bg_raw + L.q);
  bf16* sK = reinterpret_cast<bf16*>(bg_raw + L.k);
  bf16* sO = reinterpret_cast<bf16*>(bg_raw + L.dout);
  bf16* sW = reinterpret_cast<bf16*>(bg_raw + L.w);
  bf16* sUt = reinterpret_cast<bf16*>(bg_raw + L.ut);
  bf16* sU = reinterpret_cast<bf16*>(bg_raw + L.u);
  bf16* sS0 = reinterpret_cast<bf16*>(bg_raw + L.s0);
  bf16* sdST = reinterpret_cast<bf16*>(bg_raw + L.dse);
  bf16* sP = reinterpret_cast<bf16*>(bg_raw + L.P);
  bf16* sT = reinterpret_cast<bf16*>(bg_raw + L.Tb);
  bf16* sE = reinterpret_cast<bf16*>(bg_raw + L.E);
  bf16* sdU = reinterpret_cast<bf16*>(bg_raw + L.dU);
  bf16* sdW = reinterpret_cast<bf16*>(bg_raw + L.dW);
  BcSmall& sm = *reinterpret_cast<BcSmall*>(bg_raw + L.small);
  const int lbk = L.lbk;
  // this warp's partial row sums: gam's, beta's, and c_m = k^_m . dk^_m
  float* const part = reinterpret_cast<float*>(bg_raw + L.part);
  float* const wg = part + (threadIdx.x >> 5) * 64;
  float* const wb = wg + kGrWarps * 64;
  float* const wc = wb + kGrWarps * 64;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const size_t rows_bth = (size_t)a.B * a.T * a.H;
  // Tile groups, each landing on its own mbarrier (one phase per tile):
  //   0: U, dO   1: q   2: T, dU^T   3: S0, dS_e^T, W, U~   4: k (two buffers)
  // Group g of the next tile is issued (by one thread) right after the
  // barrier behind which this tile last reads group g's buffers; k, double
  // buffered, at the start of this tile.
  uint64_t* full = sm.full;
  int kbuf = 1;  // the k buffer of the current tile (the first tile's k goes to buffer 0)
  auto issue = [&](int g, const GrTile& c) {
    const uint8_t* blk = a.ws + c.bi * a.wl.block_bytes;
    fence_proxy_async_smem();  // the buffers' last generic accesses come first
    switch (g) {
      case 0:
        mbar_arrive_expect_tx(&full[0], 64 * Dv * 2 + 64 * Dv * 2);
        bulk_load(sU, blk + a.wl.off_u, 64 * Dv * 2, &full[0]);
        tma_load_tile(sO, &tm_o, &full[0], 64 * c.j, c.h, c.b);
        break;
      case 1:
        mbar_arrive_expect_tx(&full[1], 64 * Dk * 2);
        tma_load_tile(sQ, &tm_q, &full[1], 64 * c.j, c.h, c.b);
        break;
      case 2:
        mbar_arrive_expect_tx(&full[2], 64 * 64 * 2 + 64 * Dv * 2);
        bulk_load(sT, a.tinv + c.bi * 64 * 64, 64 * 64 * 2, &full[2]);
        bulk_load(sdU, a.dUT + c.bi * Dv * 64, 64 * Dv * 2, &full[2]);
        break;
      case 3:
        mbar_arrive_expect_tx(&full[3], 2 * Dk * Dv * 2 + 64 * Dk * 2 + 64 * Dv * 2);
        bulk_load(sS0, blk + a.wl.off_s, Dk * Dv * 2, &full[3]);
        bulk_load(sdST, a.dSeT + c.bi * Dv * Dk, Dv * Dk * 2, &full[3]);
        bulk_load(sW, blk + a.wl.off_w, 64 * Dk * 2, &full[3]);
        bulk_load(sUt, blk + a.wl.off_ut, 64 * Dv * 2, &full[3]);
        break;
      default:  // into the k buffer the tile after this one uses
        mbar_arrive_expect_tx(&full[4], 64 * Dk * 2);
        tma_load_tile(sK + (kbuf ^ 1) * 64 * Dk, &tm_k, &full[4], 64 * c.j, c.h, c.b);
        break;
    }
  };
  float gate_g = 0.f, gate_b = 0.f;  // row tid (< 64) of the next tile
  int gate_row = -1;
  auto load_gates = [&](const GrTile& c) {
    if (tid < 64) {
      const int t = 64 * c.j + (c.dir == 0 ? tid : 63 - tid);
      const bool valid = t < a.T;
      const size_t r = ((size_t)c.b * a.T + t) * a.H + c.h;
      gate_row = valid ? (int)r : -1;
      gate_g = valid ? __ldg(a.g + r) : 0.f;
      gate_b = valid ? __ldg(a.beta + r) : 0.f;
    }
  };

  int t = blockIdx.x;
  if (t >= ntiles) return;
  if (tid == 0) {
    for (int g = 0; g < 5; ++g) mbar_init(&full[g], 1);
    fence_mbar_init();
  }
  __syncthreads();
  {
    const GrTile c = gr_tile(a, t);
    load_gates(c);
    if (tid == 0)
      for (int g = 0; g < 5; ++g) issue(g, c);
  }
  kbuf = 0;
  for (int it = 0; t < ntiles; t += gridDim.x, ++it) {
  const GrTile cur = gr_tile(a, t);
  const bool more = t + (int)gridDim.x < ntiles;
  const GrTile nxt = gr_tile(a, more ? t + (int)gridDim.x : t);
  const int dir = cur.dir;
  float* pq = a.pq + (size_t)dir * rows_bth * Dk;
  float* pk = a.pk + (size_t)dir * rows_bth * Dk;
  float* pab = a.pab + (size_t)dir * rows_bth * 2;
  float* dvb = a.dvb + (size_t)dir * rows_bth * Dv;

  // ---- this tile's gates and zeroed partial sums; every group landed
  if (tid < 64) {
    sm.row[tid] = gate_row;
    sm.g[tid] = gate_g;
    sm.beta[tid] = gate_b;
  }
  for (int e = tid; e < 3 * kGrWarps * 64; e += kGrThreads) part[e] = 0.f;
  __syncthreads();
  if (warp == 0) gate_prefix(sm);
  {
    bool ok = true;
    for (int g = 0; g < 5; ++g) ok = mbar_wait(&full[g], it & 1, a.limit) && ok;
    if (!__syncthreads_and(ok)) {
      if (tid == 0) atomicOr(a.err, kErrTimeout);
      for (int g = 0; g < 5; ++g) mbar_wait(&full[g], it & 1, kDrainPolls);  // nothing may land after exit
      return;
    }
  }
  bf16* const sKc = sK + kbuf * 64 * Dk;  // this tile's k^
  if (more && tid == 0) issue(4, nxt);  // the other k buffer was last read by the previous tile
  normalize_rows_core(a, sQ, sKc);  // per memory row: the order of the rows does not matter
  __syncthreads();
  const float gamC = sm.gam[63], eC = expf(gamC);
  const bool rev = dir != 0;  // the tiles' time rows run against the scan
  const BMat Q = core_mat(sQ, 64, rev), K = core_mat(sKc, 64, rev), O = core_mat(sO, 64, rev);
  const BMat Wm = core_mat(sW, 64, rev), Ut = core_mat(sUt, 64, rev), Um = core_mat(sU, 64, rev);
  const BMat S0 = core_mat(sS0, Dk, false), dSTm = core_mat(sdST, Dv, false);
  const BMat dUTm = core_mat(sdU, Dv, false), Pm = row_major(sP, kLdE), dWm = row_major(sdW, lbk);
  auto none = [](int, int, float) { return 0.f; };

  // ---- 1. P = M o (Q^ K^T);  E = e^{gam_p - gam_i} K^ K^T (i < p), A = diag(beta) E
  {  // block `warp` of P and of E, interleaved (16 blocks each, one a warp)
    const int mm[2] = {(warp >> 2) << 4, (warp >> 2) << 4}, nn[2] = {(warp & 3) << 4, (warp & 3) << 4};
    float dp[2][4], de[2][4];
    zero2(dp);
    zero2(de);
    blk16x2<false, true, false, true>(mm, nn, Q, K, Dk, K, K, Dk, dp, de);
#pragma unroll
    for (int hh = 0; hh < 2; ++hh)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int m = mm[0] + tile_row(e), n = nn[0] + 8 * hh + tile_col(e);
        const float decay = n <= m ? expf(sm.gam[m] - sm.gam[n]) : 0.f;
        sP[m * kLdE + n] = __float2bfloat16_rn(decay * dp[hh][e]);
        sE[m * kLdE + n] = __float2bfloat16_rn(n < m ? decay * de[hh][e] : 0.f);
      }
  }
  __syncthreads();  // P and E complete
  // ---- 3. dK~ = U dS_e^T: dk^ starts as e^{gam_C - gam} dK~; c_m = k^_m . dk^_m
  float dk[kMaxBlocks][2][4], dq[kMaxBlocks][2][4];
#pragma unroll
  for (int i = 0; i < kMaxBlocks; ++i) {
    zero2(dk[i]);
    zero2(dq[i]);
  }
  gemm_acc2<false, false>(Dk, Dv, Um, dSTm, dk, [&](int m) { return expf(gamC - sm.gam[m]); });
  acc_row_sums(Dk, wc, [&](int i, int hh, int e, int m, int n) { return bf(sKc[cidx(m, n, 64, rev)]) * dk[i][hh][e]; });
  // ---- 5. dP = dO U^T -> dQK = M o dP (in place of P); gam gets dP o P
  gemm2<false, true, false, true>(64, 64, O, Um, Dv, O, Um, 0,
      [&](int m, int n, float v) { return n <= m ? v * bf(sP[m * kLdE + n]) : 0.f; },
      [&](int m, int n, float v) {
        sP[m * kLdE + n] = __float2bfloat16_rn(n <= m ? expf(sm.gam[m] - sm.gam[n]) * v : 0.f);
      },
      wg, wg);
  // ---- 6. Z = diag(e^gam) dO S0^T -> dq^; gam_p gets q^_p . Z_p
  gemm_acc2<false, true>(Dk, Dv, O, S0, dq, [&](int m) { return sm.eg[m]; });
  acc_row_sums(Dk, wg, [&](int i, int hh, int e, int m, int n) { return bf(sQ[cidx(m, n, 64, rev)]) * dq[i][hh][e]; });
  __syncthreads();  // dQK complete; U and dO are read no more
  if (more && tid == 0) issue(0, nxt);
  // ---- 7. dq^ += dQK K^;  8. dk^ += dQK^T Q^
  gemm_acc2<false, false>(Dk, 64, Pm, K, dq, [](int) { return 1.f; });
  gemm_acc2<true, false>(Dk, 64, Pm, Q, dk, [](int) { return 1.f; });
  store_acc(Dk, dq, pq, Dk, sm.row);
  // ---- 9. dW = -dU S0^T
  gemm2<true, true, true, true>(64, Dk, dUTm, S0, Dv, dUTm, S0, 0, none,
      [&](int m, int n, float v) { sdW[m * lbk + n] = __float2bfloat16_rn(-v); }, nullptr, nullptr);
  __syncthreads();  // q^ is read no more
  if (more && tid == 0) issue(1, nxt);
  // ---- 10. [dX_w | dX_u] solves (I + A)^T X = [dW | dU]: X = T^T [dW | dU]
  //          with the forward's own T, into the tiles of q^ and dO (neither
  //          is read again)
  bf16* sXw = reinterpret_cast<bf16*>(bg_raw + L.xw);  // dS_e^T is read no more after step 3,
  bf16* sXu = reinterpret_cast<bf16*>(bg_raw + L.xu);  // S0 after step 9
  {
    const BMat Tt = core_mat(sT, 64, false);
    gemm2<true, false, true, false>(64, Dk, Tt, dWm, 64, Tt, Tt, 0, none,
        [&](int m, int n, float v) { sXw[cidx(m, n, 64, false)] = __float2bfloat16_rn(v); }, nullptr, nullptr);
    gemm2<true, true, true, true>(64, Dv, Tt, dUTm, 64, Tt, Tt, 0, none,
        [&](int m, int n, float v) { sXu[cidx(m, n, 64, false)] = __float2bfloat16_rn(v); }, nullptr, nullptr);
  }
  __syncthreads();  // T and dU^T are read no more
  if (more && tid == 0) issue(2, nxt);
  const BMat Xw = core_mat(sXw, 64, false), Xu = core_mat(sXu, 64, false);
  // ---- 11. dk^ += diag(beta e^gam) dX_w; beta and gam from the rows of
  //          X_w = diag(beta e^gam) K^ (s_p = k^_p . dX_w_p gives e^gam_p s_p
  //          to beta_p and beta_p e^gam_p s_p to gam_p); dX_u goes out as it
  //          is (the reduction forms dv = beta dX_u and beta's v . dX_u)
  {  // one pass over this thread's elements of the 64 x Dk register blocks
    const int tn = Dk >> 4, nt = 4 * tn;
#pragma unroll
    for (int i = 0; i < kMaxBlocks; ++i) {
      const int t = warp + kGrWarps * i;
      if (t < nt) {
        const int m0 = (t / tn) << 4, n0 = (t % tn) << 4;
        float r[2] = {0.f, 0.f};  // s of rows m0 + gq and m0 + gq + 8
#pragma unroll
        for (int hh = 0; hh < 2; ++hh)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int m = m0 + tile_row(e), n = n0 + 8 * hh + tile_col(e);
            const float xw = bf(sXw[cidx(m, n, 64, false)]);
            dk[i][hh][e] = fmaf(sm.beta[m] * sm.eg[m], xw, dk[i][hh][e]);
            r[e >> 1] = fmaf(bf(sKc[cidx(m, n, 64, rev)]), xw, r[e >> 1]);
          }
#pragma unroll
        for (int off = 1; off < 4; off <<= 1) {
          r[0] += __shfl_xor_sync(0xffffffffu, r[0], off);
          r[1] += __shfl_xor_sync(0xffffffffu, r[1], off);
        }
        if ((lane & 3) == 0) {  // this warp's partial rows: e^gam s to beta, beta e^gam s to gam
          const int ma = m0 + tile_row(0), mb = m0 + tile_row(2);
          wb[ma] += sm.eg[ma] * r[0];
          wg[ma] += sm.beta[ma] * sm.eg[ma] * r[0];
          wb[mb] += sm.eg[mb] * r[1];
          wg[mb] += sm.beta[mb] * sm.eg[mb] * r[1];
        }
      }
    }
  }
  {  // dX_u rows: warp w takes rows 8 (w % 8) .. + 7 and every other slab
     // from w / 8; lane l the word l % 4 of row l / 4 (128 contiguous bytes a slab)
    const int p = 8 * (warp & 7) + (lane >> 2), r = sm.row[p];
    const uint32_t* x2 = reinterpret_cast<const uint32_t*>(sXu);
    if (r >= 0)
      for (int sl = warp >> 3; sl < Dv / 8; sl += 2) {
        float f0, f1;
        unpack_bf16x2(x2[(sl * 64 + p) * 4 + (lane & 3)], f0, f1);
        *reinterpret_cast<float2*>(dvb + (size_t)r * Dv + 8 * sl + 2 * (lane & 3)) = make_float2(f0, f1);
      }
  }
  // ---- 12. dA = -(dX_w W^T + dX_u U~^T) on i < p (warp w: block w of the
  //          64 x 64, its two operand pairs as two chains), and from it in
  //          the same pass: gam's share from A (dA o A: + to row p, - to
  //          column i), beta_p += sum_i dA_pi E_pi, and dG = dA o (beta_p
  //          e^{gam_p - gam_i}) into P
  {
    const int mm[2] = {(warp >> 2) << 4, (warp >> 2) << 4}, nn[2] = {(warp & 3) << 4, (warp & 3) << 4};
    float d1[2][4], d2[2][4];
    zero2(d1);
    zero2(d2);
    blk16x2<false, true, false, true>(mm, nn, Xw, Wm, Dk, Xu, Ut, Dv, d1, d2);
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const int n0 = nn[0] + 8 * hh;
      float cg[4], cb[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int m = mm[0] + tile_row(e), n = n0 + tile_col(e);
        const float dA = n < m ? -(d1[hh][e] + d2[hh][e]) : 0.f;
        const float E = bf(sE[m * kLdE + n]);  // zero on and above the diagonal
        cg[e] = dA * sm.beta[m] * E;
        cb[e] = dA * E;
        sP[m * kLdE + n] = __float2bfloat16_rn(n < m ? dA * sm.beta[m] * expf(sm.gam[m] - sm.gam[n]) : 0.f);
      }
      float rg0 = cg[0] + cg[1], rg1 = cg[2] + cg[3], rb0 = cb[0] + cb[1], rb1 = cb[2] + cb[3];
#pragma unroll
      for (int off = 1; off < 4; off <<= 1) {
        rg0 += __shfl_xor_sync(0xffffffffu, rg0, off);
        rg1 += __shfl_xor_sync(0xffffffffu, rg1, off);
        rb0 += __shfl_xor_sync(0xffffffffu, rb0, off);
        rb1 += __shfl_xor_sync(0xffffffffu, rb1, off);
      }
      float c0 = cg[0] + cg[2], c1 = cg[1] + cg[3];
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) {
        c0 += __shfl_xor_sync(0xffffffffu, c0, off);
        c1 += __shfl_xor_sync(0xffffffffu, c1, off);
      }
      if ((lane & 3) == 0) {  // this warp's partial rows
        wg[mm[0] + tile_row(0)] += rg0;
        wg[mm[0] + tile_row(2)] += rg1;
        wb[mm[0] + tile_row(0)] += rb0;
        wb[mm[0] + tile_row(2)] += rb1;
      }
      if (lane < 4) {
        wg[n0 + tile_col(0)] -= c0;
        wg[n0 + tile_col(1)] -= c1;
      }
    }
  }
  __syncthreads();  // dG complete; dX_w, dX_u (in the dS_e^T and S0 tiles), W and U~ are read no more
  if (more && tid == 0) issue(3, nxt);
  // ---- 13. dk^ += (dG + dG^T) K^
  gemm_acc2<false, false>(Dk, 64, Pm, K, dk, [](int) { return 1.f; });
  gemm_acc2<true, false>(Dk, 64, Pm, K, dk, [](int) { return 1.f; });
  // ---- 14. outputs: dk^, dbeta, dg = suffix sum of dgam + dgam_C
  store_acc(Dk, dk, pk, Dk, sm.row);
  __syncthreads();  // every partial row sum is done
  if (more) load_gates(nxt);
  if (tid < 3 * 64) {  // the warps' partials: dgam, dbeta, c
    const float* src = part + (tid >> 6) * kGrWarps * 64 + (tid & 63);
    float acc = 0.f;
#pragma unroll
    for (int w = 0; w < kGrWarps; ++w) acc += src[w * 64];
    (tid < 64 ? sm.dgam : tid < 128 ? sm.dbeta : sm.cK)[tid & 63] = acc;
  }
  __syncthreads();
  if (warp == 0) {
    // K~ = diag(e^{gam_C - gam}) K^: row p's exponent gives -c_p to gam_p
    // and +c_p to gam_C
    float cs = sm.cK[2 * lane] + sm.cK[2 * lane + 1];
#pragma unroll
    for (int off = 16; off; off >>= 1) cs += __shfl_xor_sync(0xffffffffu, cs, off);
    const float dC = eC * __ldg(a.dot + cur.bi) + cs;  // e^{gam_C} <dS_e, S0> (the chain's sum)
    const float d0 = sm.dgam[2 * lane] - sm.cK[2 * lane];
    const float d1 = sm.dgam[2 * lane + 1] - sm.cK[2 * lane + 1];
    float incl = d0 + d1;  // suffix sums over scan positions 2 lane, 2 lane + 1 .. 63
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
  __syncthreads();  // the next tile rewrites sm
  kbuf ^= 1;
  }
}

}  // namespace

bool bwd_chunked_fits(int Dk, int Dv) {
  return Dk <= 112 && Dv <= 112 && GradLayout(Dk, Dv).total <= 227u * 1024u;
}

namespace {
struct BwdScratch {
  size_t fwd, tinv, xt, yt, dut, dset, dot, pq, pk, pab, dvb, total;
  BwdScratch(int B, int T, int H, int Dk, int Dv, bool bidir) {
    const size_t ndir = bidir ? 2 : 1, rows = (size_t)B * T * H, NBH = (size_t)B * H;
    const size_t blocks = ndir * NBH * ((T + 63) / 64);
    auto al = [](size_t n) { return (n + 255) & ~size_t(255); };
    size_t o = 0;
    fwd = o; o += al(chunk_tc_workspace_bytes(B, T, H, Dk, Dv, bidir));
    tinv = o; o += al(blocks * 64 * 64 * 2);
    xt = o;   o += al(blocks * 64 * Dv * 2);
    yt = o;   o += al(blocks * (size_t)Dk * Dv * 2);
    dut = o;  o += al(blocks * 64 * Dv * 2);
    dset = o; o += al(blocks * (size_t)Dk * Dv * 2);
    dot = o;  o += al(blocks * 4);
    pq = o;  o += al(ndir * rows * Dk * 4);
    pk = o;  o += al(ndir * rows * Dk * 4);
    pab = o; o += al(ndir * rows * 2 * 4);
    dvb = o; o += al(ndir * rows * Dv * 4);
    total = o;
  }
};
}  // namespace

size_t bwd_chunked_workspace_bytes(int B, int T, int H, int Dk, int Dv, bool bidir) {
  return BwdScratch(B, T, H, Dk, Dv, bidir).total;
}

cudaError_t launch_backward_chunked(const BwdCall& c, void* workspace, float** pq, float** pk,
                                    float** pab, float** dvb) {
  const int ndir = c.bidir ? 2 : 1;
  const size_t NBH = (size_t)c.B * c.H;
  const int nC = (c.T + 63) / 64;
  uint8_t* base = static_cast<uint8_t*>(workspace);
  const BwdScratch W(c.B, c.T, c.H, c.Dk, c.Dv, c.bidir);
  // the forward's stages A and B fill the workspace (W, K~, U~, U, S per chunk)
  ScanArgs f;
  f.q = c.q; f.k = c.k; f.v = c.v; f.g = c.g; f.beta = c.beta;
  f.state_in = c.state_in; f.state_out = nullptr; f.out = nullptr;
  f.B = c.B; f.T = c.T; f.H = c.H; f.Dk = c.Dk; f.Dv = c.Dv;
  f.dtype = GDN_BF16; f.chunk = 64; f.bidir = c.bidir; f.gate_logits = false;
  f.stream = c.stream; f.err = c.err; f.wait_limit = c.wait_limit; f.skip_output = true;
  f.t_out = base + W.tinv;
  cudaError_t e = launch_chunk_tc(f, base + W.fwd);
  if (e != cudaSuccess) return e;

  BcArgs a;
  a.q = static_cast<const __nv_bfloat16*>(c.q);
  a.k = static_cast<const __nv_bfloat16*>(c.k);
  a.v = static_cast<const __nv_bfloat16*>(c.v);
  a.dout = static_cast<const __nv_bfloat16*>(c.d_out);
  a.g = c.g; a.beta = c.beta;
  a.d_state_out = c.d_state_out; a.d_state_in = c.d_state_in;
  a.ws = base + W.fwd;
  a.wl = chunk_tc_ws_layout(c.Dk, c.Dv);
  a.tinv = reinterpret_cast<const __nv_bfloat16*>(base + W.tinv);
  a.XT = reinterpret_cast<__nv_bfloat16*>(base + W.xt);
  a.YT = reinterpret_cast<__nv_bfloat16*>(base + W.yt);
  a.dUT = reinterpret_cast<__nv_bfloat16*>(base + W.dut);
  a.dSeT = reinterpret_cast<__nv_bfloat16*>(base + W.dset);
  a.dot = reinterpret_cast<float*>(base + W.dot);
  a.err = c.err;
  a.limit = c.wait_limit;
  a.pq = reinterpret_cast<float*>(base + W.pq);
  a.pk = reinterpret_cast<float*>(base + W.pk);
  a.pab = reinterpret_cast<float*>(base + W.pab);
  a.dvb = reinterpret_cast<float*>(base + W.dvb);
  a.B = c.B; a.T = c.T; a.H = c.H; a.Dk = c.Dk; a.Dv = c.Dv;
  a.nC = nC;
  a.NBH = (int)NBH;
  *pq = a.pq; *pk = a.pk; *pab = a.pab; *dvb = a.dvb;
  const int smem_pre = (int)PreLayout(c.Dk, c.Dv).total;
  const int smem_chain = (int)ChainSmem(c.Dk).total;
  const ChainKernel chain = chain_kernel_for(c.Dk / 16);
  // the chain copies W, K~ and e^{gam_C} of a chunk as one span
  if (a.wl.off_kt != a.wl.off_w + 128u * c.Dk || a.wl.off_decay != a.wl.off_kt + 128u * c.Dk ||
      a.wl.off_w % 16 != 0)
    return cudaErrorInvalidValue;
  const int smem_grad = (int)GradLayout(c.Dk, c.Dv).total;
  // the gradient pass copies U~, U and S0 of a chunk as one span
  if (a.wl.off_u != a.wl.off_ut + 128u * c.Dv || a.wl.off_s != a.wl.off_u + 128u * c.Dv)
    return cudaErrorInvalidValue;
  CUtensorMap tq, tk, to;
  if (!make_tile_map(&tq, c.q, c.B, c.T, c.H, c.Dk, 64) || !make_tile_map(&tk, c.k, c.B, c.T, c.H, c.Dk, 64) ||
      !make_tile_map(&to, c.d_out, c.B, c.T, c.H, c.Dv, 64))
    return cudaErrorInvalidValue;
  if ((e = cudaFuncSetAttribute(gdn_bwd_pre_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                smem_pre)) != cudaSuccess ||
      (e = cudaFuncSetAttribute(chain, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                smem_chain)) != cudaSuccess ||
      (e = cudaFuncSetAttribute(gdn_bwd_grad_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                smem_grad)) != cudaSuccess)
    return e;
  const dim3 per_chunk((unsigned)nC, (unsigned)NBH, ndir);
  {
    ProfileScope ps(c.stream, kKernBwdChunk);
    gdn_bwd_pre_kernel<<<per_chunk, kBcThreads, smem_pre, c.stream>>>(tq, tk, to, a);
  }
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  {
    ProfileScope ps(c.stream, kKernBwdChain);
    const unsigned groups = (unsigned)((c.Dv / 16 + kChSlices - 1) / kChSlices);
    chain<<<dim3(groups, (unsigned)NBH, ndir), kChThreads, smem_chain, c.stream>>>(a);
  }
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  {
    ProfileScope ps(c.stream, kKernBwdGrad);
    const int ntiles = nC * (int)NBH * ndir;
    gdn_bwd_grad_kernel<<<std::min(ntiles, num_sms()), kGrThreads, smem_grad, c.stream>>>(tq, tk, to, a,
                                                                                       ntiles);
  }
  e = cudaGetLastError();
  if (e == cudaSuccess) count_launches(3);
  return e;
}

}  // namespace gdn
