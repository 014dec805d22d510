// chunk_tc.cu -- the chunked GDN scan on sm_100a tensor cores (bf16 I/O).
//
// The pages' fused kernel runs a three-stage chunked pipeline: stage A forms
// per-chunk summaries, stage B runs the recurrent scan over chunks, stage C
// applies the state ("SANA-Streaming：基于混合扩散Transformer的实时流式视频编辑
// 系统", 方法步骤详情, fourth step).  Here the three stages are three kernels:
//
//   stage A  gdn_prep_kernel    one CTA per (chunk, b*h, direction), parallel
//   stage B  gdn_recur_kernel   one CTA per (1-4 slices of 16 state columns,
//                               b*h, direction), a dependent walk over the
//                               chunks, one warp per slice
//   stage C  gdn_output_kernel  persistent, one CTA per SM over the (chunk,
//                               b*h) tiles, both directions per tile
// launched back to back with programmatic dependent launch.
//
// Algebra (per head; a chunk holds C = 64 tokens in scan order, entered with
// state S0; gamma_r = sum of g over the chunk's tokens up to r in scan order,
// gamma_C its last value; k^ = k / |k|):
//   A_ri  = beta_r e^{gamma_r - gamma_i} k^_r . k^_i  for i before r, else 0
//   Tm    = (I + A)^-1                    (UT transform of the delta rule)
//   W     = Tm diag(beta e^gamma) K^,     U~ = Tm diag(beta) V
//   U     = U~ - W S0                     (per-token corrected values)
//   S_out = e^{gamma_C} S0 + K~^T U,      K~ = diag(e^{gamma_C - gamma}) K^
//   O     = diag(e^gamma) Q^ S0 + (Mask o Q^ K^^T) U,
//           Mask_ri = e^{gamma_r - gamma_i} for i at or before r, else 0.
// Stage A computes Tm, W, U~ and K~ (everything that does not depend on the
// state); stage B walks the chunks with the state, forming U and the next
// state (two products per chunk, d x 64 x 16 and 16 x 64 x d per slice) and
// publishing U and the chunk-start state; stage C computes O.
//
// The reverse (within-chunk backward) scan of the bidirectional mode uses the
// same memory tiles visited in the opposite order, with gamma the suffix sums
// and "before" meaning "later in memory"; both directions' outputs are summed
// in one fp32 TMEM accumulator before the single bf16 store.
//
// The contractions of stages A and C are tcgen05.mma (bf16 x bf16 -> fp32 in
// TMEM) issued by one thread from SWIZZLE_NONE core-matrix shared-memory
// layouts; q/k/v tiles arrive by TMA tensor loads, workspace tiles by bulk
// copies.  The 64 x 64 triangular inverse is a blocked solve: 16 x 16
// diagonal blocks by fp32 forward substitution, merges on tf32 mma.sync.
// Stage B's latency-bound chain uses warp-level mma.sync (bf16, fp32
// accumulate), its state in registers.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <mutex>
#include <utility>

#include "gates.cuh"
#include "gdn_internal.h"
#include "sm100.cuh"

namespace gdn {
namespace {

using namespace sm100;

constexpr int kC = 64;            // tokens per chunk
constexpr int kWideThreads = 256; // stage A: two warps per TMEM lane quadrant
constexpr int kOutThreads = 512;  // stage C: four warps per TMEM lane quadrant
constexpr int kSlab64 = kC * 16;  // bytes of one 8-column slab of a 64-row tile
constexpr long long kDrainPolls = 1LL << 40;  // drains are bounded by the 2 s timer

// ----------------------------------------------------------------- workspace
// One contiguous block per (direction, b*h, chunk), in the order the stages
// read them so that each read is a single bulk copy:
//   W     [Dk/8][64][8]   bf16                        (A writes, B reads)
//   Kt    [Dk/8][64][8]   bf16  K~                    (A writes, B reads)
//   decay {e^{gamma_C}, 0, 0, 0} fp32                 (A writes, B reads)
//   g     [64]            fp32  the tile's gates      (A writes, C reads)
//   Ut    [Dv/8][64][8]   bf16  U~                    (A writes, B reads)
//   U     [Dv/8][64][8]   bf16  U = U~ - W S0         (B writes, C reads)
//   S     [Dv/8][Dk][8]   bf16  state at chunk start  (B writes, C reads)
struct Workspace {
  uint8_t* base;
  uint8_t* tinv = nullptr;  // optional: each tile's (I + A)^-1, bf16 [8][64][8] in scan order
  size_t block_bytes;
  uint32_t off_w, off_kt, off_decay, off_g, off_ut, off_u, off_s;
  int NBH, nC, Dk, Dv;

  __host__ __device__ void layout(int dk, int dv) {
    Dk = dk;
    Dv = dv;
    off_w = 0;
    off_kt = off_w + 64u * Dk * 2;
    off_decay = off_kt + 64u * Dk * 2;
    off_g = off_decay + 16;
    off_ut = off_g + 64u * 4;
    off_u = off_ut + 64u * Dv * 2;
    off_s = off_u + 64u * Dv * 2;
    block_bytes = ((size_t)off_s + (size_t)Dk * Dv * 2 + 255) & ~size_t(255);
  }
  __device__ size_t tile(int dir, int bh, int j) const {
    return ((size_t)dir * NBH + bh) * nC + j;
  }
  __device__ uint8_t* blk(size_t tile_index) const { return base + tile_index * block_bytes; }
};

// Block-wide bounded wait: every thread polls, then all agree.  On failure
// the error word is set and the awaited operation is drained (so nothing is
// still writing shared memory when the CTA leaves).
__device__ bool block_wait(uint64_t* bar, uint32_t parity, long long limit, unsigned* err) {
  bool ok = mbar_wait(bar, parity, limit);
  ok = __syncthreads_and(ok);
  if (!ok) {
    if (threadIdx.x == 0) atomicOr(err, kErrTimeout);
    mbar_wait(bar, parity, kDrainPolls);
    __syncthreads();
  }
  return ok;
}

__device__ __forceinline__ void block_sync_async() {
  fence_proxy_async_smem();
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
}

// gamma for the 64 rows of a tile: inclusive prefix sums in memory order
// (forward) or suffix sums (reverse).  Warp 0 only.
__device__ void warp_gamma(const float* g, float* gam, int reverse) {
  const int lane = threadIdx.x & 31;
  const int r0 = reverse ? 63 - 2 * lane : 2 * lane;
  const int r1 = reverse ? 62 - 2 * lane : 2 * lane + 1;
  const float a0 = g[r0], a1 = g[r1];
  const float pair = a0 + a1;
  float incl = pair;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const float y = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += y;
  }
  const float excl = incl - pair;
  gam[r0] = excl + a0;
  gam[r1] = incl;
}

// 1 / max(|row r|, 1e-6) for a 64-row bf16 tile in [slab][64][8] layout,
// by four consecutive lanes (part = lane & 3 takes slabs part, part + 4, ...);
// every lane of the four gets the result.
__device__ float row_rnorm4(const uint8_t* tile, int r, int part, int D) {
  float ss = 0.f;
  for (int sl = part; sl < D / 8; sl += 4) {
    float x[8];
    unpack8_bf16(reinterpret_cast<const uint4*>(tile + sl * kSlab64)[r], x);
#pragma unroll
    for (int i = 0; i < 8; ++i) ss = fmaf(x[i], x[i], ss);
  }
  ss += __shfl_xor_sync(0xffffffffu, ss, 1);
  ss += __shfl_xor_sync(0xffffffffu, ss, 2);
  return 1.0f / sqrtf(fmaxf(ss, 1e-12f));
}

// ============================================================ stage A: prep
// Shared memory: K and V tiles stay for the whole tile; the solve's fp32
// scratch and the bf16 A operands TW/TU live until W and U~ are in TMEM.
// ~102 KB: two CTAs/SM.
constexpr int kLd = 68;  // fp32 row stride of the 64 x 64 scratch (16 B aligned rows)
struct PrepSmem {
  alignas(128) uint8_t K[16 * kSlab64];   // [Dk/8 slabs][64][8]
  alignas(128) uint8_t V[16 * kSlab64];
  struct alignas(128) U {
    uint8_t TW[8 * kSlab64];             // Tm diag(beta e^g / |k|), K-major A
    uint8_t TU[8 * kSlab64];             // Tm diag(beta), K-major A
    float A[64][kLd];                    // strictly lower A in scan order
    float T[64][kLd];                    // (I + A)^-1 in scan order
    float Y[64][kLd];                    // product scratch
  } u;
  float g[64], beta[64], gam[64], rn[64], csW[64], csU[64];
  float arow[64];      // beta_r |k_r|^-1 e^{gam_r - m_b(r)}       (scan order)
  float bcol[8][64];   // |k_q|^-1 e^{m_b - gam_q}, b = 8-row block (scan order)
  float dg[64][8];     // A's factor inside p's own 8-row block       (scan order)
  uint64_t tma_bar, v_bar, mma_bar;  // K tile, V tile, MMA completion
  uint32_t tmem;
};

constexpr float kLog2e = 1.4426950408889634f;

// tf32 tensor-core product on fp32 shared-memory tiles (row stride kLd):
// D(16 x 8) = sum_k A[ar + i][ac + k] * B[br + k][bc + j], k < 8 * ksteps,
// one warp, mma.sync.m16n8k8 (tf32 inputs rounded to nearest, fp32 accumulate).
__device__ __forceinline__ uint32_t to_tf32(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return r;
}
__device__ __forceinline__ void warp_mma_tf32(const float (*A)[kLd], int ar, int ac,
                                              const float (*B)[kLd], int br, int bc, int ksteps,
                                              float (&d)[4]) {
  const int lane = threadIdx.x & 31, gq = lane >> 2, tq = lane & 3;
  d[0] = d[1] = d[2] = d[3] = 0.f;
  for (int ks = 0; ks < ksteps; ++ks) {
    const int k0 = 8 * ks;
    const uint32_t a0 = to_tf32(A[ar + gq][ac + k0 + tq]);
    const uint32_t a1 = to_tf32(A[ar + gq + 8][ac + k0 + tq]);
    const uint32_t a2 = to_tf32(A[ar + gq][ac + k0 + tq + 4]);
    const uint32_t a3 = to_tf32(A[ar + gq + 8][ac + k0 + tq + 4]);
    const uint32_t b0 = to_tf32(B[br + k0 + tq][bc + gq]);
    const uint32_t b1 = to_tf32(B[br + k0 + tq + 4][bc + gq]);
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
  }
}
// Store a 16 x 8 accumulator tile (times `sign`) at C[cr .. cr+15][cc .. cc+7].
__device__ __forceinline__ void warp_store_tile(float (*C)[kLd], int cr, int cc, const float (&d)[4],
                                                float sign) {
  const int lane = threadIdx.x & 31, gq = lane >> 2, tq = lane & 3;
  *reinterpret_cast<float2*>(&C[cr + gq][cc + 2 * tq]) = make_float2(sign * d[0], sign * d[1]);
  *reinterpret_cast<float2*>(&C[cr + gq + 8][cc + 2 * tq]) = make_float2(sign * d[2], sign * d[3]);
}

// In-place blocked inverse of the unit lower-triangular 64 x 64 matrix
// I + A (A strictly lower, scan order) into T:
//   16 x 16 diagonal blocks by right-looking forward substitution in fp32
//   (one lane per column: the dependent chain is one FMA per row);
//   16 -> 32:  T_hl = -T_hh (A_hl T_ll) for the two 32 x 32 diagonal halves;
//   32 -> 64:  T_HL = -T_HH (A_HL T_LL) for the lower-left 32 x 32 block;
// the block products on tf32 tensor cores (T is rounded to bf16 right after).
__device__ void unit_lower_inverse(PrepSmem::U& u) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  float (*A)[kLd] = u.A;
  float (*T)[kLd] = u.T;
  float (*Y)[kLd] = u.Y;
  for (int i = tid; i < 64 * 16; i += kWideThreads)
    reinterpret_cast<float4*>(T[i >> 4])[i & 15] = make_float4(0.f, 0.f, 0.f, 0.f);
  __syncthreads();
  if (warp < 4 && lane < 16) {
    const int b0 = 16 * warp, j = lane;
    float acc[16];
#pragma unroll
    for (int t = 0; t < 16; ++t) acc[t] = (t == j) ? 1.f : 0.f;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const float x = acc[i];
#pragma unroll
      for (int t = i + 1; t < 16; ++t) acc[t] = fmaf(-A[b0 + t][b0 + i], x, acc[t]);
    }
#pragma unroll
    for (int t = 0; t < 16; ++t) T[b0 + t][b0 + j] = acc[t];
  }
  __syncthreads();
  // 16 -> 32: pair p = warp >> 1 (blocks (32p+16, 32p)), n-tile = warp & 1
  if (warp < 4) {
    const int pr = warp >> 1, nt = warp & 1;
    const int hb = 32 * pr + 16, lb = 32 * pr;
    float d[4];
    warp_mma_tf32(A, hb, lb, T, lb, lb + 8 * nt, 2, d);
    warp_store_tile(Y, hb, lb + 8 * nt, d, 1.f);
  }
  __syncthreads();
  if (warp < 4) {
    const int pr = warp >> 1, nt = warp & 1;
    const int hb = 32 * pr + 16, lb = 32 * pr;
    float d[4];
    warp_mma_tf32(T, hb, hb, Y, hb, lb + 8 * nt, 2, d);
    warp_store_tile(T, hb, lb + 8 * nt, d, -1.f);
  }
  __syncthreads();
  // 32 -> 64: the 32 x 32 block as 2 x 4 tiles of 16 x 8, one per warp
  {
    const int mt = warp >> 2, nt = warp & 3;
    float d[4];
    warp_mma_tf32(A, 32 + 16 * mt, 0, T, 0, 8 * nt, 4, d);
    warp_store_tile(Y, 32 + 16 * mt, 8 * nt, d, 1.f);
    __syncthreads();
    warp_mma_tf32(T, 32 + 16 * mt, 32, Y, 32, 8 * nt, 4, d);
    warp_store_tile(T, 32 + 16 * mt, 8 * nt, d, -1.f);
  }
  __syncthreads();
}

// Scan position of memory row r within a tile.
template <int REV>
__device__ __forceinline__ int scan_pos(int r) { return REV ? 63 - r : r; }

template <int REV>
__device__ bool prep_body(PrepSmem& s, const CUtensorMap* tm_k, const CUtensorMap* tm_v,
                          const void* __restrict__ g, const void* __restrict__ beta, int logits,
                          const Workspace& ws, int T, int H, long long limit, unsigned* err) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int j = blockIdx.x, bh = blockIdx.y, dir = REV;
  const int b = bh / H, h = bh - b * H;
  const int Dk = ws.Dk, Dv = ws.Dv;
  const int t0 = j * kC;
  const int nvalid = min(kC, T - t0);
  const uint32_t tm = s.tmem;

  if (tid == 0) {
    mbar_arrive_expect_tx(&s.tma_bar, (Dk / 8) * kSlab64);
    mbar_arrive_expect_tx(&s.v_bar, (Dv / 8) * kSlab64);
    tma_load_tile(s.K, tm_k, &s.tma_bar, t0, h, b);
    tma_load_tile(s.V, tm_v, &s.v_bar, t0, h, b);
  }
  if (tid < kC) {
    float gv = 0.f, bv = 0.f;  // padding rows: a = 1, beta = 0 (no effect)
    if (tid < nvalid) {
      const size_t row = ((size_t)b * T + t0 + tid) * H + h;
      if (logits) {  // the fused prologue: the gate layer's bf16 logits
        gv = gate_g_from_logit(__bfloat162float(static_cast<const __nv_bfloat16*>(g)[row]));
        bv = gate_beta_from_logit(__bfloat162float(static_cast<const __nv_bfloat16*>(beta)[row]));
      } else {
        gv = __ldg(static_cast<const float*>(g) + row);
        bv = __ldg(static_cast<const float*>(beta) + row);
      }
    }
    s.g[tid] = gv;
    s.beta[tid] = bv;
    // stage C takes the tile's gates from here, in both modes
    if (dir == 0) reinterpret_cast<float*>(ws.blk(ws.tile(0, bh, j)) + ws.off_g)[tid] = gv;
  }
  __syncthreads();
  if (warp == 0) warp_gamma(s.g, s.gam, REV);
  // V is awaited only before W / U~; a failure before that drains it too
  auto drain_v = [&]() { mbar_wait(&s.v_bar, 0, kDrainPolls); };
  if (!block_wait(&s.tma_bar, 0, limit, err)) {
    drain_v();
    return false;
  }

  // G = K K^T  (M = 64 tokens, N = 64 tokens, K = Dk), raw (unnormalised)
  // keys; the row norms below overlap it
  if (tid == 0) {
    tc_fence_after_sync();
    const uint32_t id = idesc_bf16(64, 64, 0, 0);
    for (int ks = 0; ks < Dk / 16; ++ks) {
      const uint64_t a = sdesc(smem_u32(s.K) + ks * 2 * kSlab64, kSlab64, 128);
      mma_bf16(tm, a, a, id, ks > 0);
    }
    mma_commit(&s.mma_bar);
  }
  {
    const float rn = row_rnorm4(s.K, tid >> 2, tid & 3, Dk);
    if ((tid & 3) == 0) s.rn[tid >> 2] = rn;
  }
  __syncthreads();
  const float gamC = REV ? s.gam[0] : s.gam[63];
  if (tid < kC) {
    s.csW[tid] = s.beta[tid] * expf(s.gam[tid]) * s.rn[tid];
    s.csU[tid] = s.beta[tid];
  }
  if (!block_wait(&s.mma_bar, 0, limit, err)) {
    drain_v();
    return false;
  }
  tc_fence_after_sync();

  // A[p][q] = beta_r e^{gam_r - gam_i} G_ri / (|k_r| |k_i|) for scan positions
  // q < p.  For q in an earlier 8-row block than p's block b the gate factor
  // is split at m_b = gam at b's first scan position, A = arow[p] G bcol[b][q]:
  // both exponents are <= 0, so the factors are exact (one underflows only
  // when the product does).  Inside the diagonal block the whole factor
  // beta_r e^{gam_r - gam_i} / (|k_r| |k_i|) <= 1 comes from dg[p] (the split
  // would put e^{m_b - gam_i}, up to e^{7 |g|}, in one factor).
  {
    for (int e = tid; e < 8 * 64; e += kWideThreads) {
      const int blk = e >> 6, q = e & 63;
      const int i = REV ? 63 - q : q;
      const float mb = s.gam[REV ? 63 - 8 * blk : 8 * blk];
      s.bcol[blk][q] = q < 8 * blk ? s.rn[i] * exp2f((mb - s.gam[i]) * kLog2e) : 0.f;
      const int p = e >> 3, qd = (p & ~7) + (e & 7);  // row p, column qd of its block
      const int r = REV ? 63 - p : p, id = REV ? 63 - qd : qd;
      s.dg[p][e & 7] = qd < p ? s.beta[r] * s.rn[r] * s.rn[id] * exp2f((s.gam[r] - s.gam[id]) * kLog2e)
                              : 0.f;
    }
    if (tid < 64) {
      const int p = tid, r = REV ? 63 - p : p;
      const float mb = s.gam[REV ? 63 - 8 * (p >> 3) : 8 * (p >> 3)];
      s.arow[p] = s.beta[r] * s.rn[r] * exp2f((s.gam[r] - mb) * kLog2e);
    }
    __syncthreads();
    const int quad = warp & 3, half = warp >> 2;
    const int r = 16 * quad + (lane & 15);
    const int p = scan_pos<REV>(r);
    const uint32_t lane_base = static_cast<uint32_t>(32 * quad) << 16;
    // this warp half covers scan columns q in [32 half, 32 half + 32); the
    // matching memory columns i = pos(q) form one contiguous 32-column range
    const int i0 = REV ? 32 - 32 * half : 32 * half;
    float v[32];
    tmem_ld16(tm + lane_base + i0, *reinterpret_cast<float(*)[16]>(v));
    tmem_ld16(tm + lane_base + i0 + 16, *reinterpret_cast<float(*)[16]>(v + 16));
    tmem_wait_ld();
    if (lane < 16) {
      const float* bc = s.bcol[p >> 3];
      const int pb = p & ~7;  // first column of p's own block
      float* Arow = s.u.A[p];
#pragma unroll
      for (int q4 = 0; q4 < 8; ++q4) {
        const int qb = 32 * half + 4 * q4;
        // earlier blocks: arow[p] bcol[b][q]; own block: dg[p][q - pb]; later: 0
        const bool own = (qb & ~7) == pb;
        const float sc = own ? 1.f : s.arow[p];
        const float4 b4 = *reinterpret_cast<const float4*>(own ? &s.dg[p][qb - pb] : bc + qb);
        const float bb[4] = {b4.x, b4.y, b4.z, b4.w};
        float o[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int iv = REV ? 31 - (4 * q4 + e) : 4 * q4 + e;  // index into v
          o[e] = sc * v[iv] * bb[e];
        }
        *reinterpret_cast<float4*>(Arow + qb) = make_float4(o[0], o[1], o[2], o[3]);
      }
    }
  }
  __syncthreads();
  unit_lower_inverse(s.u);
  if (ws.tinv) {  // a bf16 copy of T for the backward pass: scan order, [8][64][8] core matrices
    uint4* dst = reinterpret_cast<uint4*>(ws.tinv + ws.tile(dir, bh, j) * (64 * 64 * 2));
    for (int idx = tid; idx < 64 * 8; idx += kWideThreads) {
      const int r = idx & 63, ks = idx >> 6;
      dst[idx] = pack8_bf16(&s.u.T[r][8 * ks]);
    }
  }

  // TW[r][i] = T[pos r][pos i] beta_i e^{gam_i} / |k_i|, TU[r][i] = T[..] beta_i,
  // as bf16 K-major A operands in memory order
  for (int idx = tid; idx < 64 * 8; idx += kWideThreads) {
    const int r = idx & 63, ks = idx >> 6;
    const float* Trow = s.u.T[scan_pos<REV>(r)];
    float w[8], uu[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int i = 8 * ks + e;
      const float t = Trow[scan_pos<REV>(i)];
      w[e] = t * s.csW[i];
      uu[e] = t * s.csU[i];
    }
    reinterpret_cast<uint4*>(s.u.TW + ks * kSlab64)[r] = pack8_bf16(w);
    reinterpret_cast<uint4*>(s.u.TU + ks * kSlab64)[r] = pack8_bf16(uu);
  }
  block_sync_async();
  if (!block_wait(&s.v_bar, 0, limit, err)) return false;
  // W = TW K (N = Dk), U~ = TU V (N = Dv); K and V read MN-major (N = feature)
  if (tid == 0) {
    const uint32_t idW = idesc_bf16(64, Dk, 0, 1), idU = idesc_bf16(64, Dv, 0, 1);
    for (int ks = 0; ks < kC / 16; ++ks) {
      const uint64_t aw = sdesc(smem_u32(s.u.TW) + ks * 2 * kSlab64, kSlab64, 128);
      const uint64_t au = sdesc(smem_u32(s.u.TU) + ks * 2 * kSlab64, kSlab64, 128);
      const uint64_t bk = sdesc(smem_u32(s.K) + ks * 256, 128, kSlab64);
      const uint64_t bv = sdesc(smem_u32(s.V) + ks * 256, 128, kSlab64);
      mma_bf16(tm, aw, bk, idW, ks > 0);
      mma_bf16(tm + 128, au, bv, idU, ks > 0);
    }
    mma_commit(&s.mma_bar);
  }
  // While W and U~ compute: K~ = diag(e^{gamC - gam} / |k|) K -> workspace,
  // in the tile's own [slab][64][8] layout, and the chunk decay e^{gamC}
  const size_t tile = ws.tile(dir, bh, j);
  uint8_t* blk = ws.blk(tile);
  for (int idx = tid; idx < (Dk / 8) * kC; idx += kWideThreads) {
    const int r = idx & 63, sl = idx >> 6;
    const float sc = expf(gamC - s.gam[r]) * s.rn[r];
    float x[8];
    unpack8_bf16(reinterpret_cast<const uint4*>(s.K + sl * kSlab64)[r], x);
#pragma unroll
    for (int e = 0; e < 8; ++e) x[e] *= sc;
    reinterpret_cast<uint4*>(blk + ws.off_kt + sl * kSlab64)[r] = pack8_bf16(x);
  }
  if (tid == 0)
    *reinterpret_cast<float4*>(blk + ws.off_decay) = make_float4(expf(gamC), 0.f, 0.f, 0.f);
  if (!block_wait(&s.mma_bar, 1, limit, err)) return false;
  tc_fence_after_sync();

  // W, U~ -> workspace (bf16 [slab][64][8]).  Warps w and w + 4 share a TMEM
  // lane quadrant and split the column blocks.
  {
    const int quad = warp & 3, half = warp >> 2;
    const int r = 16 * quad + (lane & 15);
    const uint32_t lane_base = static_cast<uint32_t>(32 * quad) << 16;
    // column block cb: W's blocks [0, Dk/16) at TMEM column 16 cb, then
    // U~'s at 128 + 16 (cb - Dk/16); two TMEM loads in flight per wait
    const int nkb = Dk / 16, nb = nkb + Dv / 16;
    auto col = [&](int cb) { return cb < nkb ? 16u * cb : 128u + 16u * (cb - nkb); };
    auto put = [&](int cb, const float* v) {
      const bool isw = cb < nkb;
      const int c = isw ? cb : cb - nkb;
      uint4* G = reinterpret_cast<uint4*>(blk + (isw ? ws.off_w : ws.off_ut));
      G[(2 * c) * kC + r] = pack8_bf16(v);
      G[(2 * c + 1) * kC + r] = pack8_bf16(v + 8);
    };
    for (int cb = half; cb < nb; cb += 4) {
      float v0[16], v1[16];
      const bool two = cb + 2 < nb;
      tmem_ld16(tm + lane_base + col(cb), v0);
      if (two) tmem_ld16(tm + lane_base + col(cb + 2), v1);
      tmem_wait_ld();
      if (lane < 16) {
        put(cb, v0);
        if (two) put(cb + 2, v1);
      }
    }
  }
  return true;
}

__global__ void __launch_bounds__(kWideThreads, 2)
gdn_prep_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                const void* __restrict__ g, const void* __restrict__ beta, int logits, Workspace ws,
                int T, int H, long long limit, unsigned* err) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  PrepSmem& s = *reinterpret_cast<PrepSmem*>(smem_raw);
  const int tid = threadIdx.x;
  if (tid == 0) {
    mbar_init(&s.tma_bar, 1);
    mbar_init(&s.v_bar, 1);
    mbar_init(&s.mma_bar, 1);
    fence_mbar_init();
  }
  if ((tid >> 5) == 0) {
    tmem_alloc(&s.tmem, 256);
    tmem_relinquish();
  }
  block_sync_async();
  // Programmatic dependent launch: everything above overlaps the previous
  // kernel in the stream; nothing in global memory is touched before this.
  pdl_wait();
  pdl_trigger();
  if (blockIdx.z == 0)
    prep_body<0>(s, &tm_k, &tm_v, g, beta, logits, ws, T, H, limit, err);
  else
    prep_body<1>(s, &tm_k, &tm_v, g, beta, logits, ws, T, H, limit, err);
  tc_fence_before_sync();
  __syncthreads();
  if ((tid >> 5) == 0) tmem_dealloc(s.tmem, 256);
}

// ======================================================= stage B: recurrence
// One CTA per (one or two slices of 16 state columns, b*h, direction).  Each
// slice is walked by a group of P = min(4, Dk/16) warps (one per SM
// sub-partition); one more warp per CTA, the producer, streams each chunk's
// [W | K~ | decay] and the CTA's U~ slabs through an nst-stage ring of bulk
// copies (full / empty mbarriers) and issues the bulk stores that publish the
// groups' results.  Per chunk, transposed so that the slice's 16 state
// columns are the M = 16 rows of mma.sync.m16n8k16:
//   U^T  = U~^T - S^T W^T              (16 x 64 tokens, K = Dk)
//          warp q of the group takes 64/P of the tokens
//   S^T <- e^{gamma_C} S^T + U^T K~     (16 x Dk, K = 64 tokens)
//          warp q takes its share of the Dk state rows and keeps that part
//          of the fp32 state in its accumulator registers
// An accumulator tile pair is exactly an A-operand fragment, so between the
// two products the warps of a group only exchange bf16 fragments through a
// small shared buffer and a named barrier (U^T after the first product, S^T
// after the second).  Per-warp mma.sync issue is what bounds this stage, and
// the split gives every warp about 1/P of each product.  The chunk-start
// state S and U go to stage C through a triple-buffered staging area
// (stmatrix.trans): once a chunk's staging is complete the group tells the
// producer (mbarrier `staged`), which stores it with bulk copies and frees the
// buffer (mbarrier `freed`) when they have read it, off the chain's path.
constexpr int kChainMaxGroups = 2;
constexpr int kChainMaxStages = 6;
constexpr int kChainHeadBytes = 256;  // mbarriers and the groups' failure flags
constexpr int kChainBufs = 3;         // staging buffers per group

__host__ __device__ constexpr int chain_group_warps(int nkb) { return nkb >= 4 ? 4 : nkb >= 2 ? 2 : 1; }

struct ChainLayout {
  uint32_t wk_bytes;  // W | K~ | decay of one chunk (one bulk copy)
  uint32_t stage;     // stage stride: W | K~ | decay | the CTA's U~ slabs
  uint32_t stg_s;     // staging of S [2][Dk][8] bf16; U [2][64][8] follows
  uint32_t stg;       // one staging buffer
  uint32_t xs;        // exchange: S^T A fragments [Dk/16][32 lanes][16 B]
  uint32_t group;     // per group: staging buffers | S^T exchange | U^T exchange
  uint32_t groups;    // offset of group 0
  uint32_t total;
  __host__ __device__ ChainLayout(int Dk, int ns, int nst) {
    wk_bytes = 2u * 64 * Dk * 2 + 16;
    stage = (wk_bytes + (uint32_t)ns * 2 * kSlab64 + 127) & ~127u;
    stg_s = 2u * Dk * 16;
    stg = stg_s + 2u * kSlab64;
    xs = (uint32_t)(Dk / 16) * 512;
    group = kChainBufs * stg + xs + 4 * 512;
    groups = kChainHeadBytes + nst * stage;
    total = groups + ns * group;
  }
};

struct ChainBars {
  uint64_t full[kChainMaxStages], empty[kChainMaxStages];
  uint64_t staged[kChainBufs], freed[kChainBufs];  // per staging buffer
  int fail[kChainMaxGroups];                       // a bounded wait of the group expired
};


// What one launch of the chain kernel does (one pass of stage B):
//  * publish pass: walk each time segment of the chunk sequence from its
//    start state and publish every chunk's start state and U for stage C
//    (unsegmented: one segment, started from state_in or zero);
//  * summary pass (time-segmented scan only): walk each segment from zero
//    and, beside the Dv/16 state slices, p_slices = Dk/16 more slices that
//    start from the identity with U~ = 0: their final columns are the
//    segment's transition P (S_out = P S_in + R), the others its offset R.
struct ChainArgs {
  const float* init;   // start states [dir][seg][b*h][Dk][Dv] (dir 0 only if
                       // init_dir_stride == 0), or nullptr for zero
  size_t init_seg_stride, init_dir_stride;  // floats between segments / directions
  float* fin;          // final states, rows of fin_ld floats, or nullptr
  size_t fin_seg_stride, fin_dir_stride;
  int fin_ld;
  int fin_last_seg_only;  // publish pass: only the last segment ends the scan
  int nseg, seg_len;   // segments of seg_len chunks (the last may be shorter)
  int publish;         // 1: publish pass, 0: summary pass
  int p_slices;        // summary pass: slices past Dv/16 carry P's columns
};

// Warp q of the group walking slice s (16 state columns); gw = group index in
// the CTA.  NKB = Dk / 16.  Returns false if a bounded wait expired.
template <int NKB, bool SUMMARY>
__device__ bool chain_warp(uint8_t* smem, const ChainLayout& L, int nst, int gw, int q, int s,
                           const ChainArgs& A, const Workspace& ws, long long limit,
                           unsigned* err) {
  constexpr int P = chain_group_warps(NKB);
  constexpr int KPW = (NKB + P - 1) / P;  // most state-row k-blocks of one warp
  constexpr int TPW = 4 / P;              // 16-token blocks of one warp
  ChainBars& bars = *reinterpret_cast<ChainBars*>(smem);
  const int lane = threadIdx.x & 31, g = lane >> 2, tq = lane & 3;
  const int mi = lane >> 3, mr = lane & 7;  // ldmatrix / stmatrix: matrix, row
  const int Dk = ws.Dk, Dv = ws.Dv, nC = ws.nC;
  const int bh = blockIdx.y, dir = blockIdx.z / A.nseg, seg = blockIdx.z - dir * A.nseg;
  const int c_begin = seg * A.seg_len, n = min(A.seg_len, nC - c_begin);
  const int kb_lo = q * NKB / P, kb_hi = (q + 1) * NKB / P;  // this warp's state rows
  const int tb0 = q * TPW;                                    // this warp's tokens
  const int bar_id = 1 + gw, bar_n = 32 * P;
  const bool pcol = SUMMARY && s >= Dv / 16;       // a transition slice (summary pass)
  const int sj = pcol ? s - Dv / 16 : s;           // its 16 columns among P's or S's
  constexpr bool publish = !SUMMARY;

  // this warp's part of S^T: rows j = 16 sj + g (regs 0, 1) and + 8 (2, 3),
  // columns i = 8 nt + 2 tq (+1) for n-tiles nt of k-blocks [kb_lo, kb_hi)
  float S[2 * KPW][4];
#pragma unroll
  for (int k = 0; k < 2 * KPW; ++k) {
    const int i0 = 8 * (2 * kb_lo + k) + 2 * tq, j0 = 16 * sj + g;
    S[k][0] = S[k][1] = S[k][2] = S[k][3] = 0.f;
    if (pcol) {  // identity columns
      S[k][0] = i0 == j0 ? 1.f : 0.f;
      S[k][1] = i0 + 1 == j0 ? 1.f : 0.f;
      S[k][2] = i0 == j0 + 8 ? 1.f : 0.f;
      S[k][3] = i0 + 1 == j0 + 8 ? 1.f : 0.f;
    }
  }
  const float* init = A.init && (A.init_dir_stride || dir == 0)
                          ? A.init + dir * A.init_dir_stride + seg * A.init_seg_stride
                          : nullptr;
  if (init && !pcol) {
    const float* base = init + (size_t)bh * Dk * Dv + 16 * sj + g;
#pragma unroll
    for (int k = 0; k < 2 * KPW; ++k) {
      if (kb_lo + k / 2 < kb_hi) {
        const int i0 = 8 * (2 * kb_lo + k) + 2 * tq;
        S[k][0] = base[(size_t)i0 * Dv];
        S[k][1] = base[(size_t)(i0 + 1) * Dv];
        S[k][2] = base[(size_t)i0 * Dv + 8];
        S[k][3] = base[(size_t)(i0 + 1) * Dv + 8];
      }
    }
  }

  const uint32_t stage0 = smem_u32(smem + kChainHeadBytes);
  const uint32_t grp_u = smem_u32(smem + L.groups + gw * L.group);
  const uint32_t xs_u = grp_u + kChainBufs * L.stg, xu_u = xs_u + L.xs;
  // per-lane parts of the ldmatrix / stmatrix row addresses
  const uint32_t st_off = (uint32_t)((mi & 1) * Dk * 16 + ((mi >> 1) * 8 + mr) * 16);   // S staging
  const uint32_t su_off = (uint32_t)((mi & 1) * kSlab64 + ((mi >> 1) * 8 + mr) * 16);   // U staging, U~, W
  const uint32_t kt_off = (uint32_t)((mi >> 1) * kSlab64 + ((mi & 1) * 8 + mr) * 16);   // K~ (trans)

  // Own state rows -> bf16 A fragments, dumped to the S^T exchange and, as a
  // chunk-start state, to staging buffer sbuf (none after the last chunk).
  auto publish_state = [&](uint32_t sbuf, bool stage_it) {
#pragma unroll
    for (int k = 0; k < KPW; ++k) {
      const int kb = kb_lo + k;
      if (kb < kb_hi) {
        uint32_t a[4];
        a[0] = pack_bf16x2(S[2 * k][0], S[2 * k][1]);
        a[1] = pack_bf16x2(S[2 * k][2], S[2 * k][3]);
        a[2] = pack_bf16x2(S[2 * k + 1][0], S[2 * k + 1][1]);
        a[3] = pack_bf16x2(S[2 * k + 1][2], S[2 * k + 1][3]);
        if (stage_it) stmatrix_x4_trans(sbuf + kb * 256 + st_off, a);
        st_shared_v4(xs_u + kb * 512 + lane * 16, a);
      }
    }
  };
  publish_state(grp_u, publish);
  named_barrier(bar_id, bar_n);

  bool ok = true, okp = true;
  int lc = 0;          // chunk of this segment (its scan index is c_begin + lc)
  int st = 0, bi = 0;  // load stage and staging buffer of chunk lc
  uint32_t ph = 0;     // parity of stage st's current fill
  bool ready = false;  // chunk lc's stage was seen full ahead of time
  volatile int* fail = &bars.fail[gw];
  for (; lc < n; ++lc) {
    const uint32_t buf = grp_u + bi * L.stg;  // staging of chunk lc
    // the whole chunk-start state S^T, as A fragments over k = state rows
    uint32_t sa[NKB][4];
#pragma unroll
    for (int kb = 0; kb < NKB; ++kb) ld_shared_v4(xs_u + kb * 512 + lane * 16, sa[kb]);

    bool okw = (ready || __all_sync(0xffffffffu, mbar_wait(&bars.full[st], ph, limit))) && okp;
    const uint32_t sw = stage0 + st * L.stage;         // W
    const uint32_t sk = sw + 64u * Dk * 2;             // K~
    float u[2 * TPW][4];
    uint32_t ua_mine[TPW][4];
    if (okw) {
      const uint32_t sut = sw + L.wk_bytes + 2u * gw * kSlab64;  // this slice's U~ slabs
      // U^T = U~^T - S^T W^T over this warp's tokens: every B fragment is
      // loaded before the MMAs that use them, so the loads overlap
      uint32_t bw[NKB][TPW][4];
#pragma unroll
      for (int kb = 0; kb < NKB; ++kb)
#pragma unroll
        for (int t = 0; t < TPW; ++t) ldmatrix_x4(sw + 2 * kb * kSlab64 + (tb0 + t) * 256 + su_off, bw[kb][t]);
#pragma unroll
      for (int t = 0; t < TPW; ++t) {
        if (pcol) {  // transition columns: U~ = 0
          u[2 * t][0] = u[2 * t][1] = u[2 * t][2] = u[2 * t][3] = 0.f;
          u[2 * t + 1][0] = u[2 * t + 1][1] = u[2 * t + 1][2] = u[2 * t + 1][3] = 0.f;
          continue;
        }
        uint32_t r[4];
        ldmatrix_x4_trans(sut + (tb0 + t) * 256 + su_off, r);
        unpack_bf16x2(r[0], u[2 * t][0], u[2 * t][1]);
        unpack_bf16x2(r[1], u[2 * t][2], u[2 * t][3]);
        unpack_bf16x2(r[2], u[2 * t + 1][0], u[2 * t + 1][1]);
        unpack_bf16x2(r[3], u[2 * t + 1][2], u[2 * t + 1][3]);
      }
#pragma unroll
      for (int kb = 0; kb < NKB; ++kb) {
        uint32_t na[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) na[e] = sa[kb][e] ^ 0x80008000u;  // -S^T
#pragma unroll
        for (int t = 0; t < TPW; ++t) {
          mma_16816(u[2 * t], na, bw[kb][t][0], bw[kb][t][1]);
          mma_16816(u[2 * t + 1], na, bw[kb][t][2], bw[kb][t][3]);
        }
      }
      // this warp's U^T block(s): staged for stage C and dumped for the group
#pragma unroll
      for (int t = 0; t < TPW; ++t) {
        ua_mine[t][0] = pack_bf16x2(u[2 * t][0], u[2 * t][1]);
        ua_mine[t][1] = pack_bf16x2(u[2 * t][2], u[2 * t][3]);
        ua_mine[t][2] = pack_bf16x2(u[2 * t + 1][0], u[2 * t + 1][1]);
        ua_mine[t][3] = pack_bf16x2(u[2 * t + 1][2], u[2 * t + 1][3]);
        if (publish) stmatrix_x4_trans(buf + L.stg_s + (tb0 + t) * 256 + su_off, ua_mine[t]);
        st_shared_v4(xu_u + (tb0 + t) * 512 + lane * 16, ua_mine[t]);
      }
      if (publish) fence_proxy_async_smem();  // staging writes -> the producer's bulk stores
    }
    if (!okw && lane == 0) *fail = 1;
    named_barrier(bar_id, bar_n);
    ok = *fail == 0;
    if (!ok) break;
    // chunk lc's staging (its start state and U) is complete
    if (publish && q == 0 && lane == 0) mbar_arrive(&bars.staged[bi]);
    // S^T <- e^{gamma_C} S^T + U^T K~ over this warp's state rows (B
    // fragments first, then the MMAs)
    uint32_t bk[4][KPW][4];
#pragma unroll
    for (int kt = 0; kt < 4; ++kt)
#pragma unroll
      for (int k = 0; k < KPW; ++k)
        if (kb_lo + k < kb_hi) ldmatrix_x4_trans(sk + 2 * (kb_lo + k) * kSlab64 + kt * 256 + kt_off, bk[kt][k]);
    uint32_t ua[4][4];
#pragma unroll
    for (int kt = 0; kt < 4; ++kt) ld_shared_v4(xu_u + kt * 512 + lane * 16, ua[kt]);
    float decay;
    asm volatile("ld.shared.f32 %0, [%1];" : "=f"(decay) : "r"(sk + 64u * Dk * 2));
#pragma unroll
    for (int k = 0; k < 2 * KPW; ++k)
#pragma unroll
      for (int e = 0; e < 4; ++e) S[k][e] *= decay;
#pragma unroll
    for (int kt = 0; kt < 4; ++kt) {
#pragma unroll
      for (int k = 0; k < KPW; ++k) {
        if (kb_lo + k < kb_hi) {
          mma_16816(S[2 * k], ua[kt], bk[kt][k][0], bk[kt][k][1]);
          mma_16816(S[2 * k + 1], ua[kt], bk[kt][k][2], bk[kt][k][3]);
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&bars.empty[st]);  // this warp's reads of the stage are done
    if (++st == nst) {
      st = 0;
      ph ^= 1;
    }
    // probe the next chunk's stage while the MMAs above run
    ready = __all_sync(0xffffffffu, mbar_test_wait(&bars.full[st], ph));
    // the next chunk's start state goes to buffer (lc + 1) % 3, which the
    // producer's stores of chunk lc - 2 must have finished reading
    const bool more = lc + 1 < n;
    const int bn = bi == kChainBufs - 1 ? 0 : bi + 1;
    if (publish && more && lc >= 2)
      okp = __all_sync(0xffffffffu, mbar_wait(&bars.freed[bn], ((lc - 2) / kChainBufs) & 1, limit));
    publish_state(grp_u + bn * L.stg, publish && more && okp);
    named_barrier(bar_id, bar_n);
    bi = bn;
  }
  if (!ok) {
    if (lane == 0) atomicOr(err, kErrTimeout);
    return false;
  }
  const bool ends = !A.fin_last_seg_only || seg == A.nseg - 1;
  float* fin = A.fin && ends && (A.fin_dir_stride || dir == 0)
                   ? A.fin + dir * A.fin_dir_stride + seg * A.fin_seg_stride
                   : nullptr;
  if (fin) {
    float* base = fin + (size_t)bh * Dk * A.fin_ld + (pcol ? Dv : 0) + 16 * sj + g;
#pragma unroll
    for (int k = 0; k < 2 * KPW; ++k) {
      if (kb_lo + k / 2 < kb_hi) {
        const int i0 = 8 * (2 * kb_lo + k) + 2 * tq;
        base[(size_t)i0 * A.fin_ld] = S[k][0];
        base[(size_t)(i0 + 1) * A.fin_ld] = S[k][1];
        base[(size_t)i0 * A.fin_ld + 8] = S[k][2];
        base[(size_t)(i0 + 1) * A.fin_ld + 8] = S[k][3];
      }
    }
  }
  return true;
}

// The producer (one thread): loads the segment's chunk lc into stage lc % nst
// once the chain warps have released that stage's previous chunk and, in the
// publish pass, stores each chunk's staged S and U for the CTA's groups.
__device__ void chain_producer(uint8_t* smem, const ChainLayout& L, int nst, int active, int s0,
                               const ChainArgs& A, const Workspace& ws, long long limit,
                               unsigned* err) {
  ChainBars& bars = *reinterpret_cast<ChainBars*>(smem);
  const int bh = blockIdx.y, dir = blockIdx.z / A.nseg, seg = blockIdx.z - dir * A.nseg;
  const int nC = ws.nC, Dk = ws.Dk;
  const int c_begin = seg * A.seg_len, n = min(A.seg_len, nC - c_begin);
  uint8_t* stage0 = smem + kChainHeadBytes;
  // U~ slabs of the state slices among the CTA's (transition slices need none)
  const int ut_slices = max(0, min(s0 + active, ws.Dv / 16) - s0);
  const uint32_t ut_bytes = (uint32_t)ut_slices * 2 * kSlab64;
  auto block_of = [&](int lc) {
    const int c = c_begin + lc;
    return ws.blk(ws.tile(dir, bh, dir ? nC - 1 - c : c));
  };
  auto load = [&](int lc) -> bool {
    const int st = lc % nst;
    if (lc >= nst && !mbar_wait(&bars.empty[st], ((lc / nst) - 1) & 1, limit)) return false;
    const uint8_t* blk = block_of(lc);
    uint8_t* dst = stage0 + st * L.stage;
    mbar_arrive_expect_tx(&bars.full[st], L.wk_bytes + ut_bytes);
    bulk_load(dst, blk + ws.off_w, L.wk_bytes, &bars.full[st]);
    if (ut_bytes)
      bulk_load(dst + L.wk_bytes, blk + ws.off_ut + (size_t)s0 * 2 * kSlab64, ut_bytes, &bars.full[st]);
    return true;
  };
  int issued = 0;
  bool ok = true;
  for (; issued < n && issued < nst; ++issued) load(issued);
  for (int lc = 0; lc < n && ok; ++lc) {
    if (A.publish) {
      const int b = lc % kChainBufs;
      // chunk lc - 1's stores have read their buffer: the chain may reuse it
      // (for chunk lc + 2's start state, at the end of its chunk lc + 1)
      if (lc >= 1) {
        bulk_wait_read();
        mbar_arrive(&bars.freed[(lc - 1) % kChainBufs]);
      }
      // publish chunk lc once every group has staged it
      if (!mbar_wait(&bars.staged[b], (lc / kChainBufs) & 1, limit)) {
        ok = false;
        break;
      }
      uint8_t* blk = block_of(lc);
      for (int gw = 0; gw < active; ++gw) {
        const uint8_t* sb = smem + L.groups + gw * L.group + b * L.stg;
        bulk_store_nc(blk + ws.off_s + (size_t)(s0 + gw) * 2 * Dk * 16, sb, L.stg_s);
        bulk_store_nc(blk + ws.off_u + (size_t)(s0 + gw) * 2 * kSlab64, sb + L.stg_s, 2 * kSlab64);
      }
      bulk_commit();
    }
    // refill the stage chunk lc used with chunk lc + nst
    if (issued < n) {
      if (!load(issued)) {
        ok = false;
        break;
      }
      ++issued;
    }
  }
  bulk_wait_all();
  if (!ok) atomicOr(err, kErrTimeout);
  // nothing may still be landing in shared memory when the CTA leaves:
  // wait for the last load issued into each stage (bounded by the timer)
  for (int st = 0; st < nst && st < issued; ++st) {
    const int last = st + ((issued - 1 - st) / nst) * nst;
    mbar_wait(&bars.full[st], (last / nst) & 1, kDrainPolls);
  }
}

template <int NKB, bool SUMMARY>
__global__ void __launch_bounds__(32 * (kChainMaxGroups * 4 + 1), 1)
gdn_recur_kernel(ChainArgs A, Workspace ws, int ns, int nst, long long limit, unsigned* err) {
  constexpr int P = chain_group_warps(NKB);
  extern __shared__ __align__(128) uint8_t smem_raw[];
  ChainBars& bars = *reinterpret_cast<ChainBars*>(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int s0 = blockIdx.x * ns;
  const int nslices = ws.Dv / 16 + A.p_slices;
  const int active = min(ns, nslices - s0);  // slice groups with a slice
  const ChainLayout L(ws.Dk, ns, nst);
  if (threadIdx.x == 0) {
    for (int i = 0; i < nst; ++i) {
      mbar_init(&bars.full[i], 1);
      mbar_init(&bars.empty[i], active * P);
    }
    for (int i = 0; i < kChainBufs; ++i) {
      mbar_init(&bars.staged[i], active);
      mbar_init(&bars.freed[i], 1);
    }
    for (int i = 0; i < kChainMaxGroups; ++i) bars.fail[i] = 0;
    fence_mbar_init();
  }
  __syncthreads();
  pdl_wait();  // stage A's W, K~, U~ (or the previous pass) are complete and visible
  pdl_trigger();
  const int gw = warp / P, q = warp - gw * P;
  if (gw < active)
    chain_warp<NKB, SUMMARY>(smem_raw, L, nst, gw, q, s0 + gw, A, ws, limit, err);
  else if (warp == ns * P && lane == 0)
    chain_producer(smem_raw, L, nst, active, s0, A, ws, limit, err);
  __syncthreads();
}

// The time-segmented scan's prefix over segments (one CTA per 4 state
// columns, b*h and direction): S_0 = the scan's start state, S_{g+1} = P_g S_g
// + R_g, with the summary pass's maps [dir][seg][b*h][Dk][Dv + Dk] (row i:
// R's row i, then P's row i); writes every segment's start state S_g to
// seg_state [dir][seg][b*h][Dk][Dv].  fp32 on CUDA cores: nseg dependent
// steps of a Dk x Dk by Dk x 4 product per CTA, with P and R staged in shared
// memory by 16-byte cp.async copies (the next segment's land while this one
// computes); each thread keeps one column and Dk / 64 rows.
constexpr int kPrefixThreads = 256;
constexpr int kPrefixCols = 4;
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
struct PrefixSmem {
  float P[2][128][132];          // P_g, padded rows (double-buffered over segments)
  float R[2][128][kPrefixCols];  // this CTA's columns of R_g
  float S[128][kPrefixCols];     // this CTA's columns of the current start state
};
__global__ void __launch_bounds__(kPrefixThreads)
gdn_segment_prefix_kernel(const float* maps, const float* state_in, float* seg_state, int Dk,
                          int Dv, int NBH, int nseg) {
  extern __shared__ __align__(16) uint8_t prefix_raw[];
  PrefixSmem& sm = *reinterpret_cast<PrefixSmem*>(prefix_raw);
  constexpr int kRowGroups = kPrefixThreads / kPrefixCols;  // 64
  const int j0 = kPrefixCols * blockIdx.x, bh = blockIdx.y, dir = blockIdx.z;
  const int tid = threadIdx.x, jj = tid % kPrefixCols, rg = tid / kPrefixCols;
  const int ld = Dk + Dv;
  pdl_wait();  // the summary pass is complete and visible
  pdl_trigger();
  auto stage = [&](int sg, int buf) {  // P_g and R_g's columns -> buffer buf
    const float* M = maps + (((size_t)dir * nseg + sg) * NBH + bh) * Dk * ld;
    const int q4 = Dk / 4;  // 16-byte pieces of a P row
    for (int e = tid; e < Dk * q4; e += kPrefixThreads) {
      const int i = e / q4, c = e - i * q4;
      cp_async16(&sm.P[buf][i][4 * c], M + (size_t)i * ld + Dv + 4 * c);
    }
    for (int i = tid; i < Dk; i += kPrefixThreads) cp_async16(&sm.R[buf][i][0], M + (size_t)i * ld + j0);
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  for (int e = tid; e < Dk * kPrefixCols; e += kPrefixThreads) {
    const int i = e / kPrefixCols, j = e % kPrefixCols;
    sm.S[i][j] = (dir == 0 && state_in) ? state_in[((size_t)bh * Dk + i) * Dv + j0 + j] : 0.f;
  }
  if (nseg > 1) stage(0, 0);
  for (int sg = 0; sg < nseg; ++sg) {
    float* dst = seg_state + (((size_t)dir * nseg + sg) * NBH + bh) * Dk * Dv;
    for (int e = tid; e < Dk * kPrefixCols; e += kPrefixThreads) {
      const int i = e / kPrefixCols, j = e % kPrefixCols;
      dst[(size_t)i * Dv + j0 + j] = sm.S[i][j];
    }
    if (sg + 1 == nseg) break;
    const int buf = sg & 1;
    // this segment's copies have landed (the next segment's may still fly)
    asm volatile("cp.async.wait_group 0;" ::: "memory");
    __syncthreads();
    if (sg + 2 < nseg) stage(sg + 1, buf ^ 1);  // lands while this step computes
    // rows rg, rg + 64 (Dk <= 128): acc = R + P S, S's column loaded once per k
    const int nr = rg + kRowGroups < Dk ? 2 : (rg < Dk ? 1 : 0);
    float acc0 = rg < Dk ? sm.R[buf][rg][jj] : 0.f;
    float acc1 = nr == 2 ? sm.R[buf][rg + kRowGroups][jj] : 0.f;
    const float* P0 = sm.P[buf][rg < Dk ? rg : 0];
    const float* P1 = sm.P[buf][nr == 2 ? rg + kRowGroups : 0];
    for (int k = 0; k < Dk; k += 4) {
      const float s0 = sm.S[k][jj], s1 = sm.S[k + 1][jj], s2 = sm.S[k + 2][jj], s3 = sm.S[k + 3][jj];
      const float4 p = *reinterpret_cast<const float4*>(P0 + k);
      acc0 = fmaf(p.x, s0, fmaf(p.y, s1, fmaf(p.z, s2, fmaf(p.w, s3, acc0))));
      const float4 p1 = *reinterpret_cast<const float4*>(P1 + k);
      acc1 = fmaf(p1.x, s0, fmaf(p1.y, s1, fmaf(p1.z, s2, fmaf(p1.w, s3, acc1))));
    }
    __syncthreads();
    if (nr >= 1) sm.S[rg][jj] = acc0;
    if (nr == 2) sm.S[rg + kRowGroups][jj] = acc1;
    __syncthreads();
  }
}

// The recurrence kernel for Dk = 16 * nkb.
using RecurKernel = void (*)(ChainArgs, Workspace, int, int, long long, unsigned*);
template <bool SUMMARY>
RecurKernel recur_kernel_pass(int nkb) {
  switch (nkb) {
    case 1: return gdn_recur_kernel<1, SUMMARY>;
    case 2: return gdn_recur_kernel<2, SUMMARY>;
    case 3: return gdn_recur_kernel<3, SUMMARY>;
    case 4: return gdn_recur_kernel<4, SUMMARY>;
    case 5: return gdn_recur_kernel<5, SUMMARY>;
    case 6: return gdn_recur_kernel<6, SUMMARY>;
    case 7: return gdn_recur_kernel<7, SUMMARY>;
    default: return gdn_recur_kernel<8, SUMMARY>;
  }
}
RecurKernel recur_kernel(int nkb, bool summary = false) {
  return summary ? recur_kernel_pass<true>(nkb) : recur_kernel_pass<false>(nkb);
}

// ========================================================== stage C: output
// Persistent: one CTA per SM walks tiles t = blockIdx.x, + gridDim.x, ...
// with two input sets in shared memory, so the next tile's TMA / bulk loads
// land while the current tile computes.  Per set (offsets from Dk, Dv):
//   Q   [Dk/8][64][8]  raw q tile (TMA)
//   K   [Dk/8][64][8]  raw k tile (TMA); after P = Q K^T it holds Qs = diag(e^g) Q
//   U   [Dv/8][64][8]  U = U~ - W S0 of the current direction } one block, as in
//   S   [Dv/8][Dk][8]  state at the chunk's start             } the workspace
// then P [8][64][8] (masked, gated Q K^T, K-major A) and the scalar block.
struct OutSmall {
  float g[2][64];
  float gam[64], rnq[2][64], rnk[2][64], arow[64];  // norms per tile set
  float bcol[8][64];
  float dg[64][8];  // P's gate factor inside row r's own 8-row block (memory order)
  uint64_t tma_bar[2], ld_bar[2], mma_bar, p_bar;
  uint64_t fin_bar;  // one commit on a failed wait: every MMA issued has landed
  uint32_t tmem;
};
struct OutLayout {
  uint32_t q, k, u, s, set_bytes, p, small, total;
  __host__ __device__ OutLayout(int Dk, int Dv) {
    auto al = [](uint32_t x) { return (x + 127u) & ~127u; };
    q = 0;
    k = al(q + 64u * Dk * 2);
    u = al(k + 64u * Dk * 2);
    s = u + 64u * Dv * 2;
    set_bytes = al(s + (uint32_t)Dk * Dv * 2);
    p = 2 * set_bytes;
    small = al(p + 8u * kSlab64);
    total = al(small + (uint32_t)sizeof(OutSmall));
  }
};

__device__ __forceinline__ void cp_async4(void* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__device__ bool output_body(uint8_t* smem, const CUtensorMap* tm_q, const CUtensorMap* tm_k,
                            __nv_bfloat16* __restrict__ out, const Workspace& ws, int T, int H,
                            int ndir, long long limit, unsigned* err) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int Dk = ws.Dk, Dv = ws.Dv, nC = ws.nC;
  const int ntiles = nC * ws.NBH;
  const OutLayout L(Dk, Dv);
  OutSmall& sm = *reinterpret_cast<OutSmall*>(smem + L.small);
  uint8_t* sP = smem + L.p;
  const uint32_t tm = sm.tmem;
  const uint32_t tmP = tm, tmO = tm + 64;
  const uint32_t ubytes = kC * Dv * 2, sbytes = Dk * Dv * 2;
  // warps w, w + 4, w + 8, w + 12 share TMEM lane quadrant w % 4 and split
  // the column blocks four ways
  const int quad = warp & 3, part = warp >> 2;
  const int r = 16 * quad + (lane & 15);
  const uint32_t lane_base = static_cast<uint32_t>(32 * quad) << 16;

  auto issue_dir = [&](int set, int tile_t, int dir) {  // thread 0: U | S
    uint8_t* base = smem + set * L.set_bytes;
    const int bh = tile_t / nC, j = tile_t - bh * nC;
    const size_t tile = ws.tile(dir, bh, j);
    mbar_arrive_expect_tx(&sm.ld_bar[set], ubytes + sbytes);
    bulk_load(base + L.u, ws.blk(tile) + ws.off_u, ubytes + sbytes, &sm.ld_bar[set]);
  };
  // all threads: start loading tile `tile_t` into `set`
  auto issue_tile = [&](int set, int tile_t) {
    const int bh = tile_t / nC, j = tile_t - bh * nC;
    const int b = bh / H, h = bh - b * H, t0 = j * kC;
    if (tid == 0) {
      uint8_t* base = smem + set * L.set_bytes;
      mbar_arrive_expect_tx(&sm.tma_bar[set], 2 * (Dk / 8) * kSlab64);
      tma_load_tile(base + L.q, tm_q, &sm.tma_bar[set], t0, h, b);
      tma_load_tile(base + L.k, tm_k, &sm.tma_bar[set], t0, h, b);
      issue_dir(set, tile_t, 0);
    }
    if (tid < kC) {  // the tile's gates, as stage A formed them (0 past T)
      cp_async4(&sm.g[set][tid], ws.blk(ws.tile(0, bh, j)) + ws.off_g + 4 * tid);
      cp_async_commit();
    }
  };

  // mbarrier phase parities: bit `set` of tma_ph / ld_ph
  uint32_t tma_ph = 0, ld_ph = 0, mma_ph = 0, p_ph = 0;
  // Head of the tile in `set`: wait for its q/k tile and gates, issue
  // P = Q K^T (shared by both directions) and commit it, then the row norms,
  // which overlap it.  `one_more`: a later tile's gates are in flight too.
  // The head of tile t + 1 runs while tile t's last MMA round executes.
  auto head = [&](int set, bool one_more) -> bool {
    uint8_t* base = smem + set * L.set_bytes;
    uint8_t* sQ = base + L.q;
    uint8_t* sK = base + L.k;
    if (tid < kC) {
      if (one_more) cp_async_wait<1>();
      else cp_async_wait<0>();
    }
    if (!block_wait(&sm.tma_bar[set], (tma_ph >> set) & 1, limit, err)) return false;
    tma_ph ^= 1u << set;
    if (tid == 0) {
      tc_fence_after_sync();
      const uint32_t idP = idesc_bf16(64, 64, 0, 0);
      for (int ks = 0; ks < Dk / 16; ++ks)
        mma_bf16(tmP, sdesc(smem_u32(sQ) + ks * 2 * kSlab64, kSlab64, 128),
                 sdesc(smem_u32(sK) + ks * 2 * kSlab64, kSlab64, 128), idP, ks > 0);
      mma_commit(&sm.p_bar);
    }
    {  // 1 / |q|, 1 / |k| per row: four threads per row and tensor
      const int row = tid >> 3, part = tid & 3;
      const bool isk = (tid >> 2) & 1;
      const float rn = row_rnorm4(isk ? sK : sQ, row, part, Dk);
      if (part == 0) (isk ? sm.rnk[set] : sm.rnq[set])[row] = rn;
    }
    return true;
  };

  // On a failed wait, before leaving: one commit covering every MMA this
  // CTA issued, so none is still writing TMEM when the accumulators are freed.
  auto drain_mma = [&]() {
    if (tid == 0) mma_commit(&sm.fin_bar);
    mbar_wait(&sm.fin_bar, 0, kDrainPolls);
  };

  int k = 0;
  if (blockIdx.x < ntiles) issue_tile(0, blockIdx.x);
  if (blockIdx.x + gridDim.x < ntiles) issue_tile(1, blockIdx.x + gridDim.x);
  if (blockIdx.x < ntiles && !head(0, blockIdx.x + gridDim.x < ntiles)) {
    mbar_wait(&sm.ld_bar[0], 0, kDrainPolls);
    if (blockIdx.x + gridDim.x < ntiles) {
      mbar_wait(&sm.tma_bar[1], 0, kDrainPolls);
      mbar_wait(&sm.ld_bar[1], 0, kDrainPolls);
    }
    drain_mma();
    return false;
  }
  for (int t = blockIdx.x; t < ntiles; t += gridDim.x, ++k) {
    const int set = k & 1;
    const bool next_issued = t + gridDim.x < ntiles;
    // on a failed wait: drain the next tile's loads (its head has not run;
    // the caller drained its own barrier)
    auto drain_other = [&]() {
      if (next_issued) {
        mbar_wait(&sm.tma_bar[set ^ 1], (tma_ph >> (set ^ 1)) & 1, kDrainPolls);
        mbar_wait(&sm.ld_bar[set ^ 1], (ld_ph >> (set ^ 1)) & 1, kDrainPolls);
      }
      drain_mma();
    };
    uint8_t* base = smem + set * L.set_bytes;
    uint8_t* sQ = base + L.q;
    uint8_t* sK = base + L.k;   // then Qs
    uint8_t* sU = base + L.u;
    uint8_t* sS = base + L.s;
    const int bh = t / nC, j = t - bh * nC;
    const int b = bh / H, h = bh - b * H, t0 = j * kC;
    const int nvalid = min(kC, T - t0);

    for (int dir = 0; dir < ndir; ++dir) {
      __syncthreads();
      if (warp == 0) warp_gamma(sm.g[set], sm.gam, dir);
      __syncthreads();
      // Gate factors as in stage A: for i in an earlier 8-row block than r's
      // block b, split at m_b = gam at b's first scan position,
      // P'_ri = arow_r P_ri bcol[b][i] (both factors <= 1); inside the
      // diagonal block e^{gam_r - gam_i} is taken whole.
      for (int e = tid; e < 8 * 64; e += kOutThreads) {
        const int blk = e >> 6, i = e & 63;
        const int qpos = dir ? 63 - i : i;
        const float mb = sm.gam[dir ? 63 - 8 * blk : 8 * blk];
        sm.bcol[blk][i] = qpos < 8 * blk ? sm.rnk[set][i] * exp2f((mb - sm.gam[i]) * kLog2e) : 0.f;
        const int r = e >> 3, id = (r & ~7) + (e & 7);  // row r, column id of its block
        const bool incl = dir ? (id >= r) : (id <= r);
        sm.dg[r][e & 7] = incl ? sm.rnk[set][id] * exp2f((sm.gam[r] - sm.gam[id]) * kLog2e) : 0.f;
      }
      if (tid < 64) {
        const int p = dir ? 63 - tid : tid;
        const float mb = sm.gam[dir ? 63 - 8 * (p >> 3) : 8 * (p >> 3)];
        sm.arow[tid] = exp2f((sm.gam[tid] - mb) * kLog2e);
      }
      if (dir == 0) {
        if (!block_wait(&sm.p_bar, p_ph, limit, err)) {
          mbar_wait(&sm.ld_bar[set], (ld_ph >> set) & 1, kDrainPolls);
          drain_other();
          return false;
        }
        p_ph ^= 1;
      }
      if (!block_wait(&sm.ld_bar[set], (ld_ph >> set) & 1, limit, err)) {
        drain_other();
        return false;
      }
      ld_ph ^= 1u << set;
      tc_fence_after_sync();
      // P'_ri = (q_r . k_i) / |k_i| * e^{gam_r - gam_i} for i at or before r
      {
        float v[16];
        tmem_ld16(tmP + lane_base + 16 * part, v);
        tmem_wait_ld();
        const int c = part;
        if (lane < 16) {
          const float ar = sm.arow[r];
          const float* bc = sm.bcol[(dir ? 63 - r : r) >> 3];
          const int rb = r & ~7;  // first column of r's own block
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int i = 16 * c + e;
            // own block: dg (gate factor taken whole); elsewhere the split
            // factors (zero for columns the mask excludes)
            v[e] = (i & ~7) == rb ? v[e] * sm.dg[r][i - rb] : ar * v[e] * bc[i];
          }
          reinterpret_cast<uint4*>(sP + (2 * c) * kSlab64)[r] = pack8_bf16(v);
          reinterpret_cast<uint4*>(sP + (2 * c + 1) * kSlab64)[r] = pack8_bf16(v + 8);
        }
      }
      // Qs = diag(e^gam) Q -> sK (K is dead once P is in TMEM)
      if (lane < 16) {
        const float eg = expf(sm.gam[r]);
        for (int sl = part; sl < Dk / 8; sl += 4) {
          float x[8];
          unpack8_bf16(reinterpret_cast<const uint4*>(sQ + sl * kSlab64)[r], x);
#pragma unroll
          for (int e = 0; e < 8; ++e) x[e] *= eg;
          reinterpret_cast<uint4*>(sK + sl * kSlab64)[r] = pack8_bf16(x);
        }
      }
      block_sync_async();
      if (tid == 0) {
        // D_O (+)= Qs S0 (K = Dk) + P' U (K = 64 tokens); S and U read MN-major
        const uint32_t idO = idesc_bf16(64, Dv, 0, 1);
        for (int ks = 0; ks < Dk / 16; ++ks)
          mma_bf16(tmO, sdesc(smem_u32(sK) + ks * 2 * kSlab64, kSlab64, 128),
                   sdesc(smem_u32(sS) + ks * 256, 128, Dk * 16), idO, (dir > 0) || (ks > 0));
        for (int ks = 0; ks < kC / 16; ++ks)
          mma_bf16(tmO, sdesc(smem_u32(sP) + ks * 2 * kSlab64, kSlab64, 128),
                   sdesc(smem_u32(sU) + ks * 256, 128, kSlab64), idO, 1);
        mma_commit(&sm.mma_bar);
      }
      if (dir + 1 < ndir) {
        // the next direction rewrites P', Qs and this set's U | S
        if (!block_wait(&sm.mma_bar, mma_ph, limit, err)) {
          drain_other();
          return false;
        }
        mma_ph ^= 1;
        if (tid == 0) issue_dir(set, t, dir + 1);
      }
    }
    // the last direction's MMA round is in flight: the next tile's head
    // (its loads, P = Q K^T and norms) runs meanwhile
    if (next_issued && !head(set ^ 1, false)) {
      // head drained the next tile's q/k; its U | S and this round remain
      mbar_wait(&sm.ld_bar[set ^ 1], (ld_ph >> (set ^ 1)) & 1, kDrainPolls);
      drain_mma();
      return false;
    }
    if (!block_wait(&sm.mma_bar, mma_ph, limit, err)) {
      if (next_issued) mbar_wait(&sm.ld_bar[set ^ 1], (ld_ph >> (set ^ 1)) & 1, kDrainPolls);
      drain_mma();
      return false;
    }
    mma_ph ^= 1;
    tc_fence_after_sync();
    // O = diag(1/|q|) D_O -> out (rows of this chunk that exist)
    {
      const float rq = sm.rnq[set][r];
      float v0[16], v1[16];
      const bool has1 = part + 4 < Dv / 16;
      if (part < Dv / 16) tmem_ld16(tmO + lane_base + 16 * part, v0);
      if (has1) tmem_ld16(tmO + lane_base + 16 * (part + 4), v1);
      tmem_wait_ld();
      auto put = [&](int c, float* v) {
#pragma unroll
        for (int e = 0; e < 16; ++e) v[e] *= rq;
        uint4* o = reinterpret_cast<uint4*>(out + (((size_t)b * T + t0 + r) * H + h) * Dv + 16 * c);
        o[0] = pack8_bf16(v);
        o[1] = pack8_bf16(v + 8);
      };
      if (lane < 16 && r < nvalid) {
        if (part < Dv / 16) put(part, v0);
        if (has1) put(part + 4, v1);
      }
    }
    tc_fence_before_sync();
    __syncthreads();  // this set's buffers and the TMEM accumulators are free
    tc_fence_after_sync();
    if (t + 2 * gridDim.x < ntiles) issue_tile(set, t + 2 * gridDim.x);
  }
  return true;
}

__global__ void __launch_bounds__(kOutThreads, 1)
gdn_output_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  __nv_bfloat16* __restrict__ out, Workspace ws, int T, int H, int ndir,
                  long long limit, unsigned* err) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  const OutLayout L(ws.Dk, ws.Dv);
  OutSmall& sm = *reinterpret_cast<OutSmall*>(smem_raw + L.small);
  const int tid = threadIdx.x;
  const uint32_t ncols = 256u;  // P [0, 64), D_O [64, 64 + Dv)
  if (tid == 0) {
    mbar_init(&sm.tma_bar[0], 1);
    mbar_init(&sm.tma_bar[1], 1);
    mbar_init(&sm.ld_bar[0], 1);
    mbar_init(&sm.ld_bar[1], 1);
    mbar_init(&sm.mma_bar, 1);
    mbar_init(&sm.p_bar, 1);
    mbar_init(&sm.fin_bar, 1);
    fence_mbar_init();
  }
  if ((tid >> 5) == 0) {
    tmem_alloc(&sm.tmem, ncols);
    tmem_relinquish();
  }
  block_sync_async();
  pdl_wait();  // stage B's chunk-start states are complete and visible
  pdl_trigger();
  output_body(smem_raw, &tm_q, &tm_k, out, ws, T, H, ndir, limit, err);
  tc_fence_before_sync();
  __syncthreads();
  if ((tid >> 5) == 0) tmem_dealloc(sm.tmem, ncols);
}

// ===================================================================== host
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// A 64-token tile map of a [B, T, H, D] bf16 tensor.
bool make_map(CUtensorMap* m, const void* base, int B, int T, int H, int D) {
  return make_tile_map(m, base, B, T, H, D, kC);
}


// Opt the kernels into their dynamic shared memory, once per device.
cudaError_t set_smem_attrs() {
  constexpr int kMaxDev = 64;
  static std::mutex mu;
  static bool done[kMaxDev] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDev) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (done[dev]) return cudaSuccess;
  e = cudaFuncSetAttribute(gdn_prep_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)sizeof(PrepSmem));
  for (int nkb = 1; nkb <= 8 && e == cudaSuccess; ++nkb)
    for (int sm = 0; sm < 2 && e == cudaSuccess; ++sm)
      e = cudaFuncSetAttribute(recur_kernel(nkb, sm == 1), cudaFuncAttributeMaxDynamicSharedMemorySize,
                               227 * 1024);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(gdn_output_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)OutLayout(128, 128).total);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(gdn_segment_prefix_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)sizeof(PrefixSmem));
  if (e == cudaSuccess) done[dev] = true;
  return e;
}

// Stage B's shape: slices (16 state columns, one warp group each) per CTA
// and load-ring stages, chosen for the fewest waves of CTAs (the occupancy
// API counts how many fit an SM); among equals, one slice per CTA (its
// groups then share no issue slots), then the deepest ring.  Cached per
// (device, Dk, Dv, heads x directions).
struct ChainShape {
  int ns, nst;
};
ChainShape chain_shape(int Dk, int Dv, int heads_dirs, int sms) {
  struct Entry {
    int dev, Dk, Dv, hd;
    ChainShape shape;
  };
  static std::mutex mu;
  static Entry cache[64];
  static int used = 0;
  int dev = 0;
  cudaGetDevice(&dev);
  {
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < used; ++i)
      if (cache[i].dev == dev && cache[i].Dk == Dk && cache[i].Dv == Dv && cache[i].hd == heads_dirs)
        return cache[i].shape;
  }
  const int nslices = Dv / 16;
  const int P = chain_group_warps(Dk / 16);
  ChainShape best = {1, 2};
  long long best_waves = -1;
  for (int ns = 1; ns <= kChainMaxGroups && ns <= nslices; ns *= 2) {
    for (int nst = kChainMaxStages; nst >= 2; --nst) {
      const int smem = (int)ChainLayout(Dk, ns, nst).total;
      if (smem > 227 * 1024) continue;
      int per_sm = 0;
      if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, recur_kernel(Dk / 16), 32 * (ns * P + 1),
                                                        smem) != cudaSuccess) {
        cudaGetLastError();
        per_sm = 1;
      }
      per_sm = std::max(per_sm, 1);
      const long long ctas = (long long)((nslices + ns - 1) / ns) * heads_dirs;
      const long long waves = (ctas + (long long)sms * per_sm - 1) / ((long long)sms * per_sm);
      if (best_waves < 0 || waves < best_waves) {
        best_waves = waves;
        best = {ns, nst};
      }
    }
  }
  std::lock_guard<std::mutex> lock(mu);
  if (used < 64) cache[used++] = {dev, Dk, Dv, heads_dirs, best};
  return best;
}

// Launch with programmatic stream serialisation: the kernel may start while
// the previous kernel in the stream drains; each kernel of this path calls
// griddepcontrol.wait before its first global-memory access.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

}  // namespace

// Time segments of the chunked scan.  Segmenting pays only when a call has
// too few (head, state-slice) chains to fill the GPU and many chunks: its
// three passes do about three times the chain work, with a serial depth of
// about 2 nC / G + G chunk steps instead of nC.  A setting > 0 from
// gdn_set_time_segments forces the count (1: never segment).
int time_segments(int B, int T, int H, int Dk, int Dv, bool bidir) {
  const int nC = (T + kC - 1) / kC;
  const int forced = current_time_segments();
  int G = 1;
  if (forced > 0) {
    G = forced;
  } else {
    const long long chains = (long long)(Dv / 16) * B * H * (bidir ? 2 : 1);
    const int sms = num_sms();
    if (nC >= 64 && chains * 4 <= sms) {
      G = (int)std::lround(std::sqrt((double)nC));
      const long long per_seg = (long long)((Dv + Dk) / 16 + 1) / 2 * B * H * (bidir ? 2 : 1);
      G = (int)std::min<long long>(G, std::max<long long>(2, 2LL * sms / std::max<long long>(per_seg, 1)));
    }
  }
  G = std::max(1, std::min(G, nC / 2));
  const int seg_len = (nC + G - 1) / G;
  return (nC + seg_len - 1) / seg_len;  // no empty segment
}

bool make_tile_map(CUtensorMap* m, const void* base, int nb, int T, int H, int D, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[5] = {8, (cuuint64_t)T, (cuuint64_t)(D / 8), (cuuint64_t)H, (cuuint64_t)nb};
  const cuuint64_t strides[4] = {(cuuint64_t)H * D * 2, 16, (cuuint64_t)D * 2,
                                 (cuuint64_t)T * H * D * 2};
  const cuuint32_t box[5] = {8, (cuuint32_t)box_rows, (cuuint32_t)(D / 8), 1, 1};
  const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int num_sms() {
  constexpr int kMaxDev = 64;
  static int cached[kMaxDev] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return 148;
  if (!cached[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cached[dev] = n;
  }
  return cached[dev];
}

WsLayout chunk_tc_ws_layout(int Dk, int Dv) {
  Workspace w;
  w.layout(Dk, Dv);
  WsLayout L;
  L.block_bytes = w.block_bytes;
  L.off_w = w.off_w;
  L.off_kt = w.off_kt;
  L.off_decay = w.off_decay;
  L.off_g = w.off_g;
  L.off_ut = w.off_ut;
  L.off_u = w.off_u;
  L.off_s = w.off_s;
  return L;
}

size_t chunk_tc_workspace_bytes(int B, int T, int H, int Dk, int Dv, bool bidir) {
  const int ndir = bidir ? 2 : 1;
  const size_t tiles = (size_t)ndir * B * H * ((T + kC - 1) / kC);
  Workspace ws;
  ws.layout(Dk, Dv);
  size_t bytes = tiles * ws.block_bytes;
  const int G = time_segments(B, T, H, Dk, Dv, bidir);
  if (G > 1)  // segment maps [dir][seg][b*h][Dk][Dv + Dk] and start states [..][Dk][Dv]
    bytes += (size_t)ndir * G * B * H * Dk * ((Dv + Dk) + Dv) * sizeof(float);
  return bytes;
}

cudaError_t launch_chunk_tc(const ScanArgs& a, void* workspace) {
  cudaError_t e = set_smem_attrs();
  if (e != cudaSuccess) return e;
  const int ndir = a.bidir ? 2 : 1;
  const int nC = (a.T + kC - 1) / kC;
  const int NBH = a.B * a.H;
  Workspace ws;
  ws.base = static_cast<uint8_t*>(workspace);
  ws.tinv = static_cast<uint8_t*>(a.t_out);
  ws.layout(a.Dk, a.Dv);
  ws.NBH = NBH;
  ws.nC = nC;

  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, a.q, a.B, a.T, a.H, a.Dk) || !make_map(&mk, a.k, a.B, a.T, a.H, a.Dk) ||
      !make_map(&mv, a.v, a.B, a.T, a.H, a.Dv))
    return cudaErrorInvalidValue;

  {
    ProfileScope ps(a.stream, kKernPrep);
    e = launch_pdl(gdn_prep_kernel, dim3(nC, NBH, ndir), kWideThreads, sizeof(PrepSmem), a.stream,
                   mk, mv, a.g, a.beta, a.gate_logits ? 1 : 0, ws, a.T, a.H, a.wait_limit, a.err);
  }
  if (e != cudaSuccess) return e;
  unsigned launches = 3;
  const int nsl = a.Dv / 16, nkb = a.Dk / 16;
  const int G = time_segments(a.B, a.T, a.H, a.Dk, a.Dv, a.bidir);
  auto chain = [&](const ChainArgs& A, int slices, int groups_z) {
    ProfileScope ps(a.stream, kKernRecur);
    const ChainShape cs = chain_shape(a.Dk, 16 * slices, NBH * groups_z, num_sms());
    return launch_pdl(recur_kernel(nkb, A.publish == 0), dim3((slices + cs.ns - 1) / cs.ns, NBH, groups_z),
                      32 * (cs.ns * chain_group_warps(nkb) + 1), ChainLayout(a.Dk, cs.ns, cs.nst).total,
                      a.stream, A, ws, cs.ns, cs.nst, a.wait_limit, a.err);
  };
  ChainArgs A = {};
  A.fin_last_seg_only = 1;
  A.publish = 1;
  if (G <= 1) {  // one walk over the whole chunk sequence
    A.init = a.state_in;
    A.fin = a.state_out;
    A.fin_ld = a.Dv;
    A.nseg = 1;
    A.seg_len = nC;
    e = chain(A, nsl, ndir);
  } else {  // time-segmented: segment maps, their prefix, then every segment
    const int seg_len = (nC + G - 1) / G;
    const size_t ld = (size_t)a.Dv + a.Dk;
    float* maps = reinterpret_cast<float*>(ws.base + (size_t)ndir * NBH * nC * ws.block_bytes);
    float* seg_state = maps + (size_t)ndir * G * NBH * a.Dk * ld;
    ChainArgs S1 = {};
    S1.fin = maps;
    S1.fin_seg_stride = (size_t)NBH * a.Dk * ld;
    S1.fin_dir_stride = (size_t)G * S1.fin_seg_stride;
    S1.fin_ld = (int)ld;
    S1.nseg = G;
    S1.seg_len = seg_len;
    S1.publish = 0;
    S1.p_slices = nkb;
    e = chain(S1, nsl + nkb, ndir * G);
    if (e == cudaSuccess) {
      ProfileScope ps(a.stream, kKernSegPrefix);
      e = launch_pdl(gdn_segment_prefix_kernel, dim3(a.Dv / kPrefixCols, NBH, ndir), kPrefixThreads,
                     sizeof(PrefixSmem), a.stream, (const float*)maps, a.state_in, seg_state, a.Dk,
                     a.Dv, NBH, G);
    }
    if (e == cudaSuccess) {
      A.init = seg_state;
      A.init_seg_stride = (size_t)NBH * a.Dk * a.Dv;
      A.init_dir_stride = (size_t)G * A.init_seg_stride;
      A.fin = a.state_out;
      A.fin_ld = a.Dv;
      A.nseg = G;
      A.seg_len = seg_len;
      e = chain(A, nsl, ndir * G);
    }
    launches = 5;
  }
  if (e != cudaSuccess) return e;
  if (a.skip_output) {
    count_launches(launches - 1);
    return e;
  }
  {
    ProfileScope ps(a.stream, kKernOutput);
    e = launch_pdl(gdn_output_kernel, dim3(std::min(nC * NBH, num_sms())), kOutThreads,
                   OutLayout(a.Dk, a.Dv).total, a.stream, mq, mk,
                   static_cast<__nv_bfloat16*>(a.out), ws, a.T, a.H, ndir, a.wait_limit, a.err);
  }
  if (e == cudaSuccess) count_launches(launches);
  return e;
}

}  // namespace gdn
