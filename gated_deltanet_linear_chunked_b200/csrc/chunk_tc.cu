// chunk_tc.cu -- the chunked GDN scan on sm_100a tensor cores (bf16 I/O).
//
// The pages' fused kernel runs a three-stage chunked pipeline: stage A forms
// per-chunk summaries, stage B runs the recurrent scan over chunks, stage C
// applies the state ("SANA-Streaming：基于混合扩散Transformer的实时流式视频编辑
// 系统", 方法步骤详情, fourth step).  Here the three stages are three kernels:
//
//   stage A  gdn_prep_kernel    one CTA per (chunk, b*h, direction), parallel
//   stage B  gdn_recur_kernel   one CTA per (16 state columns, b*h, direction),
//                               a dependent walk over the chunks
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
//         = e^{gamma_C} S0 - Qc S0 + Rc,  Qc = K~^T W,  Rc = K~^T U~
//   O     = diag(e^gamma) Q^ S0 + (Mask o Q^ K^^T) U,
//           Mask_ri = e^{gamma_r - gamma_i} for i at or before r, else 0.
// Stage A computes Tm, W, U~, Qc, Rc (d x d summaries of the chunk); stage B
// runs S <- e^{gamma_C} S - Qc S + Rc (per 16-column slice, a d x d times
// d x 16 product on mma.sync per chunk) and publishes the state at each chunk
// start; stage C computes U and O.
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
#include <mutex>
#include <utility>

#include "gdn_internal.h"
#include "sm100.cuh"

namespace gdn {
namespace {

using namespace sm100;

constexpr int kC = 64;            // tokens per chunk
constexpr int kWideThreads = 256; // stage A: two warps per TMEM lane quadrant
constexpr int kOutThreads = 512;  // stage C: four warps per TMEM lane quadrant
constexpr int kSlab64 = kC * 16;  // bytes of one 8-column slab of a 64-row tile
constexpr int kRecStages = 4;  // deepest stage-B load ring (see recur_stages)
constexpr long long kDrainPolls = 1LL << 40;  // drains are bounded by the 2 s timer

// ----------------------------------------------------------------- workspace
// One contiguous block per (direction, b*h, chunk), in the order the stages
// read them so that each read is a single bulk copy:
//   Qc    [Dk/8][Dk][8]   bf16  chunk summary K~^T W          (stage B)
//   decay {e^{gamma_C}, 0, 0, 0} fp32                        (stage B)
//   Rc    [Dv/16][Dk][16] bf16  chunk summary K~^T U~ by slice (stage B)
//   W     [Dk/8][64][8]   bf16                                (stage C)
//   Ut    [Dv/8][64][8]   bf16  U~                            (stage C)
//   S     [Dv/8][Dk][8]   bf16  state at the chunk's start    (stage C)
struct Workspace {
  uint8_t* base;
  size_t block_bytes;
  uint32_t off_decay, off_rc, off_w, off_ut, off_s;
  int NBH, nC, Dk, Dv;

  __host__ __device__ void layout(int dk, int dv) {
    Dk = dk;
    Dv = dv;
    off_decay = (uint32_t)Dk * Dk * 2;
    off_rc = off_decay + 16;
    off_w = off_rc + (uint32_t)Dk * Dv * 2;
    off_ut = off_w + 64u * Dk * 2;
    off_s = off_ut + 64u * Dv * 2;
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
// scratch and the bf16 A operands TW/TU are dead once W and U~ are in TMEM,
// so the scaled B operands Wp/Up reuse their space.  ~102 KB: two CTAs/SM.
constexpr int kLd = 68;  // fp32 row stride of the 64 x 64 scratch (16 B aligned rows)
struct PrepSmem {
  alignas(128) uint8_t K[16 * kSlab64];   // [16 slabs][64][8]; slabs >= Dk/8 zero
  alignas(128) uint8_t V[16 * kSlab64];
  union alignas(128) U {
    struct {
      uint8_t TW[8 * kSlab64];             // Tm diag(beta e^g / |k|), K-major A
      uint8_t TU[8 * kSlab64];             // Tm diag(beta), K-major A
      float A[64][kLd];                    // strictly lower A in scan order
      float T[64][kLd];                    // (I + A)^-1 in scan order
      float Y[64][kLd];                    // product scratch
    } a;
    struct {
      uint8_t Wp[16 * kSlab64];            // diag(e^{gC-g}/|k|) W, MN-major B
      uint8_t Up[16 * kSlab64];            // diag(e^{gC-g}/|k|) U~, MN-major B
    } b;
  } u;
  float g[64], beta[64], gam[64], rn[64], csW[64], csU[64];
  float arow[64];      // beta_r |k_r|^-1 e^{gam_r - m_b(r)}       (scan order)
  float bcol[8][64];   // |k_q|^-1 e^{m_b - gam_q}, b = 8-row block (scan order)
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
  float (*A)[kLd] = u.a.A;
  float (*T)[kLd] = u.a.T;
  float (*Y)[kLd] = u.a.Y;
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
                          const float* __restrict__ g, const float* __restrict__ beta,
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
      gv = __ldg(g + row);
      bv = __ldg(beta + row);
    }
    s.g[tid] = gv;
    s.beta[tid] = bv;
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
  // q < p, formed as arow[p] G bcol[b(p)][q]: the gate factor is split at
  // m_b = gam at the first scan position of p's 8-row block b, so both factors
  // are bounded (|gam_r - m_b| and, inside the block, |m_b - gam_i| span at
  // most 7 tokens) and only 8 x 64 + 64 exponentials are taken per tile.
  {
    for (int e = tid; e < 8 * 64; e += kWideThreads) {
      const int blk = e >> 6, q = e & 63;
      const int i = REV ? 63 - q : q;
      const float mb = s.gam[REV ? 63 - 8 * blk : 8 * blk];
      s.bcol[blk][q] = (q < 8 * blk + 8) ? s.rn[i] * exp2f((mb - s.gam[i]) * kLog2e) : 0.f;
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
      const float ap = s.arow[p];
      const float* bc = s.bcol[p >> 3];
      float* Arow = s.u.a.A[p];
#pragma unroll
      for (int q4 = 0; q4 < 8; ++q4) {
        const int qb = 32 * half + 4 * q4;
        const float4 b4 = *reinterpret_cast<const float4*>(bc + qb);
        const float bb[4] = {b4.x, b4.y, b4.z, b4.w};
        float o[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int q = qb + e;
          const int iv = REV ? 31 - (4 * q4 + e) : 4 * q4 + e;  // index into v
          o[e] = (q < p) ? ap * v[iv] * bb[e] : 0.f;
        }
        *reinterpret_cast<float4*>(Arow + qb) = make_float4(o[0], o[1], o[2], o[3]);
      }
    }
  }
  __syncthreads();
  unit_lower_inverse(s.u);

  // TW[r][i] = T[pos r][pos i] beta_i e^{gam_i} / |k_i|, TU[r][i] = T[..] beta_i,
  // as bf16 K-major A operands in memory order
  for (int idx = tid; idx < 64 * 8; idx += kWideThreads) {
    const int r = idx & 63, ks = idx >> 6;
    const float* Trow = s.u.a.T[scan_pos<REV>(r)];
    float w[8], uu[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int i = 8 * ks + e;
      const float t = Trow[scan_pos<REV>(i)];
      w[e] = t * s.csW[i];
      uu[e] = t * s.csU[i];
    }
    reinterpret_cast<uint4*>(s.u.a.TW + ks * kSlab64)[r] = pack8_bf16(w);
    reinterpret_cast<uint4*>(s.u.a.TU + ks * kSlab64)[r] = pack8_bf16(uu);
  }
  block_sync_async();
  if (!block_wait(&s.v_bar, 0, limit, err)) return false;
  // W = TW K (N = Dk), U~ = TU V (N = Dv); K and V read MN-major (N = feature)
  if (tid == 0) {
    const uint32_t idW = idesc_bf16(64, Dk, 0, 1), idU = idesc_bf16(64, Dv, 0, 1);
    for (int ks = 0; ks < kC / 16; ++ks) {
      const uint64_t aw = sdesc(smem_u32(s.u.a.TW) + ks * 2 * kSlab64, kSlab64, 128);
      const uint64_t au = sdesc(smem_u32(s.u.a.TU) + ks * 2 * kSlab64, kSlab64, 128);
      const uint64_t bk = sdesc(smem_u32(s.K) + ks * 256, 128, kSlab64);
      const uint64_t bv = sdesc(smem_u32(s.V) + ks * 256, 128, kSlab64);
      mma_bf16(tm, aw, bk, idW, ks > 0);
      mma_bf16(tm + 128, au, bv, idU, ks > 0);
    }
    mma_commit(&s.mma_bar);
  }
  if (!block_wait(&s.mma_bar, 1, limit, err)) return false;
  tc_fence_after_sync();

  // W, U~ -> workspace (bf16 [slab][64][8]); scaled copies -> Wp, Up.
  // Warps w and w + 4 share a TMEM lane quadrant and split the column blocks.
  {
    const int quad = warp & 3, half = warp >> 2;
    const int r = 16 * quad + (lane & 15);
    const uint32_t lane_base = static_cast<uint32_t>(32 * quad) << 16;
    const size_t tile = ws.tile(dir, bh, j);
    const float sc = expf(gamC - s.gam[r]) * s.rn[r];
    // column block cb: W's blocks [0, Dk/16) at TMEM column 16 cb, then
    // U~'s at 128 + 16 (cb - Dk/16); two TMEM loads in flight per wait
    const int nkb = Dk / 16, nb = nkb + Dv / 16;
    auto col = [&](int cb) { return cb < nkb ? 16u * cb : 128u + 16u * (cb - nkb); };
    auto put = [&](int cb, const float* v) {
      const bool isw = cb < nkb;
      const int c = isw ? cb : cb - nkb;
      uint4* G = reinterpret_cast<uint4*>(ws.blk(tile) + (isw ? ws.off_w : ws.off_ut));
      uint8_t* Sp = isw ? s.u.b.Wp : s.u.b.Up;
      float sv[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) sv[e] = v[e] * sc;
      G[(2 * c) * kC + r] = pack8_bf16(v);
      G[(2 * c + 1) * kC + r] = pack8_bf16(v + 8);
      reinterpret_cast<uint4*>(Sp + (2 * c) * kSlab64)[r] = pack8_bf16(sv);
      reinterpret_cast<uint4*>(Sp + (2 * c + 1) * kSlab64)[r] = pack8_bf16(sv + 8);
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
  block_sync_async();
  const size_t tile = ws.tile(dir, bh, j);
  // Qc = K^T Wp (M = 128 >= Dk, N = Dk), Rc = K^T Up (N = Dv); K read MN-major
  // as A (M = feature; slabs >= Dk/8 are zero rows)
  if (tid == 0) {
    const uint32_t idQ = idesc_bf16(128, Dk, 1, 1), idR = idesc_bf16(128, Dv, 1, 1);
    for (int ks = 0; ks < kC / 16; ++ks) {
      const uint64_t a = sdesc(smem_u32(s.K) + ks * 256, 128, kSlab64);
      const uint64_t bw = sdesc(smem_u32(s.u.b.Wp) + ks * 256, 128, kSlab64);
      const uint64_t bu = sdesc(smem_u32(s.u.b.Up) + ks * 256, 128, kSlab64);
      mma_bf16(tm, a, bw, idQ, ks > 0);
      mma_bf16(tm + 128, a, bu, idR, ks > 0);
    }
    mma_commit(&s.mma_bar);
  }
  if (!block_wait(&s.mma_bar, 0, limit, err)) return false;
  tc_fence_after_sync();
  {
    const int quad = warp & 3, half = warp >> 2;
    const int r = 32 * quad + lane;  // TMEM lane = feature row of Qc / Rc
    const uint32_t lane_base = static_cast<uint32_t>(32 * quad) << 16;
    // Qc | decay | Rc staged in the workspace block's own layout
    uint4* Qg = reinterpret_cast<uint4*>(ws.blk(tile));
    uint4* Rg = reinterpret_cast<uint4*>(ws.blk(tile) + ws.off_rc);
    // column block cb: Qc's [0, Dk/16) at 16 cb, Rc's at 128 + 16 (cb - Dk/16)
    const int nkb = Dk / 16, nb = nkb + Dv / 16;
    auto col = [&](int cb) { return cb < nkb ? 16u * cb : 128u + 16u * (cb - nkb); };
    auto put = [&](int cb, const float* v) {
      if (cb < nkb) {
        Qg[(2 * cb) * Dk + r] = pack8_bf16(v);
        Qg[(2 * cb + 1) * Dk + r] = pack8_bf16(v + 8);
      } else {
        const int c = cb - nkb;
        Rg[(c * Dk + r) * 2] = pack8_bf16(v);
        Rg[(c * Dk + r) * 2 + 1] = pack8_bf16(v + 8);
      }
    };
    for (int cb = half; cb < nb; cb += 4) {
      float v0[16], v1[16];
      const bool two = cb + 2 < nb;
      tmem_ld16(tm + lane_base + col(cb), v0);
      if (two) tmem_ld16(tm + lane_base + col(cb + 2), v1);
      tmem_wait_ld();
      if (r < Dk) {
        put(cb, v0);
        if (two) put(cb + 2, v1);
      }
    }
    if (tid == 0)
      *reinterpret_cast<float4*>(ws.blk(tile) + ws.off_decay) = make_float4(expf(gamC), 0.f, 0.f, 0.f);
  }
  return true;
}

__global__ void __launch_bounds__(kWideThreads, 2)
gdn_prep_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                const float* __restrict__ g, const float* __restrict__ beta, Workspace ws, int T,
                int H, long long limit, unsigned* err) {
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
  {  // zero the feature slabs past Dk (rows of the M = 128 products)
    uint4* z = reinterpret_cast<uint4*>(s.K + (ws.Dk / 8) * kSlab64);
    for (int i = tid; i < (16 - ws.Dk / 8) * kSlab64 / 16; i += kWideThreads) z[i] = make_uint4(0, 0, 0, 0);
  }
  block_sync_async();
  // Programmatic dependent launch: everything above overlaps the previous
  // kernel in the stream; nothing in global memory is touched before this.
  pdl_wait();
  pdl_trigger();
  if (blockIdx.z == 0)
    prep_body<0>(s, &tm_k, &tm_v, g, beta, ws, T, H, limit, err);
  else
    prep_body<1>(s, &tm_k, &tm_v, g, beta, ws, T, H, limit, err);
  tc_fence_before_sync();
  __syncthreads();
  if ((tid >> 5) == 0) tmem_dealloc(s.tmem, 256);
}

// ======================================================= stage B: recurrence
// One CTA per (16 state columns, b*h, direction), Dk/16 warps; warp w owns
// state rows [16w, 16w + 16).  Per chunk the product Qc S (Dk x Dk times
// Dk x 16) is a dependent chain across chunks and is latency-bound: a
// tcgen05 round trip (issue 7 MMAs, commit, mbarrier, TMEM load) costs about
// 1.2k cycles for a 16-column slice and over 3k for a whole head, so this
// stage uses warp-level mma.sync.m16n8k16 (bf16 in, fp32 accumulate) with
// the fp32 state held in the accumulator registers and the bf16 copy of S
// exchanged through a double-buffered shared-memory operand: one barrier per
// chunk.  An NST-stage ring of bulk loads feeds [Qc | decay | Rc slice].
// Dynamic layout: [head 128 B] [S operand x 2: [2 n-slabs][Dk][8] bf16]
//                 [NST stages: Qc [Dk/8][Dk][8] | decay 16 B | Rc slice [Dk][16]]
struct RecSmemHead {
  uint64_t full[kRecStages];
};
constexpr int kRecHeadBytes = 128;
constexpr int kRecSBytes = 2 * 128 * 16;  // one S operand buffer at Dk = 128

__device__ __forceinline__ void ldmatrix_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
// D += A B, m16n8k16, bf16 inputs, fp32 accumulators.
__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                          uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// NKS = Dk / 16 and NST = stages of the load ring, compile-time constants so
// that the per-chunk code is straight-line.
template <int NKS, int NST>
__device__ bool recur_body(uint8_t* smem, const float* state_in, float* state_out,
                           const Workspace& ws, long long limit, unsigned* err) {
  constexpr int nst = NST;
  RecSmemHead& hd = *reinterpret_cast<RecSmemHead*>(smem);
  const int Dk = ws.Dk, Dv = ws.Dv, nC = ws.nC;
  uint8_t* Sop0 = smem + kRecHeadBytes;
  const uint32_t nslab_bytes = (uint32_t)Dk * 16;  // one n-slab [Dk][8] bf16 of the operand
  uint8_t* stage0 = Sop0 + 2 * kRecSBytes;
  const uint32_t qbytes = (uint32_t)Dk * Dk * 2, rbytes = (uint32_t)Dk * 32;
  const uint32_t stage_bytes = (qbytes + rbytes + 16 + 127) & ~127u;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int slice = blockIdx.x, bh = blockIdx.y, dir = blockIdx.z;
  // accumulator coordinates of this thread: rows rA, rA + 8; columns cA, cA + 1 (+ 8 nt)
  const int rA = 16 * warp + (lane >> 2), cA = 2 * (lane & 3);

  float S[2][4];  // [n-tile][c0..c3], fp32 state
#pragma unroll
  for (int nt = 0; nt < 2; ++nt)
#pragma unroll
    for (int i = 0; i < 4; ++i) S[nt][i] = 0.f;
  if (dir == 0 && state_in) {
    const float* base = state_in + (size_t)bh * Dk * Dv + 16 * slice;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      const float2 lo = *reinterpret_cast<const float2*>(base + (size_t)rA * Dv + 8 * nt + cA);
      const float2 hi = *reinterpret_cast<const float2*>(base + (size_t)(rA + 8) * Dv + 8 * nt + cA);
      S[nt][0] = lo.x; S[nt][1] = lo.y; S[nt][2] = hi.x; S[nt][3] = hi.y;
    }
  }
  auto issue = [&](int c) {  // one thread: load chunk c (scan order) into its stage
    const int jt = dir ? nC - 1 - c : c;
    const size_t tile = ws.tile(dir, bh, jt);
    uint8_t* st = stage0 + (c % nst) * stage_bytes;
    uint64_t* bar = &hd.full[c % nst];
    mbar_arrive_expect_tx(bar, qbytes + 16 + rbytes);
    bulk_load(st, ws.blk(tile), qbytes + 16, bar);  // Qc and decay
    bulk_load(st + qbytes + 16, ws.blk(tile) + ws.off_rc + (size_t)slice * Dk * 32, rbytes, bar);
  };
  int issued = min(nst, nC);
  if (tid == 0)
    for (int c = 0; c < issued; ++c) issue(c);

  // S (bf16) of this thread's accumulator positions -> operand buffer `buf`
  // ([n-slab][Dk rows][8]).  Its two n-slabs are exactly this slice's part of
  // the workspace copy of the chunk-start state ([Dv/8][Dk][8]), which one
  // thread then writes with a single bulk store after the next barrier.
  auto publish = [&](int buf) {
    uint8_t* Sop = Sop0 + buf * kRecSBytes;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      *reinterpret_cast<uint32_t*>(Sop + nt * nslab_bytes + rA * 16 + cA * 2) =
          pack_bf16x2(S[nt][0], S[nt][1]);
      *reinterpret_cast<uint32_t*>(Sop + nt * nslab_bytes + (rA + 8) * 16 + cA * 2) =
          pack_bf16x2(S[nt][2], S[nt][3]);
    }
  };
  const int storer = blockDim.x > 64 ? 64 : 0;
  publish(0);

  // ldmatrix row addresses (bytes in shared space) for this thread
  const int mi = lane >> 3, mr = lane & 7;
  // A: matrices (rows 0-7 | 8-15) x (k 0-7 | 8-15) of this warp's 16 rows
  const uint32_t a_off = (uint32_t)((mi >> 1) * Dk * 16 + (16 * warp + (mi & 1) * 8 + mr) * 16);
  // B (trans): matrices (k 0-7 | 8-15) x (n-slab 0 | 1)
  const uint32_t b_off = (uint32_t)((mi >> 1) * nslab_bytes + ((mi & 1) * 8 + mr) * 16);
  const uint32_t sop_u32 = smem_u32(Sop0), stage_u32 = smem_u32(stage0);

  // Software pipeline: the A fragments of Qc, the decay and the Rc slice of
  // chunk c + 1 are read into registers while chunk c's MMAs run, and
  // X = e^{gamma_C} S + Rc is formed before the product arrives, so the
  // dependent path per chunk is: barrier, B fragments, MMA, S = X - Qc S,
  // operand write.
  uint32_t af[NKS][4];
  float X[2][4];
  // wait for chunk c's stage (every thread), then read its A fragments and
  // form X from the current S
  auto prefetch = [&](int cc) -> bool {
    const int st = cc % nst;
    const bool okw = mbar_wait(&hd.full[st], (cc / nst) & 1, limit);
    const uint32_t qa = stage_u32 + st * stage_bytes + a_off;
#pragma unroll
    for (int ks = 0; ks < NKS; ++ks) ldmatrix_x4(qa + ks * 2 * Dk * 16, af[ks]);
    const uint8_t* stp = stage0 + st * stage_bytes;
    const float a = *reinterpret_cast<const float*>(stp + qbytes);
    const __nv_bfloat16* R = reinterpret_cast<const __nv_bfloat16*>(stp + qbytes + 16);
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      const __nv_bfloat162 r0 = *reinterpret_cast<const __nv_bfloat162*>(R + rA * 16 + 8 * nt + cA);
      const __nv_bfloat162 r1 = *reinterpret_cast<const __nv_bfloat162*>(R + (rA + 8) * 16 + 8 * nt + cA);
      X[nt][0] = fmaf(a, S[nt][0], __low2float(r0));
      X[nt][1] = fmaf(a, S[nt][1], __high2float(r0));
      X[nt][2] = fmaf(a, S[nt][2], __low2float(r1));
      X[nt][3] = fmaf(a, S[nt][3], __high2float(r1));
    }
    return okw;
  };

  bool ok = prefetch(0);
  int c = 0;
  for (; c < nC; ++c) {
    if (tid == storer) bulk_wait_read();  // last store done reading the buffer we reuse
    fence_proxy_async_smem();             // operand writes -> the bulk store
    if (!__syncthreads_and(ok)) break;  // S operand written, stage data visible
    if (tid == storer)
      bulk_store(ws.blk(ws.tile(dir, bh, dir ? nC - 1 - c : c)) + ws.off_s +
                     (size_t)slice * 2 * nslab_bytes,
                 Sop0 + (c & 1) * kRecSBytes, 2 * nslab_bytes);
    if (tid == 32 % blockDim.x && c >= 1 && c - 1 + nst < nC) issue(c - 1 + nst);
    if (c >= 1 && c - 1 + nst < nC) issued = c - 1 + nst + 1;
    const uint32_t sb = sop_u32 + (c & 1) * kRecSBytes + b_off;
    uint32_t bfr[NKS][4];
#pragma unroll
    for (int ks = 0; ks < NKS; ++ks) ldmatrix_x4_trans(sb + ks * 256, bfr[ks]);
    // two independent accumulator chains per n-tile (even / odd k-steps)
    float acc[2][2][4];
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[h][nt][i] = 0.f;
#pragma unroll
    for (int ks = 0; ks < NKS; ++ks) {
      mma_16816(acc[ks & 1][0], af[ks], bfr[ks][0], bfr[ks][1]);
      mma_16816(acc[ks & 1][1], af[ks], bfr[ks][2], bfr[ks][3]);
    }
    // S <- (e^{gamma_C} S + Rc) - Qc S
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int i = 0; i < 4; ++i) S[nt][i] = X[nt][i] - (acc[0][nt][i] + acc[1][nt][i]);
    if (c + 1 < nC) {
      publish((c + 1) & 1);
      ok = prefetch(c + 1);
    }
  }
  if (tid == storer) bulk_wait_all();
  if (c < nC) {  // a bounded wait expired: drain every load still in flight
    if (tid == 0) atomicOr(err, kErrTimeout);
    for (int p = c; p < issued; ++p)
      mbar_wait(&hd.full[p % nst], (p / nst) & 1, kDrainPolls);
    __syncthreads();
    return false;
  }
  if (dir == 0 && state_out) {
    float* base = state_out + (size_t)bh * Dk * Dv + 16 * slice;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      *reinterpret_cast<float2*>(base + (size_t)rA * Dv + 8 * nt + cA) = make_float2(S[nt][0], S[nt][1]);
      *reinterpret_cast<float2*>(base + (size_t)(rA + 8) * Dv + 8 * nt + cA) = make_float2(S[nt][2], S[nt][3]);
    }
  }
  return true;
}

template <int NKS, int NST>
__global__ void __launch_bounds__(256, 1)
gdn_recur_kernel(const float* state_in, float* state_out, Workspace ws, long long limit,
                 unsigned* err) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  RecSmemHead& hd = *reinterpret_cast<RecSmemHead*>(smem_raw);
  if (threadIdx.x == 0) {
    for (int i = 0; i < NST; ++i) mbar_init(&hd.full[i], 1);
    fence_mbar_init();
  }
  __syncthreads();
  pdl_wait();  // stage A's summaries are complete and visible
  pdl_trigger();
  recur_body<NKS, NST>(smem_raw, state_in, state_out, ws, limit, err);
}

// The recurrence kernel for Dk = 16 * nks with an nst-stage load ring.
using RecurKernel = void (*)(const float*, float*, Workspace, long long, unsigned*);
template <int NST>
RecurKernel recur_kernel_st(int nks) {
  switch (nks) {
    case 1: return gdn_recur_kernel<1, NST>;
    case 2: return gdn_recur_kernel<2, NST>;
    case 3: return gdn_recur_kernel<3, NST>;
    case 4: return gdn_recur_kernel<4, NST>;
    case 5: return gdn_recur_kernel<5, NST>;
    case 6: return gdn_recur_kernel<6, NST>;
    case 7: return gdn_recur_kernel<7, NST>;
    default: return gdn_recur_kernel<8, NST>;
  }
}
RecurKernel recur_kernel(int nks, int nst) {
  return nst >= 4 ? recur_kernel_st<4>(nks) : nst == 3 ? recur_kernel_st<3>(nks) : recur_kernel_st<2>(nks);
}

// ========================================================== stage C: output
// Persistent: one CTA per SM walks tiles t = blockIdx.x, + gridDim.x, ...
// with two input sets in shared memory, so the next tile's TMA / bulk loads
// land while the current tile computes.  Per set (offsets from Dk, Dv):
//   Q   [Dk/8][64][8]  raw q tile (TMA)
//   K   [Dk/8][64][8]  raw k tile (TMA); after P = Q K^T it holds Qs = diag(e^g) Q
//   W   [Dk/8][64][8]  W of the current direction     } one contiguous block,
//   Ut  [Dv/8][64][8]  U~, then U in place            } as in the workspace:
//   S   [Dv/8][Dk][8]  state at the chunk's start     } a single bulk copy
// then P [8][64][8] (masked, gated Q K^T, K-major A) and the scalar block.
struct OutSmall {
  float g[2][64];
  float gam[64], rnq[2][64], rnk[2][64], arow[64];  // norms per tile set
  float bcol[8][64];
  uint64_t tma_bar[2], ld_bar[2], mma_bar;
  uint64_t fin_bar;  // one commit on a failed wait: every MMA issued has landed
  uint32_t tmem;
};
struct OutLayout {
  uint32_t q, k, w, ut, s, set_bytes, p, small, total;
  __host__ __device__ OutLayout(int Dk, int Dv) {
    auto al = [](uint32_t x) { return (x + 127u) & ~127u; };
    q = 0;
    k = al(q + 64u * Dk * 2);
    w = al(k + 64u * Dk * 2);
    ut = w + 64u * Dk * 2;
    s = ut + 64u * Dv * 2;
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
                            const float* __restrict__ g, __nv_bfloat16* __restrict__ out,
                            const Workspace& ws, int T, int H, int ndir, long long limit,
                            unsigned* err) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int Dk = ws.Dk, Dv = ws.Dv, nC = ws.nC;
  const int ntiles = nC * ws.NBH;
  const OutLayout L(Dk, Dv);
  OutSmall& sm = *reinterpret_cast<OutSmall*>(smem + L.small);
  uint8_t* sP = smem + L.p;
  const uint32_t tm = sm.tmem;
  const uint32_t tmP = tm, tmO = tm + 64;
  const uint32_t wbytes = kC * Dk * 2, ubytes = kC * Dv * 2, sbytes = Dk * Dv * 2;
  // warps w, w + 4, w + 8, w + 12 share TMEM lane quadrant w % 4 and split
  // the column blocks four ways
  const int quad = warp & 3, part = warp >> 2;
  const int r = 16 * quad + (lane & 15);
  const uint32_t lane_base = static_cast<uint32_t>(32 * quad) << 16;

  auto issue_dir = [&](int set, int tile_t, int dir) {  // thread 0: W | U~ | S
    uint8_t* base = smem + set * L.set_bytes;
    const int bh = tile_t / nC, j = tile_t - bh * nC;
    const size_t tile = ws.tile(dir, bh, j);
    mbar_arrive_expect_tx(&sm.ld_bar[set], wbytes + ubytes + sbytes);
    bulk_load(base + L.w, ws.blk(tile) + ws.off_w, wbytes + ubytes + sbytes, &sm.ld_bar[set]);
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
    if (tid < kC) {
      if (tid < T - t0) cp_async4(&sm.g[set][tid], g + ((size_t)b * T + t0 + tid) * H + h);
      else sm.g[set][tid] = 0.f;
      cp_async_commit();
    }
  };

  // mbarrier phase parities: bit `set` of tma_ph / ld_ph
  uint32_t tma_ph = 0, ld_ph = 0, mma_ph = 0;
  // Head of the tile in `set`: wait for its q/k tile and gates, issue
  // P = Q K^T (shared by both directions), then the row norms, which overlap
  // it.  `one_more`: a later tile's gates are in flight too.  The head of
  // tile t + 1 runs while tile t's last MMA round executes.
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
  // CTA issued (P = Q K^T is issued ahead of its commit), so none is still
  // writing TMEM when the accumulators are freed.
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
    uint8_t* sW = base + L.w;
    uint8_t* sUt = base + L.ut;  // then U
    uint8_t* sS = base + L.s;
    const int bh = t / nC, j = t - bh * nC;
    const int b = bh / H, h = bh - b * H, t0 = j * kC;
    const int nvalid = min(kC, T - t0);

    for (int dir = 0; dir < ndir; ++dir) {
      // D_U: direction 0 borrows D_O's columns (D_O is first written after
      // D_U is consumed); direction 1 needs its own, [192, 320) of a
      // 512-column allocation, because D_O then holds direction 0's sum.
      const uint32_t tmU = tm + (dir == 0 ? 64u : 192u);
      __syncthreads();
      if (warp == 0) warp_gamma(sm.g[set], sm.gam, dir);
      __syncthreads();
      // Gate factors split at m_b = gam at the first scan position of each
      // 8-row block (as in stage A): P'_ri = arow_r P_ri bcol[b(r)][i].
      for (int e = tid; e < 8 * 64; e += kOutThreads) {
        const int blk = e >> 6, i = e & 63;
        const int qpos = dir ? 63 - i : i;
        const float mb = sm.gam[dir ? 63 - 8 * blk : 8 * blk];
        sm.bcol[blk][i] = (qpos < 8 * blk + 8) ? sm.rnk[set][i] * exp2f((mb - sm.gam[i]) * kLog2e) : 0.f;
      }
      if (tid < 64) {
        const int p = dir ? 63 - tid : tid;
        const float mb = sm.gam[dir ? 63 - 8 * (p >> 3) : 8 * (p >> 3)];
        sm.arow[tid] = exp2f((sm.gam[tid] - mb) * kLog2e);
      }
      if (!block_wait(&sm.ld_bar[set], (ld_ph >> set) & 1, limit, err)) {
        drain_other();
        return false;
      }
      ld_ph ^= 1u << set;
      if (tid == 0) {
        tc_fence_after_sync();
        // D_U = W S  (M = 64, N = Dv, K = Dk); S read MN-major (N = value column)
        const uint32_t idU = idesc_bf16(64, Dv, 0, 1);
        for (int ks = 0; ks < Dk / 16; ++ks)
          mma_bf16(tmU, sdesc(smem_u32(sW) + ks * 2 * kSlab64, kSlab64, 128),
                   sdesc(smem_u32(sS) + ks * 256, 128, Dk * 16), idU, ks > 0);
        mma_commit(&sm.mma_bar);
      }
      if (!block_wait(&sm.mma_bar, mma_ph, limit, err)) {
        drain_other();
        return false;
      }
      mma_ph ^= 1;
      tc_fence_after_sync();
      // U = U~ - W S, in place of U~ (MN-major B: [slab][64 tokens][8]);
      // column blocks part and part + 4 of D_U and block part of P are
      // loaded from TMEM together
      {
        float u0[16], u1[16], v[16];
        const bool has1 = part + 4 < Dv / 16;
        if (part < Dv / 16) tmem_ld16(tmU + lane_base + 16 * part, u0);
        if (has1) tmem_ld16(tmU + lane_base + 16 * (part + 4), u1);
        tmem_ld16(tmP + lane_base + 16 * part, v);
        tmem_wait_ld();
        auto sub = [&](int c, const float* d) {
          float ut[16];
          unpack8_bf16(reinterpret_cast<const uint4*>(sUt + (2 * c) * kSlab64)[r], ut);
          unpack8_bf16(reinterpret_cast<const uint4*>(sUt + (2 * c + 1) * kSlab64)[r], ut + 8);
#pragma unroll
          for (int e = 0; e < 16; ++e) ut[e] -= d[e];
          reinterpret_cast<uint4*>(sUt + (2 * c) * kSlab64)[r] = pack8_bf16(ut);
          reinterpret_cast<uint4*>(sUt + (2 * c + 1) * kSlab64)[r] = pack8_bf16(ut + 8);
        };
        if (lane < 16) {
          if (part < Dv / 16) sub(part, u0);
          if (has1) sub(part + 4, u1);
        }
        // P'_ri = (q_r . k_i) / |k_i| * e^{gam_r - gam_i} for i at or before r
        const int c = part;
        if (lane < 16) {
          const float ar = sm.arow[r];
          const float* bc = sm.bcol[(dir ? 63 - r : r) >> 3];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int i = 16 * c + e;
            const bool incl = dir ? (i >= r) : (i <= r);
            v[e] = incl ? ar * v[e] * bc[i] : 0.f;
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
        const uint32_t idO = idesc_bf16(64, Dv, 0, 1);
        for (int ks = 0; ks < Dk / 16; ++ks)
          mma_bf16(tmO, sdesc(smem_u32(sK) + ks * 2 * kSlab64, kSlab64, 128),
                   sdesc(smem_u32(sS) + ks * 256, 128, Dk * 16), idO, (dir > 0) || (ks > 0));
        for (int ks = 0; ks < kC / 16; ++ks)
          mma_bf16(tmO, sdesc(smem_u32(sP) + ks * 2 * kSlab64, kSlab64, 128),
                   sdesc(smem_u32(sUt) + ks * 256, 128, kSlab64), idO, 1);
        mma_commit(&sm.mma_bar);
      }
      if (dir + 1 < ndir) {
        if (!block_wait(&sm.mma_bar, mma_ph, limit, err)) {
          drain_other();
          return false;
        }
        mma_ph ^= 1;
        if (tid == 0) issue_dir(set, t, dir + 1);
      }
    }
    // the last direction's second round is in flight: the next tile's head
    // (its loads, P = Q K^T and norms) runs meanwhile
    if (next_issued && !head(set ^ 1, false)) {
      // head drained the next tile's q/k; its W | U~ | S and this round remain
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
                  const float* __restrict__ g, __nv_bfloat16* __restrict__ out, Workspace ws, int T,
                  int H, int ndir, long long limit, unsigned* err) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  const OutLayout L(ws.Dk, ws.Dv);
  OutSmall& sm = *reinterpret_cast<OutSmall*>(smem_raw + L.small);
  const int tid = threadIdx.x;
  const uint32_t ncols = ndir > 1 ? 512u : 256u;
  if (tid == 0) {
    mbar_init(&sm.tma_bar[0], 1);
    mbar_init(&sm.tma_bar[1], 1);
    mbar_init(&sm.ld_bar[0], 1);
    mbar_init(&sm.ld_bar[1], 1);
    mbar_init(&sm.mma_bar, 1);
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
  output_body(smem_raw, &tm_q, &tm_k, g, out, ws, T, H, ndir, limit, err);
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

// A [B, T, H, D] bf16 tensor viewed as 5-D (8 features, T, D/8 feature slabs,
// H, B) so that one box (8 x 64 tokens x D/8 slabs x 1 x 1) lands in shared
// memory exactly in the [slab][token][8] core-matrix layout of a tile.
bool make_map(CUtensorMap* m, const void* base, int B, int T, int H, int D) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[5] = {8, (cuuint64_t)T, (cuuint64_t)(D / 8), (cuuint64_t)H, (cuuint64_t)B};
  const cuuint64_t strides[4] = {(cuuint64_t)H * D * 2, 16, (cuuint64_t)D * 2,
                                 (cuuint64_t)T * H * D * 2};
  const cuuint32_t box[5] = {8, (cuuint32_t)kC, (cuuint32_t)(D / 8), 1, 1};
  const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Streaming multiprocessors of the current device (persistent grids).
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

int recur_smem_bytes(int Dk, int nst) {
  const int stage = ((Dk * Dk * 2 + Dk * 32 + 16) + 127) & ~127;
  return kRecHeadBytes + 2 * kRecSBytes + nst * stage;
}

// Stages of stage B's load ring: the full kRecStages while the grid fits one
// CTA per SM; otherwise the deepest ring (at least 2) that lets two CTAs
// share an SM, so a grid of more CTAs than SMs (both directions, many heads)
// still runs in one wave instead of two chained ones.
int recur_stages(int Dk, int ctas, int sms) {
  if (ctas <= sms) return kRecStages;
  constexpr int kHalfSm = 113 * 1024;  // per-CTA share of an SM's shared memory, two CTAs
  int nst = kRecStages;
  while (nst > 2 && recur_smem_bytes(Dk, nst) > kHalfSm) --nst;
  return nst;
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
  if (e == cudaSuccess)
    for (int nks = 1; nks <= 8 && e == cudaSuccess; ++nks)
      for (int nst = 2; nst <= kRecStages && e == cudaSuccess; ++nst)
        e = cudaFuncSetAttribute(recur_kernel(nks, nst), cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 recur_smem_bytes(128, nst));
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(gdn_output_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)OutLayout(128, 128).total);
  if (e == cudaSuccess) done[dev] = true;
  return e;
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

size_t chunk_tc_workspace_bytes(int B, int T, int H, int Dk, int Dv, bool bidir) {
  const size_t tiles = (size_t)(bidir ? 2 : 1) * B * H * ((T + kC - 1) / kC);
  Workspace ws;
  ws.layout(Dk, Dv);
  return tiles * ws.block_bytes;
}

cudaError_t launch_chunk_tc(const ScanArgs& a, void* workspace) {
  cudaError_t e = set_smem_attrs();
  if (e != cudaSuccess) return e;
  const int ndir = a.bidir ? 2 : 1;
  const int nC = (a.T + kC - 1) / kC;
  const int NBH = a.B * a.H;
  Workspace ws;
  ws.base = static_cast<uint8_t*>(workspace);
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
                   mk, mv, a.g, a.beta, ws, a.T, a.H, a.wait_limit, a.err);
  }
  if (e != cudaSuccess) return e;
  {
    ProfileScope ps(a.stream, kKernRecur);
    const int nst = recur_stages(a.Dk, (a.Dv / 16) * NBH * ndir, num_sms());
    e = launch_pdl(recur_kernel(a.Dk / 16, nst), dim3(a.Dv / 16, NBH, ndir), 32 * (a.Dk / 16),
                   recur_smem_bytes(a.Dk, nst), a.stream, a.state_in, a.state_out, ws,
                   a.wait_limit, a.err);
  }
  if (e != cudaSuccess) return e;
  {
    ProfileScope ps(a.stream, kKernOutput);
    e = launch_pdl(gdn_output_kernel, dim3(std::min(nC * NBH, num_sms())), kOutThreads,
                   OutLayout(a.Dk, a.Dv).total, a.stream, mq, mk, a.g,
                   static_cast<__nv_bfloat16*>(a.out), ws, a.T, a.H, ndir, a.wait_limit, a.err);
  }
  if (e == cudaSuccess) count_launches(3);
  return e;
}

}  // namespace gdn
