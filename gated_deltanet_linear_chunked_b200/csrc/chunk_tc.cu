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
//   stage C  gdn_output_kernel  one CTA per (chunk, b*h), both directions
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
// runs S <- e^{gamma_C} S - Qc S + Rc, one 128 x 16 x d MMA per chunk, and
// publishes the state at each chunk start; stage C computes U and O.
//
// The reverse (within-chunk backward) scan of the bidirectional mode uses the
// same memory tiles visited in the opposite order, with gamma the suffix sums
// and "before" meaning "later in memory"; both directions' outputs are summed
// in one fp32 TMEM accumulator before the single bf16 store.
//
// Every contraction is a tcgen05.mma (bf16 x bf16 -> fp32 in TMEM) issued by
// one thread from SWIZZLE_NONE core-matrix shared-memory layouts; q/k/v tiles
// arrive by TMA tensor loads, workspace tiles by bulk copies.  The 64 x 64
// triangular inverse is a blocked fp32 forward substitution on CUDA cores.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <mutex>

#include "gdn_internal.h"
#include "sm100.cuh"

namespace gdn {
namespace {

using namespace sm100;

constexpr int kC = 64;            // tokens per chunk
constexpr int kThreads = 128;
constexpr int kSlab64 = kC * 16;  // bytes of one 8-column slab of a 64-row tile
constexpr int kRecStages = 4;
constexpr long long kDrainPolls = 1LL << 40;  // drains are bounded by the 2 s timer

// ----------------------------------------------------------------- workspace
struct Workspace {
  __nv_bfloat16* W;    // [dir][bh][chunk] [Dk/8][64][8]
  __nv_bfloat16* Ut;   // [dir][bh][chunk] [Dv/8][64][8]
  __nv_bfloat16* Qc;   // [dir][bh][chunk] [Dk/8][Dk][8]
  __nv_bfloat16* Rc;   // [dir][bh][chunk] [Dv/16][Dk][16]
  __nv_bfloat16* S;    // [dir][bh][chunk] [Dv/8][Dk][8]  state at chunk start
  float* decay;        // [dir][bh][chunk] {e^{gamma_C}, 0, 0, 0} (16 B per chunk)
  int NBH, nC, Dk, Dv;

  __device__ size_t tile(int dir, int bh, int j) const {
    return ((size_t)dir * NBH + bh) * nC + j;
  }
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

// 1 / max(|row|, 1e-6) for a 64-row bf16 tile in [slab][64][8] layout.
__device__ float row_rnorm(const uint8_t* tile, int r, int D) {
  float ss = 0.f;
  for (int sl = 0; sl < D / 8; ++sl) {
    float x[8];
    unpack8_bf16(reinterpret_cast<const uint4*>(tile + sl * kSlab64)[r], x);
#pragma unroll
    for (int i = 0; i < 8; ++i) ss = fmaf(x[i], x[i], ss);
  }
  return 1.0f / sqrtf(fmaxf(ss, 1e-12f));
}

// ============================================================ stage A: prep
struct PrepSmem {
  alignas(128) uint8_t K[16 * kSlab64];   // [16 slabs][64][8]; slabs >= Dk/8 zero
  alignas(128) uint8_t V[16 * kSlab64];
  alignas(128) uint8_t TW[8 * kSlab64];   // Tm diag(beta e^g / |k|), K-major A
  alignas(128) uint8_t TU[8 * kSlab64];   // Tm diag(beta), K-major A
  alignas(128) uint8_t Wp[16 * kSlab64];  // diag(e^{gC-g}/|k|) W, MN-major B
  alignas(128) uint8_t Up[16 * kSlab64];  // diag(e^{gC-g}/|k|) U~, MN-major B
  float A[64][65];                         // strictly triangular A, then scratch
  float T[64][65];                         // (I + A)^-1
  float X[3][16][17];
  float g[64], beta[64], gam[64], rn[64], csW[64], csU[64];
  uint64_t tma_bar, mma_bar;
  uint32_t tmem;
};

// Blocked inverse of the unit triangular 64 x 64 matrix I + A (A in s.A,
// strictly lower in "scan index" p = map(r)), written to s.T.  Diagonal
// 16 x 16 blocks by forward substitution (one warp per block, one lane per
// column), then the off-diagonal blocks in order of distance from the
// diagonal: T_ij = -T_ii sum_{j<=k<i} A_ik T_kj.
__device__ void unit_triangular_inverse(PrepSmem& s, int reverse) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  auto M = [reverse](int p) { return reverse ? 63 - p : p; };  // scan index -> row
  // zero T
  for (int i = tid; i < 64 * 64; i += kThreads) s.T[i >> 6][i & 63] = 0.f;
  __syncthreads();
  // diagonal blocks
  {
    const int blk = warp, j = lane & 15;
    if (lane < 16) {
      float x[16];
#pragma unroll
      for (int t = 0; t < 16; ++t) {
        float acc = (t == j) ? 1.f : 0.f;
#pragma unroll
        for (int i = 0; i < t; ++i) acc = fmaf(-s.A[M(16 * blk + t)][M(16 * blk + i)], x[i], acc);
        x[t] = (t < j) ? 0.f : acc;
      }
#pragma unroll
      for (int t = 0; t < 16; ++t) s.T[M(16 * blk + t)][M(16 * blk + j)] = x[t];
    }
  }
  __syncthreads();
  // off-diagonal blocks by distance d = 1, 2, 3
  for (int d = 1; d <= 3; ++d) {
    const int nb = 4 - d;  // blocks (j + d, j), j = 0 .. nb-1
    for (int idx = tid; idx < nb * 256; idx += kThreads) {
      const int jb = idx >> 8, e = idx & 255, r = e >> 4, c = e & 15;
      const int ib = jb + d;
      float acc = 0.f;
      for (int kb = jb; kb < ib; ++kb)
#pragma unroll
        for (int k = 0; k < 16; ++k)
          acc = fmaf(s.A[M(16 * ib + r)][M(16 * kb + k)], s.T[M(16 * kb + k)][M(16 * jb + c)], acc);
      s.X[jb][r][c] = acc;
    }
    __syncthreads();
    for (int idx = tid; idx < nb * 256; idx += kThreads) {
      const int jb = idx >> 8, e = idx & 255, r = e >> 4, c = e & 15;
      const int ib = jb + d;
      float acc = 0.f;
#pragma unroll
      for (int k = 0; k < 16; ++k) acc = fmaf(s.T[M(16 * ib + r)][M(16 * ib + k)], s.X[jb][k][c], acc);
      s.T[M(16 * ib + r)][M(16 * jb + c)] = -acc;
    }
    __syncthreads();
  }
}

__device__ bool prep_body(PrepSmem& s, const CUtensorMap* tm_k, const CUtensorMap* tm_v,
                          const float* __restrict__ g, const float* __restrict__ beta,
                          const Workspace& ws, int T, int H, long long limit, unsigned* err) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int j = blockIdx.x, bh = blockIdx.y, dir = blockIdx.z;
  const int b = bh / H, h = bh - b * H;
  const int Dk = ws.Dk, Dv = ws.Dv;
  const int t0 = j * kC;
  const int nvalid = min(kC, T - t0);
  const uint32_t tm = s.tmem;

  if (tid == 0) {
    mbar_arrive_expect_tx(&s.tma_bar, (Dk / 8 + Dv / 8) * kSlab64);
    for (int sl = 0; sl < Dk / 8; ++sl) tma_load_4d(s.K + sl * kSlab64, tm_k, &s.tma_bar, 8 * sl, h, t0, b);
    for (int sl = 0; sl < Dv / 8; ++sl) tma_load_4d(s.V + sl * kSlab64, tm_v, &s.tma_bar, 8 * sl, h, t0, b);
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
  if (warp == 0) warp_gamma(s.g, s.gam, dir);
  if (!block_wait(&s.tma_bar, 0, limit, err)) return false;

  if (tid < kC) s.rn[tid] = row_rnorm(s.K, tid, Dk);
  // G = K K^T  (M = 64 tokens, N = 64 tokens, K = Dk), raw (unnormalised) keys
  if (tid == 0) {
    tc_fence_after_sync();
    const uint32_t id = idesc_bf16(64, 64, 0, 0);
    for (int ks = 0; ks < Dk / 16; ++ks) {
      const uint64_t a = sdesc(smem_u32(s.K) + ks * 2 * kSlab64, kSlab64, 128);
      mma_bf16(tm, a, a, id, ks > 0);
    }
    mma_commit(&s.mma_bar);
  }
  __syncthreads();
  const float gamC = dir ? s.gam[0] : s.gam[63];
  if (tid < kC) {
    const float eg = expf(s.gam[tid]);
    s.csW[tid] = s.beta[tid] * eg * s.rn[tid];
    s.csU[tid] = s.beta[tid];
  }
  if (!block_wait(&s.mma_bar, 0, limit, err)) return false;
  tc_fence_after_sync();

  // A_ri = beta_r e^{gam_r - gam_i} G_ri / (|k_r| |k_i|) for i before r
  {
    const int r = 16 * warp + (lane & 15);
    const uint32_t lane_base = static_cast<uint32_t>(32 * warp) << 16;
    for (int c = 0; c < 4; ++c) {
      float v[16];
      tmem_ld16(tm + lane_base + 16 * c, v);
      tmem_wait_ld();
      if (lane < 16) {
        const float br = s.beta[r] * s.rn[r], gr = s.gam[r];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int i = 16 * c + e;
          const bool before = dir ? (i > r) : (i < r);
          s.A[r][i] = before ? br * expf(gr - s.gam[i]) * v[e] * s.rn[i] : 0.f;
        }
      }
    }
  }
  __syncthreads();
  unit_triangular_inverse(s, dir);

  // TW = Tm diag(beta e^gam / |k|), TU = Tm diag(beta) as bf16 K-major A operands
  for (int idx = tid; idx < 64 * 8; idx += kThreads) {
    const int r = idx & 63, ks = idx >> 6;
    float w[8], u[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float t = s.T[r][8 * ks + e];
      w[e] = t * s.csW[8 * ks + e];
      u[e] = t * s.csU[8 * ks + e];
    }
    reinterpret_cast<uint4*>(s.TW + ks * kSlab64)[r] = pack8_bf16(w);
    reinterpret_cast<uint4*>(s.TU + ks * kSlab64)[r] = pack8_bf16(u);
  }
  block_sync_async();
  // W = TW K (N = Dk), U~ = TU V (N = Dv); K and V read MN-major (N = feature)
  if (tid == 0) {
    const uint32_t idW = idesc_bf16(64, Dk, 0, 1), idU = idesc_bf16(64, Dv, 0, 1);
    for (int ks = 0; ks < kC / 16; ++ks) {
      const uint64_t aw = sdesc(smem_u32(s.TW) + ks * 2 * kSlab64, kSlab64, 128);
      const uint64_t au = sdesc(smem_u32(s.TU) + ks * 2 * kSlab64, kSlab64, 128);
      const uint64_t bk = sdesc(smem_u32(s.K) + ks * 256, 128, kSlab64);
      const uint64_t bv = sdesc(smem_u32(s.V) + ks * 256, 128, kSlab64);
      mma_bf16(tm + 64, aw, bk, idW, ks > 0);
      mma_bf16(tm + 192, au, bv, idU, ks > 0);
    }
    mma_commit(&s.mma_bar);
  }
  if (!block_wait(&s.mma_bar, 1, limit, err)) return false;
  tc_fence_after_sync();

  // W, U~ -> workspace (bf16 [slab][64][8]); scaled copies -> Wp, Up
  {
    const int r = 16 * warp + (lane & 15);
    const uint32_t lane_base = static_cast<uint32_t>(32 * warp) << 16;
    const size_t tile = ws.tile(dir, bh, j);
    const float sc = expf(gamC - s.gam[r]) * s.rn[r];
    uint4* Wg = reinterpret_cast<uint4*>(ws.W + tile * kC * Dk);
    uint4* Ug = reinterpret_cast<uint4*>(ws.Ut + tile * kC * Dv);
    for (int c = 0; c < Dk / 16; ++c) {
      float v[16];
      tmem_ld16(tm + lane_base + 64 + 16 * c, v);
      tmem_wait_ld();
      if (lane < 16) {
        float sv[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) sv[e] = v[e] * sc;
        Wg[(2 * c) * kC + r] = pack8_bf16(v);
        Wg[(2 * c + 1) * kC + r] = pack8_bf16(v + 8);
        reinterpret_cast<uint4*>(s.Wp + (2 * c) * kSlab64)[r] = pack8_bf16(sv);
        reinterpret_cast<uint4*>(s.Wp + (2 * c + 1) * kSlab64)[r] = pack8_bf16(sv + 8);
      }
    }
    for (int c = 0; c < Dv / 16; ++c) {
      float v[16];
      tmem_ld16(tm + lane_base + 192 + 16 * c, v);
      tmem_wait_ld();
      if (lane < 16) {
        float sv[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) sv[e] = v[e] * sc;
        Ug[(2 * c) * kC + r] = pack8_bf16(v);
        Ug[(2 * c + 1) * kC + r] = pack8_bf16(v + 8);
        reinterpret_cast<uint4*>(s.Up + (2 * c) * kSlab64)[r] = pack8_bf16(sv);
        reinterpret_cast<uint4*>(s.Up + (2 * c + 1) * kSlab64)[r] = pack8_bf16(sv + 8);
      }
    }
  }
  block_sync_async();
  // Qc = K^T Wp (M = 128 >= Dk, N = Dk), Rc = K^T Up (N = Dv); K read MN-major
  // as A (M = feature; slabs >= Dk/8 are zero rows)
  if (tid == 0) {
    const uint32_t idQ = idesc_bf16(128, Dk, 1, 1), idR = idesc_bf16(128, Dv, 1, 1);
    for (int ks = 0; ks < kC / 16; ++ks) {
      const uint64_t a = sdesc(smem_u32(s.K) + ks * 256, 128, kSlab64);
      const uint64_t bw = sdesc(smem_u32(s.Wp) + ks * 256, 128, kSlab64);
      const uint64_t bu = sdesc(smem_u32(s.Up) + ks * 256, 128, kSlab64);
      mma_bf16(tm + 320, a, bw, idQ, ks > 0);
      mma_bf16(tm + 0, a, bu, idR, ks > 0);
    }
    mma_commit(&s.mma_bar);
  }
  if (!block_wait(&s.mma_bar, 0, limit, err)) return false;
  tc_fence_after_sync();
  {
    const int r = tid;  // TMEM lane = feature row of Qc / Rc
    const uint32_t lane_base = static_cast<uint32_t>(32 * warp) << 16;
    const size_t tile = ws.tile(dir, bh, j);
    uint4* Qg = reinterpret_cast<uint4*>(ws.Qc + tile * (size_t)Dk * Dk);
    uint4* Rg = reinterpret_cast<uint4*>(ws.Rc + tile * (size_t)Dk * Dv);
    for (int c = 0; c < Dk / 16; ++c) {
      float v[16];
      tmem_ld16(tm + lane_base + 320 + 16 * c, v);
      tmem_wait_ld();
      if (r < Dk) {
        Qg[(2 * c) * Dk + r] = pack8_bf16(v);
        Qg[(2 * c + 1) * Dk + r] = pack8_bf16(v + 8);
      }
    }
    for (int c = 0; c < Dv / 16; ++c) {
      float v[16];
      tmem_ld16(tm + lane_base + 16 * c, v);
      tmem_wait_ld();
      if (r < Dk) {
        Rg[(c * Dk + r) * 2] = pack8_bf16(v);
        Rg[(c * Dk + r) * 2 + 1] = pack8_bf16(v + 8);
      }
    }
    if (tid == 0)
      reinterpret_cast<float4*>(ws.decay)[tile] = make_float4(expf(gamC), 0.f, 0.f, 0.f);
  }
  return true;
}

__global__ void __launch_bounds__(kThreads, 1)
gdn_prep_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                const float* __restrict__ g, const float* __restrict__ beta, Workspace ws, int T,
                int H, long long limit, unsigned* err) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  PrepSmem& s = *reinterpret_cast<PrepSmem*>(smem_raw);
  const int tid = threadIdx.x;
  if (tid == 0) {
    mbar_init(&s.tma_bar, 1);
    mbar_init(&s.mma_bar, 1);
    fence_mbar_init();
  }
  if ((tid >> 5) == 0) {
    tmem_alloc(&s.tmem, 512);
    tmem_relinquish();
  }
  {  // zero the feature slabs past Dk (rows of the M = 128 products)
    uint4* z = reinterpret_cast<uint4*>(s.K + (ws.Dk / 8) * kSlab64);
    for (int i = tid; i < (16 - ws.Dk / 8) * kSlab64 / 16; i += kThreads) z[i] = make_uint4(0, 0, 0, 0);
  }
  block_sync_async();
  prep_body(s, &tm_k, &tm_v, g, beta, ws, T, H, limit, err);
  tc_fence_before_sync();
  __syncthreads();
  if ((tid >> 5) == 0) tmem_dealloc(s.tmem, 512);
}

// ======================================================= stage B: recurrence
struct RecSmemHead {
  uint64_t full[kRecStages];
  uint64_t mma_bar;
  uint32_t tmem;
};
// dynamic layout: [head (128 B)] [S operand 4 KB] [stages: Qc | Rc slice | decay]
// [2 KB tail pad: the M = 128 MMA reads up to 128 rows of Qc's last slab;
//  rows past Dk are don't-care rows of D but must lie in shared memory]
constexpr int kRecHeadBytes = 128;
constexpr int kRecSBytes = 2 * 128 * 16;

__device__ bool recur_body(uint8_t* smem, const float* state_in, float* state_out,
                           const Workspace& ws, long long limit, unsigned* err) {
  RecSmemHead& hd = *reinterpret_cast<RecSmemHead*>(smem);
  uint8_t* Ssm = smem + kRecHeadBytes;
  uint8_t* stage0 = Ssm + kRecSBytes;
  const int Dk = ws.Dk, Dv = ws.Dv, nC = ws.nC;
  const uint32_t qbytes = (uint32_t)Dk * Dk * 2, rbytes = (uint32_t)Dk * 32;
  const uint32_t stage_bytes = (qbytes + rbytes + 16 + 127) & ~127u;
  const int tid = threadIdx.x, warp = tid >> 5;
  const int slice = blockIdx.x, bh = blockIdx.y, dir = blockIdx.z;
  const int r = tid;
  const uint32_t tm = hd.tmem;

  float S[16];
#pragma unroll
  for (int e = 0; e < 16; ++e) S[e] = 0.f;
  if (dir == 0 && state_in && r < Dk) {
    const float4* p = reinterpret_cast<const float4*>(state_in + ((size_t)bh * Dk + r) * Dv + 16 * slice);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float4 v = p[q];
      S[4 * q] = v.x; S[4 * q + 1] = v.y; S[4 * q + 2] = v.z; S[4 * q + 3] = v.w;
    }
  }
  auto issue = [&](int c) {  // thread 0: load chunk c (scan order) into its stage
    const int jt = dir ? nC - 1 - c : c;
    const size_t tile = ws.tile(dir, bh, jt);
    uint8_t* st = stage0 + (c % kRecStages) * stage_bytes;
    mbar_arrive_expect_tx(&hd.full[c % kRecStages], qbytes + rbytes + 16);
    bulk_load(st, ws.Qc + tile * (size_t)Dk * Dk, qbytes, &hd.full[c % kRecStages]);
    bulk_load(st + qbytes, ws.Rc + tile * (size_t)Dk * Dv + (size_t)slice * Dk * 16, rbytes,
              &hd.full[c % kRecStages]);
    bulk_load(st + qbytes + rbytes, ws.decay + 4 * tile, 16, &hd.full[c % kRecStages]);
  };
  int issued = 0;
  if (tid == 0)
    for (; issued < kRecStages && issued < nC; ++issued) issue(issued);
  issued = min(kRecStages, nC);

  const uint32_t id = idesc_bf16(128, 16, 0, 1);
  const uint32_t lane_base = static_cast<uint32_t>(32 * warp) << 16;
  for (int c = 0; c < nC; ++c) {
    const int jt = dir ? nC - 1 - c : c;
    const size_t tile = ws.tile(dir, bh, jt);
    // publish S at the start of this chunk: MMA operand + workspace for stage C
    if (r < Dk) {
      const uint4 lo = pack8_bf16(S), hi = pack8_bf16(S + 8);
      reinterpret_cast<uint4*>(Ssm)[r] = lo;
      reinterpret_cast<uint4*>(Ssm + 2048)[r] = hi;
      uint4* Sg = reinterpret_cast<uint4*>(ws.S + tile * (size_t)Dk * Dv);
      Sg[(2 * slice) * Dk + r] = lo;
      Sg[(2 * slice + 1) * Dk + r] = hi;
    }
    block_sync_async();
    if (tid == 0 && c >= 1 && c - 1 + kRecStages < nC) issue(c - 1 + kRecStages);
    if (c >= 1 && c - 1 + kRecStages < nC) issued = c - 1 + kRecStages + 1;
    const int st = c % kRecStages;
    if (!block_wait(&hd.full[st], (c / kRecStages) & 1, limit, err)) {
      for (int p = c + 1; p < issued; ++p)
        mbar_wait(&hd.full[p % kRecStages], (p / kRecStages) & 1, kDrainPolls);
      return false;
    }
    const uint8_t* Qst = stage0 + st * stage_bytes;
    if (tid == 0) {
      tc_fence_after_sync();
      for (int ks = 0; ks < Dk / 16; ++ks) {
        const uint64_t a = sdesc(smem_u32(Qst) + ks * 2 * Dk * 16, Dk * 16, 128);
        const uint64_t bd = sdesc(smem_u32(Ssm) + ks * 256, 128, 2048);
        mma_bf16(tm, a, bd, id, ks > 0);
      }
      mma_commit(&hd.mma_bar);
    }
    if (!block_wait(&hd.mma_bar, c & 1, limit, err)) {
      for (int p = c + 1; p < issued; ++p)
        mbar_wait(&hd.full[p % kRecStages], (p / kRecStages) & 1, kDrainPolls);
      return false;
    }
    tc_fence_after_sync();
    float D[16];
    tmem_ld16(tm + lane_base, D);
    tmem_wait_ld();
    if (r < Dk) {
      float R[16];
      const uint4* Rs = reinterpret_cast<const uint4*>(Qst + qbytes);
      unpack8_bf16(Rs[2 * r], R);
      unpack8_bf16(Rs[2 * r + 1], R + 8);
      const float a = *reinterpret_cast<const float*>(Qst + qbytes + rbytes);
#pragma unroll
      for (int e = 0; e < 16; ++e) S[e] = fmaf(a, S[e], R[e] - D[e]);
    }
  }
  if (dir == 0 && state_out && r < Dk) {
    float4* p = reinterpret_cast<float4*>(state_out + ((size_t)bh * Dk + r) * Dv + 16 * slice);
#pragma unroll
    for (int q = 0; q < 4; ++q) p[q] = make_float4(S[4 * q], S[4 * q + 1], S[4 * q + 2], S[4 * q + 3]);
  }
  return true;
}

__global__ void __launch_bounds__(kThreads, 1)
gdn_recur_kernel(const float* state_in, float* state_out, Workspace ws, long long limit,
                 unsigned* err) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  RecSmemHead& hd = *reinterpret_cast<RecSmemHead*>(smem_raw);
  const int tid = threadIdx.x;
  if (tid == 0) {
    for (int i = 0; i < kRecStages; ++i) mbar_init(&hd.full[i], 1);
    mbar_init(&hd.mma_bar, 1);
    fence_mbar_init();
  }
  if ((tid >> 5) == 0) {
    tmem_alloc(&hd.tmem, 32);
    tmem_relinquish();
  }
  block_sync_async();
  recur_body(smem_raw, state_in, state_out, ws, limit, err);
  tc_fence_before_sync();
  __syncthreads();
  if ((tid >> 5) == 0) tmem_dealloc(hd.tmem, 32);
}

// ========================================================== stage C: output
struct OutSmem {
  alignas(128) uint8_t Q[16 * kSlab64];   // raw q tile [slab][64][8]
  alignas(128) uint8_t K[16 * kSlab64];   // raw k tile
  alignas(128) uint8_t W[16 * kSlab64];   // W of this direction
  alignas(128) uint8_t Ut[16 * kSlab64];  // U~ of this direction
  alignas(128) uint8_t S[16 * 128 * 16];  // state at chunk start [Dv/8][Dk][8]
  alignas(128) uint8_t P[8 * kSlab64];    // masked, gated Q K^T, K-major A
  alignas(128) uint8_t U[16 * kSlab64];   // U, MN-major B
  alignas(128) uint8_t Qs[16 * kSlab64];  // diag(e^gamma) Q, K-major A
  float g[64], gam[64], rnq[64], rnk[64];
  uint64_t tma_bar, ld_bar, mma_bar;
  uint32_t tmem;
};

__device__ bool output_body(OutSmem& s, const CUtensorMap* tm_q, const CUtensorMap* tm_k,
                            const float* __restrict__ g, __nv_bfloat16* __restrict__ out,
                            const Workspace& ws, int T, int H, int ndir, long long limit,
                            unsigned* err) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int j = blockIdx.x, bh = blockIdx.y;
  const int b = bh / H, h = bh - b * H;
  const int Dk = ws.Dk, Dv = ws.Dv;
  const int t0 = j * kC;
  const int nvalid = min(kC, T - t0);
  const uint32_t tm = s.tmem;
  const uint32_t tmO = tm, tmU = tm + 128, tmP = tm + 256;
  const uint32_t wbytes = kC * Dk * 2, ubytes = kC * Dv * 2, sbytes = Dk * Dv * 2;
  auto issue_dir = [&](int dir) {
    const size_t tile = ws.tile(dir, bh, j);
    mbar_arrive_expect_tx(&s.ld_bar, wbytes + ubytes + sbytes);
    bulk_load(s.W, ws.W + tile * kC * Dk, wbytes, &s.ld_bar);
    bulk_load(s.Ut, ws.Ut + tile * kC * Dv, ubytes, &s.ld_bar);
    bulk_load(s.S, ws.S + tile * (size_t)Dk * Dv, sbytes, &s.ld_bar);
  };
  if (tid == 0) {
    mbar_arrive_expect_tx(&s.tma_bar, 2 * (Dk / 8) * kSlab64);
    for (int sl = 0; sl < Dk / 8; ++sl) {
      tma_load_4d(s.Q + sl * kSlab64, tm_q, &s.tma_bar, 8 * sl, h, t0, b);
      tma_load_4d(s.K + sl * kSlab64, tm_k, &s.tma_bar, 8 * sl, h, t0, b);
    }
    issue_dir(0);
  }
  if (tid < kC) s.g[tid] = (tid < nvalid) ? __ldg(g + ((size_t)b * T + t0 + tid) * H + h) : 0.f;
  if (!block_wait(&s.tma_bar, 0, limit, err)) {
    mbar_wait(&s.ld_bar, 0, kDrainPolls);
    return false;
  }
  if (tid < kC) {
    s.rnq[tid] = row_rnorm(s.Q, tid, Dk);
    s.rnk[tid] = row_rnorm(s.K, tid, Dk);
  }
  uint32_t mma_phase = 0;
  const int r = 16 * warp + (lane & 15);
  const uint32_t lane_base = static_cast<uint32_t>(32 * warp) << 16;
  for (int dir = 0; dir < ndir; ++dir) {
    __syncthreads();
    if (warp == 0) warp_gamma(s.g, s.gam, dir);
    if (!block_wait(&s.ld_bar, dir & 1, limit, err)) return false;
    if (tid == 0) {
      tc_fence_after_sync();
      if (dir == 0) {  // P = Q K^T, shared by both directions
        const uint32_t idP = idesc_bf16(64, 64, 0, 0);
        for (int ks = 0; ks < Dk / 16; ++ks)
          mma_bf16(tmP, sdesc(smem_u32(s.Q) + ks * 2 * kSlab64, kSlab64, 128),
                   sdesc(smem_u32(s.K) + ks * 2 * kSlab64, kSlab64, 128), idP, ks > 0);
      }
      // D_U = W S  (M = 64, N = Dv, K = Dk); S read MN-major (N = value column)
      const uint32_t idU = idesc_bf16(64, Dv, 0, 1);
      for (int ks = 0; ks < Dk / 16; ++ks)
        mma_bf16(tmU, sdesc(smem_u32(s.W) + ks * 2 * kSlab64, kSlab64, 128),
                 sdesc(smem_u32(s.S) + ks * 256, 128, Dk * 16), idU, ks > 0);
      mma_commit(&s.mma_bar);
    }
    if (!block_wait(&s.mma_bar, mma_phase & 1, limit, err)) return false;
    ++mma_phase;
    tc_fence_after_sync();
    // U = U~ - W S  -> s.U (MN-major B: [slab][64 tokens][8])
    for (int c = 0; c < Dv / 16; ++c) {
      float v[16];
      tmem_ld16(tmU + lane_base + 16 * c, v);
      tmem_wait_ld();
      if (lane < 16) {
        float ut[16];
        unpack8_bf16(reinterpret_cast<const uint4*>(s.Ut + (2 * c) * kSlab64)[r], ut);
        unpack8_bf16(reinterpret_cast<const uint4*>(s.Ut + (2 * c + 1) * kSlab64)[r], ut + 8);
#pragma unroll
        for (int e = 0; e < 16; ++e) ut[e] -= v[e];
        reinterpret_cast<uint4*>(s.U + (2 * c) * kSlab64)[r] = pack8_bf16(ut);
        reinterpret_cast<uint4*>(s.U + (2 * c + 1) * kSlab64)[r] = pack8_bf16(ut + 8);
      }
    }
    // P'_ri = (q_r . k_i) / |k_i| * e^{gam_r - gam_i} for i at or before r
    for (int c = 0; c < 4; ++c) {
      float v[16];
      tmem_ld16(tmP + lane_base + 16 * c, v);
      tmem_wait_ld();
      if (lane < 16) {
        const float gr = s.gam[r];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int i = 16 * c + e;
          const bool incl = dir ? (i >= r) : (i <= r);
          v[e] = incl ? v[e] * s.rnk[i] * expf(gr - s.gam[i]) : 0.f;
        }
        reinterpret_cast<uint4*>(s.P + (2 * c) * kSlab64)[r] = pack8_bf16(v);
        reinterpret_cast<uint4*>(s.P + (2 * c + 1) * kSlab64)[r] = pack8_bf16(v + 8);
      }
    }
    // Qs = diag(e^gam) Q
    if (lane < 16) {
      const float eg = expf(s.gam[r]);
      for (int sl = 0; sl < Dk / 8; ++sl) {
        float x[8];
        unpack8_bf16(reinterpret_cast<const uint4*>(s.Q + sl * kSlab64)[r], x);
#pragma unroll
        for (int e = 0; e < 8; ++e) x[e] *= eg;
        reinterpret_cast<uint4*>(s.Qs + sl * kSlab64)[r] = pack8_bf16(x);
      }
    }
    block_sync_async();
    if (tid == 0) {
      const uint32_t idO = idesc_bf16(64, Dv, 0, 1);
      for (int ks = 0; ks < Dk / 16; ++ks)
        mma_bf16(tmO, sdesc(smem_u32(s.Qs) + ks * 2 * kSlab64, kSlab64, 128),
                 sdesc(smem_u32(s.S) + ks * 256, 128, Dk * 16), idO, (dir > 0) || (ks > 0));
      for (int ks = 0; ks < kC / 16; ++ks)
        mma_bf16(tmO, sdesc(smem_u32(s.P) + ks * 2 * kSlab64, kSlab64, 128),
                 sdesc(smem_u32(s.U) + ks * 256, 128, kSlab64), idO, 1);
      mma_commit(&s.mma_bar);
    }
    if (!block_wait(&s.mma_bar, mma_phase & 1, limit, err)) return false;
    ++mma_phase;
    if (dir + 1 < ndir && tid == 0) issue_dir(dir + 1);
  }
  tc_fence_after_sync();
  // O = diag(1/|q|) D_O -> out (rows of this chunk that exist)
  {
    const float rq = s.rnq[r];
    for (int c = 0; c < Dv / 16; ++c) {
      float v[16];
      tmem_ld16(tmO + lane_base + 16 * c, v);
      tmem_wait_ld();
      if (lane < 16 && r < nvalid) {
#pragma unroll
        for (int e = 0; e < 16; ++e) v[e] *= rq;
        uint4* o = reinterpret_cast<uint4*>(out + (((size_t)b * T + t0 + r) * H + h) * Dv + 16 * c);
        o[0] = pack8_bf16(v);
        o[1] = pack8_bf16(v + 8);
      }
    }
  }
  return true;
}

__global__ void __launch_bounds__(kThreads, 1)
gdn_output_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const float* __restrict__ g, __nv_bfloat16* __restrict__ out, Workspace ws, int T,
                  int H, int ndir, long long limit, unsigned* err) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  OutSmem& s = *reinterpret_cast<OutSmem*>(smem_raw);
  const int tid = threadIdx.x;
  if (tid == 0) {
    mbar_init(&s.tma_bar, 1);
    mbar_init(&s.ld_bar, 1);
    mbar_init(&s.mma_bar, 1);
    fence_mbar_init();
  }
  if ((tid >> 5) == 0) {
    tmem_alloc(&s.tmem, 512);
    tmem_relinquish();
  }
  block_sync_async();
  output_body(s, &tm_q, &tm_k, g, out, ws, T, H, ndir, limit, err);
  tc_fence_before_sync();
  __syncthreads();
  if ((tid >> 5) == 0) tmem_dealloc(s.tmem, 512);
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

// [B, T, H, D] bf16 tensor; box = 8 features x 1 head x 64 tokens x 1 batch.
bool make_map(CUtensorMap* m, const void* base, int B, int T, int H, int D) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
  const cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2, (cuuint64_t)T * H * D * 2};
  const cuuint32_t box[4] = {8, 1, (cuuint32_t)kC, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

int recur_smem_bytes(int Dk) {
  const int stage = ((Dk * Dk * 2 + Dk * 32 + 16) + 127) & ~127;
  return kRecHeadBytes + kRecSBytes + kRecStages * stage + 2048;
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
    e = cudaFuncSetAttribute(gdn_recur_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             recur_smem_bytes(128));
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(gdn_output_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)sizeof(OutSmem));
  if (e == cudaSuccess) done[dev] = true;
  return e;
}

}  // namespace

size_t chunk_tc_workspace_bytes(int B, int T, int H, int Dk, int Dv, bool bidir) {
  const size_t tiles = (size_t)(bidir ? 2 : 1) * B * H * ((T + kC - 1) / kC);
  return align256(tiles * kC * Dk * 2) + align256(tiles * kC * Dv * 2) +
         align256(tiles * (size_t)Dk * Dk * 2) + align256(tiles * (size_t)Dk * Dv * 2) +
         align256(tiles * (size_t)Dk * Dv * 2) + align256(tiles * 16);
}

cudaError_t launch_chunk_tc(const ScanArgs& a, void* workspace) {
  cudaError_t e = set_smem_attrs();
  if (e != cudaSuccess) return e;
  const int ndir = a.bidir ? 2 : 1;
  const int nC = (a.T + kC - 1) / kC;
  const int NBH = a.B * a.H;
  const size_t tiles = (size_t)ndir * NBH * nC;
  Workspace ws;
  uint8_t* p = static_cast<uint8_t*>(workspace);
  ws.W = reinterpret_cast<__nv_bfloat16*>(p);  p += align256(tiles * kC * a.Dk * 2);
  ws.Ut = reinterpret_cast<__nv_bfloat16*>(p); p += align256(tiles * kC * a.Dv * 2);
  ws.Qc = reinterpret_cast<__nv_bfloat16*>(p); p += align256(tiles * (size_t)a.Dk * a.Dk * 2);
  ws.Rc = reinterpret_cast<__nv_bfloat16*>(p); p += align256(tiles * (size_t)a.Dk * a.Dv * 2);
  ws.S = reinterpret_cast<__nv_bfloat16*>(p);  p += align256(tiles * (size_t)a.Dk * a.Dv * 2);
  ws.decay = reinterpret_cast<float*>(p);
  ws.NBH = NBH; ws.nC = nC; ws.Dk = a.Dk; ws.Dv = a.Dv;

  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, a.q, a.B, a.T, a.H, a.Dk) || !make_map(&mk, a.k, a.B, a.T, a.H, a.Dk) ||
      !make_map(&mv, a.v, a.B, a.T, a.H, a.Dv))
    return cudaErrorInvalidValue;

  {
    ProfileScope ps(a.stream, kKernPrep);
    gdn_prep_kernel<<<dim3(nC, NBH, ndir), kThreads, sizeof(PrepSmem), a.stream>>>(
        mk, mv, a.g, a.beta, ws, a.T, a.H, a.wait_limit, a.err);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  {
    ProfileScope ps(a.stream, kKernRecur);
    gdn_recur_kernel<<<dim3(a.Dv / 16, NBH, ndir), kThreads, recur_smem_bytes(a.Dk), a.stream>>>(
        a.state_in, a.state_out, ws, a.wait_limit, a.err);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  {
    ProfileScope ps(a.stream, kKernOutput);
    gdn_output_kernel<<<dim3(nC, NBH), kThreads, sizeof(OutSmem), a.stream>>>(
        mq, mk, a.g, static_cast<__nv_bfloat16*>(a.out), ws, a.T, a.H, ndir, a.wait_limit, a.err);
  }
  e = cudaGetLastError();
  if (e == cudaSuccess) count_launches(3);
  return e;
}

}  // namespace gdn
