// sink_window_attn.cu -- the hybrid DiT's softmax blocks: one streaming
// chunk's queries attend to a persistent sink and a sliding window of chunks
// ("SANA-Streaming：基于混合扩散Transformer的实时流式视频编辑系统", 核心方法:
// softmax blocks among the GDN blocks, each with a sliding window plus a
// persistent sink, so that memory stays fixed).  The keys a query in chunk c
// sees are whole chunks: the stream's first n_sink chunks and the last
// `window` chunks (c included); the chunk's own keys and values are written
// into the block's KV cache during the same pass.
//
//   out = softmax(Q K^T / sqrt(D)) V   over the visible keys, per (b, h)
//
// One CTA per 128 query rows of one (b, h), two CTAs per SM.  The work is a
// dense contraction, so it runs on tcgen05 with TMEM accumulators, online
// softmax between the two products (the streaming form of softmax that keeps
// a running maximum and sum per row):
//   warp 4 (one lane)  TMA producer: the Q tile, then 64-key K and V tiles of
//                      every visible chunk through two 2-stage rings; it also
//                      stores the current chunk's K and V tiles that match
//                      this CTA's query rows into the cache slot of chunk c.
//   warp 5 (one lane)  MMA issuer: S_j = Q K_j^T (M 128, N 64) into one of two
//                      TMEM S buffers, then O += P_{j-1} V_{j-1} (M 128, N D).
//   warps 0-3          softmax, one query row per thread (its TMEM lane): row
//                      maximum, p = 2^(s log2e / sqrt(D) - m), row sum, P as
//                      bf16 to shared memory; O is rescaled in TMEM only when
//                      the running maximum grows by more than 2^8 (otherwise
//                      p may reach 2^8, which fp32 sums and bf16 P hold
//                      exactly as well); at the end O / l goes out through
//                      shared memory and one TMA store.
// Every wait is bounded; a wait that gives up sets the error word, and the
// CTA drains its copies and MMAs before it frees TMEM and leaves.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <mutex>

#include "gdn_internal.h"
#include "sm100.cuh"

namespace gdn {
namespace {

using namespace sm100;

constexpr int kQRows = 128;          // query rows per CTA = TMEM lanes
constexpr int kKRows = 64;           // keys per tile
constexpr int kStages = 2;           // K/V ring depth
constexpr int kThreads = 192;        // softmax warps 0-3, producer 4, MMA 5
constexpr uint32_t kTmemCols = 256;  // S0 [0, 64) | S1 [64, 128) | O [128, 128 + D)
constexpr float kRescaleLog2 = 8.f;  // headroom of the running maximum
constexpr long long kDrainPolls = 1LL << 40;  // drains are bounded by the 2 s timer

struct SwaParams {
  int Tc, H, D, nslot;
  int nseg, tiles_per_seg;
  int seg_slot[kSwaMaxSeg];  // cache slot of each visible chunk; -1: this chunk (the inputs)
  int append_slot;           // cache slot this chunk is written to
  float scale_log2;          // log2(e) / sqrt(D)
  long long limit;
  unsigned* err;
};

struct SwaBars {
  uint64_t q_full;
  uint64_t k_full[kStages], k_empty[kStages], v_full[kStages], v_empty[kStages];
  uint64_t s_full[2], s_free[2];
  uint64_t p_full, pv_done, drain;
  uint32_t tmem;
  int abort;
};

// Shared memory: Q [D/8][128][8] (later the output tile), the K/V ring
// (per stage K [D/8][64][8] | V [D/8][64][8]), P [8][128][8], barriers.
struct SwaLayout {
  uint32_t q, kv, kv_stage, v_off, p, bars, total;
};
__host__ __device__ inline SwaLayout swa_layout(int D) {
  SwaLayout L;
  L.q = 0;
  L.kv = kQRows * D * 2;
  L.v_off = kKRows * D * 2;
  L.kv_stage = 2 * L.v_off;
  L.p = L.kv + kStages * L.kv_stage;
  L.bars = L.p + kQRows * kKRows * 2;
  L.total = L.bars + 256;
  return L;
}
static_assert(sizeof(SwaBars) <= 256, "barrier block");

__global__ void __launch_bounds__(kThreads, 2)
gdn_sink_window_kernel(const __grid_constant__ CUtensorMap tm_q,
                       const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v,
                       const __grid_constant__ CUtensorMap tm_kc,
                       const __grid_constant__ CUtensorMap tm_vc,
                       const __grid_constant__ CUtensorMap tm_out,
                       const __grid_constant__ SwaParams P) {
  extern __shared__ __align__(128) uint8_t smem[];
  const SwaLayout L = swa_layout(P.D);
  SwaBars& bar = *reinterpret_cast<SwaBars*>(smem + L.bars);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int qt = blockIdx.x, bh = blockIdx.y, b = bh / P.H, h = bh - b * P.H;
  const int q0 = qt * kQRows, D = P.D, tps = P.tiles_per_seg;
  const int ntiles = P.nseg * tps;
  volatile int* abort_flag = &bar.abort;

  if (tid == 0) {
    mbar_init(&bar.q_full, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bar.k_full[s], 1);
      mbar_init(&bar.k_empty[s], 1);
      mbar_init(&bar.v_full[s], 1);
      mbar_init(&bar.v_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar.s_full[s], 1);
      mbar_init(&bar.s_free[s], 128);
    }
    mbar_init(&bar.p_full, 128);
    mbar_init(&bar.pv_done, 1);
    mbar_init(&bar.drain, 1);
    bar.abort = 0;
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(&bar.tmem, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tm = bar.tmem;
  auto fail = [&]() {
    *abort_flag = 1;
    atomicOr(P.err, kErrTimeout);
  };

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    // K runs one tile ahead of V: K_j is free once S_j is done, V_j only
    // once P_j V_j is, so the two rings refill independently.
    if (lane == 0) {
      uint8_t* sq = smem + L.q;
      mbar_arrive_expect_tx(&bar.q_full, kQRows * D * 2);
      tma_load_tile(sq, &tm_q, &bar.q_full, q0, h, b);
      const int cache_bs = b * P.nslot;
      // per ring (0: K, 1: V): loads issued into each stage, and the first
      // row of a tile still to be stored from the stage into the cache (-1)
      uint32_t loads[2][kStages];
      int append_row[2][kStages];
      for (int x = 0; x < 2; ++x)
        for (int st = 0; st < kStages; ++st) {
          loads[x][st] = 0;
          append_row[x][st] = -1;
        }
      auto stage_ptr = [&](int x, int st) { return smem + L.kv + st * L.kv_stage + x * L.v_off; };
      auto full = [&](int x, int st) { return x ? &bar.v_full[st] : &bar.k_full[st]; };
      auto append = [&](int x, int st) {
        // the load has landed (it was consumed, or is waited for here)
        if (!mbar_wait(full(x, st), (loads[x][st] - 1) & 1, P.limit)) {
          fail();
          return false;
        }
        tma_store_tile(x ? &tm_vc : &tm_kc, stage_ptr(x, st), append_row[x][st], h,
                       cache_bs + P.append_slot);
        bulk_commit();
        append_row[x][st] = -1;
        return true;
      };
      // tile j of ring x into its stage
      auto issue = [&](int x, int j) {
        const int st = j % kStages;
        if (j >= kStages) {
          uint64_t* empty = x ? &bar.v_empty[st] : &bar.k_empty[st];
          if (!mbar_wait(empty, (j / kStages - 1) & 1, P.limit)) {
            fail();
            return false;
          }
          if (append_row[x][st] >= 0) {
            if (!append(x, st)) return false;
            bulk_wait_read();  // the store has read the stage before it is refilled
          }
        }
        const int seg = j / tps, t = j - seg * tps, r0 = t * kKRows;
        const int slot = P.seg_slot[seg];
        mbar_arrive_expect_tx(full(x, st), kKRows * D * 2);
        if (slot < 0) {
          tma_load_tile(stage_ptr(x, st), x ? &tm_v : &tm_k, full(x, st), r0, h, b);
          if (P.append_slot >= 0 && r0 / kQRows == qt) append_row[x][st] = r0;
        } else {
          tma_load_tile(stage_ptr(x, st), x ? &tm_vc : &tm_kc, full(x, st), r0, h, cache_bs + slot);
        }
        ++loads[x][st];
        return true;
      };
      for (int j = 0; j <= ntiles; ++j) {
        if (*abort_flag) break;
        if (j < ntiles && !issue(0, j)) break;
        if (j >= 1 && !issue(1, j - 1)) break;
      }
      // stores still owed (a chunk of a few tiles), then drain every load
      for (int x = 0; x < 2; ++x)
        for (int st = 0; st < kStages; ++st)
          if (append_row[x][st] >= 0 && !*abort_flag) append(x, st);
      for (int x = 0; x < 2; ++x)
        for (int st = 0; st < kStages; ++st)
          if (loads[x][st]) mbar_wait(full(x, st), (loads[x][st] - 1) & 1, kDrainPolls);
      bulk_wait_all();
    }
  } else if (warp == 5) {
    // ----------------------------------------------------------- MMA issue
    if (lane == 0) {
      const uint32_t idS = idesc_bf16(kQRows, kKRows, 0, 0);
      const uint32_t idO = idesc_bf16(kQRows, D, 0, 1);
      const uint32_t qa = smem_u32(smem + L.q), pa = smem_u32(smem + L.p);
      constexpr uint32_t kQSlab = kQRows * 16, kKSlab = kKRows * 16;
      bool ok = mbar_wait(&bar.q_full, 0, P.limit);
      if (!ok) fail();
      tc_fence_after_sync();
      for (int j = 0; ok && j <= ntiles; ++j) {
        if (*abort_flag) break;
        if (j < ntiles) {
          const int s = j % kStages, sb = j & 1;
          if (!mbar_wait(&bar.k_full[s], (j / kStages) & 1, P.limit) ||
              (j >= 2 && !mbar_wait(&bar.s_free[sb], ((j >> 1) - 1) & 1, P.limit))) {
            fail();
            break;
          }
          tc_fence_after_sync();
          const uint32_t ka = smem_u32(smem + L.kv + s * L.kv_stage);
          // S_j = Q K_j^T: both K-major, K = D in steps of 16
          for (int ks = 0; ks < D / 16; ++ks)
            mma_bf16(tm + sb * kKRows, sdesc(qa + ks * 2 * kQSlab, kQSlab, 128),
                     sdesc(ka + ks * 2 * kKSlab, kKSlab, 128), idS, ks > 0);
          mma_commit(&bar.s_full[sb]);
          mma_commit(&bar.k_empty[s]);
        }
        if (j >= 1) {
          const int jp = j - 1, s = jp % kStages;
          if (!mbar_wait(&bar.v_full[s], (jp / kStages) & 1, P.limit) ||
              !mbar_wait(&bar.p_full, jp & 1, P.limit)) {
            fail();
            break;
          }
          tc_fence_after_sync();
          const uint32_t va = smem_u32(smem + L.kv + s * L.kv_stage + L.v_off);
          // O += P V: P K-major (K = 64 keys), V MN-major (N = D)
          for (int ks = 0; ks < kKRows / 16; ++ks)
            mma_bf16(tm + 2 * kKRows, sdesc(pa + ks * 2 * kQSlab, kQSlab, 128),
                     sdesc(va + ks * 256, 128, kKSlab), idO, (jp > 0) || (ks > 0));
          mma_commit(&bar.pv_done);
          mma_commit(&bar.v_empty[s]);
        }
      }
      // every MMA issued has completed before TMEM and shared memory go
      mma_commit(&bar.drain);
      mbar_wait(&bar.drain, 0, kDrainPolls);
    }
  } else {
    // ------------------------------------------------------------- softmax
    const int r = tid;  // query row within the tile = TMEM lane
    const uint32_t lrow = tm + ((uint32_t)(warp * 32) << 16);
    const uint32_t tO = lrow + 2 * kKRows;
    uint8_t* sp = smem + L.p;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < ntiles; ++j) {
      const int sb = j & 1;
      if (__any_sync(~0u, *abort_flag != 0)) {
        ok = false;
        break;
      }
      if (!__all_sync(~0u, mbar_wait(&bar.s_full[sb], (j >> 1) & 1, P.limit))) {
        if (lane == 0) fail();
        ok = false;
        break;
      }
      tc_fence_after_sync();
      float s[kKRows];
#pragma unroll
      for (int c = 0; c < kKRows / 16; ++c)
        tmem_ld16(lrow + sb * kKRows + 16 * c, *reinterpret_cast<float(*)[16]>(s + 16 * c));
      tmem_wait_ld();
      tc_fence_before_sync();
      mbar_arrive(&bar.s_free[sb]);

      const int t = j % tps;
      const int nvalid = min(kKRows, P.Tc - t * kKRows);
      if (nvalid < kKRows) {  // the ragged last tile of a chunk (warp-uniform)
#pragma unroll
        for (int i = 0; i < kKRows; ++i)
          if (i >= nvalid) s[i] = -INFINITY;
      }
      // row maximum and, below, row sum as eight independent chains each
      float acc[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] = fmaxf(s[e], s[e + 8]);
#pragma unroll
      for (int i = 16; i < kKRows; i += 8)
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = fmaxf(acc[e], s[i + e]);
      float mx = fmaxf(fmaxf(fmaxf(acc[0], acc[1]), fmaxf(acc[2], acc[3])),
                       fmaxf(fmaxf(acc[4], acc[5]), fmaxf(acc[6], acc[7])));
      mx *= P.scale_log2;
      float m_new = m_run, alpha = 1.f;
      bool resc = false;
      if (mx > m_run + kRescaleLog2) {
        m_new = mx;
        alpha = ex2_approx(m_run - m_new);  // 0 on the first tile
        resc = j > 0;
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] = 0.f;
#pragma unroll
      for (int i = 0; i < kKRows; ++i) {
        s[i] = ex2_approx(fmaf(s[i], P.scale_log2, -m_new));
        acc[i & 7] += s[i];
      }
      const float rs = ((acc[0] + acc[1]) + (acc[2] + acc[3])) + ((acc[4] + acc[5]) + (acc[6] + acc[7]));
      // P and O belong to the previous tile's P V until it completes
      if (j > 0) {
        if (!__all_sync(~0u, mbar_wait(&bar.pv_done, (j - 1) & 1, P.limit))) {
          if (lane == 0) fail();
          ok = false;
          break;
        }
        tc_fence_after_sync();
      }
      if (__any_sync(~0u, resc)) {
        const float a = resc ? alpha : 1.f;
        for (int c0 = 0; c0 < D; c0 += 16) {
          float o[16];
          tmem_ld16(tO + c0, o);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 16; ++e) o[e] *= a;
          tmem_st16(tO + c0, o);
        }
        tmem_wait_st();
      }
      l_run = l_run * alpha + rs;
      m_run = m_new;
#pragma unroll
      for (int sl = 0; sl < kKRows / 8; ++sl)
        reinterpret_cast<uint4*>(sp + sl * kQRows * 16)[r] = pack8_bf16(s + 8 * sl);
      fence_proxy_async_smem();
      tc_fence_before_sync();
      mbar_arrive(&bar.p_full);
    }
    if (ok && ntiles > 0 &&
        !__all_sync(~0u, mbar_wait(&bar.pv_done, (ntiles - 1) & 1, P.limit))) {
      if (lane == 0) fail();
      ok = false;
    }
    // all 128 rows agree before the tile is stored
    ok = named_barrier_and(1, 128, ok);
    if (ok) {
      tc_fence_after_sync();
      // every S MMA has completed, so the Q buffer takes the output tile
      uint8_t* so = smem + L.q;
      const float inv = 1.f / l_run;
      for (int c0 = 0; c0 < D; c0 += 16) {
        float o[16];
        tmem_ld16(tO + c0, o);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 16; ++e) o[e] *= inv;
        reinterpret_cast<uint4*>(so + (c0 / 8) * kQRows * 16)[r] = pack8_bf16(o);
        reinterpret_cast<uint4*>(so + (c0 / 8 + 1) * kQRows * 16)[r] = pack8_bf16(o + 8);
      }
      fence_proxy_async_smem();
      named_barrier(1, 128);
      if (tid == 0) {
        tma_store_tile(&tm_out, so, q0, h, b);
        bulk_commit();
        bulk_wait_all();
      }
    }
  }
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after_sync();
    tmem_dealloc(tm, kTmemCols);
  }
}

cudaError_t set_attr_once(int smem_bytes) {
  constexpr int kMaxDev = 64;
  static std::mutex mu;
  static int done[kMaxDev] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  if (dev >= 0 && dev < kMaxDev && done[dev] >= smem_bytes) return cudaSuccess;
  // the largest layout (D = 128) once, so every D after it is covered
  const int bytes = (int)swa_layout(128).total;
  e = cudaFuncSetAttribute(gdn_sink_window_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && dev >= 0 && dev < kMaxDev) done[dev] = bytes;
  (void)smem_bytes;
  return e;
}

}  // namespace

int sink_window_slot(int chunk, int n_sink, int window) {
  return chunk < n_sink ? chunk : n_sink + (chunk - n_sink) % window;
}

cudaError_t launch_sink_window(const SwaCall& c) {
  SwaParams P;
  P.Tc = c.Tc;
  P.H = c.H;
  P.D = c.D;
  P.nslot = c.n_sink + c.window;
  P.tiles_per_seg = (c.Tc + kKRows - 1) / kKRows;
  // the chunk itself first (its tiles are the ones stored into the cache),
  // then every other visible chunk in stream order
  P.nseg = 0;
  P.seg_slot[P.nseg++] = -1;
  for (int m = 0; m < c.chunk; ++m)
    if (m < c.n_sink || m > c.chunk - c.window) P.seg_slot[P.nseg++] = sink_window_slot(m, c.n_sink, c.window);
  P.append_slot = sink_window_slot(c.chunk, c.n_sink, c.window);
  P.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)c.D));
  P.limit = c.limit;
  P.err = c.err;

  CUtensorMap mq, mk, mv, mkc, mvc, mo;
  if (!make_tile_map(&mq, c.q, c.B, c.Tc, c.H, c.D, kQRows) ||
      !make_tile_map(&mk, c.k, c.B, c.Tc, c.H, c.D, kKRows) ||
      !make_tile_map(&mv, c.v, c.B, c.Tc, c.H, c.D, kKRows) ||
      !make_tile_map(&mkc, c.k_cache, c.B * P.nslot, c.Tc, c.H, c.D, kKRows) ||
      !make_tile_map(&mvc, c.v_cache, c.B * P.nslot, c.Tc, c.H, c.D, kKRows) ||
      !make_tile_map(&mo, c.out, c.B, c.Tc, c.H, c.D, kQRows))
    return cudaErrorInvalidValue;
  const SwaLayout L = swa_layout(c.D);
  cudaError_t e = set_attr_once((int)L.total);
  if (e != cudaSuccess) return e;
  const dim3 grid((c.Tc + kQRows - 1) / kQRows, c.B * c.H);
  {
    ProfileScope ps(c.stream, kKernSinkWindow);
    gdn_sink_window_kernel<<<grid, kThreads, L.total, c.stream>>>(mq, mk, mv, mkc, mvc, mo, P);
  }
  e = cudaGetLastError();
  if (e == cudaSuccess) count_launches(1);
  return e;
}

}  // namespace gdn
