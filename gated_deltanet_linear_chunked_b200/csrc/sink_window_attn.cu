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
// One CTA per 256 query rows of one (b, h): two 128-row query tiles that
// share every K and V tile loaded (halving the K/V traffic per flop), one CTA
// per SM holding all 512 TMEM columns.  The work is a dense contraction, so
// it runs on tcgen05 with TMEM accumulators, online softmax between the two
// products (the streaming form of softmax that keeps a running maximum and
// sum per row):
//   warp 8 (one lane)  TMA producer: the Q tiles, then 64-key K and V tiles of
//                      every visible chunk through two 4-stage rings; it also
//                      stores the current chunk's K and V tiles that match
//                      this CTA's query rows into the cache slot of chunk c.
//   warps 9, 10        MMA issue, one lane per query tile g: per key tile j,
//                      S_gj = Q_g K_j^T (M 128, N 64) into one of two TMEM S
//                      buffers of tile g, then O_g += P_g,j-1 V_j-1 (M 128, N D).
//                      Two issuing threads, because each bounded wait costs
//                      the issuing thread about as long as an MMA takes; the
//                      tensor pipe interleaves their MMAs.
//   warps 0-3, 4-7     softmax of query tiles 0 and 1, one row per thread (its
//                      TMEM lane): row maximum, p = 2^(s log2e / sqrt(D) - m),
//                      row sum, P as bf16 to shared memory; O is rescaled in
//                      TMEM only when the running maximum grows by more than
//                      2^8 (otherwise p may reach 2^8, which fp32 sums and bf16
//                      P hold as well as 1); at the end O / l goes out through
//                      shared memory and one TMA store per tile.
// The two warpgroups alternate on the tensor pipe: while one computes its
// softmax the MMAs of the other run.  Every wait is bounded; a wait that gives
// up sets the error word, and the CTA drains its copies and MMAs before it
// frees TMEM and leaves.
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

constexpr int kQTiles = 2;                     // 128-row query tiles per CTA
constexpr int kQRows = 128;                    // rows per query tile = TMEM lanes
constexpr int kKRows = 64;                     // keys per tile
constexpr int kStages = 4;                     // K and V ring depth
constexpr int kSoftmaxWarps = 4 * kQTiles;
constexpr int kProducerWarp = kSoftmaxWarps;
constexpr int kMmaWarp = kSoftmaxWarps + 1;    // first MMA warp: one per query tile
constexpr int kThreads = 32 * (kSoftmaxWarps + 1 + kQTiles);
constexpr uint32_t kTileCols = 256;            // per query tile: S0 [0,64) | S1 [64,128) | O [128, 128+D)
constexpr uint32_t kTmemCols = kTileCols * kQTiles;
constexpr uint32_t kMinSmem = 116 * 1024;      // more than half an SM: one CTA per SM
constexpr float kRescaleLog2 = 8.f;            // headroom of the running maximum
constexpr long long kDrainPolls = 1LL << 40;   // drains are bounded by the 2 s timer

// 2^x for a pair of x <= 2^8 on the FMA pipe, so that the special-function
// unit's ex2 is not the only source of exponentials: Cody and Waite's range
// reduction x = n + f (n = round(x) by adding and subtracting 1.5 * 2^23, f in
// [-1/2, 1/2]) with 2^f from a degree-3 polynomial whose coefficients were
// fitted here to 2^f on [-1/2, 1/2] by weighted least squares in relative
// error (Lawson's iteration); its largest relative error is 7.5e-5, far under
// the bf16 rounding of P.  2^n enters by adding n to the exponent field.
// Inputs are clamped at -125 (2^-125 stands for 0, as ex2 gives for -inf).
__device__ __forceinline__ uint64_t exp2_poly2(uint64_t x) {
  float x0, x1;
  f2_unpack(x, x0, x1);
  const uint64_t xc = f2_pack(fmaxf(x0, -125.f), fmaxf(x1, -125.f));
  const uint64_t magic = f2_pack(12582912.f, 12582912.f);
  const uint64_t t = f2_add(xc, magic);                        // n in the low bits
  const uint64_t n = f2_add(t, f2_pack(-12582912.f, -12582912.f));
  const uint64_t f = f2_fma(n, f2_pack(-1.f, -1.f), xc);       // x - n
  uint64_t p = f2_fma(f2_pack(0.0551716648f, 0.0551716648f), f,
                      f2_pack(0.2426111251f, 0.2426111251f));
  p = f2_fma(p, f, f2_pack(0.6932609677f, 0.6932609677f));
  p = f2_fma(p, f, f2_pack(0.9999280572f, 0.9999280572f));
  float p0, p1, t0, t1;
  f2_unpack(p, p0, p1);
  f2_unpack(t, t0, t1);
  return f2_pack(__uint_as_float(__float_as_uint(p0) + (__float_as_uint(t0) << 23)),
                 __uint_as_float(__float_as_uint(p1) + (__float_as_uint(t1) << 23)));
}

struct SwaParams {
  int Tc, H, D, nslot;
  // work units: blockIdx.x < pair_units is the pair of query tiles
  // (bh, blockIdx.x % pairs_per_bh); beyond, each later pair is split into
  // two single-tile units (fewer query rows in the last wave of CTAs)
  int pairs_per_bh, pair_units;
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
  uint64_t s_full[kQTiles][2], s_free[kQTiles][2];
  uint64_t p_full[kQTiles], pv_done[kQTiles];
  uint64_t drain[kQTiles];
  uint32_t tmem;
  int abort;
};

// Shared memory: Q tiles [g][D/8][128][8] (later the output tiles), the K and
// V rings (per stage K [D/8][64][8] | V [D/8][64][8]), P [g][8][128][8],
// barriers.
struct SwaLayout {
  uint32_t q, q_tile, kv, kv_stage, v_off, p, p_tile, bars, total;
};
__host__ __device__ inline SwaLayout swa_layout(int D) {
  SwaLayout L;
  L.q = 0;
  L.q_tile = kQRows * D * 2;
  L.kv = kQTiles * L.q_tile;
  L.v_off = kKRows * D * 2;
  L.kv_stage = 2 * L.v_off;
  L.p = L.kv + kStages * L.kv_stage;
  L.p_tile = kQRows * kKRows * 2;
  L.bars = L.p + kQTiles * L.p_tile;
  L.total = L.bars + 256;
  if (L.total < kMinSmem) L.total = kMinSmem;
  return L;
}
static_assert(sizeof(SwaBars) <= 256, "barrier block");

template <int NK>  // D / 16
__global__ void __launch_bounds__(kThreads, 1)
gdn_sink_window_kernel(const __grid_constant__ CUtensorMap tm_q,
                       const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v,
                       const __grid_constant__ CUtensorMap tm_kc,
                       const __grid_constant__ CUtensorMap tm_vc,
                       const __grid_constant__ CUtensorMap tm_out,
                       const __grid_constant__ SwaParams P) {
  extern __shared__ __align__(128) uint8_t smem[];
  constexpr int D = 16 * NK;
  const SwaLayout L = swa_layout(D);
  SwaBars& bar = *reinterpret_cast<SwaBars*>(smem + L.bars);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  int pair_index, q0, nq;  // query tiles present: nq of 128 rows from row q0
  if ((int)blockIdx.x < P.pair_units) {
    pair_index = blockIdx.x;
    q0 = (pair_index % P.pairs_per_bh) * kQTiles * kQRows;
    nq = min(kQTiles, (P.Tc - q0 + kQRows - 1) / kQRows);
  } else {
    const int u = blockIdx.x - P.pair_units;
    pair_index = P.pair_units + u / kQTiles;
    q0 = (pair_index % P.pairs_per_bh) * kQTiles * kQRows + (u % kQTiles) * kQRows;
    nq = q0 < P.Tc ? 1 : 0;
  }
  if (nq == 0) return;  // the missing half of a ragged pair (uniform over the CTA)
  const int bh = pair_index / P.pairs_per_bh, b = bh / P.H, h = bh - b * P.H;
  const int tps = P.tiles_per_seg;
  const int ntiles = P.nseg * tps;
  volatile int* abort_flag = &bar.abort;

  if (tid == 0) {
    mbar_init(&bar.q_full, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bar.k_full[s], 1);
      mbar_init(&bar.k_empty[s], nq);  // one release per MMA warp in use
      mbar_init(&bar.v_full[s], 1);
      mbar_init(&bar.v_empty[s], nq);
    }
    for (int g = 0; g < kQTiles; ++g) {
      for (int s = 0; s < 2; ++s) {
        mbar_init(&bar.s_full[g][s], 1);
        mbar_init(&bar.s_free[g][s], 128);
      }
      mbar_init(&bar.p_full[g], 128);
      mbar_init(&bar.pv_done[g], 1);
      mbar_init(&bar.drain[g], 1);
    }
    bar.abort = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
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

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------ producer
    // K runs one tile ahead of V: K_j is free once the S MMAs of tile j are
    // done, V_j only once the P V MMAs are, so the rings refill independently.
    if (lane == 0) {
      mbar_arrive_expect_tx(&bar.q_full, nq * L.q_tile);
      for (int g = 0; g < nq; ++g)
        tma_load_tile(smem + L.q + g * L.q_tile, &tm_q, &bar.q_full, q0 + g * kQRows, h, b);
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
          if (P.append_slot >= 0 && r0 >= q0 && r0 < q0 + nq * kQRows) append_row[x][st] = r0;
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
  } else if (warp >= kMmaWarp) {
    // ----------------------------------------------------------- MMA issue
    const int g = warp - kMmaWarp;
    if (lane == 0 && g < nq) {
      constexpr uint32_t kQSlab = kQRows * 16, kKSlab = kKRows * 16;
      const uint32_t idS = idesc_bf16(kQRows, kKRows, 0, 0);
      const uint32_t idO = idesc_bf16(kQRows, D, 0, 1);
      const uint32_t tS = tm + g * kTileCols, tOg = tS + 2 * kKRows;
      // descriptors of stage 0 / this tile; a stage or a K step moves only
      // the start-address field (addresses >> 4)
      const uint64_t dq = sdesc(smem_u32(smem + L.q + g * L.q_tile), kQSlab, 128);
      const uint64_t dp = sdesc(smem_u32(smem + L.p + g * L.p_tile), kQSlab, 128);
      const uint64_t dk = sdesc(smem_u32(smem + L.kv), kKSlab, 128);
      const uint64_t dv = sdesc(smem_u32(smem + L.kv + L.v_off), 128, kKSlab);
      const uint64_t dstage = L.kv_stage >> 4;
      bool ok = mbar_wait(&bar.q_full, 0, P.limit);
      if (!ok) fail();
      tc_fence_after_sync();
      for (int j = 0; ok && j <= ntiles; ++j) {
        if (*abort_flag) break;
        if (j < ntiles) {
          const int s = j % kStages, sb = j & 1;
          if (!mbar_wait(&bar.k_full[s], (j / kStages) & 1, P.limit) ||
              (j >= 2 && !mbar_wait(&bar.s_free[g][sb], ((j >> 1) - 1) & 1, P.limit))) {
            fail();
            break;
          }
          tc_fence_after_sync();
          // S_gj = Q_g K_j^T: both K-major, K = D in steps of 16
          const uint64_t dks = dk + s * dstage;
#pragma unroll
          for (int ks = 0; ks < NK; ++ks)
            mma_bf16(tS + sb * kKRows, dq + ks * (2 * kQSlab >> 4), dks + ks * (2 * kKSlab >> 4), idS,
                     ks > 0);
          mma_commit(&bar.s_full[g][sb]);
          mma_commit(&bar.k_empty[s]);
        }
        if (j >= 1) {
          const int jp = j - 1, s = jp % kStages;
          if (!mbar_wait(&bar.v_full[s], (jp / kStages) & 1, P.limit) ||
              !mbar_wait(&bar.p_full[g], jp & 1, P.limit)) {
            fail();
            break;
          }
          tc_fence_after_sync();
          // O_g += P_g V: P K-major (K = 64 keys), V MN-major (N = D)
          const uint64_t dvs = dv + s * dstage;
#pragma unroll
          for (int ks = 0; ks < kKRows / 16; ++ks)
            mma_bf16(tOg, dp + ks * (2 * kQSlab >> 4), dvs + ks * (256 >> 4), idO,
                     (jp > 0) || (ks > 0));
          mma_commit(&bar.pv_done[g]);
          mma_commit(&bar.v_empty[s]);
        }
      }
      // every MMA issued has completed before TMEM and shared memory go
      mma_commit(&bar.drain[g]);
      mbar_wait(&bar.drain[g], 0, kDrainPolls);
    }
  } else if ((warp >> 2) < nq) {
    // ------------------------------------------------------------- softmax
    const int g = warp >> 2;
    const int r = tid & (kQRows - 1);  // query row within the tile = TMEM lane
    const uint32_t lrow = tm + g * kTileCols + ((uint32_t)((warp & 3) * 32) << 16);
    const uint32_t tO = lrow + 2 * kKRows;
    uint8_t* sp = smem + L.p + g * L.p_tile;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < ntiles; ++j) {
      const int sb = j & 1;
      if (__any_sync(~0u, *abort_flag != 0)) {
        ok = false;
        break;
      }
      if (!__all_sync(~0u, mbar_wait(&bar.s_full[g][sb], (j >> 1) & 1, P.limit))) {
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
      mbar_arrive(&bar.s_free[g][sb]);

      const int t = j % tps;
      const int nvalid = min(kKRows, P.Tc - t * kKRows);
      if (nvalid < kKRows) {  // the ragged last tile of a chunk (warp-uniform)
#pragma unroll
        for (int i = 0; i < kKRows; ++i)
          if (i >= nvalid) s[i] = -INFINITY;
      }
      // row maximum: eight independent chains of three-input maxima over
      // columns 0-23, 24-39, 40-55, then 56-63
      static_assert(kKRows == 64, "the maximum's column pattern");
      float acc[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] = fmax3(s[e], s[e + 8], s[e + 16]);
#pragma unroll
      for (int i = 24; i + 16 <= 56; i += 16)
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = fmax3(acc[e], s[i + e], s[i + 8 + e]);
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] = fmaxf(acc[e], s[56 + e]);
      float mx = fmax3(fmax3(acc[0], acc[1], acc[2]), fmax3(acc[3], acc[4], acc[5]), fmaxf(acc[6], acc[7]));
      mx *= P.scale_log2;
      float m_new = m_run, alpha = 1.f;
      bool resc = false;
      if (mx > m_run + kRescaleLog2) {
        m_new = mx;
        alpha = ex2_approx(m_run - m_new);  // 0 on the first tile
        resc = j > 0;
      }
      // p = 2^(s c - m), two at a time: one pair in four on the FMA pipe,
      // the rest on the special-function unit; P packed to bf16 as it goes
      const uint64_t c2 = f2_pack(P.scale_log2, P.scale_log2), nm2 = f2_pack(-m_new, -m_new);
      uint64_t sum2[4] = {0, 0, 0, 0};  // packed +0.0f pairs
      uint32_t pk[kKRows / 2];
#pragma unroll
      for (int i = 0; i < kKRows; i += 2) {
        const uint64_t x = f2_fma(f2_pack(s[i], s[i + 1]), c2, nm2);
        uint64_t p2;
        if ((i & 7) == 6) {
          p2 = exp2_poly2(x);
        } else {
          float a, c;
          f2_unpack(x, a, c);
          p2 = f2_pack(ex2_approx(a), ex2_approx(c));
        }
        sum2[(i >> 1) & 3] = f2_add(sum2[(i >> 1) & 3], p2);
        float a, c;
        f2_unpack(p2, a, c);
        pk[i >> 1] = pack_bf16x2(a, c);
      }
      const uint64_t sa = f2_add(f2_add(sum2[0], sum2[1]), f2_add(sum2[2], sum2[3]));
      float rs0, rs1;
      f2_unpack(sa, rs0, rs1);
      const float rs = rs0 + rs1;
      // P and O belong to the previous tile's P V until it completes
      if (j > 0) {
        if (!__all_sync(~0u, mbar_wait(&bar.pv_done[g], (j - 1) & 1, P.limit))) {
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
        reinterpret_cast<uint4*>(sp + sl * kQRows * 16)[r] =
            make_uint4(pk[4 * sl], pk[4 * sl + 1], pk[4 * sl + 2], pk[4 * sl + 3]);
      fence_proxy_async_smem();
      tc_fence_before_sync();
      mbar_arrive(&bar.p_full[g]);
    }
    if (ok && ntiles > 0 &&
        !__all_sync(~0u, mbar_wait(&bar.pv_done[g], (ntiles - 1) & 1, P.limit))) {
      if (lane == 0) fail();
      ok = false;
    }
    // all 128 rows of the tile agree before it is stored
    ok = named_barrier_and(1 + g, kQRows, ok);
    if (ok) {
      tc_fence_after_sync();
      // every S MMA has completed, so the tile's Q buffer takes its output
      uint8_t* so = smem + L.q + g * L.q_tile;
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
      named_barrier(1 + g, kQRows);
      if (r == 0) {
        tma_store_tile(&tm_out, so, q0 + g * kQRows, h, b);
        bulk_commit();
        bulk_wait_all();
      }
    }
  }
  tc_fence_before_sync();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after_sync();
    tmem_dealloc(tm, kTmemCols);
  }
}

template <int NK>
cudaError_t launch_nk(dim3 grid, cudaStream_t stream, const CUtensorMap& mq, const CUtensorMap& mk,
                      const CUtensorMap& mv, const CUtensorMap& mkc, const CUtensorMap& mvc,
                      const CUtensorMap& mo, const SwaParams& P) {
  // opt in to the dynamic shared memory once per device
  constexpr int kMaxDev = 64;
  static std::mutex mu;
  static bool done[kMaxDev] = {};
  const int bytes = (int)swa_layout(16 * NK).total;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (dev < 0 || dev >= kMaxDev || !done[dev]) {
      e = cudaFuncSetAttribute(gdn_sink_window_kernel<NK>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               bytes);
      if (e != cudaSuccess) return e;
      if (dev >= 0 && dev < kMaxDev) done[dev] = true;
    }
  }
  ProfileScope ps(stream, kKernSinkWindow);
  gdn_sink_window_kernel<NK><<<grid, kThreads, bytes, stream>>>(mq, mk, mv, mkc, mvc, mo, P);
  return cudaSuccess;
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
  // one CTA per SM: a pair of query tiles per CTA, except that when the
  // pairs overfill the first wave by less than half, the overflow's worth of
  // pairs run as single tiles so that the second wave is half as long
  P.pairs_per_bh = (c.Tc + kQTiles * kQRows - 1) / (kQTiles * kQRows);
  const int pairs = P.pairs_per_bh * c.B * c.H;
  const int sms = num_sms();
  int split = 0;
  if (pairs > sms && 2 * (pairs - sms) <= sms) split = pairs - sms;
  P.pair_units = pairs - split;
  const dim3 grid(P.pair_units + kQTiles * split);
  cudaError_t e = cudaSuccess;
  switch (c.D / 16) {
    case 1: e = launch_nk<1>(grid, c.stream, mq, mk, mv, mkc, mvc, mo, P); break;
    case 2: e = launch_nk<2>(grid, c.stream, mq, mk, mv, mkc, mvc, mo, P); break;
    case 3: e = launch_nk<3>(grid, c.stream, mq, mk, mv, mkc, mvc, mo, P); break;
    case 4: e = launch_nk<4>(grid, c.stream, mq, mk, mv, mkc, mvc, mo, P); break;
    case 5: e = launch_nk<5>(grid, c.stream, mq, mk, mv, mkc, mvc, mo, P); break;
    case 6: e = launch_nk<6>(grid, c.stream, mq, mk, mv, mkc, mvc, mo, P); break;
    case 7: e = launch_nk<7>(grid, c.stream, mq, mk, mv, mkc, mvc, mo, P); break;
    case 8: e = launch_nk<8>(grid, c.stream, mq, mk, mv, mkc, mvc, mo, P); break;
    default: return cudaErrorInvalidValue;
  }
  if (e != cudaSuccess) return e;
  e = cudaGetLastError();
  if (e == cudaSuccess) count_launches(1);
  return e;
}

}  // namespace gdn
