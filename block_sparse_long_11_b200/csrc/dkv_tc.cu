// Backward, key side: dK and dV of the MoBA forward with the selection held
// fixed, on the 5th-generation tensor cores (tcgen05 + TMEM).
//
// Page cited by title: "同一天，DeepSeek和月之暗面發表了關于改進注意力機制的論文"
// (MoBA write-up), opening list: trainable block-sparse attention -- the top-k
// gate passes no gradient; over the chosen keys the attention is ordinary
// softmax attention.  Per query row r with upstream dout_r and the forward's
// lse_r, for every key u the row attends:
//   p_ru = exp(scale q_r.k_u - lse_r),  dp_ru = dout_r . v_u,
//   D_r = dout_r . out_r,  ds_ru = p_ru (dp_ru - D_r),
//   dv_u = sum_r p_ru dout_r,  dk_u = scale sum_r ds_ru q_r.
//
// Work unit: one tile of 128 keys of one block (one kv head).  The keys of
// block b for kv head g are attended by exactly two sets of rows: the rows
// the scheduler routed to bucket (b, g) (b one of their past blocks), and the
// rows of block b itself for the query heads of g (own block, token-level
// causal mask).  The unit streams all of them in tiles of 64 rows, so it
// holds every contribution to its keys and writes dk, dv directly (no
// atomics).  Per row tile, with the keys as the TMEM lanes (M = 128 keys):
//   S^T  = K_tile Q_rows^T      (SS: both operands K-major in shared memory)
//   dP^T = V_tile dO_rows^T     (SS)
//   P^T = exp2(S^T * scale log2 e - lse_r log2 e) under the masks,
//   dS^T = P^T (dP^T - D_r), written back over S^T / dP^T as packed bf16;
//   dV += P^T dO_rows,  dK += dS^T Q_rows   (TS: P^T / dS^T read from TMEM,
//                                            the row tiles MN-major in smem).
// Two row tiles are in flight (TMEM ping-pong): while the P^T / dS^T warps
// work on tile c, the tensor cores compute S^T / dP^T of tile c + 1 and then
// dV / dK of tile c.  TMEM columns: S^T of buffer b at [64 b, 64 b + 64),
// dP^T at [128 + 64 b, ...), dV and dK after them (d each).
//
// Row tiles arrive as whole TMA boxes.  A routed tile is 64 consecutive
// rows of the packed copy that dkv_pack_kernel makes first: the Q and dO
// rows of the bucket entries in entry order (with -lse log2 e and D beside
// them), so a bucket's rows are contiguous.  (Gathering the scattered rows
// into shared memory inside this kernel -- four-row TMA gathers or cp.async
// -- cost about as much as all its tensor-core and softmax work together;
// loading the same bytes as boxes costs a tenth of that.)  An own-block tile
// is 64 consecutive tokens of one query head, a box of the 3D view
// [T, Hq, d] of q / dout itself.  The packed copy is bounded: entries are
// packed and processed in chunks; the first chunk's launch also takes the
// own rows and writes dk, dv, later chunks add their routed rows to them in
// launch order (the result does not depend on the chunking's timing).
//
// Warp roles (12 warps): warp 0 loads the unit's K and V tiles with TMA;
// warp 1 issues the MMAs (one elected lane); warps 2 / 3 load the Q / dO
// row tiles (a 4-deep ring) and warp 2 the rows' lse, D and causal limit;
// warps 4-11 compute P^T and dS^T (warps 4-7 the row columns [0, 32) of a
// tile, warps 8-11 [32, 64), each warp the 32 keys of its TMEM lane
// quarter) and write the unit's dK, dV out.  Every mbarrier wait is bounded
// as in the forward kernel.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "kernels.h"
#include "tc_ptx.cuh"

namespace moba {
namespace {
using namespace tc;

constexpr int kRows = 64;   // rows per row tile (N of the S^T / dP^T MMAs)
constexpr int kKeys = 128;  // keys per unit (TMEM lanes)
constexpr int kRing = 4;    // gathered row tiles in flight
constexpr int kThreads = 384;
constexpr long long kWaitBudget = 4000000000LL;
constexpr uint32_t kTmemCols = 512;
constexpr int kNoLimit = 0x7ffffffe;  // past rows see every key of the block
constexpr int kNoKey = 0x7fffffff;    // a lane past the block end: above every row's limit

template <int D>
struct DkvSmem {
  alignas(1024) __nv_bfloat16 kt[kKeys * D];    // K tile: A of S^T
  alignas(1024) __nv_bfloat16 vt[kKeys * D];    // V tile: A of dP^T
  alignas(1024) __nv_bfloat16 q[kRing][kRows * D];  // gathered Q rows: B of S^T and of dK
  alignas(1024) __nv_bfloat16 g[kRing][kRows * D];  // gathered dO rows: B of dP^T and of dV
  // per row of a tile (read four columns at a time by the P^T / dS^T warps)
  alignas(16) float nlse2[kRing][kRows];  // -lse * log2(e)
  alignas(16) float dd[kRing][kRows];     // D = dout . out
  alignas(16) int lim[kRing][kRows];      // last in-block key the row sees (-1: padding row)
  uint64_t kv_full, kv_empty;
  uint64_t q_full[kRing], g_full[kRing];   // row-tile ring: Q rows (+ lse, D, limit) / dO rows landed
  uint64_t t_empty[kRing];                 // row-tile ring slot free
  uint64_t s_full[2];                      // [TMEM buffer]: S^T and dP^T are in TMEM
  uint64_t p_full[2];                      // [TMEM buffer]: P^T and dS^T are back (8 warps)
  uint64_t acc_full, acc_empty;    // the unit's dK, dV done / read out (8 warps)
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

__device__ __forceinline__ uint32_t bar(const uint64_t& b) { return smem_addr(&b); }

// One box of a 2D tensor map at (c0, c1).
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const void* tmap, uint32_t bar, int c0,
                                            int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];\n" ::"r"(dst),
      "l"(tmap), "r"(bar), "r"(c0), "r"(c1)
      : "memory");
}

// Packed rows of a chunk of bucket entries [e_lo, e_lo + cap): entry e's Q
// and dO rows go to row e - e_lo of qp / gp, and (-lse log2 e, D) of its row
// to ld[e - e_lo].  The 64 rows after the chunk's last entry are zeroed, so
// a row tile that runs past it reads finite values (its rows are masked).
template <int D>
__global__ void __launch_bounds__(256) dkv_pack_kernel(
    const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ dout,
    const float* __restrict__ lse, const float* __restrict__ dvec, Workspace ws,
    __nv_bfloat16* __restrict__ qp, __nv_bfloat16* __restrict__ gp, float2* __restrict__ ld,
    int Hkv, int topk, int e_lo, int cap) {
  const DevPlan* plan = ws.plan;
  if (plan->err != 0) return;
  const int e_all = ws.bucket_off[plan->nfull_total * Hkv];
  const int n = max(0, min(cap, e_all - e_lo));  // entries of this chunk
  const int lane = threadIdx.x & 31;
  constexpr int kChunks = D / 8;  // 16-byte pieces of a row
  const long long nwarps = (long long)gridDim.x * (blockDim.x >> 5);
  for (long long w = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5; w < n + 64;
       w += nwarps) {
    const int i = (int)w;  // packed row
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    float2 l2 = make_float2(0.f, 0.f);
    const bool live = i < n;
    long long row = 0;
    if (live) {
      const int ent = ws.entries[e_lo + i];
      const bool ok_ = MOBA_INDEX_OK(plan, ent >= 0 && ent / topk < ws.rows_cap, kSiteDkvEntry);
      row = ok_ ? ent / topk : 0;
    }
    const bool is_q = lane < 16;
    const int cc = lane & 15;
    if (cc < kChunks) {
      if (live) v = *reinterpret_cast<const uint4*>((is_q ? q : dout) + row * D + cc * 8);
      *reinterpret_cast<uint4*>((is_q ? qp : gp) + (long long)i * D + cc * 8) = v;
    }
    if (lane == 0) {
      if (live) l2 = make_float2(-lse[row] * 1.4426950408889634f, dvec[row]);
      ld[i] = l2;
    }
  }
}

// One unit: key tile kt of global block gb, kv head g.
struct DkvUnit {
  int gb, g, kt, start, len;
  int e0, e1;      // the bucket's routed entries in this chunk, e0 = e1 if none
  int npast;       // row tiles of routed rows
  int nown;        // own-row tiles per query head of the group
  int ntiles;      // npast + G * nown (0: nothing to do)
};

__device__ __forceinline__ DkvUnit decode_dkv(int u, const Workspace& ws, int Hkv, int G, int B,
                                              int e_lo, int cap, int first) {
  DkvUnit U;
  const int nkt = (B + kKeys - 1) / kKeys;
  U.kt = u % nkt;
  int v = u / nkt;
  U.g = v % Hkv;
  U.gb = v / Hkv;
  U.len = ws.blk_len[U.gb];
  U.start = ws.blk_start[U.gb];
  U.e0 = U.e1 = 0;
  U.npast = U.nown = U.ntiles = 0;
  if (U.kt * kKeys >= U.len) return U;
  if (U.len == B) {  // a full block: its bucket of routed rows
    const int b = (ws.blk_fullbase[U.gb] + ws.blk_j[U.gb]) * Hkv + U.g;
    if (MOBA_INDEX_OK(ws.plan,
                      b >= 0 && b < ws.nbk_cap && ws.bucket_off[b] >= 0 &&
                          ws.bucket_off[b] <= ws.bucket_off[b + 1] &&
                          ws.bucket_off[b + 1] <= ws.entries_cap,
                      kSiteDkvBucket)) {  // else every role drops the routed rows
      // the part of the bucket inside this chunk of packed entries
      U.e0 = max(ws.bucket_off[b], e_lo);
      U.e1 = max(U.e0, (int)min((long long)ws.bucket_off[b + 1], (long long)e_lo + cap));
    }
  }
  U.npast = (U.e1 - U.e0 + kRows - 1) / kRows;
  U.nown = first ? (U.len - U.kt * kKeys + kRows - 1) / kRows : 0;
  U.ntiles = U.npast + G * U.nown;
  return U;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    dkv_tc_kernel(const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
                  const __grid_constant__ CUtensorMap tmqp, const __grid_constant__ CUtensorMap tmgp,
                  const __grid_constant__ CUtensorMap tmq3, const __grid_constant__ CUtensorMap tmg3,
                  const float2* __restrict__ ld, const float* __restrict__ lse,
                  const float* __restrict__ dvec, Workspace ws, float* __restrict__ dk,
                  float* __restrict__ dv, int Hq, int Hkv, int B, float scale_log2, float scale,
                  int e_lo, int cap, int first) {
  extern __shared__ unsigned char smem_raw[];
  DkvSmem<D>& sm = *reinterpret_cast<DkvSmem<D>*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  DevPlan* plan = ws.plan;
  if (plan->err != 0) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = Hq / Hkv;
  const int n_units = plan->nblk_total * Hkv * ((B + kKeys - 1) / kKeys);
  constexpr uint32_t kRegionK = kKeys * 128;  // bytes of one 64-column region of a K / V tile
  constexpr uint32_t kRegionR = kRows * 128;  // ... and of a row tile
  constexpr uint32_t kTileBytes = kKeys * D * 2;

  if (threadIdx.x == 0) {
    mbar_init(bar(sm.kv_full), 1);
    mbar_init(bar(sm.kv_empty), 1);
    for (int s = 0; s < kRing; ++s) {
      mbar_init(bar(sm.q_full[s]), 1);
      mbar_init(bar(sm.g_full[s]), 1);
      mbar_init(bar(sm.t_empty[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(sm.s_full[b]), 1);
      mbar_init(bar(sm.p_full[b]), 8);
    }
    mbar_init(bar(sm.acc_full), 1);
    mbar_init(bar(sm.acc_empty), 8);
    mbar_init(bar(sm.drain), 1);
    sm.abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_addr(&sm.tmem_base), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  volatile int* abort = &sm.abort_flag;

  if (warp == 0) {
    // ------------------------------------------------------------ K/V loader
    if (lane == 0) {
      prefetch_tmap(&tmk);
      prefetch_tmap(&tmv);
      bool ok = true;
      int nu = 0;
      for (int u = blockIdx.x; ok && u < n_units; u += gridDim.x) {
        const DkvUnit U = decode_dkv(u, ws, Hkv, G, B, e_lo, cap, first);
        if (U.ntiles == 0) continue;
        if (!(ok = mbar_wait(bar(sm.kv_empty), (uint32_t)(nu & 1) ^ 1u, abort, kWaitBudget))) break;
        mbar_arrive_expect_tx(bar(sm.kv_full), 2 * kTileBytes);
        for (int h = 0; h < D / 64; ++h) {
          tma_load_3d(smem_addr(sm.kt) + h * kRegionK, &tmk, bar(sm.kv_full), 64 * h, U.g,
                      U.start + U.kt * kKeys);
          tma_load_3d(smem_addr(sm.vt) + h * kRegionK, &tmv, bar(sm.kv_full), 64 * h, U.g,
                      U.start + U.kt * kKeys);
        }
        ++nu;
      }
      if (!ok && nu > 0) {  // the copies issued last must land before the CTA exits
        int dummy = 0;
        mbar_wait(bar(sm.kv_full), (uint32_t)((nu - 1) & 1), &dummy, kWaitBudget);
      }
    }
  } else if (warp == 2 || warp == 3) {
    // ------------------------------------------------------------ row tiles
    // warp 2: Q tiles and the rows' -lse log2 e, D and causal limit; warp 3:
    // dO tiles.  One TMA box per 64-column region, completing on the warp's
    // own barrier of the ring slot; the rows' scalars are read one tile ahead.
    const CUtensorMap* tmp = warp == 2 ? &tmqp : &tmgp;
    const CUtensorMap* tm3 = warp == 2 ? &tmq3 : &tmg3;
    if (lane == 0) {
      prefetch_tmap(tmp);
      prefetch_tmap(tm3);
    }
    constexpr int RPL = kRows / 32;  // rows per lane
    // walks the CTA's row tiles across its units
    struct TileIt {
      int u, m;
      DkvUnit U;
      bool valid;
    };
    auto advance = [&](TileIt& it) {
      ++it.m;
      while (it.valid && it.m >= it.U.ntiles) {
        it.u += gridDim.x;
        if (it.u >= n_units) {
          it.valid = false;
          break;
        }
        it.U = decode_dkv(it.u, ws, Hkv, G, B, e_lo, cap, first);
        it.m = 0;
      }
    };
    // the scalars of a tile's rows (masked rows: limit -1, zeros)
    auto scalars_of = [&](const TileIt& it, float* nl, float* dd, int* lim) {
#pragma unroll
      for (int i = 0; i < RPL; ++i) {
        const int r = lane + 32 * i;
        nl[i] = dd[i] = 0.f;
        lim[i] = -1;
        if (it.m < it.U.npast) {
          const int e = it.U.e0 + it.m * kRows + r;
          if (e < it.U.e1) {
            const float2 l2 = ld[e - e_lo];
            nl[i] = l2.x;
            dd[i] = l2.y;
            lim[i] = kNoLimit;
          }
        } else {
          const int mm = it.m - it.U.npast;
          const int hh = mm / it.U.nown;
          const int y = it.U.kt * kKeys + (mm % it.U.nown) * kRows + r;  // in-block position
          if (y < it.U.len) {
            const long long row = (long long)(it.U.start + y) * Hq + it.U.g * G + hh;
            nl[i] = -lse[row] * 1.4426950408889634f;
            dd[i] = dvec[row];
            lim[i] = y;
          }
        }
      }
    };
    TileIt cur;
    cur.u = blockIdx.x;
    cur.m = -1;
    cur.valid = cur.u < n_units;
    if (cur.valid) cur.U = decode_dkv(cur.u, ws, Hkv, G, B, e_lo, cap, first);
    advance(cur);
    float nl[RPL], dd[RPL];
    int lim[RPL];
    if (warp == 2 && cur.valid) scalars_of(cur, nl, dd, lim);
    bool ok = true;
    long long c = 0;  // row tiles issued
    while (ok && cur.valid) {
      const int s = (int)(c % kRing);
      ok = __all_sync(0xffffffffu, mbar_wait(bar(sm.t_empty[s]), (uint32_t)((c / kRing) & 1) ^ 1u,
                                             abort, kWaitBudget));
      if (!ok) break;
      const uint32_t full = bar(warp == 2 ? sm.q_full[s] : sm.g_full[s]);
      if (warp == 2) {
#pragma unroll
        for (int i = 0; i < RPL; ++i) {
          sm.nlse2[s][lane + 32 * i] = nl[i];
          sm.dd[s][lane + 32 * i] = dd[i];
          sm.lim[s][lane + 32 * i] = lim[i];
        }
      }
      __syncwarp();
      if (lane == 0) {
        mbar_arrive_expect_tx(full, kRows * D * 2);
        const uint32_t base = smem_addr(warp == 2 ? sm.q[s] : sm.g[s]);
        if (cur.m < cur.U.npast) {  // packed rows of the bucket's entries
          const int p0 = cur.U.e0 + cur.m * kRows - e_lo;
#pragma unroll
          for (int h = 0; h < D / 64; ++h) tma_load_2d(base + h * kRegionR, tmp, full, 64 * h, p0);
        } else {  // 64 tokens of one query head of the block
          const int mm = cur.m - cur.U.npast;
          const int head = cur.U.g * G + mm / cur.U.nown;
          const int t0 = cur.U.start + cur.U.kt * kKeys + (mm % cur.U.nown) * kRows;
#pragma unroll
          for (int h = 0; h < D / 64; ++h)
            tma_load_3d(base + h * kRegionR, tm3, full, 64 * h, head, t0);
        }
      }
      __syncwarp();
      ++c;
      advance(cur);
      if (warp == 2 && cur.valid) scalars_of(cur, nl, dd, lim);  // used next iteration
    }
    if (!ok) {  // the loads issued last must land before the CTA exits
      int dummy = 0;
      for (long long cc = (c > kRing ? c - kRing : 0); cc < c; ++cc)
        mbar_wait(bar(warp == 2 ? sm.q_full[cc % kRing] : sm.g_full[cc % kRing]),
                  (uint32_t)((cc / kRing) & 1), &dummy, kWaitBudget);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    bool ok = true;
    auto wait_all = [&](uint32_t b, uint32_t par) -> bool {
      const bool r = __all_sync(0xffffffffu, mbar_wait(b, par, abort, kWaitBudget));
      tc_fence_after();
      return r;
    };
    auto commit = [&](const uint64_t& b) {
      if (elect_one()) umma_commit(bar(b));
      __syncwarp();
    };
    constexpr uint32_t idesc_s = idesc_bf16(128, kRows, 0, 0);  // keys x rows, K = d
    constexpr uint32_t idesc_a = idesc_bf16(128, D, 0, 1);      // keys x d, K = rows
    const uint64_t kdesc = sdesc_sw128(smem_addr(sm.kt), 16, 1024);
    const uint64_t vdesc = sdesc_sw128(smem_addr(sm.vt), 16, 1024);
    // S^T and dP^T of row tile c into TMEM buffer c & 1
    auto issue_sd = [&](long long cc) -> bool {
      const int s = (int)(cc % kRing);
      const uint32_t b = (uint32_t)(cc & 1);
      if (!wait_all(bar(sm.q_full[s]), (uint32_t)((cc / kRing) & 1)) ||
          !wait_all(bar(sm.g_full[s]), (uint32_t)((cc / kRing) & 1)))
        return false;
      const uint64_t qk = sdesc_sw128(smem_addr(sm.q[s]), 16, 1024);
      const uint64_t gk = sdesc_sw128(smem_addr(sm.g[s]), 16, 1024);
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t ok_ = (uint64_t)(((kk >> 2) * kRegionK + (kk & 3) * 32) >> 4);
          const uint64_t or_ = (uint64_t)(((kk >> 2) * kRegionR + (kk & 3) * 32) >> 4);
          umma_ss(tmem + 64u * b, kdesc + ok_, qk + or_, idesc_s, kk > 0);
          umma_ss(tmem + 128u + 64u * b, vdesc + ok_, gk + or_, idesc_s, kk > 0);
        }
      }
      __syncwarp();
      commit(sm.s_full[b]);
      return true;
    };
    // dV += P^T dO, dK += dS^T Q of row tile c: K = 64 rows in 4 steps of 16;
    // P^T / dS^T packed bf16, rows [32 h, 32 h + 32) in columns [32 h, 32 h + 16)
    // of the buffer (each half of the P^T warps writes inside its own columns)
    auto issue_acc = [&](long long cc, bool first) -> bool {
      const int s = (int)(cc % kRing);
      const uint32_t b = (uint32_t)(cc & 1);
      if (!wait_all(bar(sm.p_full[b]), (uint32_t)((cc >> 1) & 1))) return false;
      const uint64_t gm = sdesc_sw128(smem_addr(sm.g[s]), kRegionR, 1024);
      const uint64_t qm = sdesc_sw128(smem_addr(sm.q[s]), kRegionR, 1024);
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < kRows / 16; ++kk) {
          const uint32_t acol = 64u * b + (uint32_t)(32 * (kk >> 1) + 8 * (kk & 1));
          const uint32_t acc = (!first || kk > 0) ? 1u : 0u;
          umma_ts(tmem + 256u, tmem + acol, gm + (uint64_t)(kk * 128), idesc_a, acc);
          umma_ts(tmem + 256u + D, tmem + 128u + acol, qm + (uint64_t)(kk * 128), idesc_a, acc);
        }
      }
      __syncwarp();
      commit(sm.t_empty[s]);
      return true;
    };
    long long c = 0;
    int nu = 0;
    for (int u = blockIdx.x; ok && u < n_units; u += gridDim.x) {
      const DkvUnit U = decode_dkv(u, ws, Hkv, G, B, e_lo, cap, first);
      if (U.ntiles == 0) continue;
      if (!(ok = wait_all(bar(sm.kv_full), (uint32_t)(nu & 1)))) break;
      if (!(ok = issue_sd(c))) break;
      for (int m = 0; m < U.ntiles; ++m, ++c) {
        // the next tile's S^T / dP^T go to the other buffer while this tile's
        // P^T / dS^T are computed; then this tile's dV / dK
        if (m + 1 < U.ntiles && !(ok = issue_sd(c + 1))) break;
        if (m + 1 == U.ntiles) commit(sm.kv_empty);  // the unit's last read of K / V
        if (m == 0 && !(ok = wait_all(bar(sm.acc_empty), (uint32_t)(nu & 1) ^ 1u))) break;
        if (!(ok = issue_acc(c, m == 0))) break;
      }
      if (!ok) break;
      commit(sm.acc_full);
      ++nu;
    }
    commit(sm.drain);  // every MMA issued must finish before TMEM is freed
    int dummy = 0;
    mbar_wait(bar(sm.drain), 0, &dummy, kWaitBudget);
  } else {
    // ------------------------------------------------------------ P^T, dS^T, epilogue
    const int quad = warp & 3;             // TMEM lanes 32 quad .. 32 quad + 31
    const int half = (warp - 4) >> 2;      // row columns [32 half, 32 half + 32) of a tile
    const int kl = quad * 32 + lane;       // key of the tile (TMEM lane)
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const uint64_t sc2 = f32x2(scale_log2, scale_log2);
    bool ok = true;
    long long c = 0;
    int nu = 0;
    for (int u = blockIdx.x; ok && u < n_units; u += gridDim.x) {
      const DkvUnit U = decode_dkv(u, ws, Hkv, G, B, e_lo, cap, first);
      if (U.ntiles == 0) continue;
      const int kpos = U.kt * kKeys + kl;  // in-block key position
      const bool kvalid = kpos < U.len;
      const int kposv = kvalid ? kpos : kNoKey;  // a key past the block end sees no row
      for (int m = 0; m < U.ntiles; ++m, ++c) {
        const int s = (int)(c % kRing);
        const uint32_t b = (uint32_t)(c & 1);
        ok = __all_sync(0xffffffffu, mbar_wait(bar(sm.s_full[b]), (uint32_t)((c >> 1) & 1), abort,
                                               kWaitBudget));
        if (!ok) break;
        tc_fence_after();
        // the warp's 32 row columns; the packed P / dS land in the first 16
        // of them, which this warp has read already
        const uint32_t scol = tmem + lane_off + 64u * b + 32u * half;
        uint32_t sv[32], pv[32];
        tmem_ld32(scol, sv);
        tmem_ld32(scol + 128, pv);
        tmem_ld_wait();
        reg_fence32(sv);
        reg_fence32(pv);
        uint32_t pk[16], dk2[16];
#pragma unroll
        for (int y = 0; y < 8; ++y) {  // four row columns per step
          const int c0 = 32 * half + 4 * y;
          const float4 nl = *reinterpret_cast<const float4*>(&sm.nlse2[s][c0]);
          const float4 dd4 = *reinterpret_cast<const float4*>(&sm.dd[s][c0]);
          const int4 lm = *reinterpret_cast<const int4*>(&sm.lim[s][c0]);
          float a0, a1, a2, a3;
          fma2(__uint_as_float(sv[4 * y]), __uint_as_float(sv[4 * y + 1]), sc2, f32x2(nl.x, nl.y),
               a0, a1);
          fma2(__uint_as_float(sv[4 * y + 2]), __uint_as_float(sv[4 * y + 3]), sc2,
               f32x2(nl.z, nl.w), a2, a3);
          const float p0 = kposv <= lm.x ? ex2(a0) : 0.f;
          const float p1 = kposv <= lm.y ? ex2(a1) : 0.f;
          const float p2 = kposv <= lm.z ? ex2(a2) : 0.f;
          const float p3 = kposv <= lm.w ? ex2(a3) : 0.f;
          pk[2 * y] = pack_bf16x2(p0, p1);
          pk[2 * y + 1] = pack_bf16x2(p2, p3);
          dk2[2 * y] = pack_bf16x2(p0 * (__uint_as_float(pv[4 * y]) - dd4.x),
                                   p1 * (__uint_as_float(pv[4 * y + 1]) - dd4.y));
          dk2[2 * y + 1] = pack_bf16x2(p2 * (__uint_as_float(pv[4 * y + 2]) - dd4.z),
                                       p3 * (__uint_as_float(pv[4 * y + 3]) - dd4.w));
        }
        tmem_st16(scol, pk);
        tmem_st16(scol + 128, dk2);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(sm.p_full[b]));
      }
      if (!ok) break;
      // epilogue: warps 4-7 write dV, warps 8-11 dK (x scale) of their 32 keys
      ok = __all_sync(0xffffffffu, mbar_wait(bar(sm.acc_full), (uint32_t)(nu & 1), abort, kWaitBudget));
      if (!ok) break;
      tc_fence_after();
      float* dst = (half == 0 ? dv : dk) + ((long long)(U.start + min(kpos, U.len - 1)) * Hkv + U.g) * D;
      const float mul = half == 0 ? 1.f : scale;
      const uint32_t acol = tmem + lane_off + 256u + (uint32_t)(half * D);
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t o[32];
        tmem_ld32(acol + cc * 32, o);
        tmem_ld_wait();
        if (kvalid) {
          float4* d4 = reinterpret_cast<float4*>(dst + cc * 32);
#pragma unroll
          for (int x = 0; x < 8; ++x) {
            float4 r = make_float4(__uint_as_float(o[4 * x]) * mul, __uint_as_float(o[4 * x + 1]) * mul,
                                   __uint_as_float(o[4 * x + 2]) * mul,
                                   __uint_as_float(o[4 * x + 3]) * mul);
            if (!first) {  // a later chunk: add to what the earlier ones wrote
              const float4 a = d4[x];
              r.x += a.x;
              r.y += a.y;
              r.z += a.z;
              r.w += a.w;
            }
            d4[x] = r;
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(sm.acc_empty));
      ++nu;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  if (threadIdx.x == 0 && sm.abort_flag) raise_error(plan, kErrTimeout, blockIdx.x);
}

// ---------------------------------------------------------------- host side
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult qr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &qr) ==
            cudaSuccess &&
        qr == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// 3D map over a [T, Hkv, d] bf16 tensor; a box is 128 tokens x 1 head x 64
// dims, landing in shared memory as 128 rows of 128 bytes, 128B-swizzled.
bool make_map(CUtensorMap* m, const void* base, int T, int Hkv, int D) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)Hkv, (cuuint64_t)T};
  cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)Hkv * D * 2};
  cuuint32_t box[3] = {64, 1, (cuuint32_t)kKeys};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2D map over `rows` packed bf16 rows of d; a box is 64 rows x 64 dims,
// landing as 64 rows of 128 bytes, 128B-swizzled.
bool make_packed_map(CUtensorMap* m, const void* base, long long rows, int D) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)D * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)kRows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3D map over the [T, Hq, d] bf16 q or dout; a box is 64 tokens x 1 head x
// 64 dims.
bool make_head_map(CUtensorMap* m, const void* base, int T, int Hq, int D) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)Hq, (cuuint64_t)T};
  cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)Hq * D * 2};
  cuuint32_t box[3] = {64, 1, (cuuint32_t)kRows};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D>
cudaError_t launch(const void* q, const void* k, const void* v, const void* dout, const float* lse,
                   const float* dvec, const Sizes& z, const Workspace& ws, const DkvPack& pk,
                   float* dk, float* dv, float scale, int num_sms, cudaStream_t st) {
  if (pk.cap < 1 || z.entries_max >= (1LL << 31)) return cudaErrorInvalidValue;
  CUtensorMap mk, mv, mqp, mgp, mq3, mg3;
  if (!make_map(&mk, k, z.T, z.Hkv, D) || !make_map(&mv, v, z.T, z.Hkv, D) ||
      !make_packed_map(&mqp, pk.qp, (long long)pk.cap + kRows, D) ||
      !make_packed_map(&mgp, pk.gp, (long long)pk.cap + kRows, D) ||
      !make_head_map(&mq3, q, z.T, z.Hq, D) || !make_head_map(&mg3, dout, z.T, z.Hq, D))
    return cudaErrorInvalidValue;
  const size_t smem = sizeof(DkvSmem<D>) + 1024;
  cudaError_t e = cudaFuncSetAttribute(dkv_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  const auto* qb = static_cast<const __nv_bfloat16*>(q);
  const auto* gb = static_cast<const __nv_bfloat16*>(dout);
  // chunks of packed entries up to the largest possible entry count
  for (long long e_lo = 0, ci = 0; e == cudaSuccess && (ci == 0 || e_lo < z.entries_max);
       e_lo += pk.cap, ++ci) {
    dkv_pack_kernel<D><<<num_sms * 8, 256, 0, st>>>(qb, gb, lse, dvec, ws, pk.qp, pk.gp, pk.ld,
                                                    z.Hkv, z.topk, (int)e_lo, pk.cap);
    if ((e = cudaGetLastError()) != cudaSuccess) break;
    dkv_tc_kernel<D><<<num_sms, kThreads, smem, st>>>(
        mk, mv, mqp, mgp, mq3, mg3, pk.ld, lse, dvec, ws, dk, dv, z.Hq, z.Hkv, z.B,
        scale * 1.4426950408889634f, scale, (int)e_lo, pk.cap, ci == 0 ? 1 : 0);
    e = cudaGetLastError();
  }
  return e;
}

}  // namespace

cudaError_t launch_backward_dkv(const void* q, const void* k, const void* v, const void* dout,
                                const float* lse, const float* dvec, const Sizes& z,
                                const Workspace& ws, const DkvPack& pk, float* dk, float* dv,
                                float scale, int num_sms, cudaStream_t st) {
  if (z.d == 128)
    return launch<128>(q, k, v, dout, lse, dvec, z, ws, pk, dk, dv, scale, num_sms, st);
  return launch<64>(q, k, v, dout, lse, dvec, z, ws, pk, dk, dv, scale, num_sms, st);
}

}  // namespace moba
