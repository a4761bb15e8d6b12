// Backward, query side: dQ of the MoBA forward with the selection held
// fixed, on the 5th-generation tensor cores (tcgen05 + TMEM).
//
// Page cited by title: "同一天，DeepSeek和月之暗面發表了關于改進注意力機制的論文"
// (MoBA write-up), opening list: trainable block-sparse attention (the gate
// passes no gradient).  For a query row r and each block it attends (its
// past blocks and its own block under the causal mask):
//   p_ru = exp(scale q_r.k_u - lse_r),  ds_ru = p_ru (dout_r . v_u - D_r),
//   dq_r(block) = scale sum_u ds_ru k_u,   D_r = dout_r . out_r.
// Each (row, selected block) result goes to the row's partial slot (fp32);
// the slots are summed in ascending block order by a separate pass, so dq is
// the same from run to run.
//
// Work unit: 128 rows -- routed rows of one bucket (block b, kv head g) from
// the scheduler's list, or 128 consecutive tokens of one query head in their
// own block -- against the block's keys, 64 per step (rows = TMEM lanes):
//   S  = Q_rows K_half^T,  dP = dO_rows V_half^T      (SS, K-major operands)
//   dS = exp2(S * scale log2 e - lse_r log2 e) (dP - D_r) under the masks,
//        written back over S as packed bf16,
//   dQ += dS K_half                                    (TS, K_half MN-major).
// Two steps are in flight (TMEM ping-pong): S / dP of step n + 1 and dQ of
// step n run while the dS warps work on step n.  Q and dO stay in TMEM for
// the whole unit as the A operands of S and dP (TS MMAs: only the K / V
// halves are read from shared memory), which frees the staging tile early.
// TMEM columns: S of buffer b at [64 b, 64 b + 64), dP at
// [128 + 64 b, ...), dQ [256, 256 + d), Q [384, 384 + d / 2), dO after it
// (bf16 pairs).  K and V arrive in tiles of 128 keys (two steps each).
//
// Warp roles (12 warps): warp 0 streams K and V tiles with TMA (two-stage
// ring); warp 1 issues the MMAs; warps 2 / 3 gather the unit's Q / dO rows
// (cp.async, 128-byte swizzle) into a staging tile, with the rows' slot,
// causal limit, lse and D; warps 4-11 move the staged rows into TMEM (each
// warp its 32 rows, half of d), compute dS (warps 4-7 keys [0, 32), warps
// 8-11 keys [32, 64) of each step, each warp the 32 rows of its TMEM lane
// quarter) and write the unit's dQ rows out.  The staging tile is free once
// its rows are in TMEM, so the next unit's gather overlaps this unit.  Every
// mbarrier wait is bounded.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "kernels.h"
#include "tc_ptx.cuh"

namespace moba {
namespace {
using namespace tc;

constexpr int kRows = 128;  // rows per unit (TMEM lanes)
constexpr int kKeys = 128;  // keys per K/V tile (two 64-key steps)
constexpr int kStages = 2;  // K/V ring depth (each stage a K and a V tile)
constexpr int kThreads = 384;
constexpr long long kWaitBudget = 4000000000LL;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kQCol = 384;  // TMEM column of Q (dO follows at kQCol + d / 2)

template <int D>
struct DqSmem {
  alignas(1024) __nv_bfloat16 q[kRows * D];   // staged Q rows (then in TMEM: A of S)
  alignas(1024) __nv_bfloat16 g[kRows * D];   // staged dO rows (then in TMEM: A of dP)
  alignas(1024) __nv_bfloat16 kt[kStages][kKeys * D];
  alignas(1024) __nv_bfloat16 vt[kStages][kKeys * D];
  // per row of the unit, double buffered by unit parity: partial slot (-1:
  // padding row), last in-block key it sees, dq row when written directly
  // (-1: through the partial slot), lse * log2(e), D
  int pid[2][kRows], lim[2][kRows], drow[2][kRows];
  float lse2[2][kRows], dd[2][kRows];
  int unit_key0[2], unit_g[2], unit_nkv[2];
  int rowid[2][kRows];  // [gather warp - 2]: row (t * Hq + h) of each row of the unit
  uint64_t kv_full[kStages], kv_empty[kStages];
  uint64_t q_full, q_empty;  // staging tile gathered / moved into TMEM (8 warps)
  uint64_t qt_full;          // the unit's Q and dO are in TMEM (8 warps)
  uint64_t s_full[2], p_full[2];  // [TMEM buffer]
  uint64_t acc_full, acc_empty;
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

__device__ __forceinline__ uint32_t bar(const uint64_t& b) { return smem_addr(&b); }

struct DqUnit {
  int kind;  // 0 = routed rows of a bucket, 1 = own block, -1 = nothing in this chunk
  int key0, g, nkv, lim;
  int e0, e_end;
  int y0, h, slot, len;
};

__device__ __forceinline__ DqUnit decode_dq(int u, int n_past, const Workspace& ws, int Hq, int Hkv,
                                            int topk, int B, int t0, int t1) {
  DqUnit U;
  if (u < n_past) {
    const int2 tile = ws.tiles[u];
    const int b = tile.x;
    if (!MOBA_INDEX_OK(ws.plan,
                       b >= 0 && b < ws.nbk_cap && tile.y >= 0 &&
                           ws.bucket_off[b + 1] <= ws.entries_cap,
                       kSiteDqTile)) {
      U.kind = -1;  // every role skips the unit
      return U;
    }
    const int fb = b / Hkv;
    U.kind = 0;
    U.e0 = tile.y;
    U.e_end = ws.bucket_off[b + 1];
    U.g = b - fb * Hkv;
    U.key0 = ws.full_start[fb];
    U.nkv = (B + kKeys - 1) / kKeys;
    U.lim = B - 1;
    U.y0 = U.h = U.slot = U.len = 0;
    return U;
  }
  const int G = Hq / Hkv;
  const int nu_blk = (B + kRows - 1) / kRows;
  int v = u - n_past;
  const int hh = v % G;
  v /= G;
  const int i = v % nu_blk;
  v /= nu_blk;
  const int g = v % Hkv;
  const int gb = v / Hkv;
  const int len = ws.blk_len[gb];
  const int start = ws.blk_start[gb];
  U.kind = 1;
  U.y0 = i * kRows;
  U.key0 = start;
  U.g = g;
  U.h = g * G + hh;
  U.len = len;
  U.lim = len - 1;
  U.slot = min(topk, ws.blk_j[gb] + 1) - 1;
  const int rows_end = min(len, U.y0 + kRows);
  U.nkv = (rows_end + kKeys - 1) / kKeys;
  U.e0 = U.e_end = 0;
  if (U.y0 >= len || start + U.y0 >= t1 || start + rows_end <= t0) U.kind = -1;
  return U;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    dq_tc_kernel(const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
                 const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ dout,
                 const float* __restrict__ lse, const float* __restrict__ dvec, Workspace ws,
                 float* __restrict__ dq_part, float* __restrict__ dq, int Hq, int Hkv, int topk,
                 int B, int t0, int t1, float scale_log2, float scale) {
  extern __shared__ unsigned char smem_raw[];
  DqSmem<D>& sm = *reinterpret_cast<DqSmem<D>*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  DevPlan* plan = ws.plan;
  if (plan->err != 0) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_past = plan->ntiles;
  const int n_units = n_past + plan->nblk_total * Hq * ((B + kRows - 1) / kRows);
  constexpr uint32_t kRegion = kRows * 128;
  constexpr uint32_t kTileBytes = kKeys * D * 2;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar(sm.kv_full[s]), 1);
      mbar_init(bar(sm.kv_empty[s]), 1);
    }
    mbar_init(bar(sm.q_full), 2);
    mbar_init(bar(sm.q_empty), 8);
    mbar_init(bar(sm.qt_full), 8);
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
      long long j = 0;  // K/V stages filled
      for (int u = blockIdx.x; ok && u < n_units; u += gridDim.x) {
        const DqUnit U = decode_dq(u, n_past, ws, Hq, Hkv, topk, B, t0, t1);
        if (U.kind < 0) continue;
        for (int n = 0; ok && n < U.nkv; ++n, ++j) {
          const int s = (int)(j % kStages);
          if (!(ok = mbar_wait(bar(sm.kv_empty[s]), (uint32_t)((j / kStages) & 1) ^ 1u, abort,
                               kWaitBudget)))
            break;
          mbar_arrive_expect_tx(bar(sm.kv_full[s]), 2 * kTileBytes);
          for (int h = 0; h < D / 64; ++h) {
            tma_load_3d(smem_addr(sm.kt[s]) + h * kRegion, &tmk, bar(sm.kv_full[s]), 64 * h, U.g,
                        U.key0 + n * kKeys);
            tma_load_3d(smem_addr(sm.vt[s]) + h * kRegion, &tmv, bar(sm.kv_full[s]), 64 * h, U.g,
                        U.key0 + n * kKeys);
          }
        }
      }
      if (!ok) {
        int dummy = 0;
        for (long long jj = (j > kStages ? j - kStages : 0); jj < j; ++jj)
          mbar_wait(bar(sm.kv_full[jj % kStages]), (uint32_t)((jj / kStages) & 1), &dummy,
                    kWaitBudget);
      }
    }
  } else if (warp == 2 || warp == 3) {
    // ------------------------------------------------------------ row gather
    const __nv_bfloat16* src = warp == 2 ? q : dout;
    const uint32_t base = smem_addr(warp == 2 ? sm.q : sm.g);
    bool ok = true;
    int k = 0;  // units gathered
    for (int u = blockIdx.x; ok && u < n_units; u += gridDim.x) {
      const DqUnit U = decode_dq(u, n_past, ws, Hq, Hkv, topk, B, t0, t1);
      if (U.kind < 0) continue;
      ok = __all_sync(0xffffffffu, mbar_wait(bar(sm.q_empty), (uint32_t)(k & 1) ^ 1u, abort,
                                             kWaitBudget));
      if (!ok) break;
      const int ib = k & 1;
      // the lane's four rows: every index load first, then the dependent loads
      // and the copies (a cp.async is a compiler barrier)
      long long row[kRows / 32];
      int p_id[kRows / 32], lim[kRows / 32], drow[kRows / 32];
#pragma unroll
      for (int i = 0; i < kRows / 32; ++i) {
        const int r = lane + 32 * i;
        drow[i] = -1;
        if (U.kind == 0) {
          const int e = U.e0 + r;
          int ent = ws.entries[min(e, U.e_end - 1)];
          const bool ok_ = MOBA_INDEX_OK(
              ws.plan, ent >= 0 && ent < (t1 - t0) * Hq * topk, kSiteDqEntry);
          if (!ok_) ent = 0;  // a padding row
          p_id[i] = e < U.e_end && ok_ ? ent : -1;
          lim[i] = U.lim;
          row[i] = (long long)t0 * Hq + ent / topk;
        } else {
          const int tl = U.y0 + r;
          const int tok = U.key0 + min(tl, U.len - 1);
          const bool in = tl < U.len && tok >= t0 && tok < t1;
          p_id[i] = in ? ((tok - t0) * Hq + U.h) * topk + U.slot : -1;
          lim[i] = min(tl, U.len - 1);
          row[i] = (long long)tok * Hq + U.h;
          if (in && U.slot == 0) drow[i] = (int)row[i];  // the row's only slot: straight to dq
        }
      }
      if (warp == 2) {
        float l2[kRows / 32], dv_[kRows / 32];
#pragma unroll
        for (int i = 0; i < kRows / 32; ++i) {
          l2[i] = lse[row[i]] * 1.4426950408889634f;
          dv_[i] = dvec[row[i]];
        }
#pragma unroll
        for (int i = 0; i < kRows / 32; ++i) {
          const int r = lane + 32 * i;
          sm.pid[ib][r] = p_id[i];
          sm.lim[ib][r] = lim[i];
          sm.drow[ib][r] = drow[i];
          sm.lse2[ib][r] = l2[i];
          sm.dd[ib][r] = dv_[i];
        }
      }
      // copies with the 16-byte chunks of a row on consecutive lanes
#pragma unroll
      for (int i = 0; i < kRows / 32; ++i) sm.rowid[warp - 2][lane + 32 * i] = (int)row[i];
      __syncwarp();
#pragma unroll 8
      for (int x = lane; x < kRows * (D / 8); x += 32) {
        const int r = x / (D / 8), cc = x % (D / 8);
        cp_async16(base + (cc >> 3) * kRegion + r * 128 + (((cc & 7) ^ (r & 7)) << 4),
                   src + (long long)sm.rowid[warp - 2][r] * D + cc * 8);
      }
      if (warp == 2 && lane == 0) {
        sm.unit_nkv[ib] = U.nkv;
        sm.unit_key0[ib] = U.key0;
        sm.unit_g[ib] = U.g;
      }
      cp_async_commit_wait_all();
      fence_proxy_async();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(sm.q_full));
      ++k;
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
    constexpr int kStep = 64;                                   // keys per step
    constexpr uint32_t idesc_s = idesc_bf16(128, kStep, 0, 0);  // rows x keys, K = d
    constexpr uint32_t idesc_q = idesc_bf16(128, D, 0, 1);      // rows x d, K = keys
    // step n (global counter jn) uses key half (jn & 1) of K/V tile jn >> 1
    // (ring slot (jn >> 1) % kStages) and TMEM buffer jn & 1
    auto issue_sd = [&](long long jn) -> bool {
      const long long jt = jn >> 1;
      const int s = (int)(jt % kStages);
      const uint32_t b = (uint32_t)(jn & 1);
      if ((jn & 1) == 0 && !wait_all(bar(sm.kv_full[s]), (uint32_t)((jt / kStages) & 1)))
        return false;
      const uint64_t kdesc = sdesc_sw128(smem_addr(sm.kt[s]), 16, 1024);
      const uint64_t vdesc = sdesc_sw128(smem_addr(sm.vt[s]), 16, 1024);
      const uint32_t kh = (uint32_t)(jn & 1) * (kStep * 128);  // byte offset of the key half
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (uint32_t)((kk >> 2) * kRegion + (kk & 3) * 32);
          umma_ts(tmem + 64u * b, tmem + kQCol + 8u * kk, kdesc + ((off + kh) >> 4), idesc_s,
                  kk > 0);
          umma_ts(tmem + 128u + 64u * b, tmem + kQCol + D / 2 + 8u * kk, vdesc + ((off + kh) >> 4),
                  idesc_s, kk > 0);
        }
      }
      __syncwarp();
      commit(sm.s_full[b]);
      return true;
    };
    // dQ += dS K over the step's 64 keys in 4 steps of 16; dS packed bf16,
    // keys [32 h, 32 h + 32) in columns [32 h, 32 h + 16) of the buffer
    auto issue_q = [&](long long jn, bool first) -> bool {
      const long long jt = jn >> 1;
      const int s = (int)(jt % kStages);
      const uint32_t b = (uint32_t)(jn & 1);
      if (!wait_all(bar(sm.p_full[b]), (uint32_t)((jn >> 1) & 1))) return false;
      const uint64_t km = sdesc_sw128(smem_addr(sm.kt[s]), kRegion, 1024);
      const uint64_t kh = (uint64_t)((jn & 1) * (kStep * 128 / 16));
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < kStep / 16; ++kk) {
          const uint32_t acol = 64u * b + (uint32_t)(32 * (kk >> 1) + 8 * (kk & 1));
          umma_ts(tmem + 256u, tmem + acol, km + kh + (uint64_t)(kk * 128), idesc_q,
                  (!first || kk > 0) ? 1u : 0u);
        }
      }
      __syncwarp();
      if (jn & 1) commit(sm.kv_empty[s]);  // both halves of the tile are done
      return true;
    };
    long long j = 0;  // steps (64 keys) issued
    int k = 0;
    for (int u = blockIdx.x; ok && u < n_units; u += gridDim.x) {
      const DqUnit U = decode_dq(u, n_past, ws, Hq, Hkv, topk, B, t0, t1);
      if (U.kind < 0) continue;
      if (!(ok = wait_all(bar(sm.qt_full), (uint32_t)(k & 1)))) break;  // Q, dO in TMEM
      const int nst = 2 * U.nkv;
      if (!(ok = issue_sd(j))) break;
      for (int n = 0; n < nst; ++n, ++j) {
        if (n + 1 < nst && !(ok = issue_sd(j + 1))) break;
        if (n == 0 && !(ok = wait_all(bar(sm.acc_empty), (uint32_t)(k & 1) ^ 1u))) break;
        if (!(ok = issue_q(j, n == 0))) break;
      }
      if (!ok) break;
      commit(sm.acc_full);
      ++k;
    }
    commit(sm.drain);
    int dummy = 0;
    mbar_wait(bar(sm.drain), 0, &dummy, kWaitBudget);
  } else {
    // ------------------------------------------------------------ dS, epilogue
    const int quad = warp & 3;          // TMEM lanes (rows) 32 quad .. 32 quad + 31
    const int half = (warp - 4) >> 2;   // keys [32 half, 32 half + 32) of a step
    const int row = quad * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const uint64_t sc2 = f32x2(scale_log2, scale_log2);
    // moves unit kk's staged Q and dO (the warp's 32 rows, half of d) into
    // TMEM as bf16 pairs, then frees the staging tile
    auto stage_to_tmem = [&](int kk) -> bool {
      if (!__all_sync(0xffffffffu, mbar_wait(bar(sm.q_full), (uint32_t)(kk & 1), abort,
                                             kWaitBudget)))
        return false;
      constexpr int kHalf = D / 16;  // 16-byte pieces in half a row
      uint32_t vq[4 * kHalf], vg[4 * kHalf];
      const char* qs = reinterpret_cast<const char*>(sm.q);
      const char* gs = reinterpret_cast<const char*>(sm.g);
#pragma unroll
      for (int i = 0; i < kHalf; ++i) {
        const int cc = half * kHalf + i;
        const uint32_t off = (cc >> 3) * kRegion + row * 128 + (((cc & 7) ^ (row & 7)) << 4);
        const uint4 a = *reinterpret_cast<const uint4*>(qs + off);
        const uint4 c = *reinterpret_cast<const uint4*>(gs + off);
        vq[4 * i] = a.x, vq[4 * i + 1] = a.y, vq[4 * i + 2] = a.z, vq[4 * i + 3] = a.w;
        vg[4 * i] = c.x, vg[4 * i + 1] = c.y, vg[4 * i + 2] = c.z, vg[4 * i + 3] = c.w;
      }
      const uint32_t qcol = tmem + lane_off + kQCol + (uint32_t)(half * (D / 4));
      if constexpr (D == 128) {
        tmem_st32(qcol, vq);
        tmem_st32(qcol + D / 2, vg);
      } else {
        tmem_st16(qcol, vq);
        tmem_st16(qcol + D / 2, vg);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(bar(sm.q_empty));
        mbar_arrive(bar(sm.qt_full));
      }
      return true;
    };
    auto next_unit = [&](int v) -> int {
      for (; v < n_units; v += gridDim.x)
        if (decode_dq(v, n_past, ws, Hq, Hkv, topk, B, t0, t1).kind >= 0) break;
      return v;
    };
    bool ok = true;
    long long j = 0;
    int k = 0;
    int u = next_unit(blockIdx.x);
    if (u < n_units) ok = stage_to_tmem(0);
    while (ok && u < n_units) {
      const DqUnit U = decode_dq(u, n_past, ws, Hq, Hkv, topk, B, t0, t1);
      const int ib = k & 1;
      int p_id = -1, lim = -1, drow = -1;
      float nlse = 0.f, Dr = 0.f;
      const int nst = 2 * U.nkv;
      for (int n = 0; n < nst; ++n, ++j) {
        const uint32_t b = (uint32_t)(j & 1);
        ok = __all_sync(0xffffffffu, mbar_wait(bar(sm.s_full[b]), (uint32_t)((j >> 1) & 1), abort,
                                               kWaitBudget));
        if (!ok) break;
        tc_fence_after();
        if (n == 0) {  // the unit's row record (gathered before its first S)
          p_id = sm.pid[ib][row];
          lim = p_id >= 0 ? sm.lim[ib][row] : -1;
          drow = sm.drow[ib][row];
          nlse = -sm.lse2[ib][row];
          Dr = sm.dd[ib][row];
        }
        const uint64_t nl2 = f32x2(nlse, nlse);
        // the warp's 32 keys; packed dS lands in the first 16 of its columns
        const uint32_t scol = tmem + lane_off + 64u * b + 32u * half;
        uint32_t sv[32], pv[32];
        tmem_ld32(scol, sv);
        tmem_ld32(scol + 128, pv);
        tmem_ld_wait();
        reg_fence32(sv);
        reg_fence32(pv);
        const int kbase = n * 64 + 32 * half;  // in-block key of column 0
        uint32_t dk2[16];
#pragma unroll
        for (int x = 0; x < 16; ++x) {
          float a0, a1;
          fma2(__uint_as_float(sv[2 * x]), __uint_as_float(sv[2 * x + 1]), sc2, nl2, a0, a1);
          const float p0 = kbase + 2 * x <= lim ? ex2(a0) : 0.f;
          const float p1 = kbase + 2 * x + 1 <= lim ? ex2(a1) : 0.f;
          dk2[x] = pack_bf16x2(p0 * (__uint_as_float(pv[2 * x]) - Dr),
                               p1 * (__uint_as_float(pv[2 * x + 1]) - Dr));
        }
        tmem_st16(scol, dk2);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(sm.p_full[b]));
      }
      if (!ok) break;
      // the next unit's Q and dO into TMEM (this unit's last S / dP are done),
      // so its MMAs can start while this unit's dQ is written out
      const int u_next = next_unit(u + gridDim.x);
      if (u_next < n_units && !(ok = stage_to_tmem(k + 1))) break;
      // epilogue: dims [half * D / 2, (half + 1) * D / 2) of the warp's rows
      ok = __all_sync(0xffffffffu, mbar_wait(bar(sm.acc_full), (uint32_t)(k & 1), abort, kWaitBudget));
      if (!ok) break;
      tc_fence_after();
      float* dst = drow >= 0 ? dq + (long long)drow * D
                             : dq_part + (long long)(p_id < 0 ? 0 : p_id) * D;
      const uint32_t acol = tmem + lane_off + 256u + (uint32_t)(half * (D / 2));
#pragma unroll
      for (int cc = 0; cc < D / 64; ++cc) {
        uint32_t o[32];
        tmem_ld32(acol + cc * 32, o);
        tmem_ld_wait();
        if (p_id >= 0) {
          float4* d4 = reinterpret_cast<float4*>(dst + half * (D / 2) + cc * 32);
#pragma unroll
          for (int x = 0; x < 8; ++x)
            d4[x] = make_float4(__uint_as_float(o[4 * x]) * scale, __uint_as_float(o[4 * x + 1]) * scale,
                                __uint_as_float(o[4 * x + 2]) * scale,
                                __uint_as_float(o[4 * x + 3]) * scale);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(sm.acc_empty));
      ++k;
      u = u_next;
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

template <int D>
cudaError_t launch(const void* q, const void* k, const void* v, const void* dout, const float* lse,
                   const float* dvec, const Sizes& z, const Workspace& ws, float* dq_part,
                   float* dq, int t0, int t1, float scale, int num_sms, cudaStream_t st) {
  CUtensorMap mk, mv;
  if (!make_map(&mk, k, z.T, z.Hkv, D) || !make_map(&mv, v, z.T, z.Hkv, D))
    return cudaErrorInvalidValue;
  const size_t smem = sizeof(DqSmem<D>) + 1024;
  cudaError_t e = cudaFuncSetAttribute(dq_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  dq_tc_kernel<D><<<num_sms, kThreads, smem, st>>>(
      mk, mv, static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(dout), lse,
      dvec, ws, dq_part, dq, z.Hq, z.Hkv, z.topk, z.B, t0, t1, scale * 1.4426950408889634f, scale);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_backward_dq(const void* q, const void* k, const void* v, const void* dout,
                               const float* lse, const float* dvec, const Sizes& z,
                               const Workspace& ws, float* dq_part, float* dq, int t0, int t1,
                               float scale, int num_sms, cudaStream_t st) {
  if (z.d == 128)
    return launch<128>(q, k, v, dout, lse, dvec, z, ws, dq_part, dq, t0, t1, scale, num_sms, st);
  return launch<64>(q, k, v, dout, lse, dvec, z, ws, dq_part, dq, t0, t1, scale, num_sms, st);
}

}  // namespace moba
