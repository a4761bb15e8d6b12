// Block attention on the 5th-generation tensor cores (tcgen05 + TMEM).
//
// Page cited by title: "同一天，DeepSeek和月之暗面發表了關于改進注意力機制的論文"
// (MoBA write-up), section "MoBA：將 MoE 原理應用于注意力機制", step 3: the
// attention output of every KV block with the query tokens routed to it (the
// pages run it with variable-length FlashAttention); and the explainer
// "月球計畫 AI 研究介紹混合區塊注意力 (MoBA)...", section "技術細節與優勢": the
// query's own block is always attended, under the causal mask.
//
// One persistent kernel walks two kinds of work unit (256 rows each, as two
// 128-row tiles that share every K/V tile):
//   * past units: up to 256 gathered (token, head) rows of one bucket (full
//     block b, kv head g) from the scheduler's list, against all B keys of b;
//   * own units: 256 consecutive tokens of one query head inside their own
//     block, against keys 0 .. t of that block (token-level causal mask).
// Units u = blockIdx.x, blockIdx.x + gridDim.x, ... (past units first).
//
// Warp roles (12 warps):
//   warp 0      K/V loader: streams K and V tiles of 128 keys with TMA (3D
//               tensor map over [T, Hkv, d]) into a 4-stage ring.
//   warps 2, 3  Q gather of tile 0 / tile 1: cp.async of the scattered rows
//               into the 128-byte-swizzled K-major layout.
//   warp 1      MMA issuer (one thread): S_t = Q_t K^T (SS form, both
//               K-major) and O_t += P_t V (TS form: P read from TMEM, V
//               MN-major in smem), ping-ponging the two tiles so the tensor
//               cores stay busy while the other tile's softmax runs.
//   warps 4-7   softmax of tile 0, warps 8-11 softmax of tile 1: one row per
//               thread (TMEM lane = row), online softmax in base 2, P written
//               back over S as packed bf16 and handed over in two key halves,
//               so PV on keys [64, 128) runs while the exps of [0, 64) are
//               computed (the second half of the row-max pass stays in
//               registers and is exponentiated first); the running max only
//               moves (and O is rescaled in TMEM) when it grows by more than
//               2^8.
// TMEM columns: S0 [0,128), S1 [128,256), O0 and O1 after them (d each).
// tcgen05.ld/st are warp-collective: every branch around them is warp-uniform.
// Every mbarrier wait is bounded; a wait that gives up raises the abort flag,
// all roles leave their loops, in-flight copies and MMAs are drained, TMEM is
// freed, and the kernel reports MOBA_ERR_TIMEOUT through the error word.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "kernels.h"
#include "tc_ptx.cuh"


namespace moba {
namespace {
using namespace tc;

constexpr int kRows = 128;     // rows per Q tile = TMEM lanes
constexpr int kKeys = 128;     // keys per K/V tile
constexpr int kStages = 4;     // K/V ring depth
constexpr int kThreads = 384;  // 12 warps
constexpr int kUnitRows = 2 * kRows;
constexpr long long kWaitBudget = 4000000000LL;  // clock cycles (~2 s)
// Budget of the waits in the bounded-wait test (moba_debug_attention_wait_test);
// the drain waits keep kWaitBudget.
constexpr long long kTestWaitBudget = 2000000LL;  // ~1 ms
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleThreshold = 8.0f;  // log2 units
// Unit information is published one unit ahead; a buffer is written again
// three units later, when every reader of its previous contents has
// provably moved past them (the gather needs the last QK of the unit in
// between, which needs every P of the unit before it).
constexpr int kInfoBufs = 3;

template <int D>
struct TcSmem {
  alignas(1024) __nv_bfloat16 q[2][kRows * D];
  alignas(1024) __nv_bfloat16 kv[kStages][kKeys * D];
  int qrow[2][kRows];  // gather scratch: q row (t * Hq + h) of each row of tile t
  // per-unit information published by the gather warp of each tile, in
  // kInfoBufs buffers by unit index: K/V tiles of the unit (0 = no more
  // units) and, per row, the partial slot (-1 = padding row) and the last key
  // to keep
  int unit_nkv[2][kInfoBufs];
  int unit_key0[kInfoBufs], unit_g[kInfoBufs];  // first key and kv head (tile 0's gather)
  int2 rowinfo[2][kInfoBufs][kRows];

  uint64_t kv_full[kStages], kv_empty[kStages];
  uint64_t q_full[2], q_empty[2], s_full[2], o_full[2], o_empty[2];
  uint64_t info_full[2][kInfoBufs];  // [tile][unit % kInfoBufs]: unit_nkv / rowinfo written
  uint64_t p_full[2][2];  // [tile][phase]: P of keys [64, 128) / [0, 64) is in TMEM
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

template <int D>
constexpr size_t tc_smem_bytes() {
  return sizeof(TcSmem<D>) + 1024;
}

__device__ __forceinline__ uint32_t bar(const uint64_t& b) { return smem_addr(&b); }


// What one work unit covers.  Every role decodes units the same way.
struct Unit {
  int kind;   // 0 = past (gathered rows), 1 = own block (causal), -1 = nothing to do
  int key0;   // first token of the K/V block
  int g;      // kv head
  int nkv;    // K/V tiles visited
  int lim;    // past: last valid key (B - 1); own: block length - 1
  int e0, e_end;               // past: entry range of the unit
  int y0, h, slot;             // own: first row (block-local token), query head, partial slot
};

__device__ __forceinline__ Unit decode_unit(int u, int n_past, const Workspace& ws, int Hq, int Hkv,
                                            int topk, int B, int t0, int t1, int full) {
  Unit U;
  if (full) {
    // Dense causal attention: the plan cut every sequence into blocks of
    // kUnitRows tokens; unit = one such block x one query head, against every
    // key from the sequence start, latest blocks (the longest units) first.
    const int gb = ws.plan->nblk_total - 1 - u / Hq;
    const int jb = ws.blk_j[gb];
    const int len = ws.blk_len[gb];
    U.kind = 1;
    U.h = u % Hq;
    U.g = U.h / (Hq / Hkv);
    U.y0 = jb * kUnitRows;
    U.key0 = ws.blk_start[gb] - U.y0;
    U.lim = U.y0 + len - 1;
    U.slot = 0;
    U.nkv = (U.y0 + len + kKeys - 1) / kKeys;
    U.e0 = U.e_end = 0;
    return U;
  }
  if (u < n_past) {
    const int2 tile = ws.tiles[u];
    const int b = tile.x;
    if (!MOBA_INDEX_OK(ws.plan,
                       b >= 0 && b < ws.nbk_cap && tile.y >= 0 &&
                           ws.bucket_off[b + 1] <= ws.entries_cap,
                       kSiteAttnTile)) {
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
    U.y0 = U.h = U.slot = 0;
  } else {
    const int G = Hq / Hkv;
    const int nu_blk = (B + kUnitRows - 1) / kUnitRows;
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
    U.y0 = i * kUnitRows;
    U.key0 = start;
    U.g = g;
    U.h = g * G + hh;
    U.lim = len - 1;
    U.slot = min(topk, ws.blk_j[gb] + 1) - 1;
    const int rows_end = min(len, U.y0 + kUnitRows);
    U.nkv = (rows_end + kKeys - 1) / kKeys;
    U.e0 = U.e_end = 0;
    if (U.y0 >= len || start + U.y0 >= t1 || start + rows_end <= t0) U.kind = -1;
  }
  return U;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tmk,
                        const __grid_constant__ CUtensorMap tmv,
                        const __nv_bfloat16* __restrict__ q, Workspace ws, int Hq, int Hkv,
                        int topk, int B, int t0, int t1, float scale_log2, int full,
                        long long budget, int wait_test) {
  extern __shared__ unsigned char smem_raw[];
  TcSmem<D>& sm = *reinterpret_cast<TcSmem<D>*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  DevPlan* plan = ws.plan;
  if (plan->err != 0) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_past = plan->ntiles;
  const int n_units = full ? plan->nblk_total * Hq
                           : n_past + plan->nblk_total * Hq * ((B + kUnitRows - 1) / kUnitRows);
  constexpr uint32_t kTileBytes = kKeys * D * 2;
  constexpr uint32_t kRegion = kRows * 128;  // bytes of one 64-column swizzled region

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar(sm.kv_full[s]), 1);
      mbar_init(bar(sm.kv_empty[s]), 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(bar(sm.q_full[t]), 32);
      mbar_init(bar(sm.q_empty[t]), 1);
      for (int b = 0; b < kInfoBufs; ++b) mbar_init(bar(sm.info_full[t][b]), 32);
      mbar_init(bar(sm.s_full[t]), 1);
      mbar_init(bar(sm.p_full[t][0]), 4);   // the tile's 4 softmax warps
      mbar_init(bar(sm.p_full[t][1]), 4);
      mbar_init(bar(sm.o_full[t]), 1);
      mbar_init(bar(sm.o_empty[t]), 4);
    }
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

  if ((warp == 2 || warp == 3) && wait_test) {
    // Test of the bounded waits: the gather warps publish nothing, so every
    // other role's first wait (for a unit record) runs out before anything is
    // copied or issued, and the kernel must report MOBA_ERR_TIMEOUT.
  } else if (warp == 2 || warp == 3) {
    // ------------------------------------------------------------ Q gather (tile warp - 2)
    // Decodes the units of this CTA one ahead of the MMA and softmax warps:
    // while unit k is being computed, the rows of unit k + 1 are resolved and
    // published (unit_nkv, rowinfo; info_full), then its Q rows are copied as
    // soon as the tile's last QK of unit k has read the previous ones.  A
    // final record with nkv = 0 tells the consumers that no unit is left.
    const int t = warp - 2;
    uint32_t q_empty_par = 1;
    bool ok = true;
    int k = 0;  // units published
    int u = blockIdx.x;
    // resolve the next unit with work at or after u (nkv = 0 when none is left)
    auto publish_next = [&]() {
      Unit U;
      U.kind = -1;
      for (; u < n_units; u += gridDim.x) {
        U = decode_unit(u, n_past, ws, Hq, Hkv, topk, B, t0, t1, full);
        if (U.kind >= 0) break;
      }
      const int buf = k % kInfoBufs;
      if (u < n_units) {
        for (int r = lane; r < kRows; r += 32) {
          int p_id, lim, qr;
          if (U.kind == 0) {
            const int e = U.e0 + t * kRows + r;
            int ent = ws.entries[min(e, U.e_end - 1)];
#ifdef MOBA_DEBUG
            if (ws.poison == 1 && e == U.e0) ent = -1 - ent;  // planted: a slot outside the chunk
#endif
            const bool ent_ok = MOBA_INDEX_OK(
                ws.plan, ent >= 0 && ent < (t1 - t0) * Hq * topk, kSiteAttnEntry);
            if (!ent_ok) ent = 0;  // a padding row
            p_id = e < U.e_end && ent_ok ? ent : -1;
            lim = U.lim;
            qr = t0 * Hq + ent / topk;
          } else {
            const int tl = U.y0 + t * kRows + r;
            const int tok = U.key0 + tl;
            p_id = (tl <= U.lim && tok >= t0 && tok < t1)
                       ? ((tok - t0) * Hq + U.h) * topk + U.slot : -1;
            lim = min(tl, U.lim);
            qr = (U.key0 + min(tl, U.lim)) * Hq + U.h;
          }
          sm.qrow[t][r] = qr;
          sm.rowinfo[t][buf][r] = make_int2(p_id, lim);
        }
        if (lane == 0) {
          sm.unit_nkv[t][buf] = U.nkv;
          if (t == 0) {
            sm.unit_key0[buf] = U.key0;
            sm.unit_g[buf] = U.g;
          }
        }
      } else if (lane == 0) {
        sm.unit_nkv[t][buf] = 0;
      }
      __syncwarp();
      mbar_arrive(bar(sm.info_full[t][buf]));
    };
    publish_next();
    while (ok && u < n_units) {
      ok = __all_sync(0xffffffffu,
                      mbar_wait(bar(sm.q_empty[t]), q_empty_par, abort, budget));
      if (!ok) break;
      q_empty_par ^= 1;
      const uint32_t qt = smem_addr(sm.q[t]);
#pragma unroll 4
      for (int idx = lane; idx < kRows * (D / 8); idx += 32) {
        const int r = idx / (D / 8), c = idx % (D / 8);
        const uint32_t dst = qt + (c >> 3) * kRegion + r * 128 + ((((c & 7) ^ (r & 7))) << 4);
        cp_async16(dst, q + (long long)sm.qrow[t][r] * D + c * 8);
      }
      cp_async_commit_wait_all();
      fence_proxy_async();
      mbar_arrive(bar(sm.q_full[t]));
      __syncwarp();
      ++k;
      u += gridDim.x;
      publish_next();
    }
  } else if (warp == 0) {
    // ------------------------------------------------------------ K/V loader
    long long j = 0;  // K/V tiles issued so far (ring position)
    bool ok = true;
    if (lane == 0) {
      prefetch_tmap(&tmk);
      prefetch_tmap(&tmv);
      // units as the gather warps publish them (the next unit is known while
      // the current one still streams)
      for (int k = 0; ok; ++k) {
        const int buf = k % kInfoBufs;
        if (!(ok = mbar_wait(bar(sm.info_full[0][buf]), (uint32_t)((k / kInfoBufs) & 1), abort,
                             budget)))
          break;
        const int nkv = sm.unit_nkv[0][buf];
        if (nkv == 0) break;
        const int ug = sm.unit_g[buf], ukey0 = sm.unit_key0[buf];
        for (int n = 0; ok && n < nkv; ++n) {
          for (int kind = 0; kind < 2; ++kind) {
            const int slot = (int)(j % kStages);
            const uint32_t par = (uint32_t)((j / kStages) & 1) ^ 1u;
            if (!(ok = mbar_wait(bar(sm.kv_empty[slot]), par, abort, budget))) break;
            mbar_arrive_expect_tx(bar(sm.kv_full[slot]), kTileBytes);
            const uint32_t dst = smem_addr(sm.kv[slot]);
            for (int h = 0; h < D / 64; ++h)
              tma_load_3d(dst + h * kRegion, kind == 0 ? (const void*)&tmk : (const void*)&tmv,
                          bar(sm.kv_full[slot]), 64 * h, ug, ukey0 + n * kKeys);
            ++j;
          }
        }
      }
      if (!ok) {
        // let the copies already issued land before the CTA can exit
        for (long long jj = (j > kStages ? j - kStages : 0); jj < j; ++jj) {
          int dummy = 0;
          mbar_wait(bar(sm.kv_full[jj % kStages]), (uint32_t)((jj / kStages) & 1), &dummy,
                    kWaitBudget);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs this converged, so descriptors and barrier phases are
    // warp-uniform values; one elected lane issues each tcgen05 instruction.
    {
      uint32_t q_full_par[2] = {0, 0}, p_full_par[2] = {0, 0}, o_empty_par[2] = {1, 1};
      long long j = 0;
      bool ok = true;
      constexpr uint32_t idesc_qk = idesc_bf16(128, kKeys, 0, 0);
      constexpr uint32_t idesc_pv = idesc_bf16(128, D, 0, 1);
      auto wait_all = [&](uint32_t b, uint32_t par) -> bool {
        return __all_sync(0xffffffffu, mbar_wait(b, par, abort, budget));
      };
      auto kv_wait = [&](long long jj) -> bool {
        bool r = wait_all(bar(sm.kv_full[jj % kStages]), (uint32_t)((jj / kStages) & 1));
        tc_fence_after();
        return r;
      };
      auto commit = [&](const uint64_t& b) {
        if (elect_one()) umma_commit(bar(b));
        __syncwarp();
      };
      // descriptor start addresses advance in 16-byte units: k-step kk of a
      // K-major tile starts (kk / 4) regions and (kk % 4) * 32 bytes in; k-step
      // kk of the MN-major V tile starts kk * 16 rows of 128 bytes in
      const uint64_t qdesc[2] = {sdesc_sw128(smem_addr(sm.q[0]), 16, 1024),
                                 sdesc_sw128(smem_addr(sm.q[1]), 16, 1024)};
      const uint32_t kv0 = smem_addr(sm.kv[0]);
      constexpr uint32_t kSlotBytes = kKeys * D * 2;
      auto issue_qk = [&](int t, int slot) {
        const uint64_t qd = qdesc[t];
        const uint64_t kd = sdesc_sw128(kv0 + slot * kSlotBytes, 16, 1024);
        const uint32_t dt = tmem + (uint32_t)t * 128u;
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t off = (uint64_t)(((kk >> 2) * kRegion + (kk & 3) * 32) >> 4);
            umma_ss(dt, qd + off, kd + off, idesc_qk, kk > 0);
          }
        }
        __syncwarp();
      };
      // PV over keys [64 * kh, 64 * kh + 64): P of those keys is packed in TMEM
      // columns [64 * kh, 64 * kh + 32) of the tile's S columns.  The softmax
      // hands over key half 1 first (phase 0), then key half 0 (phase 1).
      auto issue_pv = [&](int t, int slot, int phase, bool acc) {
        const int kh = 1 - phase;
        const uint64_t vd = sdesc_sw128(kv0 + slot * kSlotBytes, kRegion, 1024);
        const uint32_t dt = tmem + 256u + (uint32_t)t * D;
        const uint32_t pt = tmem + (uint32_t)t * 128u + 64u * kh;
        if (elect_one()) {
#pragma unroll
          for (int k4 = 0; k4 < 4; ++k4) {
            const int kk = 4 * kh + k4;
            umma_ts(dt, pt + k4 * 8, vd + (uint64_t)(kk * 128), idesc_pv,
                    (acc || phase > 0 || k4 > 0) ? 1u : 0u);
          }
        }
        __syncwarp();
      };
      // The units of the CTA run back to back: the QK of a tile's first step
      // of unit k + 1 is issued right after that tile's last PV of unit k, so
      // the tile ping-pong does not drain at unit boundaries.
      auto unit_nkv = [&](int k, int& nkv) -> bool {
        const int buf = k % kInfoBufs;
        const bool r = wait_all(bar(sm.info_full[0][buf]), (uint32_t)((k / kInfoBufs) & 1));
        nkv = sm.unit_nkv[0][buf];
        return r;
      };
      int k = 0, nkv = 0;
      ok = unit_nkv(0, nkv);
      if (ok && nkv > 0) {
        if (!(ok = kv_wait(j))) nkv = 0;
        const int kslot0 = (int)(j % kStages);
        for (int t = 0; t < 2 && nkv > 0; ++t) {
          if (!(ok = wait_all(bar(sm.q_full[t]), q_full_par[t]))) {
            nkv = 0;
            break;
          }
          q_full_par[t] ^= 1;
          tc_fence_after();
          issue_qk(t, kslot0);
          commit(sm.s_full[t]);
          if (nkv == 1) commit(sm.q_empty[t]);
        }
        if (nkv > 0) {
          commit(sm.kv_empty[kslot0]);
          ++j;
        }
      }
      while (ok && nkv > 0) {
        int nkv_next = 0;
        for (int n = 0; ok && n < nkv; ++n) {
          const long long jv = j;  // V_n; waited for right before its first PV
          const int vslot = (int)(j % kStages);
          ++j;
          const bool last = n + 1 == nkv;
          if (last && !(ok = unit_nkv(k + 1, nkv_next))) break;
          const bool more = !last || nkv_next > 0;  // a QK follows: K_{n+1} or the next unit's K_0
          const int kslot = (int)(j % kStages);
          for (int t = 0; t < 2; ++t) {
            for (int half = 0; half < 2; ++half) {
              if (!(ok = wait_all(bar(sm.p_full[t][half]), p_full_par[t]))) break;
              tc_fence_after();
              if (n == 0 && half == 0) {
                if (!(ok = wait_all(bar(sm.o_empty[t]), o_empty_par[t]))) break;
                o_empty_par[t] ^= 1;
                tc_fence_after();
              }
              if (t == 0 && half == 0 && !(ok = kv_wait(jv))) break;
              issue_pv(t, vslot, half, n > 0);
            }
            if (!ok) break;
            p_full_par[t] ^= 1;
            if (last) commit(sm.o_full[t]);
            if (more) {
              if (last) {  // the next unit's Q tile t
                if (!(ok = wait_all(bar(sm.q_full[t]), q_full_par[t]))) break;
                q_full_par[t] ^= 1;
                tc_fence_after();
              }
              if (t == 0 && !(ok = kv_wait(j))) break;
              issue_qk(t, kslot);
              commit(sm.s_full[t]);
              // the tile's last QK of a unit frees its Q tile for the gather
              if (last ? nkv_next == 1 : n + 2 == nkv) commit(sm.q_empty[t]);
            }
          }
          if (!ok) break;
          commit(sm.kv_empty[vslot]);
          if (more) {
            commit(sm.kv_empty[kslot]);
            ++j;
          }
        }
        ++k;
        nkv = nkv_next;
      }
      // every MMA issued must finish before TMEM is freed
      commit(sm.drain);
      int dummy = 0;
      mbar_wait(bar(sm.drain), 0, &dummy, kWaitBudget);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax + epilogue
    const int t = (warp - 4) >> 2;
    const int row = (warp & 3) * 32 + lane;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t s_addr = tmem + lane_off + (uint32_t)t * 128u;
    const uint32_t o_addr = tmem + lane_off + 256u + (uint32_t)t * D;
    uint32_t s_par = 0, o_par = 0;
    bool ok = true;
    for (int k = 0; ok; ++k) {
      const int buf = k % kInfoBufs;
      ok = __all_sync(0xffffffffu, mbar_wait(bar(sm.info_full[t][buf]), (uint32_t)((k / kInfoBufs) & 1),
                                             abort, budget));
      if (!ok) break;
      const int nkv = sm.unit_nkv[t][buf];
      if (nkv == 0) break;
      const int2 ri = sm.rowinfo[t][buf][row];
      const int p_id = ri.x, lim = ri.y;
      float m_used = -INFINITY, l = 0.f;
      for (int n = 0; n < nkv; ++n) {
        ok = __all_sync(0xffffffffu, mbar_wait(bar(sm.s_full[t]), s_par, abort, budget));
        if (!ok) break;
        s_par ^= 1;
        tc_fence_after();
        const int keep = lim - n * kKeys;  // last key column to keep (causal or short block)
        // pass 1: row max, streaming S from TMEM 64 columns at a time (the
        // scores are never all live in registers); key half 1 stays in sv
        uint32_t sv[64];
        float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
        auto load_half = [&](int hh) {
          tmem_ld32(s_addr + hh * 64, sv);
          tmem_ld32(s_addr + hh * 64 + 32, sv + 32);
        };
        auto wait_half = [&]() {
          tmem_ld_wait();
          reg_fence32(sv);
          reg_fence32(sv + 32);
        };
        auto mask_half = [&](int hh) {
          if (keep < hh * 64 + 63) {
#pragma unroll
            for (int c = 0; c < 64; ++c)
              if (hh * 64 + c > keep) sv[c] = __float_as_uint(-INFINITY);
          }
        };
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          load_half(hh);
          wait_half();
          mask_half(hh);
#pragma unroll
          for (int c = 0; c < 64; c += 2)
            mx4[(c >> 1) & 3] = max3(mx4[(c >> 1) & 3], __uint_as_float(sv[c]), __uint_as_float(sv[c + 1]));
        }
        const float mxs = fmaxf(max3(mx4[0], mx4[1], mx4[2]), mx4[3]) * scale_log2;
        float alpha = 1.f;
        if (n == 0) {
          m_used = mxs;
        } else if (mxs > m_used + kRescaleThreshold) {
          // the running max only moves when the row max grows by more than 2^8
          alpha = ex2(m_used - mxs);
          m_used = mxs;
          l *= alpha;
        }
        // pass 2: P = exp2(s * scale_log2 - m) as bf16 pairs, key half 1 first
        // (still in registers), then key half 0 (read again).  P of key half h
        // goes to columns [64 h, 64 h + 32), which hold scores of that half
        // already in registers, and is handed to the MMA thread half by half.
        // Packed pairs: (s0, s1) * scale_log2 - m in one f32x2 FMA, the row sum
        // in paired accumulators.
        const uint64_t sc2 = f32x2(scale_log2, scale_log2);
        const uint64_t nm2 = f32x2(-m_used, -m_used);
        float ls[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        auto exp_half = [&](int hh) {
#pragma unroll
          for (int cc = 0; cc < 2; ++cc) {
            uint32_t pk[16];
#pragma unroll
            for (int x = 0; x < 16; ++x) {
              float x0, x1;
              fma2(__uint_as_float(sv[cc * 32 + 2 * x]), __uint_as_float(sv[cc * 32 + 2 * x + 1]),
                   sc2, nm2, x0, x1);
              const float a = ex2(x0);
              const float b = ex2(x1);
              add2(ls[2 * (x & 3)], ls[2 * (x & 3) + 1], a, b);
              pk[x] = pack_bf16x2(a, b);
            }
            tmem_st16(s_addr + hh * 64 + cc * 16, pk);
          }
        };
        auto hand_over = [&](int phase) {
          tmem_st_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(sm.p_full[t][phase]));
        };
        exp_half(1);
        if (__any_sync(0xffffffffu, alpha != 1.f)) {  // warp-uniform: tcgen05.ld/st below
          // rescale O in TMEM before any PV of this step (the PV of the previous
          // step has completed: it was issued before the QK that filled S)
#pragma unroll 1
          for (int c = 0; c < D / 32; ++c) {
            uint32_t o[32];
            tmem_ld32(o_addr + c * 32, o);
            tmem_ld_wait();
#pragma unroll
            for (int x = 0; x < 32; ++x) o[x] = __float_as_uint(__uint_as_float(o[x]) * alpha);
            tmem_st32(o_addr + c * 32, o);
          }
        }
        load_half(0);  // in flight while the stores of P (key half 1) settle
        hand_over(0);
        wait_half();
        mask_half(0);
        exp_half(0);
        hand_over(1);
        l += ((ls[0] + ls[1]) + (ls[2] + ls[3])) + ((ls[4] + ls[5]) + (ls[6] + ls[7]));
      }
      if (!ok) break;
      // epilogue: O / l -> bf16 partial slot, lse
      ok = __all_sync(0xffffffffu, mbar_wait(bar(sm.o_full[t]), o_par, abort, budget));
      if (!ok) break;
      o_par ^= 1;
      tc_fence_after();
      const float inv = 1.f / l;
      __nv_bfloat16* dst = ws.part_o + (long long)(p_id < 0 ? 0 : p_id) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(o_addr + c * 32, o);
        tmem_ld_wait();
        if (p_id >= 0) {
          uint32_t w[16];
#pragma unroll
          for (int x = 0; x < 16; ++x)
            w[x] = pack_bf16x2(__uint_as_float(o[2 * x]) * inv, __uint_as_float(o[2 * x + 1]) * inv);
          uint4* d4 = reinterpret_cast<uint4*>(dst + c * 32);
#pragma unroll
          for (int x = 0; x < 4; ++x) d4[x] = make_uint4(w[4 * x], w[4 * x + 1], w[4 * x + 2], w[4 * x + 3]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(sm.o_empty[t]));
      if (p_id >= 0) ws.part_lse[p_id] = (m_used + __log2f(l)) * 0.6931471805599453f;
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
bool make_kv_map(CUtensorMap* m, const void* base, int T, int Hkv, int D) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)Hkv, (cuuint64_t)T};
  cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)Hkv * D * 2};
  cuuint32_t box[3] = {64, 1, (cuuint32_t)kKeys};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int D>
cudaError_t launch_tc(const void* q, const void* k, const void* v, const Sizes& z,
                      const Workspace& ws, int t0, int t1, float scale_log2, int full, int num_sms,
                      cudaStream_t st) {
  CUtensorMap mk, mv;
  if (!make_kv_map(&mk, k, z.T, z.Hkv, D) || !make_kv_map(&mv, v, z.T, z.Hkv, D))
    return cudaErrorInvalidValue;
  const size_t smem = tc_smem_bytes<D>();
  cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem);
  if (e != cudaSuccess) return e;
  const int grid = num_sms;
  const int wait_test = attn_wait_test();
  attn_tc_kernel<D><<<grid, kThreads, smem, st>>>(
      mk, mv, static_cast<const __nv_bfloat16*>(q), ws, z.Hq, z.Hkv, z.topk, z.B, t0, t1,
      scale_log2, full, wait_test ? kTestWaitBudget : kWaitBudget, wait_test);
  return cudaGetLastError();
}

}  // namespace

int attn_unit_rows() { return kUnitRows; }

namespace {
int g_attn_wait_test = 0;
}
void set_attn_wait_test(int on) { g_attn_wait_test = on ? 1 : 0; }
int attn_wait_test() { return g_attn_wait_test; }

cudaError_t launch_attn(const void* q, const void* k, const void* v, const Sizes& z,
                        const Workspace& ws, int t0, int t1, float scale_log2, int num_sms,
                        cudaStream_t st) {
  if (z.d == 128) return launch_tc<128>(q, k, v, z, ws, t0, t1, scale_log2, 0, num_sms, st);
  return launch_tc<64>(q, k, v, z, ws, t0, t1, scale_log2, 0, num_sms, st);
}

cudaError_t launch_attn_full(const void* q, const void* k, const void* v, const Sizes& z,
                             const Workspace& ws, float scale_log2, int num_sms, cudaStream_t st) {
  if (z.d == 128) return launch_tc<128>(q, k, v, z, ws, 0, z.T, scale_log2, 1, num_sms, st);
  return launch_tc<64>(q, k, v, z, ws, 0, z.T, scale_log2, 1, num_sms, st);
}

}  // namespace moba
