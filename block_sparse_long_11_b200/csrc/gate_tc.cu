// Gate on the tensor cores: block scores q . Kbar with tcgen05, top-k on the
// CUDA cores straight from TMEM.
//
// Pages cited by title:
//  [W] "同一天，DeepSeek和月之暗面發表了關于改進注意力機制的論文", section
//      "MoBA：將 MoE 原理應用于注意力機制": parameter-free top-k gate, step 1
//      (assign query tokens to KV blocks under the causal mask).
//  [E] "月球計畫 AI 研究介紹混合區塊注意力 (MoBA)...", section "技術細節與優勢":
//      affinity of the query with an aggregated representation (the mean) of
//      each block's keys; the best blocks are kept; the own block is always in.
//
// Scores.  Kbar is split as hi = bf16(Kbar), lo = bf16(Kbar - hi) (residual
// below 2^-18 |Kbar|), and S = Q hi^T + Q lo^T accumulates in fp32 in TMEM:
// near-fp32 scores from bf16 MMAs (q itself is exact in bf16).
//
// Selection of the topk - 1 best past blocks per row (score descending, ties
// to the lower index), without moving indices around:
//   pass 1: a branch-free max/min network keeps the topk - 1 largest VALUES;
//           tau = the smallest of them;
//   pass 2: scan the scores again in index order and emit every block with
//           s > tau, then blocks with s == tau (lowest index first) until
//           topk - 1 are out.  The result is already ascending; the own block
//           j is appended last.
// With at most 256 past blocks (scores stay in TMEM), pass 1 first takes the
// maxima of 32 interleaved groups of blocks, whose (topk - 1)-th largest,
// tau0, bounds tau from below; the scores >= tau0 (about topk of them for
// random scores) go with their block indices into a short list in shared
// memory, in block order; pass 1 proper and pass 2 then run over the list
// only.  A warp with a row whose list overflows (many equal scores) runs
// both passes over all scores instead.  Beyond 256 past blocks the chunks
// are recomputed for pass 2, and the passes change: pass 1 keeps only the
// group maxima, and pass 2 runs only the scores above tau0 through a sorted
// list carrying indices.
//
// Work tile: 128 consecutive tokens of one query head inside one block (all
// rows share j and the kv head).  Warp roles: warp 0 loads Q tiles and Kbar
// chunks of 128 blocks with TMA; warp 1 (one thread) issues the MMAs; warps
// 4-7 and 8-11 are two top-k warpgroups taking tiles in turn, each owning 256
// TMEM columns (two score buffers of 128 blocks).  Waits are bounded as in the
// attention kernel.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "kernels.h"
#include "tc_ptx.cuh"

namespace moba {
namespace {
using namespace tc;

constexpr int kRows = 128;      // tokens per tile
constexpr int kChunk = 128;     // past blocks per score chunk
constexpr int kCand = 24;       // candidate list per row (at most 256 past blocks)
constexpr int kThreads = 384;
constexpr long long kWaitBudget = 4000000000LL;

template <int D>
struct GateSmem {
  alignas(1024) __nv_bfloat16 q[2][kRows * D];            // Q ring
  alignas(1024) __nv_bfloat16 kb[2][2][kChunk * D];       // Kbar ring: [stage][hi, lo]
  // per row of each top-k warpgroup: the scores above the lower bound tau0
  // and their block indices, in block order ([warpgroup][entry][row])
  float cand_v[2][kCand][kRows];
  uint8_t cand_i[2][kCand][kRows];
  uint64_t q_full[2], q_empty[2], kb_full[2], kb_empty[2];
  uint64_t sc_full[2][2], sc_empty[2][2];                 // [warpgroup][buffer]
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

struct Tile {
  int kind;    // 0 = scored, 1 = trivial (every block 0..j), -1 = nothing
  int gb, g, h, y0, len, start, j, fbase;
};

__device__ __forceinline__ Tile decode_tile(int u, const Workspace& ws, int Hq, int Hkv, int B,
                                            int topk) {
  const int G = Hq / Hkv;
  const int nty = (B + kRows - 1) / kRows;
  Tile T;
  int v = u;
  const int hh = v % G;
  v /= G;
  const int y = v % nty;
  v /= nty;
  T.g = v % Hkv;
  T.gb = v / Hkv;
  T.h = T.g * G + hh;
  T.y0 = y * kRows;
  T.len = ws.blk_len[T.gb];
  T.start = ws.blk_start[T.gb];
  T.j = ws.blk_j[T.gb];
  T.fbase = ws.blk_fullbase[T.gb];
  T.kind = T.y0 >= T.len ? -1 : (T.j + 1 <= topk ? 1 : 0);
  return T;
}

__device__ __forceinline__ uint32_t bar(const uint64_t& b) { return smem_addr(&b); }

template <int D, int MAXK>
__global__ void __launch_bounds__(kThreads, 1)
    gate_tc_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmh,
                   const __grid_constant__ CUtensorMap tml, Workspace ws, int32_t* __restrict__ idx,
                   int Hq, int Hkv, int B, int topk) {
  extern __shared__ unsigned char smem_raw[];
  GateSmem<D>& sm = *reinterpret_cast<GateSmem<D>*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  DevPlan* plan = ws.plan;
  if (plan->err != 0) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_tiles = plan->nblk_total * Hq * ((B + kRows - 1) / kRows);
  constexpr uint32_t kRegion = 128 * 128;  // one 64-column swizzled region of 128 rows
  constexpr uint32_t kQBytes = kRows * D * 2;
  constexpr uint32_t kKbBytes = 2 * kChunk * D * 2;

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(sm.q_full[s]), 1);
      mbar_init(bar(sm.q_empty[s]), 1);
      mbar_init(bar(sm.kb_full[s]), 1);
      mbar_init(bar(sm.kb_empty[s]), 1);
      for (int b = 0; b < 2; ++b) {
        mbar_init(bar(sm.sc_full[s][b]), 1);
        mbar_init(bar(sm.sc_empty[s][b]), kRows);
      }
    }
    mbar_init(bar(sm.drain), 1);
    sm.abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_addr(&sm.tmem_base), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  volatile int* abort = &sm.abort_flag;

  if (warp == 0) {
    // ------------------------------------------------------------ loader
    if (lane == 0) {
      prefetch_tmap(&tmq);
      prefetch_tmap(&tmh);
      prefetch_tmap(&tml);
      long long nq = 0, nk = 0;
      bool ok = true;
      for (int u = blockIdx.x; ok && u < n_tiles; u += gridDim.x) {
        const Tile T = decode_tile(u, ws, Hq, Hkv, B, topk);
        if (T.kind != 0) continue;
        const int slot = (int)(nq & 1);
        if (!(ok = mbar_wait(bar(sm.q_empty[slot]), (uint32_t)((nq >> 1) & 1) ^ 1u, abort,
                             kWaitBudget)))
          break;
        mbar_arrive_expect_tx(bar(sm.q_full[slot]), kQBytes);
        for (int r = 0; r < D / 64; ++r)
          tma_load_3d(smem_addr(sm.q[slot]) + r * kRegion, &tmq, bar(sm.q_full[slot]), 64 * r, T.h,
                      T.start + T.y0);
        ++nq;
        const int nch = (T.j + kChunk - 1) / kChunk;
        const int jobs = nch <= 2 ? nch : 2 * nch;
        for (int m = 0; ok && m < jobs; ++m) {
          const int c = m % nch;
          const int ks = (int)(nk & 1);
          if (!(ok = mbar_wait(bar(sm.kb_empty[ks]), (uint32_t)((nk >> 1) & 1) ^ 1u, abort,
                               kWaitBudget)))
            break;
          mbar_arrive_expect_tx(bar(sm.kb_full[ks]), kKbBytes);
          for (int r = 0; r < D / 64; ++r) {
            tma_load_3d(smem_addr(sm.kb[ks][0]) + r * kRegion, &tmh, bar(sm.kb_full[ks]), 64 * r,
                        T.g, T.fbase + c * kChunk);
            tma_load_3d(smem_addr(sm.kb[ks][1]) + r * kRegion, &tml, bar(sm.kb_full[ks]), 64 * r,
                        T.g, T.fbase + c * kChunk);
          }
          ++nk;
        }
      }
      if (!ok) {  // let issued copies land before exit
        int dummy = 0;
        for (long long i = (nq > 2 ? nq - 2 : 0); i < nq; ++i)
          mbar_wait(bar(sm.q_full[i & 1]), (uint32_t)((i >> 1) & 1), &dummy, kWaitBudget);
        for (long long i = (nk > 2 ? nk - 2 : 0); i < nk; ++i)
          mbar_wait(bar(sm.kb_full[i & 1]), (uint32_t)((i >> 1) & 1), &dummy, kWaitBudget);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(128, kChunk, 0, 0);
      long long nq = 0, nk = 0, ntile = 0;
      uint32_t sc_empty_par[2][2] = {{1, 1}, {1, 1}};
      bool ok = true;
      for (int u = blockIdx.x; ok && u < n_tiles; u += gridDim.x) {
        const Tile T = decode_tile(u, ws, Hq, Hkv, B, topk);
        if (T.kind < 0) continue;
        const int wg = (int)(ntile & 1);
        ++ntile;
        if (T.kind != 0) continue;
        const int qs = (int)(nq & 1);
        if (!(ok = mbar_wait(bar(sm.q_full[qs]), (uint32_t)((nq >> 1) & 1), abort, kWaitBudget)))
          break;
        tc_fence_after();
        const int nch = (T.j + kChunk - 1) / kChunk;
        const int jobs = nch <= 2 ? nch : 2 * nch;
        for (int m = 0; ok && m < jobs; ++m) {
          const int b = nch <= 2 ? m : (m & 1);
          const int ks = (int)(nk & 1);
          if (!(ok = mbar_wait(bar(sm.kb_full[ks]), (uint32_t)((nk >> 1) & 1), abort, kWaitBudget)))
            break;
          if (!(ok = mbar_wait(bar(sm.sc_empty[wg][b]), sc_empty_par[wg][b], abort, kWaitBudget)))
            break;
          sc_empty_par[wg][b] ^= 1;
          tc_fence_after();
          const uint32_t d_tmem = tmem + (uint32_t)wg * 256u + (uint32_t)b * 128u;
          const uint32_t qa = smem_addr(sm.q[qs]);
#pragma unroll
          for (int part = 0; part < 2; ++part) {
            const uint32_t ka = smem_addr(sm.kb[ks][part]);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t off = (kk >> 2) * kRegion + (kk & 3) * 32;
              umma_ss(d_tmem, sdesc_sw128(qa + off, 16, 1024), sdesc_sw128(ka + off, 16, 1024),
                      idesc, (part > 0 || kk > 0) ? 1u : 0u);
            }
          }
          umma_commit(bar(sm.sc_full[wg][b]));
          umma_commit(bar(sm.kb_empty[ks]));
          ++nk;
        }
        if (!ok) break;
        umma_commit(bar(sm.q_empty[qs]));
        ++nq;
      }
      umma_commit(bar(sm.drain));
      int dummy = 0;
      mbar_wait(bar(sm.drain), 0, &dummy, kWaitBudget);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ top-k warpgroups
    const int wg = (warp - 4) >> 2;
    const int row = (warp & 3) * 32 + lane;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const int km1 = topk - 1;
    uint32_t sc_full_par[2] = {0, 0};
    long long ntile = 0;
    bool ok = true;
    for (int u = blockIdx.x; ok && u < n_tiles; u += gridDim.x) {
      const Tile T = decode_tile(u, ws, Hq, Hkv, B, topk);
      if (T.kind < 0) continue;
      const bool mine = (ntile & 1) == wg;
      ++ntile;
      if (!mine) continue;
      const int tl = T.y0 + row;
      const bool valid = tl < T.len;
      int32_t* out = idx + ((long long)(T.start + (valid ? tl : 0)) * Hq + T.h) * topk;
      if (T.kind == 1) {
        if (valid)
          for (int p = 0; p < topk; ++p) out[p] = p <= T.j ? p : -1;
        continue;
      }
      const int j = T.j;
      const int nch = (j + kChunk - 1) / kChunk;
      // wait for the score buffer of job m, read 32 columns at a time
      auto wait_buf = [&](int b) -> bool {
        bool r = __all_sync(0xffffffffu, mbar_wait(bar(sm.sc_full[wg][b]), sc_full_par[b], abort,
                                                   kWaitBudget));
        sc_full_par[b] ^= 1;
        tc_fence_after();
        return r;
      };
      auto release_buf = [&](int b) {
        tc_fence_before();
        mbar_arrive(bar(sm.sc_empty[wg][b]));
      };
      if (nch > 2) {
        // More than 256 past blocks: the score chunks are computed twice
        // anyway, so pass 1 only takes the maxima of 32 interleaved groups
        // (column x of every 32-column load); the km1-th largest of them,
        // tau0, is a lower bound on the km1-th largest score (km1 groups,
        // each holding a score >= tau0).  Pass 2 feeds only scores >= tau0,
        // in ascending block order, into a sorted list that carries the
        // indices (strict comparisons: an equal later score never passes an
        // earlier one), so the list ends as the exact selection.
        float gm[32];
#pragma unroll
        for (int x = 0; x < 32; ++x) gm[x] = -INFINITY;
        for (int c = 0; ok && c < nch; ++c) {
          const int b = c & 1;
          if (!(ok = wait_buf(b))) break;
          const uint32_t base = tmem + lane_off + (uint32_t)wg * 256u + (uint32_t)b * 128u;
          const int ncol = min(kChunk, j - c * kChunk);
#pragma unroll 1
          for (int sub = 0; sub < kChunk / 32; ++sub) {
            if (sub * 32 >= ncol) break;
            uint32_t s[32];
            tmem_ld32(base + sub * 32, s);
            tmem_ld_wait();
            const int nvalid = ncol - sub * 32;
#pragma unroll
            for (int x = 0; x < 32; ++x)
              if (x < nvalid) gm[x] = fmaxf(gm[x], __uint_as_float(s[x]));
          }
          release_buf(b);
        }
        if (!ok) break;
        float a[MAXK];
#pragma unroll
        for (int p = 0; p < MAXK; ++p) a[p] = -INFINITY;
#pragma unroll
        for (int x = 0; x < 32; x += 2) {
          const float hi = fmaxf(gm[x], gm[x + 1]), lo = fminf(gm[x], gm[x + 1]);
          float na[MAXK];
          na[0] = fmaxf(a[0], hi);
          if (MAXK > 1) na[1 % MAXK] = max3(a[1 % MAXK], fminf(a[0], hi), lo);
#pragma unroll
          for (int p = 2; p < MAXK; ++p) na[p] = max3(a[p], fminf(a[p - 1], hi), fminf(a[p - 2], lo));
#pragma unroll
          for (int p = 0; p < MAXK; ++p)
            if (p < km1) a[p] = na[p];
        }
        float tau0 = a[0];
#pragma unroll
        for (int p = 0; p < MAXK; ++p)
          if (p < km1) tau0 = a[p];
        float av[MAXK];
        int ai[MAXK];
#pragma unroll
        for (int p = 0; p < MAXK; ++p) {
          av[p] = -INFINITY;
          ai[p] = 0x7fffffff;
        }
        for (int c = 0; ok && c < nch; ++c) {
          const int b = (nch + c) & 1;  // job nch + c
          if (!(ok = wait_buf(b))) break;
          const uint32_t base = tmem + lane_off + (uint32_t)wg * 256u + (uint32_t)b * 128u;
          const int ncol = min(kChunk, j - c * kChunk);
#pragma unroll 1
          for (int sub = 0; sub < kChunk / 32; ++sub) {
            if (sub * 32 >= ncol) break;
            uint32_t s[32];
            tmem_ld32(base + sub * 32, s);
            tmem_ld_wait();
            const int nvalid = ncol - sub * 32;
            float thr = av[0];
#pragma unroll
            for (int p = 0; p < MAXK; ++p)
              if (p < km1) thr = av[p];  // the current km1-th best
            uint32_t mask = 0;
#pragma unroll
            for (int x = 0; x < 32; ++x) {
              const float v = __uint_as_float(s[x]);
              mask |= (x < nvalid && v >= tau0 && v > thr) ? (1u << x) : 0u;
            }
            while (__any_sync(0xffffffffu, mask != 0u)) {
              const int x = mask ? __ffs(mask) - 1 : 0;
              float v = -INFINITY;
#pragma unroll
              for (int y = 0; y < 32; ++y) v = (y == x) ? __uint_as_float(s[y]) : v;
              if (!mask) v = -INFINITY;
              mask &= mask - 1u;
              const int bi = c * kChunk + sub * 32 + x;
#pragma unroll
              for (int p = MAXK - 1; p >= 1; --p) {
                if (p < km1) {
                  const bool up = v > av[p - 1], in = v > av[p];
                  const float nv = up ? av[p - 1] : (in ? v : av[p]);
                  const int ni = up ? ai[p - 1] : (in ? bi : ai[p]);
                  av[p] = nv;
                  ai[p] = ni;
                }
              }
              if (v > av[0]) {
                av[0] = v;
                ai[0] = bi;
              }
            }
          }
          release_buf(b);
        }
        if (!ok) break;
        if (valid) {
          // ascending block order: each winner's rank among the winners
#pragma unroll
          for (int p = 0; p < MAXK; ++p) {
            if (p < km1) {
              int rank = 0;
#pragma unroll
              for (int o = 0; o < MAXK; ++o)
                if (o < km1) rank += ai[o] < ai[p] ? 1 : 0;
              out[rank] = min(ai[p], j - 1);  // (j - 1 only if the scores held NaNs)
            }
          }
          out[km1] = j;
        }
        continue;
      }
      // two sorted candidates hi >= lo merged into the descending list a
      // (every position from the old list: no serial chain)
      auto merge_pair = [&](float* a, float v0, float v1) {
        const float hi = fmaxf(v0, v1), lo = fminf(v0, v1);
        float na[MAXK];
        na[0] = fmaxf(a[0], hi);
        if (MAXK > 1) na[1 % MAXK] = max3(a[1 % MAXK], fminf(a[0], hi), lo);
#pragma unroll
        for (int p = 2; p < MAXK; ++p) na[p] = max3(a[p], fminf(a[p - 1], hi), fminf(a[p - 2], lo));
#pragma unroll
        for (int p = 0; p < MAXK; ++p)
          if (p < km1) a[p] = na[p];
      };
      bool acquired = false;  // score buffers already waited for by the list path
      if (nch <= 2) {
        // pass 1a: the maxima of 32 interleaved groups (column x of every
        // 32-column load); their km1-th largest, tau0, is at most tau
        float gm[32];
#pragma unroll
        for (int x = 0; x < 32; ++x) gm[x] = -INFINITY;
        for (int c = 0; ok && c < nch; ++c) {
          if (!(ok = wait_buf(c))) break;
          const uint32_t base = tmem + lane_off + (uint32_t)wg * 256u + (uint32_t)c * 128u;
          const int ncol = min(kChunk, j - c * kChunk);
#pragma unroll 1
          for (int sub = 0; sub < kChunk / 32; ++sub) {
            if (sub * 32 >= ncol) break;
            uint32_t s[32];
            tmem_ld32(base + sub * 32, s);
            tmem_ld_wait();
            const int nvalid = ncol - sub * 32;
#pragma unroll
            for (int x = 0; x < 32; ++x)
              if (x < nvalid) gm[x] = fmaxf(gm[x], __uint_as_float(s[x]));
          }
        }
        if (!ok) break;
        acquired = true;
        float g[MAXK];
#pragma unroll
        for (int p = 0; p < MAXK; ++p) g[p] = -INFINITY;
#pragma unroll
        for (int x = 0; x < 32; x += 2) merge_pair(g, gm[x], gm[x + 1]);
        float tau0 = g[0];
#pragma unroll
        for (int p = 0; p < MAXK; ++p)
          if (p < km1) tau0 = g[p];
        // pass 1b: every score >= tau0, with its block, into the row's list
        int n = 0;
        for (int c = 0; c < nch; ++c) {
          const uint32_t base = tmem + lane_off + (uint32_t)wg * 256u + (uint32_t)c * 128u;
          const int ncol = min(kChunk, j - c * kChunk);
#pragma unroll 1
          for (int sub = 0; sub < kChunk / 32; ++sub) {
            if (sub * 32 >= ncol) break;
            uint32_t s[32];
            tmem_ld32(base + sub * 32, s);
            tmem_ld_wait();
            const int nvalid = ncol - sub * 32;
#pragma unroll
            for (int x = 0; x < 32; ++x) {
              const float v = __uint_as_float(s[x]);
              if (x < nvalid && v >= tau0) {
                if (n < kCand) {
                  sm.cand_v[wg][n][row] = v;
                  sm.cand_i[wg][n][row] = (uint8_t)(c * kChunk + sub * 32 + x);
                }
                ++n;
              }
            }
          }
        }
        if (!__any_sync(0xffffffffu, n > kCand)) {
          // pass 1 and pass 2 over the list (it holds every score >= tau)
          float a[MAXK];
#pragma unroll
          for (int p = 0; p < MAXK; ++p) a[p] = -INFINITY;
#pragma unroll 1
          for (int i = 0; i < n; i += 2)
            merge_pair(a, sm.cand_v[wg][i][row],
                       i + 1 < n ? sm.cand_v[wg][i + 1][row] : -INFINITY);
          float tau = a[0];
          int gt = 0;
#pragma unroll
          for (int p = 0; p < MAXK; ++p)
            if (p < km1) tau = a[p];
#pragma unroll
          for (int p = 0; p < MAXK; ++p)
            if (p < km1 && a[p] > tau) ++gt;
          int need_eq = km1 - gt;
          int cnt = 0;
#pragma unroll 1
          for (int i = 0; i < n; ++i) {
            const float v = sm.cand_v[wg][i][row];
            bool take = v > tau || (v == tau && need_eq > 0);
            if (take && !(v > tau)) --need_eq;
            take = take && cnt < km1;
            if (take && valid) out[cnt] = sm.cand_i[wg][i][row];
            cnt += take ? 1 : 0;
          }
          for (int b = 0; b < nch; ++b) release_buf(b);
          if (valid) out[km1] = j;
          continue;
        }
        // a row of this warp holds more than kCand scores >= tau0 (many equal
        // scores): both passes over every score
      }
      float a[MAXK];
#pragma unroll
      for (int p = 0; p < MAXK; ++p) a[p] = -INFINITY;
      // pass 1: the km1 largest values
      for (int c = 0; ok && c < nch; ++c) {
        const int b = nch <= 2 ? c : (c & 1);
        if (!acquired && !(ok = wait_buf(b))) break;
        const uint32_t base = tmem + lane_off + (uint32_t)wg * 256u + (uint32_t)b * 128u;
        const int ncol = min(kChunk, j - c * kChunk);
#pragma unroll 1
        for (int sub = 0; sub < kChunk / 32; ++sub) {
          if (sub * 32 >= ncol) break;  // uniform across the warpgroup
          uint32_t s[32];
          tmem_ld32(base + sub * 32, s);
          tmem_ld_wait();
          const int nvalid = ncol - sub * 32;
          // two candidates per step: for a list sorted descending and a pair
          // hi >= lo, the merged list is new[p] = max(a[p], min(a[p-1], hi),
          // min(a[p-2], lo)) (a[-1] = a[-2] = +inf); every position comes
          // from the old list, so the step has no serial chain
#pragma unroll
          for (int x = 0; x < 32; x += 2) {
            const float v0 = x < nvalid ? __uint_as_float(s[x]) : -INFINITY;
            const float v1 = x + 1 < nvalid ? __uint_as_float(s[x + 1]) : -INFINITY;
            const float hi = fmaxf(v0, v1), lo = fminf(v0, v1);
            float na[MAXK];
            na[0] = fmaxf(a[0], hi);
            if (MAXK > 1) na[1 % MAXK] = max3(a[1 % MAXK], fminf(a[0], hi), lo);
#pragma unroll
            for (int p = 2; p < MAXK; ++p) na[p] = max3(a[p], fminf(a[p - 1], hi), fminf(a[p - 2], lo));
#pragma unroll
            for (int p = 0; p < MAXK; ++p)
              if (p < km1) a[p] = na[p];
          }
        }
        if (nch > 2) release_buf(b);
      }
      if (!ok) break;
      float tau = a[0];
      int gt = 0;
#pragma unroll
      for (int p = 0; p < MAXK; ++p)
        if (p < km1) tau = a[p];
#pragma unroll
      for (int p = 0; p < MAXK; ++p)
        if (p < km1 && a[p] > tau) ++gt;
      int need_eq = km1 - gt;
      int cnt = 0;
      // pass 2: emit indices in ascending order
      for (int c = 0; ok && c < nch; ++c) {
        const int b = nch <= 2 ? c : ((nch + c) & 1);  // job nch + c when recomputed
        if (nch > 2 && !(ok = wait_buf(b))) break;
        const uint32_t base = tmem + lane_off + (uint32_t)wg * 256u + (uint32_t)b * 128u;
        const int ncol = min(kChunk, j - c * kChunk);
#pragma unroll 1
        for (int sub = 0; sub < kChunk / 32; ++sub) {
          if (sub * 32 >= ncol) break;
          uint32_t s[32];
          tmem_ld32(base + sub * 32, s);
          tmem_ld_wait();
          const int nvalid = ncol - sub * 32;
#pragma unroll
          for (int x = 0; x < 32; ++x) {
            const float v = __uint_as_float(s[x]);
            bool take = x < nvalid && (v > tau || (v == tau && need_eq > 0));
            if (take && !(v > tau)) --need_eq;
            take = take && cnt < km1;
            if (take && valid) out[cnt] = c * kChunk + sub * 32 + x;
            cnt += take ? 1 : 0;
          }
        }
        if (nch > 2) release_buf(b);
      }
      if (!ok) break;
      if (nch <= 2)
        for (int b = 0; b < nch; ++b) release_buf(b);
      if (valid) out[km1] = j;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
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

// 3D map over a [rows, heads, d] bf16 tensor, boxes of 128 rows x 1 head x 64 dims
bool make_map(CUtensorMap* m, const void* base, long long rows, int heads, int D) {
  auto fn = encode_fn();
  if (!fn || rows <= 0) return false;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)heads, (cuuint64_t)rows};
  cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)heads * D * 2};
  cuuint32_t box[3] = {64, 1, 128};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, int MAXK>
cudaError_t launch(const void* q, int32_t* idx, const Sizes& z, const Workspace& ws, int num_sms,
                   cudaStream_t st) {
  CUtensorMap mq, mh, ml;
  if (!make_map(&mq, q, z.T, z.Hq, D) || !make_map(&mh, ws.kbar_hi, z.nfull_max, z.Hkv, D) ||
      !make_map(&ml, ws.kbar_lo, z.nfull_max, z.Hkv, D))
    return cudaErrorInvalidValue;
  const size_t smem = sizeof(GateSmem<D>) + 1024;
  cudaError_t e = cudaFuncSetAttribute(gate_tc_kernel<D, MAXK>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  gate_tc_kernel<D, MAXK><<<num_sms, kThreads, smem, st>>>(mq, mh, ml, ws, idx, z.Hq, z.Hkv, z.B,
                                                           z.topk);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_d(const void* q, int32_t* idx, const Sizes& z, const Workspace& ws,
                     int num_sms, cudaStream_t st) {
  const int km1 = z.topk - 1;
  if (km1 <= 2) return launch<D, 2>(q, idx, z, ws, num_sms, st);
  if (km1 <= 4) return launch<D, 4>(q, idx, z, ws, num_sms, st);
  if (km1 <= 8) return launch<D, 8>(q, idx, z, ws, num_sms, st);
  if (km1 <= 11) return launch<D, 11>(q, idx, z, ws, num_sms, st);
  return launch<D, 15>(q, idx, z, ws, num_sms, st);
}

}  // namespace

bool gate_tc_supported(const Sizes& z) { return z.nfull_max > 0 && z.topk >= 2 && z.topk <= 16; }

cudaError_t launch_gate_tc(const void* q, int32_t* idx, const Sizes& z, const Workspace& ws,
                           int num_sms, cudaStream_t st) {
  if (z.d == 128) return launch_d<128>(q, idx, z, ws, num_sms, st);
  return launch_d<64>(q, idx, z, ws, num_sms, st);
}

}  // namespace moba
