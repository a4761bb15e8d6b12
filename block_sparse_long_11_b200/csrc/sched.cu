// Scheduler and merge kernels of the MoBA forward.
//
// Page cited by title: "同一天，DeepSeek和月之暗面發表了關于改進注意力機制的論文"
// (MoBA write-up), section "MoBA：將 MoE 原理應用于注意力機制", the five
// implementation steps: (2) order the query tokens by their assigned KV block,
// (4) put the attention outputs back in the original order, (5) merge the
// outputs of a query's blocks with online softmax.
//
// Step 2 is a counting sort of the gate's past selections by bucket
// (full block, kv head): histogram -> exclusive scan -> scatter.  Step 4 needs
// no pass of its own: every partial output is written straight to the slot of
// its (row, selection) pair, and step 5 reads a row's slots in ascending
// block order.
#include "common.cuh"
#include "kernels.h"

namespace moba {

// Bins of the shared-memory histogram: past blocks j of a query block.  A
// sequence with more than kSmemBins blocks uses global atomics directly.
constexpr int kSmemBins = 4096;

// grid (nblk_max, ceil(B/128), Hkv), 128 threads: one thread per token, looping
// over the Hq/Hkv query heads of kv head g.  All rows of a CTA sit in the same
// block j of the same sequence and map to buckets (fbase + i, g), i < j, so
// the CTA histograms them in shared memory and touches each global counter
// once.  MODE 0 counts entries per bucket; MODE 1 reserves a contiguous range
// per bucket and scatters the partial-slot ids into it.
template <int MODE>
__global__ void __launch_bounds__(128) sched_bucket_kernel(const int32_t* __restrict__ idx,
                                                           Workspace ws, int Hq, int Hkv,
                                                           int topk, int t0, int t1) {
  __shared__ int s_hist[kSmemBins];
  __shared__ int s_base[MODE == 1 ? kSmemBins : 1];
  const DevPlan* plan = ws.plan;
  const int gb = blockIdx.x;
  if (plan->err != 0 || gb >= plan->nblk_total) return;
  const int len = ws.blk_len[gb];
  const int y0 = blockIdx.y * 128;
  if (y0 >= len) return;
  const int bstart = ws.blk_start[gb];
  if (bstart + y0 >= t1 || bstart + min(len, y0 + 128) <= t0) return;
  const int j = ws.blk_j[gb];
  const int nsel = min(topk, j + 1);
  if (nsel <= 1) return;
  const int g = blockIdx.z;
  const int G = Hq / Hkv;
  const int fbase = ws.blk_fullbase[gb];
  const int tl = y0 + threadIdx.x;
  const int t = bstart + tl;
  const bool row_ok = tl < len && t >= t0 && t < t1;
  const bool use_smem = j <= kSmemBins;

  if (!use_smem) {  // very long sequences at small block sizes: global atomics
    if (!row_ok) return;
    for (int hh = 0; hh < G; ++hh) {
      const int h = g * G + hh;
      const int32_t* row = idx + ((long long)t * Hq + h) * topk;
      const int pbase = ((t - t0) * Hq + h) * topk;
      for (int s = 0; s < nsel - 1; ++s) {
        const int i = row[s];
        if (i < 0 || i >= j) continue;
        const int bucket = (fbase + i) * Hkv + g;
        if (MODE == 0)
          atomicAdd(&ws.bucket_count[bucket], 1);
        else {
          const int pos = atomicAdd(&ws.bucket_cursor[bucket], 1);
          if (MOBA_INDEX_OK(ws.plan, pos >= 0 && pos < ws.entries_cap, kSiteSchedEntry))
            ws.entries[pos] = pbase + s;
        }
      }
    }
    return;
  }
  for (int i = threadIdx.x; i < j; i += 128) s_hist[i] = 0;
  __syncthreads();
  if (row_ok) {
    for (int hh = 0; hh < G; ++hh) {
      const int32_t* row = idx + ((long long)t * Hq + g * G + hh) * topk;
      for (int s = 0; s < nsel - 1; ++s) {
        const int i = row[s];
        if (i >= 0 && i < j) atomicAdd(&s_hist[i], 1);
      }
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < j; i += 128) {
    const int c = s_hist[i];
    if (c == 0) continue;
    const int bucket = (fbase + i) * Hkv + g;
    if (MODE == 0) {
      atomicAdd(&ws.bucket_count[bucket], c);
    } else {
      s_base[i] = atomicAdd(&ws.bucket_cursor[bucket], c);
      s_hist[i] = 0;  // reused as the running rank inside this CTA's range
    }
  }
  if (MODE == 0) return;
  __syncthreads();
  if (row_ok) {
    for (int hh = 0; hh < G; ++hh) {
      const int h = g * G + hh;
      const int32_t* row = idx + ((long long)t * Hq + h) * topk;
      const int pbase = ((t - t0) * Hq + h) * topk;
      for (int s = 0; s < nsel - 1; ++s) {
        const int i = row[s];
        if (i >= 0 && i < j) {
          const int pos = s_base[i] + atomicAdd(&s_hist[i], 1);
          if (MOBA_INDEX_OK(ws.plan, pos >= 0 && pos < ws.entries_cap, kSiteSchedEntry))
            ws.entries[pos] = pbase + s;
        }
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Stable fill, for the backward's schedule over every token: dK and dV sum
// over a bucket's rows in their order in the bucket, so that order is made
// the ascending one -- (token, head) -- for the result to be the same from
// run to run.  A bucket (full block f, kv head g) owns a segment of cm with
// one slot per scheduler CTA that can route to it: CTAs (block gb, 128-token
// slice y, g) of f's sequence with gb after f, in token order (slot
// (j(gb) - j(f) - 1) * nyb + y).  MODE 0 writes each CTA's count into its
// slot (and the bucket totals); sched_runs_kernel turns every segment into
// the start of each CTA's run inside the bucket; MODE 1 places each entry at
// its run start plus its rank inside the CTA in (token, head) order.
// The CTA's buckets i < j are taken kStableBins at a time through a
// shared-memory table of per-thread (= per-token) counts.
// ---------------------------------------------------------------------------
constexpr int kStableBins = 128;

__device__ __forceinline__ long long cm_slot(const Workspace& ws, int fb, int g, int Hkv, int nyb) {
  return (ws.full_cm[fb] * Hkv + (long long)g * ws.full_nlater[fb]) * nyb;
}

template <int MODE>
__global__ void __launch_bounds__(128) sched_stable_kernel(const int32_t* __restrict__ idx,
                                                           Workspace ws, int Hq, int Hkv,
                                                           int topk, int nyb, int t0, int t1) {
  __shared__ uint16_t s_cnt[kStableBins][128];
  __shared__ int s_run[kStableBins];
  const DevPlan* plan = ws.plan;
  const int gb = blockIdx.x;
  if (plan->err != 0 || gb >= plan->nblk_total) return;
  const int len = ws.blk_len[gb];
  const int y0 = blockIdx.y * 128;
  if (y0 >= len) return;
  const int bstart = ws.blk_start[gb];
  if (bstart + y0 >= t1 || bstart + min(len, y0 + 128) <= t0) return;
  const int j = ws.blk_j[gb];
  const int nsel = min(topk, j + 1);
  if (nsel <= 1) return;
  const int g = blockIdx.z;
  const int G = Hq / Hkv;
  const int fbase = ws.blk_fullbase[gb];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int tl = y0 + tid;
  const int t = bstart + tl;
  const bool row_ok = tl < len && t >= t0 && t < t1;
  for (int i0 = 0; i0 < j; i0 += kStableBins) {
    const int nbin = min(kStableBins, j - i0);
    for (int i = 0; i < nbin; ++i) s_cnt[i][tid] = 0;  // the thread's own column
    if (row_ok) {
      for (int hh = 0; hh < G; ++hh) {
        const int32_t* row = idx + ((long long)t * Hq + g * G + hh) * topk;
        for (int s = 0; s < nsel - 1; ++s) {
          const int i = row[s] - i0;
          if (i >= 0 && i < nbin && row[s] < j) ++s_cnt[i][tid];
        }
      }
    }
    __syncthreads();
    // per bucket: the CTA's count (MODE 0) or exclusive ranks along the
    // tokens and the run start (MODE 1); lane l covers tokens 4 l .. 4 l + 3
    for (int i = warp; i < nbin; i += 4) {
      const int fb = fbase + i0 + i;
      const long long slot = cm_slot(ws, fb, g, Hkv, nyb) + (long long)(j - (i0 + i) - 1) * nyb +
                             blockIdx.y;
      const bool slot_ok =
          MOBA_INDEX_OK(plan, slot >= 0 && slot < ws.cm_cap, kSiteSchedEntry);
      int c[4], sum = 0;
#pragma unroll
      for (int e = 0; e < 4; ++e) sum += (c[e] = s_cnt[i][4 * lane + e]);
      int ex = sum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, ex, o);
        if (lane >= o) ex += v;
      }
      const int total = __shfl_sync(0xffffffffu, ex, 31);
      ex -= sum;
      if (MODE == 0) {
        if (lane == 0 && total > 0 && slot_ok) {
          ws.cm[slot] = total;
          atomicAdd(&ws.bucket_count[fb * Hkv + g], total);
        }
      } else {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          s_cnt[i][4 * lane + e] = (uint16_t)ex;
          ex += c[e];
        }
        if (lane == 0) s_run[i] = slot_ok ? ws.cm[slot] : -1;
      }
    }
    __syncthreads();
    if (MODE == 1 && row_ok) {
      for (int hh = 0; hh < G; ++hh) {
        const int h = g * G + hh;
        const int32_t* row = idx + ((long long)t * Hq + h) * topk;
        const int pbase = ((t - t0) * Hq + h) * topk;
        for (int s = 0; s < nsel - 1; ++s) {
          const int i = row[s] - i0;
          if (i < 0 || i >= nbin || row[s] >= j || s_run[i] < 0) continue;
          const int pos = s_run[i] + s_cnt[i][tid]++;
          if (MOBA_INDEX_OK(plan, pos >= 0 && pos < ws.entries_cap, kSiteSchedEntry))
            ws.entries[pos] = pbase + s;
        }
      }
    }
    __syncthreads();
  }
}

// Stable fill: one warp per bucket turns its segment of CTA counts into run
// starts (the bucket's offset plus an exclusive scan in token order).
__global__ void sched_runs_kernel(Workspace ws, int Hkv, int nyb) {
  const DevPlan* plan = ws.plan;
  if (plan->err != 0) return;
  const int lane = threadIdx.x & 31;
  const int b = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (b >= plan->nfull_total * Hkv) return;
  const int fb = b / Hkv, g = b - fb * Hkv;
  const long long base = cm_slot(ws, fb, g, Hkv, nyb);
  const int n = ws.full_nlater[fb] * nyb;
  if (!MOBA_INDEX_OK(plan, base >= 0 && base + n <= ws.cm_cap, kSiteSchedEntry)) return;
  int carry = ws.bucket_off[b];
  for (int c0 = 0; c0 < n; c0 += 32) {
    const int v = c0 + lane < n ? ws.cm[base + c0 + lane] : 0;
    int ex = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, ex, o);
      if (lane >= o) ex += u;
    }
    if (c0 + lane < n) ws.cm[base + c0 + lane] = carry + ex - v;
    carry += __shfl_sync(0xffffffffu, ex, 31);
  }
}

// One CTA of 1024 threads: exclusive scans of entries and of tiles per bucket.
__global__ void __launch_bounds__(1024) sched_scan_kernel(Workspace ws, int Hkv, int unit_rows) {
  __shared__ int s_e[1024];
  __shared__ int s_t[1024];
  DevPlan* plan = ws.plan;
  if (plan->err != 0) return;
  const int nbk = plan->nfull_total * Hkv;
  const int tid = threadIdx.x;
  int carry_e = 0, carry_t = 0;
  for (int base = 0; base < nbk; base += 1024) {
    int b = base + tid;
    int c = b < nbk ? ws.bucket_count[b] : 0;
    int nt = (c + unit_rows - 1) / unit_rows;
    s_e[tid] = c;
    s_t[tid] = nt;
    __syncthreads();
    for (int off = 1; off < 1024; off <<= 1) {
      int ve = tid >= off ? s_e[tid - off] : 0;
      int vt = tid >= off ? s_t[tid - off] : 0;
      __syncthreads();
      s_e[tid] += ve;
      s_t[tid] += vt;
      __syncthreads();
    }
    if (b < nbk) {
      int eo = carry_e + s_e[tid] - c;
      ws.bucket_off[b] = eo;
      ws.bucket_cursor[b] = eo;
      ws.tile_off[b] = carry_t + s_t[tid] - nt;
    }
    carry_e += s_e[1023];
    carry_t += s_t[1023];
    __syncthreads();
  }
  if (tid == 0) {
    ws.bucket_off[nbk] = carry_e;
    ws.tile_off[nbk] = carry_t;
    plan->ntiles = carry_t;
  }
}

// Work list: unit i of bucket b covers entries
// [off_b + unit_rows * i, min(off_b + unit_rows * (i + 1), off_{b+1})).
__global__ void sched_tiles_kernel(Workspace ws, int Hkv, int unit_rows) {
  const DevPlan* plan = ws.plan;
  if (plan->err != 0) return;
  const int nbk = plan->nfull_total * Hkv;
  for (int b = blockIdx.x * blockDim.x + threadIdx.x; b < nbk; b += gridDim.x * blockDim.x) {
    int e0 = ws.bucket_off[b], e1 = ws.bucket_off[b + 1];
    int t = ws.tile_off[b];
    for (int e = e0; e < e1; e += unit_rows, ++t) ws.tiles[t] = make_int2(b, e);
  }
}

// ---------------------------------------------------------------------------
// merge (step 5): one warp per (token, head) row of the chunk.
//   m = max_s lse_s, w_s = exp(lse_s - m), out = sum_s w_s o_s / sum_s w_s,
//   lse = m + ln(sum_s w_s), over the row's slots in ascending block order.
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) merge_kernel(const int32_t* __restrict__ idx, Workspace ws,
                                                    __nv_bfloat16* __restrict__ out,
                                                    float* __restrict__ lse_out, int Hq, int topk,
                                                    int t0, int t1) {
  if (ws.plan->err != 0) return;
  const int lane = threadIdx.x & 31;
  const long long nrows = (long long)(t1 - t0) * Hq;
  const long long r = (long long)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  if (r >= nrows) return;
  const long long grow = (long long)t0 * Hq + r;  // t * Hq + h
  const int32_t* sel = idx + grow * topk;
  int nsel = __popc(__ballot_sync(0xffffffffu, lane < topk && sel[lane] >= 0));
  if (topk > 32) nsel += __popc(__ballot_sync(0xffffffffu, lane + 32 < topk && sel[lane + 32] >= 0));
  const long long p0 = r * topk;
  float m = -INFINITY;
  for (int s = lane; s < nsel; s += 32) m = fmaxf(m, ws.part_lse[p0 + s]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  constexpr int PER = D / 32;  // dims per lane: 4 (d=128) or 2 (d=64)
  float acc[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) acc[e] = 0.f;
  float wsum = 0.f;
  for (int s = 0; s < nsel; ++s) {
    float w = __expf(ws.part_lse[p0 + s] - m);
    wsum += w;
    const __nv_bfloat16* o = ws.part_o + (p0 + s) * D + lane * PER;
    if (PER == 4) {
      uint2 v = *reinterpret_cast<const uint2*>(o);
      float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&v.x));
      float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&v.y));
      acc[0] = fmaf(w, a.x, acc[0]);
      acc[1] = fmaf(w, a.y, acc[1]);
      acc[2 % PER] = fmaf(w, b.x, acc[2 % PER]);
      acc[3 % PER] = fmaf(w, b.y, acc[3 % PER]);
    } else {
      float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(o));
      acc[0] = fmaf(w, a.x, acc[0]);
      acc[1 % PER] = fmaf(w, a.y, acc[1 % PER]);
    }
  }
  const float inv = 1.0f / wsum;
  __nv_bfloat16* dst = out + grow * D + lane * PER;
  if (PER == 4) {
    __nv_bfloat162 a = __floats2bfloat162_rn(acc[0] * inv, acc[1] * inv);
    __nv_bfloat162 b = __floats2bfloat162_rn(acc[2 % PER] * inv, acc[3 % PER] * inv);
    uint2 v;
    v.x = *reinterpret_cast<uint32_t*>(&a);
    v.y = *reinterpret_cast<uint32_t*>(&b);
    *reinterpret_cast<uint2*>(dst) = v;
  } else {
    *reinterpret_cast<__nv_bfloat162*>(dst) = __floats2bfloat162_rn(acc[0] * inv, acc[1 % PER] * inv);
  }
  if (lane == 0) lse_out[grow] = m + logf(wsum);
}

// ---------------------------------------------------------------------------
cudaError_t launch_sched(const int32_t* idx, const Sizes& z, const Workspace& ws, int t0, int t1,
                         int unit_rows, cudaStream_t st, bool stable) {
  cudaError_t e = cudaMemsetAsync(ws.bucket_count, 0, sizeof(int) * (z.nbk_max + 1), st);
  if (e != cudaSuccess) return e;
  const int nyb = (z.B + 127) / 128;
  dim3 grid(z.nblk_max, nyb, z.Hkv);
  stable = stable && ws.cm_cap > 0;
  if (stable) {
    e = cudaMemsetAsync(ws.cm, 0, sizeof(int) * (size_t)ws.cm_cap, st);
    if (e != cudaSuccess) return e;
    sched_stable_kernel<0><<<grid, 128, 0, st>>>(idx, ws, z.Hq, z.Hkv, z.topk, nyb, t0, t1);
  } else {
    sched_bucket_kernel<0><<<grid, 128, 0, st>>>(idx, ws, z.Hq, z.Hkv, z.topk, t0, t1);
  }
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  sched_scan_kernel<<<1, 1024, 0, st>>>(ws, z.Hkv, unit_rows);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (stable) {
    const long long threads = 32LL * z.nbk_max;
    sched_runs_kernel<<<(unsigned)((threads + 255) / 256 > 0 ? (threads + 255) / 256 : 1), 256, 0,
                        st>>>(ws, z.Hkv, nyb);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    sched_stable_kernel<1><<<grid, 128, 0, st>>>(idx, ws, z.Hq, z.Hkv, z.topk, nyb, t0, t1);
  } else {
    sched_bucket_kernel<1><<<grid, 128, 0, st>>>(idx, ws, z.Hq, z.Hkv, z.topk, t0, t1);
  }
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  int nb = (z.nbk_max + 255) / 256;
  sched_tiles_kernel<<<nb > 0 ? nb : 1, 256, 0, st>>>(ws, z.Hkv, unit_rows);
  return cudaGetLastError();
}

cudaError_t launch_merge(const int32_t* idx, void* out, float* lse, const Sizes& z,
                         const Workspace& ws, int t0, int t1, cudaStream_t st) {
  long long rows = (long long)(t1 - t0) * z.Hq;
  if (rows <= 0) return cudaSuccess;
  long long blocks = (rows + 7) / 8;
  __nv_bfloat16* o = static_cast<__nv_bfloat16*>(out);
  if (z.d == 128)
    merge_kernel<128><<<(unsigned)blocks, 256, 0, st>>>(idx, ws, o, lse, z.Hq, z.topk, t0, t1);
  else
    merge_kernel<64><<<(unsigned)blocks, 256, 0, st>>>(idx, ws, o, lse, z.Hq, z.topk, t0, t1);
  return cudaGetLastError();
}

}  // namespace moba
