// Plan, block mean-pool and gate kernels of the MoBA forward.
//
// Pages cited by title:
//  [W] "同一天，DeepSeek和月之暗面發表了關于改進注意力機制的論文", section
//      "MoBA：將 MoE 原理應用于注意力機制": context cut into blocks, parameter-free
//      top-k gate, step 1 (assign queries to KV blocks under the causal mask).
//  [E] "月球計畫 AI 研究介紹混合區塊注意力 (MoBA)...", section "技術細節與優勢":
//      score against an aggregated representation of a block's keys (read as
//      their mean), own block always selected, no future block.
#include "common.cuh"
#include "kernels.h"

namespace moba {

// ---------------------------------------------------------------------------
// plan: validate cu_seqlens, number the blocks of every sequence.
// One CTA of 1024 threads.  Blocks restart at every sequence start; a short
// last block is numbered but has no mean (it is only ever an own block).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(1024) plan_kernel(const int* __restrict__ cu, int n_seqs, int T,
                                                    int B, Workspace ws, int nblk_max,
                                                    int nfull_max) {
  __shared__ int s_bad;
  __shared__ int s_scan_b[1024];
  __shared__ int s_scan_f[1024];
  const int tid = threadIdx.x;
  if (tid == 0) s_bad = -1;
  __syncthreads();
  for (int s = tid; s < n_seqs; s += blockDim.x) {
    int a = cu[s], b = cu[s + 1];
    bool bad = (b < a) || (s == 0 && a != 0) || (s == n_seqs - 1 && b != T) || a < 0 || b > T;
    if (bad) atomicMax(&s_bad, s);
  }
  __syncthreads();
  if (s_bad >= 0) {
    if (tid == 0) {
      raise_error(ws.plan, kErrBadSeqlens, s_bad);
      ws.plan->nblk_total = 0;
      ws.plan->nfull_total = 0;
      ws.plan->ntiles = 0;
    }
    return;
  }
  int carry_b = 0, carry_f = 0;
  for (int base = 0; base < n_seqs; base += blockDim.x) {
    int s = base + tid;
    int nb = 0, nf = 0;
    if (s < n_seqs) {
      int L = cu[s + 1] - cu[s];
      nb = (L + B - 1) / B;
      nf = L / B;
    }
    s_scan_b[tid] = nb;
    s_scan_f[tid] = nf;
    __syncthreads();
    for (int off = 1; off < (int)blockDim.x; off <<= 1) {
      int vb = tid >= off ? s_scan_b[tid - off] : 0;
      int vf = tid >= off ? s_scan_f[tid - off] : 0;
      __syncthreads();
      s_scan_b[tid] += vb;
      s_scan_f[tid] += vf;
      __syncthreads();
    }
    if (s < n_seqs) {
      ws.seq_blk_base[s] = carry_b + s_scan_b[tid] - nb;
      ws.seq_full_base[s] = carry_f + s_scan_f[tid] - nf;
    }
    carry_b += s_scan_b[blockDim.x - 1];
    carry_f += s_scan_f[blockDim.x - 1];
    __syncthreads();
  }
  if (tid == 0) {
    ws.seq_blk_base[n_seqs] = carry_b;
    ws.seq_full_base[n_seqs] = carry_f;
    ws.plan->nblk_total = carry_b <= nblk_max ? carry_b : 0;
    ws.plan->nfull_total = carry_f <= nfull_max ? carry_f : 0;
    ws.plan->ntiles = 0;
  }
  __syncthreads();
  if (carry_b > nblk_max || carry_f > nfull_max) return;  // impossible after validation
  long long pairs = 0;  // full_cm of the sequence's first full block
  for (int s = 0; s < n_seqs; ++s) {
    int a = cu[s], L = cu[s + 1] - a;
    int nb = (L + B - 1) / B;
    int nf = L / B;
    int bb = ws.seq_blk_base[s], fb = ws.seq_full_base[s];
    for (int i = tid; i < nb; i += blockDim.x) {
      int gb = bb + i;
      ws.blk_start[gb] = a + i * B;
      ws.blk_len[gb] = min(B, L - i * B);
      ws.blk_j[gb] = i;
      ws.blk_fullbase[gb] = fb;
      if ((i + 1) * B <= L) {
        ws.full_start[fb + i] = a + i * B;
        if (ws.full_cm) {  // blocks after full block i: nb - 1 - i; their sum over i' < i
          ws.full_nlater[fb + i] = nb - 1 - i;
          ws.full_cm[fb + i] = pairs + (long long)i * (nb - 1) - (long long)i * (i - 1) / 2;
        }
      }
    }
    pairs += (long long)nf * (nb - 1) - (long long)nf * (nf - 1) / 2;
  }
}

// ---------------------------------------------------------------------------
// pool, pass 1: partial key sums over one of kPoolSplit row slices of a full
// block.  grid (nfull_max, kPoolSplit, ceil(Hkv*d/8 / 256)), 256 threads.
// Each thread reads 16-byte vectors of 8 bf16 keys; rows of a token are
// contiguous over all kv heads, so a warp reads 512 contiguous bytes.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) pool_partial_kernel(const __nv_bfloat16* __restrict__ k,
                                                           Workspace ws, int Hkv, int d, int B) {
  const DevPlan* plan = ws.plan;
  const int fb = blockIdx.x;
  if (plan->err != 0 || fb >= plan->nfull_total) return;
  const int cols8 = Hkv * d / 8;
  const int per = min(cols8, 256);
  const int rgroups = 256 / per;
  const int tid = threadIdx.x;
  const int rg = tid / per;
  const int c8 = blockIdx.z * 256 + tid % per;
  const int rows = B / kPoolSplit;
  const long long r0 = (long long)ws.full_start[fb] + (long long)blockIdx.y * rows;
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;
  const bool active = rg < rgroups && c8 < cols8;
  if (active) {
    const uint4* src = reinterpret_cast<const uint4*>(k) + r0 * cols8 + c8;
    int r = rg;
    for (; r + 3 * rgroups < rows; r += 4 * rgroups) {
      uint4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) v[u] = __ldg(src + (long long)(r + u * rgroups) * cols8);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v[u]);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          float2 f = __bfloat1622float2(h[e]);
          acc[2 * e] += f.x;
          acc[2 * e + 1] += f.y;
        }
      }
    }
    for (; r < rows; r += rgroups) {
      uint4 v = __ldg(src + (long long)r * cols8);
      const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float2 f = __bfloat1622float2(h[e]);
        acc[2 * e] += f.x;
        acc[2 * e + 1] += f.y;
      }
    }
  }
  __shared__ float red[256 * 8];
#pragma unroll
  for (int e = 0; e < 8; ++e) red[tid * 8 + e] = acc[e];
  __syncthreads();
  if (rg == 0 && c8 < cols8) {
    float s[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) s[e] = acc[e];
    for (int g = 1; g < rgroups; ++g) {
#pragma unroll
      for (int e = 0; e < 8; ++e) s[e] += red[(g * per + tid) * 8 + e];
    }
    float* dst = ws.pool_part + ((long long)fb * kPoolSplit + blockIdx.y) * (Hkv * d) + c8 * 8;
#pragma unroll
    for (int e = 0; e < 8; ++e) dst[e] = s[e];
  }
}

// pool, pass 2: sum the slices in a fixed order, divide by B, and emit the
// fp32 mean plus its bf16 hi/lo split (hi = bf16(m), lo = bf16(m - hi)).
__global__ void pool_finish_kernel(Workspace ws, int Hkv, int d, int B) {
  const DevPlan* plan = ws.plan;
  if (plan->err != 0) return;
  const long long n = (long long)plan->nfull_total * Hkv * d;
  const int cols = Hkv * d;
  const float inv = 1.0f / (float)B;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x) {
    long long fb = i / cols;
    int c = (int)(i % cols);
    const float* p = ws.pool_part + fb * kPoolSplit * cols + c;
    float s = 0.f;
#pragma unroll
    for (int u = 0; u < kPoolSplit; ++u) s += p[(long long)u * cols];
    float m = s * inv;
    ws.kbar[i] = m;
    __nv_bfloat16 hi = __float2bfloat16_rn(m);
    ws.kbar_hi[i] = hi;
    ws.kbar_lo[i] = __float2bfloat16_rn(m - __bfloat162float(hi));
  }
}

// ---------------------------------------------------------------------------
// gate (CUDA cores, fp32): one thread per (token, head) row.
// grid (nblk_max, ceil(B/128), Hq), 128 threads: all rows of a CTA share the
// block j and kv head g, so they share the candidate set Kbar[0..j-1, g].
// Streaming top-(topk-1): a register list sorted by (score desc, index asc);
// a new score enters only if strictly larger than the current last entry
// (scanning in ascending index order makes equal later scores lose the tie).
// ---------------------------------------------------------------------------
template <int D, int MAXK>
__global__ void __launch_bounds__(128) gate_simt_kernel(const __nv_bfloat16* __restrict__ q,
                                                        Workspace ws, int32_t* __restrict__ idx,
                                                        int Hq, int Hkv, int topk) {
  constexpr int CH = 32;  // mean keys staged per round
  __shared__ __align__(16) float s_kbar[CH * D];
  const DevPlan* plan = ws.plan;
  const int gb = blockIdx.x;
  if (plan->err != 0 || gb >= plan->nblk_total) return;
  const int len = ws.blk_len[gb];
  const int tl = blockIdx.y * 128 + threadIdx.x;
  if (blockIdx.y * 128 >= len) return;
  const bool valid = tl < len;
  const long long t = ws.blk_start[gb] + (valid ? tl : 0);
  const int j = ws.blk_j[gb];
  const int h = blockIdx.z;
  const int g = h / (Hq / Hkv);
  int32_t* out = idx + (t * Hq + h) * topk;

  if (j + 1 <= topk) {  // every block 0..j is selected
    if (valid)
      for (int p = 0; p < topk; ++p) out[p] = p <= j ? p : -1;
    return;
  }
  const int km1 = topk - 1;
  if (km1 == 0) {  // top-1: only the own block
    if (valid) out[0] = j;
    return;
  }
  float qv[D];
  {
    const uint4* src = reinterpret_cast<const uint4*>(q + (t * Hq + h) * D);
#pragma unroll
    for (int c = 0; c < D / 8; ++c) {
      uint4 v = __ldg(src + c);
      const __nv_bfloat162* hp = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float2 f = __bfloat1622float2(hp[e]);
        qv[c * 8 + 2 * e] = f.x;
        qv[c * 8 + 2 * e + 1] = f.y;
      }
    }
  }
  float vals[MAXK];
  int ids[MAXK];
#pragma unroll
  for (int p = 0; p < MAXK; ++p) {
    vals[p] = -INFINITY;
    ids[p] = 0x7fffffff;
  }
  const int fbase = ws.blk_fullbase[gb];
  for (int i0 = 0; i0 < j; i0 += CH) {
    const int n = min(CH, j - i0);
    __syncthreads();
    for (int e = threadIdx.x; e < n * (D / 4); e += 128) {
      int r = e / (D / 4), c4 = e % (D / 4);
      reinterpret_cast<float4*>(s_kbar)[e] = reinterpret_cast<const float4*>(
          ws.kbar + ((long long)(fbase + i0 + r) * Hkv + g) * D)[c4];
    }
    __syncthreads();
    for (int r = 0; r < n; ++r) {
      const float4* kb = reinterpret_cast<const float4*>(s_kbar + r * D);
      float s0 = 0.f, s1 = 0.f;
#pragma unroll
      for (int c = 0; c < D / 4; c += 2) {
        float4 a = kb[c], b = kb[c + 1];
        s0 = fmaf(qv[4 * c + 0], a.x, s0);
        s0 = fmaf(qv[4 * c + 1], a.y, s0);
        s0 = fmaf(qv[4 * c + 2], a.z, s0);
        s0 = fmaf(qv[4 * c + 3], a.w, s0);
        s1 = fmaf(qv[4 * c + 4], b.x, s1);
        s1 = fmaf(qv[4 * c + 5], b.y, s1);
        s1 = fmaf(qv[4 * c + 6], b.z, s1);
        s1 = fmaf(qv[4 * c + 7], b.w, s1);
      }
      float s = s0 + s1;
      int id = i0 + r;
      if (s > vals[km1 - 1]) {
        // carry the new entry down the list; an entry moves below another only
        // when it is smaller, or equal with a larger index.
        float cv = s;
        int ci = id;
#pragma unroll
        for (int p = 0; p < MAXK; ++p) {
          if (p < km1) {
            bool take = (cv > vals[p]) || (cv == vals[p] && ci < ids[p]);
            float tv = vals[p];
            int ti = ids[p];
            vals[p] = take ? cv : tv;
            ids[p] = take ? ci : ti;
            cv = take ? tv : cv;
            ci = take ? ti : ci;
          }
        }
      }
    }
  }
  if (!valid) return;
  // report ascending: sort the kept past indices, then the own block j.
#pragma unroll
  for (int a = 0; a < MAXK; ++a) {
#pragma unroll
    for (int b = a + 1; b < MAXK; ++b) {
      if (b < km1) {
        int x = ids[a], y = ids[b];
        ids[a] = min(x, y);
        ids[b] = max(x, y);
      }
    }
  }
#pragma unroll
  for (int p = 0; p < MAXK; ++p)
    if (p < km1) out[p] = ids[p];
  out[km1] = j;
}

// ---------------------------------------------------------------------------
// host launchers
// ---------------------------------------------------------------------------
cudaError_t launch_plan(const int* cu, const Sizes& z, const Workspace& ws, cudaStream_t st) {
  plan_kernel<<<1, 1024, 0, st>>>(cu, z.n_seqs, z.T, z.B, ws, z.nblk_max, z.nfull_max);
  return cudaGetLastError();
}

cudaError_t launch_pool(const void* k, const Sizes& z, const Workspace& ws, cudaStream_t st) {
  if (z.nfull_max == 0) return cudaSuccess;
  int cols8 = z.Hkv * z.d / 8;
  dim3 grid(z.nfull_max, kPoolSplit, (cols8 + 255) / 256);
  pool_partial_kernel<<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(k), ws, z.Hkv, z.d,
                                             z.B);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  long long n = (long long)z.nfull_max * z.Hkv * z.d;
  int blocks = (int)((n + 255) / 256);
  if (blocks > 148 * 16) blocks = 148 * 16;
  pool_finish_kernel<<<blocks, 256, 0, st>>>(ws, z.Hkv, z.d, z.B);
  return cudaGetLastError();
}

cudaError_t launch_gate(const void* q, int32_t* idx, const Sizes& z, const Workspace& ws,
                        cudaStream_t st) {
  dim3 grid(z.nblk_max, (z.B + 127) / 128, z.Hq);
  const __nv_bfloat16* qp = static_cast<const __nv_bfloat16*>(q);
  if (z.d == 128) {
    if (z.topk <= 16)
      gate_simt_kernel<128, 15><<<grid, 128, 0, st>>>(qp, ws, idx, z.Hq, z.Hkv, z.topk);
    else
      gate_simt_kernel<128, 63><<<grid, 128, 0, st>>>(qp, ws, idx, z.Hq, z.Hkv, z.topk);
  } else {
    if (z.topk <= 16)
      gate_simt_kernel<64, 15><<<grid, 128, 0, st>>>(qp, ws, idx, z.Hq, z.Hkv, z.topk);
    else
      gate_simt_kernel<64, 63><<<grid, 128, 0, st>>>(qp, ws, idx, z.Hq, z.Hkv, z.topk);
  }
  return cudaGetLastError();
}

}  // namespace moba
