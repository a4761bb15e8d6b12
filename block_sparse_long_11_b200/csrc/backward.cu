// Backward of the MoBA forward with the selection held fixed: dq, dk, dv of
// sum(dout * out).
//
// Pages cited by title: "同一天，DeepSeek和月之暗面發表了關于改進注意力機制的論文"
// (MoBA write-up), opening list: trainable block-sparse attention -- the top-k
// gate passes no gradient; over the chosen keys the attention is ordinary
// softmax attention, whose derivative is, per query row with upstream dout:
//   p_u = exp(scale q.k_u - lse), D = dout . out, dp_u = dout . v_u,
//   ds_u = p_u (dp_u - D), dq += scale ds_u k_u, dk_u += scale ds_u q,
//   dv_u += p_u dout.
//
// First version, on the CUDA cores: one warp per (query row, selected slot)
// walks the block's keys (the own block up to the row's token) in chunks of
// 32 rows read whole (lane = d/32 dims, coalesced); the q.k and dout.v dots
// of a chunk are finished by a transposing shuffle reduction (lane i ends
// with key i); dq, dk and dv are accumulated with fp32 atomics (dk, dv sum
// over the query heads of a kv head, dq over the row's slots).  Correctness
// first: the tensor-core backward replaces it.
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace moba {
namespace {

constexpr int kBwdWarps = 8;

__device__ __forceinline__ float bf(const __nv_bfloat16 x) { return __bfloat162float(x); }

// 32 partial sums per lane -> lane i holds the warp-wide sum of element i
__device__ __forceinline__ float transpose_reduce(float* part) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int w = 16; w >= 1; w >>= 1) {
    const bool up = (lane & w) != 0;
#pragma unroll
    for (int i = 0; i < w; ++i) {
      const float send = up ? part[i] : part[i + w];
      const float keep = up ? part[i + w] : part[i];
      part[i] = keep + __shfl_xor_sync(0xffffffffu, send, w);
    }
  }
  return part[0];
}

template <int D>
__global__ void __launch_bounds__(32 * kBwdWarps) backward_kernel(
    const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
    const __nv_bfloat16* __restrict__ v, const __nv_bfloat16* __restrict__ out,
    const float* __restrict__ lse, const __nv_bfloat16* __restrict__ dout,
    const int32_t* __restrict__ idx, const int32_t* __restrict__ cu, int n_seqs, int T, int Hq,
    int Hkv, int B, int topk, float scale, float* __restrict__ dq, float* __restrict__ dk,
    float* __restrict__ dv) {
  constexpr int PER = D / 32;
  const int lane = threadIdx.x & 31;
  const long long item = (long long)blockIdx.x * kBwdWarps + (threadIdx.x >> 5);
  if (item >= (long long)T * Hq * topk) return;
  const int slot = (int)(item % topk);
  const long long row = item / topk;  // t * Hq + h
  const int t = (int)(row / Hq), h = (int)(row % Hq);
  const int g = h / (Hq / Hkv);
  const int b = idx[row * topk + slot];
  if (b < 0) return;
  // the row's sequence (binary search over cu_seqlens)
  int lo = 0, hi = n_seqs - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (cu[mid] <= t) lo = mid; else hi = mid - 1;
  }
  const int a = cu[lo];
  if (a < 0 || a > t) return;  // (malformed cu_seqlens: nothing is read)
  const int tl = t - a;
  if (b > tl / B) return;  // not a block the row may attend
  const int k0 = a + b * B;
  const int k1 = min(a + b * B + B, t + 1);  // own block: up to the row's token
  float qv[PER], gv[PER], dqa[PER];
  float Dd = 0.f;
#pragma unroll
  for (int e = 0; e < PER; ++e) {
    qv[e] = bf(q[row * D + lane * PER + e]);
    gv[e] = bf(dout[row * D + lane * PER + e]);
    Dd = fmaf(gv[e], bf(out[row * D + lane * PER + e]), Dd);
    dqa[e] = 0.f;
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) Dd += __shfl_xor_sync(0xffffffffu, Dd, off);
  const float l = lse[row];
  const long long stride = (long long)Hkv * D;
  for (int base = k0; base < k1; base += 32) {
    float ps[32], pd[32];
    float kr[32][PER];
#pragma unroll
    for (int kk = 0; kk < 32; ++kk) {
      const long long u = min(base + kk, k1 - 1);
      const __nv_bfloat16* kp = k + u * stride + (long long)g * D + lane * PER;
      const __nv_bfloat16* vp = v + u * stride + (long long)g * D + lane * PER;
      float s = 0.f, dp = 0.f;
#pragma unroll
      for (int e = 0; e < PER; ++e) {
        kr[kk][e] = bf(kp[e]);
        s = fmaf(qv[e], kr[kk][e], s);
        dp = fmaf(gv[e], bf(vp[e]), dp);
      }
      ps[kk] = s;
      pd[kk] = dp;
    }
    const float s_me = transpose_reduce(ps);
    const float dp_me = transpose_reduce(pd);
    const bool valid = base + lane < k1;
    const float p = valid ? expf(scale * s_me - l) : 0.f;
    const float ds = p * (dp_me - Dd);
    const int n = min(32, k1 - base);
    for (int kk = 0; kk < n; ++kk) {
      const float pk = __shfl_sync(0xffffffffu, p, kk);
      const float dsk = __shfl_sync(0xffffffffu, ds, kk);
      const long long u = base + kk;
      float* dkp = dk + u * stride + (long long)g * D + lane * PER;
      float* dvp = dv + u * stride + (long long)g * D + lane * PER;
#pragma unroll
      for (int e = 0; e < PER; ++e) {
        dqa[e] = fmaf(scale * dsk, kr[kk][e], dqa[e]);
        atomicAdd(dkp + e, scale * dsk * qv[e]);
        atomicAdd(dvp + e, pk * gv[e]);
      }
    }
  }
#pragma unroll
  for (int e = 0; e < PER; ++e) atomicAdd(dq + row * D + lane * PER + e, dqa[e]);
}

}  // namespace

cudaError_t launch_backward(const void* q, const void* k, const void* v, const void* out,
                            const float* lse, const void* dout, const int32_t* idx,
                            const int32_t* cu, int n_seqs, int T, int Hq, int Hkv, int d, int B,
                            int topk, float scale, float* dq, float* dk, float* dv,
                            cudaStream_t st) {
  cudaError_t e = cudaMemsetAsync(dq, 0, sizeof(float) * (size_t)T * Hq * d, st);
  if (e == cudaSuccess) e = cudaMemsetAsync(dk, 0, sizeof(float) * (size_t)T * Hkv * d, st);
  if (e == cudaSuccess) e = cudaMemsetAsync(dv, 0, sizeof(float) * (size_t)T * Hkv * d, st);
  if (e != cudaSuccess || T == 0) return e;
  const long long items = (long long)T * Hq * topk;
  const unsigned grid = (unsigned)((items + kBwdWarps - 1) / kBwdWarps);
  const auto* qb = static_cast<const __nv_bfloat16*>(q);
  const auto* kb = static_cast<const __nv_bfloat16*>(k);
  const auto* vb = static_cast<const __nv_bfloat16*>(v);
  const auto* ob = static_cast<const __nv_bfloat16*>(out);
  const auto* gb = static_cast<const __nv_bfloat16*>(dout);
  if (d == 128)
    backward_kernel<128><<<grid, 32 * kBwdWarps, 0, st>>>(qb, kb, vb, ob, lse, gb, idx, cu, n_seqs,
                                                          T, Hq, Hkv, B, topk, scale, dq, dk, dv);
  else
    backward_kernel<64><<<grid, 32 * kBwdWarps, 0, st>>>(qb, kb, vb, ob, lse, gb, idx, cu, n_seqs,
                                                         T, Hq, Hkv, B, topk, scale, dq, dk, dv);
  return cudaGetLastError();
}

}  // namespace moba
