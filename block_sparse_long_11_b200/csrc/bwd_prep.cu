// Row-wise passes of the backward around the tensor-core kernels
// (dkv_tc.cu, dq_tc.cu).
//
// Page cited by title: "同一天，DeepSeek和月之暗面發表了關于改進注意力機制的論文"
// (MoBA write-up), opening list: trainable block-sparse attention.
//   prep:  D_r = dout_r . out_r for every row (t, h), and a check of the
//          row's selection -- the forward's idx: ascending block indices of
//          the row's sequence, each in 0..j, the own block j last, min(topk,
//          j + 1) of them, -1 after.  A row that breaks it raises
//          MOBA_ERR_BAD_SELECTION (nothing downstream would write it).
//   merge: dq_r = sum over the row's slots, in ascending block order, of the
//          dQ kernel's fp32 partials (rows with one slot were written
//          directly).
#include "common.cuh"
#include "kernels.h"

namespace moba {
namespace {

template <int D>
__global__ void __launch_bounds__(256) bwd_prep_kernel(
    const __nv_bfloat16* __restrict__ out, const __nv_bfloat16* __restrict__ dout,
    const int32_t* __restrict__ idx, const int32_t* __restrict__ cu, int n_seqs, int Hq, int B,
    int topk, float* __restrict__ dvec, DevPlan* plan, long long nrows) {
  if (plan->err != 0) return;
  const int lane = threadIdx.x & 31;
  const long long r = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (r >= nrows) return;
  constexpr int PER = D / 32;
  float acc = 0.f;
#pragma unroll
  for (int e = 0; e < PER; ++e)
    acc = fmaf(__bfloat162float(dout[r * D + lane * PER + e]),
               __bfloat162float(out[r * D + lane * PER + e]), acc);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane == 0) dvec[r] = acc;
  // the row's selection
  const int t = (int)(r / Hq);
  int lo = 0, hi = n_seqs - 1;  // cu_seqlens was checked by the plan
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (cu[mid] <= t) lo = mid; else hi = mid - 1;
  }
  const int j = (t - cu[lo]) / B;
  const int want = min(topk, j + 1);
  const int32_t* sel = idx + r * topk;
  bool bad = false;
  for (int p = lane; p < topk; p += 32) {
    const int v = sel[p];
    if (p < want) {
      const int prev = p > 0 ? sel[p - 1] : -1;
      bad |= v < 0 || v > j || v <= prev || (p == want - 1 && v != j);
    } else {
      bad |= v != -1;
    }
  }
  if (__any_sync(0xffffffffu, bad) && lane == 0) raise_error(plan, kErrBadSelection, (int)r);
}

template <int D>
__global__ void __launch_bounds__(256) dq_merge_kernel(const int32_t* __restrict__ idx,
                                                       const float* __restrict__ part,
                                                       float* __restrict__ dq, const DevPlan* plan,
                                                       int Hq, int topk, int t0, int t1) {
  if (plan->err != 0) return;
  const int lane = threadIdx.x & 31;
  const long long nrows = (long long)(t1 - t0) * Hq;
  const long long r = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (r >= nrows) return;
  const long long grow = (long long)t0 * Hq + r;
  const int32_t* sel = idx + grow * topk;
  int nsel = __popc(__ballot_sync(0xffffffffu, lane < topk && sel[lane] >= 0));
  if (topk > 32) nsel += __popc(__ballot_sync(0xffffffffu, lane + 32 < topk && sel[lane + 32] >= 0));
  if (nsel <= 1) return;  // written by the dQ kernel
  constexpr int PER = D / 32;
  float acc[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) acc[e] = 0.f;
  const float* p0 = part + r * topk * D + lane * PER;
  for (int s = 0; s < nsel; ++s) {
#pragma unroll
    for (int e = 0; e < PER; ++e) acc[e] += p0[(long long)s * D + e];
  }
#pragma unroll
  for (int e = 0; e < PER; ++e) dq[grow * D + lane * PER + e] = acc[e];
}

}  // namespace

cudaError_t launch_bwd_prep(const void* out, const void* dout, const int32_t* idx,
                            const int32_t* cu, const Sizes& z, float* dvec, DevPlan* plan,
                            cudaStream_t st) {
  const long long nrows = (long long)z.T * z.Hq;
  if (nrows == 0) return cudaSuccess;
  const unsigned grid = (unsigned)((nrows + 7) / 8);
  const auto* o = static_cast<const __nv_bfloat16*>(out);
  const auto* g = static_cast<const __nv_bfloat16*>(dout);
  if (z.d == 128)
    bwd_prep_kernel<128><<<grid, 256, 0, st>>>(o, g, idx, cu, z.n_seqs, z.Hq, z.B, z.topk, dvec,
                                               plan, nrows);
  else
    bwd_prep_kernel<64><<<grid, 256, 0, st>>>(o, g, idx, cu, z.n_seqs, z.Hq, z.B, z.topk, dvec,
                                              plan, nrows);
  return cudaGetLastError();
}

cudaError_t launch_dq_merge(const int32_t* idx, const float* part, float* dq, const Sizes& z,
                            const DevPlan* plan, int t0, int t1, cudaStream_t st) {
  const long long rows = (long long)(t1 - t0) * z.Hq;
  if (rows <= 0) return cudaSuccess;
  const unsigned grid = (unsigned)((rows + 7) / 8);
  if (z.d == 128)
    dq_merge_kernel<128><<<grid, 256, 0, st>>>(idx, part, dq, plan, z.Hq, z.topk, t0, t1);
  else
    dq_merge_kernel<64><<<grid, 256, 0, st>>>(idx, part, dq, plan, z.Hq, z.topk, t0, t1);
  return cudaGetLastError();
}

}  // namespace moba
