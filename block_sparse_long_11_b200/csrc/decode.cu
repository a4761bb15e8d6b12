// Decode: one new query token per sequence against a padded KV cache, with the
// gate's block means kept incrementally.
//
// Pages cited by title:
//  [W] "同一天，DeepSeek和月之暗面發表了關于改進注意力機制的論文", section
//      "MoBA：將 MoE 原理應用于注意力機制": top-k gate over block means,
//      attention to the chosen blocks, log-sum-exp merge of the per-block
//      results (the same five steps as the prefill, for one query row).
//  [S] "MoBA: Mixture of Block Attention for Long-Context LLMs", section
//      "Limitations": generation still runs full attention there; this path
//      gives the sparse forward for generated tokens.
//
// A decode step for sequence s whose cache now holds L tokens (the new
// token's k and v already written at position t = L - 1) computes exactly the
// prefill forward's output row t of the sequence's first L tokens: the gate
// scores q against the means of the full blocks i < j = t / B, keeps the
// (topk - 1) best (ties to the lower index) plus the own block j, and the
// query attends every key of the chosen past blocks and keys jB .. t of its
// own block.  When the new token fills block j, its mean is added to the
// cache after the gate (the query never scores its own block).
//
// Kernels (all memory-bound; CUDA cores, no tensor cores):
//   decode_gate_kernel   one CTA per (sequence, query head): 4 warps score the
//                        past blocks (mean rows read whole, transposing
//                        shuffle reduction) into shared memory, then topk - 1
//                        rounds of a warp arg-max with the lower-index
//                        tie-break, indices ascending.
//   decode_attn_kernel   one CTA per (sequence, query head, selected slot,
//                        part of the block: blocks of 2048 keys or more are cut
//                        into parts of ~1024 keys so the grid fills the GPU in
//                        several waves); items of one (sequence, kv head)
//                        adjacent so the heads of a group read the same block
//                        while it is in L2; 8 warps split the part's keys in
//                        chunks of 32 read as whole rows (lane = 4 dims, so
//                        every load is coalesced), q . k finished by a
//                        transposing shuffle reduction (lane i ends with key
//                        i), online softmax in base 2, warps combined in
//                        shared memory.
//                        The CTA that finishes a row's last part (an atomic
//                        count per row) merges the row's parts (log-sum-exp,
//                        ascending block order) into out and lse.
//   decode_kbar_kernel   block means of every full block (init), fp64
//                        accumulation; a step's new filled block is averaged
//                        by the gate kernel (row slices over the sequence's
//                        CTAs, summed in order by the last one).
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace moba {
namespace {

constexpr int kGateWarps = 4;
constexpr int kAttnWarps = 8;

__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }

// ---------------------------------------------------------------------------
// gate
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(32 * kGateWarps) decode_gate_kernel(
    const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ kc,
    float* __restrict__ kbar, const int32_t* __restrict__ seqlens, int32_t* __restrict__ idx,
    double* __restrict__ kb_part, int* __restrict__ seq_done, DevPlan* plan, int n_seqs,
    int max_len, int max_blocks, int Hq, int Hkv, int B, int topk) {
  constexpr int PER = D / 32;  // dims per lane
  extern __shared__ float sc[];  // [max_blocks] scores of the past blocks
  __shared__ int win[64];        // the topk - 1 winners
  __shared__ int s_last;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int w = blockIdx.x;  // (sequence, query head)
  const int s = w / Hq, h = w % Hq, g = h / (Hq / Hkv);
  int32_t* sel = idx + (long long)w * topk;
  const int L = seqlens[s];
  if (L < 1 || L > max_len) {
    if (threadIdx.x == 0) raise_error(plan, kErrBadSeqlens, s);
    for (int p = threadIdx.x; p < topk; p += blockDim.x) sel[p] = -1;
    return;
  }
  // The new token filled block i = L / B - 1: its mean joins the cache for
  // later steps (this step's gate reads only blocks below i).  The Hq CTAs of
  // the sequence each sum a slice of the block's rows in fp64; the last one
  // to finish adds the slices in order (deterministic) and writes the mean.
  if (L % B == 0 && L / B - 1 < max_blocks) {
    const int i = L / B - 1;
    const int cols = Hkv * D;
    const int per = (B + Hq - 1) / Hq;
    const int r0 = min(B, h * per), r1 = min(B, r0 + per);
    const __nv_bfloat16* src = kc + ((long long)s * max_len + (long long)i * B) * cols;
    double* mine = kb_part + ((long long)s * Hq + h) * cols;
    for (int c = threadIdx.x; c < cols; c += blockDim.x) {
      double acc = 0.0;
#pragma unroll 8
      for (int r = r0; r < r1; ++r) acc += (double)__bfloat162float(src[(long long)r * cols + c]);
      mine[c] = acc;
    }
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) s_last = atomicAdd(&seq_done[s], 1) == Hq - 1;
    __syncthreads();
    if (s_last) {
      __threadfence();
      for (int c = threadIdx.x; c < cols; c += blockDim.x) {
        double acc = 0.0;
        for (int hh = 0; hh < Hq; ++hh) acc += __ldcg(kb_part + ((long long)s * Hq + hh) * cols + c);
        kbar[((long long)s * max_blocks + i) * cols + c] = (float)(acc / B);
      }
    }
  }
  const int t = L - 1, j = t / B;
  if (j + 1 <= topk) {  // every block 0..j
    for (int p = threadIdx.x; p < topk; p += blockDim.x) sel[p] = p <= j ? p : -1;
    return;
  }
  // scores: each warp takes chunks of 32 blocks and reads their mean rows
  // whole (lane = PER dims, coalesced); a transposing shuffle reduction
  // leaves lane i with block (chunk + i)'s score
  float qv[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) qv[e] = __bfloat162float(q[(long long)w * D + lane * PER + e]);
  const float* kb = kbar + ((long long)s * max_blocks * Hkv + g) * D + lane * PER;
  for (int c0 = warp * 32; c0 < j; c0 += 32 * kGateWarps) {
    float part[32];
#pragma unroll
    for (int k8 = 0; k8 < 32; k8 += 8) {
      float rv[8][PER];
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const float* r = kb + (long long)min(c0 + k8 + kk, j - 1) * Hkv * D;
        if (PER == 4) {
          const float4 v = __ldg(reinterpret_cast<const float4*>(r));
          rv[kk][0] = v.x;
          rv[kk][1 % PER] = v.y;
          rv[kk][2 % PER] = v.z;
          rv[kk][3 % PER] = v.w;
        } else {
          const float2 v = __ldg(reinterpret_cast<const float2*>(r));
          rv[kk][0] = v.x;
          rv[kk][1 % PER] = v.y;
        }
      }
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        float a = qv[0] * rv[kk][0];
#pragma unroll
        for (int e = 1; e < PER; ++e) a = fmaf(qv[e], rv[kk][e], a);
        part[k8 + kk] = a;
      }
    }
#pragma unroll
    for (int wd = 16; wd >= 1; wd >>= 1) {
      const bool up = (lane & wd) != 0;
#pragma unroll
      for (int i = 0; i < wd; ++i) {
        const float send = up ? part[i] : part[i + wd];
        const float keep = up ? part[i + wd] : part[i];
        part[i] = keep + __shfl_xor_sync(0xffffffffu, send, wd);
      }
    }
    if (c0 + lane < j) sc[c0 + lane] = part[0];
  }
  __syncthreads();
  if (warp != 0) return;
  // topk - 1 rounds of arg-max (score descending, index ascending); the
  // winner of a round leaves the race
  const int K = topk - 1;
  for (int r = 0; r < K; ++r) {
    float bv = -INFINITY;
    int bi = 0x7fffffff;
    for (int i = lane; i < j; i += 32) {
      const float v = sc[i];
      if (v > bv) {  // ascending i per lane: the first of equal values stays
        bv = v;
        bi = i;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (ov > bv || (ov == bv && oi < bi)) {
        bv = ov;
        bi = oi;
      }
    }
    if (lane == 0) {
      win[r] = bi;
      if (bi < j) sc[bi] = -INFINITY;  // (no winner only if scores are NaN)
    }
    __syncwarp();
  }
  // ascending block order: each winner's rank among the winners
  for (int p = lane; p < K; p += 32) {
    const int me = win[p];
    int rank = 0;
    for (int o = 0; o < K; ++o) rank += win[o] < me ? 1 : 0;
    sel[rank] = me;
  }
  if (lane == 0) sel[K] = j;
}

// ---------------------------------------------------------------------------
// attention of one (sequence, query head) to one selected block
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(32 * kAttnWarps) decode_attn_kernel(
    const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ kc,
    const __nv_bfloat16* __restrict__ vc, const int32_t* __restrict__ seqlens,
    const int32_t* __restrict__ idx, float* __restrict__ part_o, float* __restrict__ part_lse,
    __nv_bfloat16* __restrict__ out, float* __restrict__ lse, int* __restrict__ row_done,
    const DevPlan* plan, int max_len, int Hq, int Hkv, int B, int topk, int nsplit,
    float scale_log2) {
  constexpr int PER = D / 32;  // dims per lane in p . v
  __shared__ int s_last;
  __shared__ float s_w[kAttnWarps * 32];
  __shared__ float qs[D];
  __shared__ float wm[kAttnWarps], wl[kAttnWarps];
  __shared__ float wo[kAttnWarps][D];
  if (plan->err != 0) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // item = (((s * Hkv + g) * topk + slot) * nsplit + part) * G + hh
  const int G = Hq / Hkv;
  int v = blockIdx.x;
  const int hh = v % G;
  v /= G;
  const int part = v % nsplit;
  v /= nsplit;
  const int slot = v % topk;
  v /= topk;
  const int g = v % Hkv;
  const int s = v / Hkv;
  const int h = g * G + hh;
  const long long row = (long long)s * Hq + h;
  const int b = idx[row * topk + slot];
  const int t = seqlens[s] - 1;
  if (b < 0) return;  // unused slot: not one of the row's parts
  const long long p_id = (row * topk + slot) * nsplit + part;
  const int span = (B + nsplit - 1) / nsplit;  // keys of this part of the block
  const int k0 = b * B + part * span;
  // own block: keys up to t (b > t / B only for a selection of NaN scores)
  const bool b_ok = MOBA_INDEX_OK(plan, b < (max_len + B - 1) / B, kSiteDecodeBlock);
  const int k1 = b_ok && b <= t / B ? min(min(k0 + span, b * B + B), t + 1) : k0;
  if (k1 <= k0) {  // a part of the own block after the query: contributes nothing
    for (int c = threadIdx.x; c < D; c += blockDim.x) part_o[p_id * D + c] = 0.f;
    if (threadIdx.x == 0) part_lse[p_id] = -INFINITY;
  } else {
  for (int c = threadIdx.x; c < D; c += blockDim.x)
    qs[c] = __bfloat162float(q[row * D + c]) * scale_log2;
  __syncthreads();
  const long long stride = (long long)Hkv * D;  // elements per cache token
  const __nv_bfloat16* kbase = kc + ((long long)s * max_len) * stride + (long long)g * D;
  const __nv_bfloat16* vbase = vc + ((long long)s * max_len) * stride + (long long)g * D;
  float m = -INFINITY, l = 0.f;
  float o[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) o[e] = 0.f;
  // Chunks of 32 keys per warp.  K and V rows are read whole by the warp
  // (lane = PER dims of the row: coalesced), so q . k leaves each lane with
  // partial dots of all 32 keys; a transposing butterfly (16 + 8 + 4 + 2 + 1
  // shuffles) then leaves lane i with the full dot of key i.  Rows past the
  // end are clamped to the last valid key and get weight 0.
  float qv[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) qv[e] = qs[lane * PER + e];
  auto row_ld = [&](const __nv_bfloat16* basep, int key) -> uint2 {
    const __nv_bfloat16* r = basep + (long long)min(key, k1 - 1) * stride + lane * PER;
    uint2 v;
    if (PER == 4) {
      v = __ldg(reinterpret_cast<const uint2*>(r));
    } else {
      v.x = __ldg(reinterpret_cast<const unsigned int*>(r));
      v.y = 0u;
    }
    return v;
  };
  for (int base = k0 + warp * 32; base < k1; base += 32 * kAttnWarps) {
    float part[32];
#pragma unroll
    for (int k8 = 0; k8 < 32; k8 += 16) {
      uint2 kv[16];
#pragma unroll
      for (int kk = 0; kk < 16; ++kk) kv[kk] = row_ld(kbase, base + k8 + kk);
#pragma unroll
      for (int kk = 0; kk < 16; ++kk) {
        float a = qv[0] * bf16_lo(kv[kk].x);
        a = fmaf(qv[1 % PER], bf16_hi(kv[kk].x), a);
        if (PER == 4) {
          a = fmaf(qv[2 % PER], bf16_lo(kv[kk].y), a);
          a = fmaf(qv[3 % PER], bf16_hi(kv[kk].y), a);
        }
        part[k8 + kk] = a;
      }
    }
    // transposing reduction: at width w the lane keeps the half of its w
    // partial sums whose key has the lane's bit w/2 ... and adds the partner's
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
    const float x = base + lane < k1 ? part[0] : -INFINITY;
    float cm = x;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, off));
    const float mn = fmaxf(m, cm);
    const float alpha = exp2f(m - mn);  // m = -inf on the first chunk: alpha = 0
    const float p = exp2f(x - mn);
    l = l * alpha + p;
#pragma unroll
    for (int e = 0; e < PER; ++e) o[e] *= alpha;
    m = mn;
#pragma unroll
    for (int k8 = 0; k8 < 32; k8 += 16) {
      uint2 vv[16];
#pragma unroll
      for (int kk = 0; kk < 16; ++kk) vv[kk] = row_ld(vbase, base + k8 + kk);
#pragma unroll
      for (int kk = 0; kk < 16; ++kk) {
        const float pk = __shfl_sync(0xffffffffu, p, k8 + kk);
        o[0] = fmaf(pk, bf16_lo(vv[kk].x), o[0]);
        o[1 % PER] = fmaf(pk, bf16_hi(vv[kk].x), o[1 % PER]);
        if (PER == 4) {
          o[2 % PER] = fmaf(pk, bf16_lo(vv[kk].y), o[2 % PER]);
          o[3 % PER] = fmaf(pk, bf16_hi(vv[kk].y), o[3 % PER]);
        }
      }
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) l += __shfl_xor_sync(0xffffffffu, l, off);
  if (lane == 0) {
    wm[warp] = m;
    wl[warp] = l;
  }
#pragma unroll
  for (int e = 0; e < PER; ++e) wo[warp][lane * PER + e] = o[e];
  __syncthreads();
  float mt = -INFINITY;
#pragma unroll
  for (int w2 = 0; w2 < kAttnWarps; ++w2) mt = fmaxf(mt, wm[w2]);
  float lt = 0.f;
  float sc_w[kAttnWarps];
#pragma unroll
  for (int w2 = 0; w2 < kAttnWarps; ++w2) {
    sc_w[w2] = wm[w2] == -INFINITY ? 0.f : exp2f(wm[w2] - mt);  // a warp with no keys adds 0
    lt += wl[w2] * sc_w[w2];
  }
  for (int c = threadIdx.x; c < D; c += blockDim.x) {
    float acc = 0.f;
#pragma unroll
    for (int w2 = 0; w2 < kAttnWarps; ++w2) acc += wo[w2][c] * sc_w[w2];
    part_o[p_id * D + c] = acc / lt;
  }
  if (threadIdx.x == 0) part_lse[p_id] = (mt + log2f(lt)) * 0.6931471805599453f;
  }
  // The CTA that delivers a row's last part merges the row's parts (log-sum-
  // exp, ascending block order) into out / lse and re-arms the row's counter.
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    const int32_t* srow = idx + row * topk;
    int nsel = 0;
    for (int c = 0; c < topk; ++c) nsel += srow[c] >= 0 ? 1 : 0;
    s_last = atomicAdd(&row_done[row], 1) == nsel * nsplit - 1 ? nsel * nsplit : 0;
  }
  __syncthreads();
  const int np = s_last;
  if (np == 0) return;
  __threadfence();
  const long long p0 = row * topk * nsplit;
  float m = -INFINITY;
  for (int c = 0; c < np; ++c) m = fmaxf(m, __ldcg(part_lse + p0 + c));
  // weights of the parts, then one output column per thread
  float wsum = 0.f;
  for (int c = threadIdx.x; c < np; c += blockDim.x) s_w[c] = expf(__ldcg(part_lse + p0 + c) - m);
  __syncthreads();
  for (int c = 0; c < np; ++c) wsum += s_w[c];
  for (int c = threadIdx.x; c < D; c += blockDim.x) {
    float acc = 0.f;
    for (int i = 0; i < np; ++i) acc = fmaf(s_w[i], __ldcg(part_o + (p0 + i) * D + c), acc);
    out[row * D + c] = __float2bfloat16(acc / wsum);
  }
  if (threadIdx.x == 0) {
    lse[row] = m + logf(wsum);
    row_done[row] = 0;
  }
}

// ---------------------------------------------------------------------------
// block means (fp64 accumulation over the block's keys, one thread per column)
// grid (max_blocks or 1, n_seqs, ceil(Hkv * D / 256)); step mode: only the
// block the new token filled
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) decode_kbar_kernel(const __nv_bfloat16* __restrict__ kc,
                                                          const int32_t* __restrict__ seqlens,
                                                          float* __restrict__ kbar, DevPlan* plan,
                                                          int max_len, int max_blocks, int Hkv,
                                                          int D, int B, int step) {
  const int s = blockIdx.y;
  const int L = seqlens[s];
  if (L < 1 || L > max_len) {
    if (threadIdx.x == 0 && blockIdx.x == 0 && blockIdx.z == 0) raise_error(plan, kErrBadSeqlens, s);
    return;
  }
  int i;
  if (step) {
    if (L % B != 0) return;
    i = L / B - 1;
  } else {
    i = blockIdx.x;
    if (i >= L / B) return;
  }
  if (i >= max_blocks) return;
  const int cols = Hkv * D;
  const int c = blockIdx.z * blockDim.x + threadIdx.x;
  if (c >= cols) return;
  const __nv_bfloat16* src = kc + ((long long)s * max_len + (long long)i * B) * cols + c;
  double acc = 0.0;
  for (int r = 0; r < B; ++r) acc += (double)__bfloat162float(src[(long long)r * cols]);
  kbar[((long long)s * max_blocks + i) * cols + c] = (float)(acc / B);
}

}  // namespace

// ---------------------------------------------------------------------------
cudaError_t launch_decode_kbar(const void* k_cache, const int32_t* seqlens, float* kbar,
                               DevPlan* plan, int n_seqs, int max_len, int Hkv, int d, int B,
                               bool step, cudaStream_t st) {
  const int max_blocks = max_len / B;
  if (max_blocks == 0 || n_seqs == 0) return cudaSuccess;
  dim3 grid(step ? 1 : max_blocks, n_seqs, (Hkv * d + 255) / 256);
  decode_kbar_kernel<<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(k_cache), seqlens,
                                           kbar, plan, max_len, max_blocks, Hkv, d, B,
                                           step ? 1 : 0);
  return cudaGetLastError();
}

// Parts per selected block: ~1024 keys each, at most 256 parts per row (the
// merging CTA keeps one weight per part in shared memory).
int decode_splits(int B, int topk) {
  int n = B >= 2048 ? B / 1024 : 1;
  const int cap = 32 * kAttnWarps / topk;
  return n < cap ? n : (cap > 1 ? cap : 1);
}

size_t decode_gate_smem(int max_len, int B, int d) {
  (void)d;
  return sizeof(float) * (size_t)(max_len / B + 1);
}

template <int D>
static cudaError_t decode_run(const void* q, const void* k_cache, const void* v_cache,
                              const int32_t* seqlens, float* kbar, void* out, float* lse,
                              int32_t* idx, float* part_o, float* part_lse, int* row_done,
                              double* kb_part, int* seq_done, DevPlan* plan,
                              int n_seqs, int max_len, int Hq, int Hkv, int B, int topk,
                              float scale_log2, cudaStream_t st) {
  const int max_blocks = max_len / B;
  const int rows = n_seqs * Hq;
  const size_t smem = decode_gate_smem(max_len, B, D);
  cudaError_t e = cudaSuccess;
  if (smem > 48 * 1024)
    e = cudaFuncSetAttribute(decode_gate_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
  if (e != cudaSuccess) return e;
  decode_gate_kernel<D><<<rows, 32 * kGateWarps, smem, st>>>(
      static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k_cache), kbar,
      seqlens, idx, kb_part, seq_done, plan, n_seqs, max_len, max_blocks, Hq, Hkv, B, topk);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const int nsplit = decode_splits(B, topk);
  decode_attn_kernel<D><<<(unsigned)(rows * topk * nsplit), 32 * kAttnWarps, 0, st>>>(
      static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k_cache),
      static_cast<const __nv_bfloat16*>(v_cache), seqlens, idx, part_o, part_lse,
      static_cast<__nv_bfloat16*>(out), lse, row_done, plan, max_len, Hq, Hkv, B, topk, nsplit,
      scale_log2);
  return cudaGetLastError();
}

cudaError_t launch_decode(const void* q, const void* k_cache, const void* v_cache,
                          const int32_t* seqlens, float* kbar, void* out, float* lse, int32_t* idx,
                          float* part_o, float* part_lse, int* row_done, double* kb_part,
                          int* seq_done, DevPlan* plan, int n_seqs, int max_len,
                          int Hq, int Hkv, int d, int B, int topk, float scale_log2,
                          cudaStream_t st) {
  if (d == 128)
    return decode_run<128>(q, k_cache, v_cache, seqlens, kbar, out, lse, idx, part_o, part_lse,
                           row_done, kb_part, seq_done, plan, n_seqs, max_len, Hq, Hkv, B, topk,
                           scale_log2, st);
  return decode_run<64>(q, k_cache, v_cache, seqlens, kbar, out, lse, idx, part_o, part_lse,
                        row_done, kb_part, seq_done, plan, n_seqs, max_len, Hq, Hkv, B, topk,
                        scale_log2, st);
}

}  // namespace moba
