// Block attention with warp-level mma.sync (m16n8k16, bf16 in, fp32 accumulate).
//
// Page cited by title: "同一天，DeepSeek和月之暗面發表了關于改進注意力機制的論文"
// (MoBA write-up), section "MoBA：將 MoE 原理應用于注意力機制", step 3: the
// attention output of every KV block with the query tokens assigned to it.
//
// Two tile kinds, one kernel body:
//  * PAST  (OWN = false): 128 gathered (token, head) rows of one bucket
//    (full block, kv head) against all B keys of that block, no mask.
//  * OWN   (OWN = true):  128 consecutive tokens of one head inside their own
//    block, keys 0..t (token-level causal mask).
// Each row's normalised output (bf16) and log-sum-exp (fp32) go to its
// partial slot; the merge kernel combines a row's slots.
//
// CTA: 8 warps x 16 rows, K/V tiles of 64 keys double-buffered with cp.async,
// 16-byte chunks XOR-swizzled by (row & 7) so ldmatrix is conflict-free.
#include "common.cuh"
#include "kernels.h"

namespace moba {
namespace {

constexpr int BM = 128;  // rows per CTA
constexpr int BN = 64;   // keys per K/V tile

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(dst), "l"(src));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N));
}
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void mma16816(float* c, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// byte offset of 16-byte chunk c of row r in a [rows][D] bf16 tile
template <int D>
__device__ __forceinline__ uint32_t swz(int r, int c) {
  return static_cast<uint32_t>(r * (D * 2) + ((c ^ (r & 7)) << 4));
}

template <int D>
struct Smem {
  __nv_bfloat16 q[BM * D];
  __nv_bfloat16 k[2][BN * D];
  __nv_bfloat16 v[2][BN * D];
  int qrow[BM];   // t * Hq + h of each row
  int part[BM];   // partial slot id, -1 = row not written
  int lim[BM];    // last key (block-local) the row may attend
};

template <int D, bool OWN>
__global__ void __launch_bounds__(256) attn_mma_kernel(const __nv_bfloat16* __restrict__ q,
                                                       const __nv_bfloat16* __restrict__ k,
                                                       const __nv_bfloat16* __restrict__ v,
                                                       Workspace ws, int Hq, int Hkv, int topk,
                                                       int B, int t0, int t1, float scale_log2) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  Smem<D>& sm = *reinterpret_cast<Smem<D>*>(smem_raw);
  const DevPlan* plan = ws.plan;
  if (plan->err != 0) return;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  constexpr int CH = D / 8;  // 16-byte chunks per row

  int n_units = OWN ? 1 : plan->ntiles;
  for (int unit = OWN ? 0 : blockIdx.x; unit < n_units; unit += OWN ? 1 : gridDim.x) {
    int key_start, g, nkeys;
    // ---- tile description -------------------------------------------------
    if (OWN) {
      const int gb = blockIdx.x;
      if (gb >= plan->nblk_total) return;
      const int len = ws.blk_len[gb];
      const int y0 = blockIdx.y * BM;
      if (y0 >= len) return;
      const int bstart = ws.blk_start[gb];
      if (bstart + y0 >= t1 || bstart + min(len, y0 + BM) <= t0) return;
      const int h = blockIdx.z;
      g = h / (Hq / Hkv);
      key_start = bstart;
      nkeys = min(len, y0 + BM);
      const int j = ws.blk_j[gb];
      const int slot = min(topk, j + 1) - 1;
      if (tid < BM) {
        int tl = y0 + tid;
        int tt = bstart + min(tl, len - 1);
        bool ok = tl < len && tt >= t0 && tt < t1;
        sm.qrow[tid] = tt * Hq + h;
        sm.part[tid] = ok ? ((tt - t0) * Hq + h) * topk + slot : -1;
        sm.lim[tid] = tl < len ? tl : len - 1;
      }
    } else {
      const int2 tile = ws.tiles[unit];
      const int b = tile.x, e0 = tile.y;
      const int e1 = min(e0 + BM, ws.bucket_off[b + 1]);
      const int fb = b / Hkv;
      g = b - fb * Hkv;
      key_start = ws.full_start[fb];
      nkeys = B;
      if (tid < BM) {
        int e = e0 + min(tid, e1 - e0 - 1);
        int p = ws.entries[e];
        sm.qrow[tid] = t0 * Hq + p / topk;
        sm.part[tid] = tid < e1 - e0 ? p : -1;
        sm.lim[tid] = B - 1;
      }
    }
    __syncthreads();

    // ---- loads ----------------------------------------------------------------
    const long long kv_stride = (long long)Hkv * D;
    const __nv_bfloat16* kbase = k + (long long)key_start * kv_stride + (long long)g * D;
    const __nv_bfloat16* vbase = v + (long long)key_start * kv_stride + (long long)g * D;
    auto load_kv = [&](int n, int buf) {
      const int kmax = nkeys - 1;
      for (int c = tid; c < BN * CH; c += 256) {
        int r = c / CH, ch = c % CH;
        int u = min(n * BN + r, kmax);
        cp_async16(smem_u32(sm.k[buf]) + swz<D>(r, ch), kbase + u * kv_stride + ch * 8);
        cp_async16(smem_u32(sm.v[buf]) + swz<D>(r, ch), vbase + u * kv_stride + ch * 8);
      }
    };
    for (int c = tid; c < BM * CH; c += 256) {
      int r = c / CH, ch = c % CH;
      cp_async16(smem_u32(sm.q) + swz<D>(r, ch), q + (long long)sm.qrow[r] * D + ch * 8);
    }
    load_kv(0, 0);
    cp_async_commit();

    const int ntiles_kv = (nkeys + BN - 1) / BN;
    const int r0 = warp * 16 + (lane >> 2);  // this thread's two rows: r0, r0 + 8
    const int lim0 = sm.lim[r0], lim1 = sm.lim[r0 + 8];
    uint32_t qf[D / 16][4];
    float oacc[D / 8][4];
#pragma unroll
    for (int i = 0; i < D / 8; ++i) oacc[i][0] = oacc[i][1] = oacc[i][2] = oacc[i][3] = 0.f;
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;

    for (int n = 0; n < ntiles_kv; ++n) {
      if (n + 1 < ntiles_kv) {
        load_kv(n + 1, (n + 1) & 1);
        cp_async_commit();
        cp_async_wait<1>();
      } else {
        cp_async_wait<0>();
      }
      __syncthreads();
      if (n == 0) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          int mi = lane >> 3;
          int row = warp * 16 + (mi & 1) * 8 + (lane & 7);
          ldsm_x4(smem_u32(sm.q) + swz<D>(row, kk * 2 + (mi >> 1)), qf[kk][0], qf[kk][1],
                  qf[kk][2], qf[kk][3]);
        }
      }
      const uint32_t ks = smem_u32(sm.k[n & 1]);
      const uint32_t vs = smem_u32(sm.v[n & 1]);
      // S = Q K^T : 16 rows x 64 keys per warp
      float s[BN / 8][4];
#pragma unroll
      for (int i = 0; i < BN / 8; ++i) s[i][0] = s[i][1] = s[i][2] = s[i][3] = 0.f;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
#pragma unroll
        for (int np = 0; np < BN / 16; ++np) {
          int mi = lane >> 3;
          int key = np * 16 + (mi >> 1) * 8 + (lane & 7);
          uint32_t b0, b1, b2, b3;
          ldsm_x4(ks + swz<D>(key, kk * 2 + (mi & 1)), b0, b1, b2, b3);
          mma16816(s[2 * np], qf[kk], b0, b1);
          mma16816(s[2 * np + 1], qf[kk], b2, b3);
        }
      }
      // online softmax in base 2
      float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
      for (int i = 0; i < BN / 8; ++i) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          int u = n * BN + i * 8 + (lane & 3) * 2 + e;
          float a = s[i][e] * scale_log2, b = s[i][2 + e] * scale_log2;
          if (OWN) {
            if (u > lim0) a = -INFINITY;
            if (u > lim1) b = -INFINITY;
          }
          s[i][e] = a;
          s[i][2 + e] = b;
          mx0 = fmaxf(mx0, a);
          mx1 = fmaxf(mx1, b);
        }
      }
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
      const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
      const float base0 = mn0 == -INFINITY ? 0.f : mn0;
      const float base1 = mn1 == -INFINITY ? 0.f : mn1;
      const float al0 = exp2f(m0 - base0), al1 = exp2f(m1 - base1);
      m0 = mn0;
      m1 = mn1;
      float rs0 = 0.f, rs1 = 0.f;
#pragma unroll
      for (int i = 0; i < BN / 8; ++i) {
        s[i][0] = exp2f(s[i][0] - base0);
        s[i][1] = exp2f(s[i][1] - base0);
        s[i][2] = exp2f(s[i][2] - base1);
        s[i][3] = exp2f(s[i][3] - base1);
        rs0 += s[i][0] + s[i][1];
        rs1 += s[i][2] + s[i][3];
      }
      l0 = l0 * al0 + rs0;
      l1 = l1 * al1 + rs1;
#pragma unroll
      for (int i = 0; i < D / 8; ++i) {
        oacc[i][0] *= al0;
        oacc[i][1] *= al0;
        oacc[i][2] *= al1;
        oacc[i][3] *= al1;
      }
      // O += P V
#pragma unroll
      for (int kk = 0; kk < BN / 16; ++kk) {
        uint32_t a[4];
        a[0] = pack_bf16(s[2 * kk][0], s[2 * kk][1]);
        a[1] = pack_bf16(s[2 * kk][2], s[2 * kk][3]);
        a[2] = pack_bf16(s[2 * kk + 1][0], s[2 * kk + 1][1]);
        a[3] = pack_bf16(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
        for (int dp = 0; dp < D / 16; ++dp) {
          int mi = lane >> 3;
          int key = kk * 16 + (mi & 1) * 8 + (lane & 7);
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(vs + swz<D>(key, dp * 2 + (mi >> 1)), b0, b1, b2, b3);
          mma16816(oacc[2 * dp], a, b0, b1);
          mma16816(oacc[2 * dp + 1], a, b2, b3);
        }
      }
      __syncthreads();
    }
    // ---- epilogue: normalise, write the partial slot ----------------------------
    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
    const int p0 = sm.part[r0], p1 = sm.part[r0 + 8];
    const float inv0 = 1.f / l0, inv1 = 1.f / l1;
    constexpr float kLn2 = 0.6931471805599453f;
#pragma unroll
    for (int i = 0; i < D / 8; ++i) {
      int col = i * 8 + (lane & 3) * 2;
      if (p0 >= 0)
        *reinterpret_cast<uint32_t*>(ws.part_o + (long long)p0 * D + col) =
            pack_bf16(oacc[i][0] * inv0, oacc[i][1] * inv0);
      if (p1 >= 0)
        *reinterpret_cast<uint32_t*>(ws.part_o + (long long)p1 * D + col) =
            pack_bf16(oacc[i][2] * inv1, oacc[i][3] * inv1);
    }
    if ((lane & 3) == 0) {
      if (p0 >= 0) ws.part_lse[p0] = (m0 + log2f(l0)) * kLn2;
      if (p1 >= 0) ws.part_lse[p1] = (m1 + log2f(l1)) * kLn2;
    }
    __syncthreads();
  }
}

template <int D, bool OWN>
cudaError_t launch_one(dim3 grid, const void* q, const void* k, const void* v, const Sizes& z,
                       const Workspace& ws, int t0, int t1, float scale_log2, cudaStream_t st) {
  const size_t smem = sizeof(Smem<D>);
  cudaError_t e = cudaFuncSetAttribute(attn_mma_kernel<D, OWN>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  attn_mma_kernel<D, OWN><<<grid, 256, smem, st>>>(
      static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
      static_cast<const __nv_bfloat16*>(v), ws, z.Hq, z.Hkv, z.topk, z.B, t0, t1, scale_log2);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_past(const void* q, const void* k, const void* v, const Sizes& z,
                             const Workspace& ws, int t0, int t1, float scale_log2,
                             int num_sms, cudaStream_t st) {
  if (z.nfull_max == 0 || z.topk < 2) return cudaSuccess;
  int grid = num_sms * 2;
  if (grid > z.ntiles_max) grid = z.ntiles_max > 0 ? z.ntiles_max : 1;
  if (z.d == 128)
    return launch_one<128, false>(dim3(grid), q, k, v, z, ws, t0, t1, scale_log2, st);
  return launch_one<64, false>(dim3(grid), q, k, v, z, ws, t0, t1, scale_log2, st);
}

cudaError_t launch_attn_own(const void* q, const void* k, const void* v, const Sizes& z,
                            const Workspace& ws, int t0, int t1, float scale_log2,
                            cudaStream_t st) {
  dim3 grid(z.nblk_max, (z.B + BM - 1) / BM, z.Hq);
  if (z.d == 128) return launch_one<128, true>(grid, q, k, v, z, ws, t0, t1, scale_log2, st);
  return launch_one<64, true>(grid, q, k, v, z, ws, t0, t1, scale_log2, st);
}

}  // namespace moba
