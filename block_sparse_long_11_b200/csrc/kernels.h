// Host-side launchers of the MoBA kernels (internal to the library).
#pragma once
#include "common.cuh"

namespace moba {

// Workspace guards of the MOBA_DEBUG build (at most kMaxGuards per call).
constexpr int kMaxGuards = 32;
constexpr int kGuardWords = 64;  // 256 bytes
struct Guards {
  int n;
  uint32_t* p[kMaxGuards];
};
cudaError_t launch_guard_fill(const Guards& gs, cudaStream_t st);
cudaError_t launch_guard_check(const Guards& gs, DevPlan* plan, cudaStream_t st);

cudaError_t launch_plan(const int* cu, const Sizes& z, const Workspace& ws, cudaStream_t st);
cudaError_t launch_pool(const void* k, const Sizes& z, const Workspace& ws, cudaStream_t st);
cudaError_t launch_gate(const void* q, int32_t* idx, const Sizes& z, const Workspace& ws,
                        cudaStream_t st);
bool gate_tc_supported(const Sizes& z);
cudaError_t launch_gate_tc(const void* q, int32_t* idx, const Sizes& z, const Workspace& ws,
                           int num_sms, cudaStream_t st);
// stable: every bucket's entries in ascending (token, head) order (needs
// ws.cm; without it, or with stable = false, the order inside a bucket is
// whatever the fill's atomics give)
cudaError_t launch_sched(const int32_t* idx, const Sizes& z, const Workspace& ws, int t0, int t1,
                         int unit_rows, cudaStream_t st, bool stable = false);
// Attention of every routed row to its past blocks and of every token to its
// own block (causal), one persistent tcgen05 kernel; writes the partial slots.
int attn_unit_rows();
// Test of the attention kernel's bounded waits (see moba_debug_attention_wait_test).
void set_attn_wait_test(int on);
int attn_wait_test();
cudaError_t launch_attn(const void* q, const void* k, const void* v, const Sizes& z,
                        const Workspace& ws, int t0, int t1, float scale_log2, int num_sms,
                        cudaStream_t st);
// Dense causal attention with the same kernel: the plan must cut the
// sequences into blocks of attn_unit_rows() tokens; ws.part_o / ws.part_lse
// are the caller's out / lse and z.topk is 1.
cudaError_t launch_attn_full(const void* q, const void* k, const void* v, const Sizes& z,
                             const Workspace& ws, float scale_log2, int num_sms, cudaStream_t st);
// Decode (one new query per sequence against a padded KV cache).
cudaError_t launch_decode_kbar(const void* k_cache, const int32_t* seqlens, float* kbar,
                               DevPlan* plan, int n_seqs, int max_len, int Hkv, int d, int B,
                               bool step, cudaStream_t st);
size_t decode_gate_smem(int max_len, int B, int d);
int decode_splits(int B, int topk);  // parts per selected block in the decode attention
cudaError_t launch_decode(const void* q, const void* k_cache, const void* v_cache,
                          const int32_t* seqlens, float* kbar, void* out, float* lse, int32_t* idx,
                          float* part_o, float* part_lse, int* row_done, double* kb_part,
                          int* seq_done, DevPlan* plan, int n_seqs, int max_len, int Hq, int Hkv,
                          int d, int B, int topk, float scale_log2, cudaStream_t st);
// Backward with the selection held fixed (tensor cores): D = dout . out per
// row and a check of the selection; dK / dV per key tile over the whole
// sequence's bucket lists (written directly); dQ per query chunk as fp32
// partial slots, then their sum in slot order.
cudaError_t launch_bwd_prep(const void* out, const void* dout, const int32_t* idx,
                            const int32_t* cu, const Sizes& z, float* dvec, DevPlan* plan,
                            cudaStream_t st);
// Packed row buffers of the dK / dV kernel: Q and dO rows of `cap` bucket
// entries (plus 64 zero rows after the last), and their (-lse log2 e, D).
struct DkvPack {
  __nv_bfloat16* qp;  // [cap + 64, d]
  __nv_bfloat16* gp;  // [cap + 64, d]
  float2* ld;         // [cap + 64]
  int cap;
};
cudaError_t launch_backward_dkv(const void* q, const void* k, const void* v, const void* dout,
                                const float* lse, const float* dvec, const Sizes& z,
                                const Workspace& ws, const DkvPack& pk, float* dk, float* dv,
                                float scale, int num_sms, cudaStream_t st);
cudaError_t launch_backward_dq(const void* q, const void* k, const void* v, const void* dout,
                               const float* lse, const float* dvec, const Sizes& z,
                               const Workspace& ws, float* dq_part, float* dq, int t0, int t1,
                               float scale, int num_sms, cudaStream_t st);
cudaError_t launch_dq_merge(const int32_t* idx, const float* part, float* dq, const Sizes& z,
                            const DevPlan* plan, int t0, int t1, cudaStream_t st);
cudaError_t launch_merge(const int32_t* idx, void* out, float* lse, const Sizes& z,
                         const Workspace& ws, int t0, int t1, cudaStream_t st);

}  // namespace moba
