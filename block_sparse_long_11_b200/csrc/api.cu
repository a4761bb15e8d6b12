// C ABI of the MoBA forward: argument checks, workspace carving and the launch
// sequence.  Declared in include/moba.h.
//
// Launch sequence of moba_forward (all on the caller's stream, no host sync):
//   plan -> pool (2 kernels) -> gate -> per query chunk:
//   scheduler (count, scan, scatter, unit list) -> block attention (past blocks
//   and own block, one tcgen05 kernel) -> merge.
#include <math.h>
#include <string.h>

#include <mutex>

#include "../../include/moba.h"
#include "common.cuh"
#include "kernels.h"

namespace moba {
namespace {

constexpr long long kAlign = 256;

#ifdef MOBA_DEBUG
constexpr long long kGuardBytes = 4LL * kGuardWords;
int g_poison = 0;  // moba_debug_poison's mode
#else
constexpr long long kGuardBytes = 0;
#endif

// Lays the regions of a workspace out one after another at kAlign
// boundaries.  In MOBA_DEBUG builds every region is followed by a guard,
// recorded in `guards` when the guard lies inside the first `owned` bytes
// (owned < 0: all of them).
struct Carver {
  char* base;
  Guards* guards;
  long long owned;
  long long off = 0;
  Carver(char* b, Guards* g, long long own) : base(b), guards(g), owned(own) {
    if (guards) guards->n = 0;
  }
  char* take(long long bytes) {
    char* p = base ? base + off : nullptr;
    off = align_up(off + (bytes > 0 ? bytes : 0), kAlign);
    if (kGuardBytes > 0) {
      if (guards && base && guards->n < kMaxGuards && (owned < 0 || off + kGuardBytes <= owned))
        guards->p[guards->n++] = reinterpret_cast<uint32_t*>(base + off);
      off = align_up(off + kGuardBytes, kAlign);
    }
    return p;
  }
};

// Capacities the MOBA_DEBUG index checks test against.
void set_caps(const Sizes& z, Workspace* ws) {
  ws->rows_cap = (long long)z.T * z.Hq;
  ws->entries_cap = z.entries_max;
  ws->nbk_cap = z.nbk_max;
  ws->cm_cap = 0;
#ifdef MOBA_DEBUG
  ws->poison = g_poison;
#else
  ws->poison = 0;
#endif
}

// MOBA_DEBUG: fill a call's guards before its first kernel (and plant the
// overwrite of moba_debug_poison mode 2) / check them after its last one.
cudaError_t guards_begin(const Guards& g, cudaStream_t st) {
#ifdef MOBA_DEBUG
  cudaError_t e = launch_guard_fill(g, st);
  if (e == cudaSuccess && g_poison == 2 && g.n > 0) e = cudaMemsetAsync(g.p[0], 0, 4, st);
  return e;
#else
  (void)g;
  (void)st;
  return cudaSuccess;
#endif
}

cudaError_t guards_end(const Guards& g, DevPlan* plan, cudaStream_t st) {
#ifdef MOBA_DEBUG
  return launch_guard_check(g, plan, st);
#else
  (void)g;
  (void)plan;
  (void)st;
  return cudaSuccess;
#endif
}

moba_status check_args(int T, int n_seqs, int Hq, int Hkv, int d, int B, int topk) {
  if (T < 0 || n_seqs < 1 || Hq < 1 || Hkv < 1 || topk < 1 || B < 1) return MOBA_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return MOBA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return MOBA_ERR_UNSUPPORTED;
  if (B % 64 != 0 || B > 65536) return MOBA_ERR_UNSUPPORTED;
  if (topk > 64) return MOBA_ERR_UNSUPPORTED;
  if ((long long)T * Hq >= (1LL << 31)) return MOBA_ERR_UNSUPPORTED;
  if ((long long)T * Hq * topk >= (1LL << 40)) return MOBA_ERR_UNSUPPORTED;
  return MOBA_OK;
}

moba_status make_sizes(int T, int n_seqs, int Hq, int Hkv, int d, int B, int topk, int chunk,
                       Sizes* z) {
  moba_status s = check_args(T, n_seqs, Hq, Hkv, d, B, topk);
  if (s != MOBA_OK) return s;
  if (chunk < 0) return MOBA_ERR_INVALID_ARG;
  z->T = T;
  z->n_seqs = n_seqs;
  z->Hq = Hq;
  z->Hkv = Hkv;
  z->d = d;
  z->B = B;
  z->topk = topk;
  z->chunk = (chunk == 0 || chunk > T) ? T : chunk;
  if (z->chunk < 1) z->chunk = 1;
  if ((long long)z->chunk * Hq * topk >= (1LL << 31)) return MOBA_ERR_UNSUPPORTED;
  z->nfull_max = T / B;
  long long nblk = (long long)T / B + n_seqs;
  if (nblk >= (1LL << 31)) return MOBA_ERR_UNSUPPORTED;
  z->nblk_max = (int)nblk;
  long long nbk = (long long)z->nfull_max * Hkv;
  if (nbk >= (1LL << 30)) return MOBA_ERR_UNSUPPORTED;
  z->nbk_max = (int)nbk;
  z->entries_max = (long long)z->chunk * Hq * (topk - 1);
  long long nt = z->entries_max / kTileRows + z->nbk_max + 1;
  if (nt >= (1LL << 31)) return MOBA_ERR_UNSUPPORTED;
  z->ntiles_max = (int)nt;
  z->part_rows = (long long)z->chunk * Hq * topk;
  return MOBA_OK;
}

// Carves the workspace.  gate_end receives the bytes the gate alone needs.
long long carve(const Sizes& z, char* base, Workspace* w, long long* gate_end,
                Guards* guards = nullptr, long long owned = -1) {
  Carver c(base, guards, owned);
  auto take = [&](long long bytes) -> char* { return c.take(bytes); };
  Workspace ws;
  memset(&ws, 0, sizeof(ws));
  ws.plan = reinterpret_cast<DevPlan*>(take(sizeof(DevPlan)));
  ws.seq_blk_base = reinterpret_cast<int*>(take(4LL * (z.n_seqs + 1)));
  ws.seq_full_base = reinterpret_cast<int*>(take(4LL * (z.n_seqs + 1)));
  ws.blk_start = reinterpret_cast<int*>(take(4LL * z.nblk_max));
  ws.blk_len = reinterpret_cast<int*>(take(4LL * z.nblk_max));
  ws.blk_j = reinterpret_cast<int*>(take(4LL * z.nblk_max));
  ws.blk_fullbase = reinterpret_cast<int*>(take(4LL * z.nblk_max));
  ws.full_start = reinterpret_cast<int*>(take(4LL * z.nfull_max));
  const long long nk = (long long)z.nfull_max * z.Hkv * z.d;
  ws.pool_part = reinterpret_cast<float*>(take(4LL * nk * kPoolSplit));
  ws.kbar = reinterpret_cast<float*>(take(4LL * nk));
  ws.kbar_hi = reinterpret_cast<__nv_bfloat16*>(take(2LL * nk));
  ws.kbar_lo = reinterpret_cast<__nv_bfloat16*>(take(2LL * nk));
  if (gate_end) *gate_end = c.off;
  ws.idx = reinterpret_cast<int32_t*>(take(4LL * z.T * z.Hq * z.topk));
  ws.bucket_count = reinterpret_cast<int*>(take(4LL * (z.nbk_max + 1)));
  ws.bucket_off = reinterpret_cast<int*>(take(4LL * (z.nbk_max + 1)));
  ws.bucket_cursor = reinterpret_cast<int*>(take(4LL * (z.nbk_max + 1)));
  ws.tile_off = reinterpret_cast<int*>(take(4LL * (z.nbk_max + 1)));
  ws.entries = reinterpret_cast<int*>(take(4LL * z.entries_max));
  ws.tiles = reinterpret_cast<int2*>(take(8LL * z.ntiles_max));
  ws.part_o = reinterpret_cast<__nv_bfloat16*>(take(2LL * z.part_rows * z.d));
  ws.part_lse = reinterpret_cast<float*>(take(4LL * z.part_rows));
  set_caps(z, &ws);
  if (w) *w = ws;
  return c.off;
}


// Sizes and workspace of the dense causal path: the plan's per-block arrays
// with blocks of attn_unit_rows() tokens, nothing else.
moba_status make_sizes_full(int T, int n_seqs, int Hq, int Hkv, int d, Sizes* z) {
  moba_status s = make_sizes(T, n_seqs, Hq, Hkv, d, attn_unit_rows(), 1, 0, z);
  if (s != MOBA_OK) return s;
  if ((long long)z->nblk_max * Hq >= (1LL << 31)) return MOBA_ERR_UNSUPPORTED;
  return MOBA_OK;
}

long long carve_full(const Sizes& z, char* base, Workspace* w, Guards* guards = nullptr,
                     long long owned = -1) {
  Carver c(base, guards, owned);
  auto take = [&](long long bytes) -> char* { return c.take(bytes); };
  Workspace ws;
  memset(&ws, 0, sizeof(ws));
  ws.plan = reinterpret_cast<DevPlan*>(take(sizeof(DevPlan)));
  ws.seq_blk_base = reinterpret_cast<int*>(take(4LL * (z.n_seqs + 1)));
  ws.seq_full_base = reinterpret_cast<int*>(take(4LL * (z.n_seqs + 1)));
  ws.blk_start = reinterpret_cast<int*>(take(4LL * z.nblk_max));
  ws.blk_len = reinterpret_cast<int*>(take(4LL * z.nblk_max));
  ws.blk_j = reinterpret_cast<int*>(take(4LL * z.nblk_max));
  ws.blk_fullbase = reinterpret_cast<int*>(take(4LL * z.nblk_max));
  ws.full_start = reinterpret_cast<int*>(take(4LL * z.nfull_max));
  set_caps(z, &ws);
  if (w) *w = ws;
  return c.off;
}

// Decode: argument checks and workspace (error word, selection, partials).
moba_status check_decode(int n_seqs, int max_len, int Hq, int Hkv, int d, int B, int topk) {
  if (n_seqs < 1 || max_len < 1 || Hq < 1 || Hkv < 1 || B < 1 || topk < 1)
    return MOBA_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return MOBA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return MOBA_ERR_UNSUPPORTED;
  if (B % 64 != 0 || B > 65536 || topk > 64) return MOBA_ERR_UNSUPPORTED;
  if ((long long)n_seqs * Hq * topk * decode_splits(B, topk) >= (1LL << 31))
    return MOBA_ERR_UNSUPPORTED;
  if ((long long)n_seqs * max_len * Hkv * d >= (1LL << 40)) return MOBA_ERR_UNSUPPORTED;
  if (decode_gate_smem(max_len, B, d) > 200 * 1024) return MOBA_ERR_UNSUPPORTED;
  return MOBA_OK;
}

struct DecodeWs {
  DevPlan* plan;
  int* row_done;  // [n_seqs * Hq] parts delivered per row (zeroed by every call)
  int* seq_done;  // [n_seqs] row slices of a filled block summed (zeroed by every call)
  long long zero_bytes;  // plan .. seq_done, cleared by one memset
  double* kb_part;  // [n_seqs, Hq, Hkv * d] per-slice sums of a filled block
  int32_t* idx;
  float* part_o;
  float* part_lse;
};

long long carve_decode(int n_seqs, int Hq, int Hkv, int d, int B, int topk, char* base,
                       DecodeWs* w, Guards* guards = nullptr, long long owned = -1) {
  Carver c(base, guards, owned);
  auto take = [&](long long bytes) -> char* { return c.take(bytes); };
  const long long slots = (long long)n_seqs * Hq * topk;
  const long long parts = slots * decode_splits(B, topk);
  DecodeWs ws;
  ws.plan = reinterpret_cast<DevPlan*>(take(sizeof(DevPlan)));
  ws.row_done = reinterpret_cast<int*>(take(4LL * n_seqs * Hq));
  ws.seq_done = reinterpret_cast<int*>(take(4LL * n_seqs));
  ws.zero_bytes = c.off;
  ws.kb_part = reinterpret_cast<double*>(take(8LL * n_seqs * Hq * Hkv * d));
  ws.idx = reinterpret_cast<int32_t*>(take(4LL * slots));
  ws.part_o = reinterpret_cast<float*>(take(4LL * parts * d));
  ws.part_lse = reinterpret_cast<float*>(take(4LL * parts));
  if (w) *w = ws;
  return c.off;
}

int sm_count() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

moba_status cuda_status(cudaError_t e) { return e == cudaSuccess ? MOBA_OK : MOBA_ERR_CUDA; }

// Backward workspace: the plan's block tables, the bucket lists of the whole
// sequence set (every routed row of every bucket: the dK / dV kernel needs
// them all at once), D per row, and the dQ partial slots of one query chunk.
struct BwdWs {
  Workspace ws;
  float* dvec;     // [T * Hq] dout . out
  float* dq_part;  // [chunk * Hq * topk, d] fp32
  DkvPack pack;    // the dK / dV kernel's packed rows of one chunk of entries
};

// Entries per chunk of the dK / dV kernel's packed rows: every entry when the
// buffers stay within 8 GiB, else as many as fit.
int dkv_pack_cap(const Sizes& z) {
  const long long per = 4LL * z.d + 8;  // Q and dO rows (bf16) and (-lse log2 e, D)
  long long cap = (8LL << 30) / per;
  if (z.entries_max < cap) cap = z.entries_max;
  return (int)(cap < 64 ? 64 : cap);
}

// Slots of the stable fill's count table: (bucket, scheduler CTA) pairs, at
// most N (N - 1) / 2 (full block, later block) pairs for N blocks, times the
// kv heads and the 128-token slices of a block.  0 (the unstable fill) when
// the table would pass 1 GiB or a CTA's per-bucket ranks could pass 16 bits.
long long stable_fill_slots(const Sizes& z) {
  const long long N = z.nblk_max;
  const long long n = N * (N - 1) / 2 * z.Hkv * ((z.B + 127) / 128);
  if (n > (1LL << 28) || z.Hq / z.Hkv > 511) return 0;
  return n;
}

long long carve_bwd(const Sizes& zf, const Sizes& zc, char* base, BwdWs* w,
                    Guards* guards = nullptr, long long owned = -1) {
  Carver c(base, guards, owned);
  auto take = [&](long long bytes) -> char* { return c.take(bytes); };
  BwdWs b;
  memset(&b, 0, sizeof(b));
  Workspace& ws = b.ws;
  ws.plan = reinterpret_cast<DevPlan*>(take(sizeof(DevPlan)));
  ws.seq_blk_base = reinterpret_cast<int*>(take(4LL * (zf.n_seqs + 1)));
  ws.seq_full_base = reinterpret_cast<int*>(take(4LL * (zf.n_seqs + 1)));
  ws.blk_start = reinterpret_cast<int*>(take(4LL * zf.nblk_max));
  ws.blk_len = reinterpret_cast<int*>(take(4LL * zf.nblk_max));
  ws.blk_j = reinterpret_cast<int*>(take(4LL * zf.nblk_max));
  ws.blk_fullbase = reinterpret_cast<int*>(take(4LL * zf.nblk_max));
  ws.full_start = reinterpret_cast<int*>(take(4LL * zf.nfull_max));
  ws.full_nlater = reinterpret_cast<int*>(take(4LL * zf.nfull_max));
  ws.full_cm = reinterpret_cast<long long*>(take(8LL * zf.nfull_max));
  const long long ncm = stable_fill_slots(zf);
  ws.cm = reinterpret_cast<int*>(take(4LL * ncm));
  ws.bucket_count = reinterpret_cast<int*>(take(4LL * (zf.nbk_max + 1)));
  ws.bucket_off = reinterpret_cast<int*>(take(4LL * (zf.nbk_max + 1)));
  ws.bucket_cursor = reinterpret_cast<int*>(take(4LL * (zf.nbk_max + 1)));
  ws.tile_off = reinterpret_cast<int*>(take(4LL * (zf.nbk_max + 1)));
  ws.entries = reinterpret_cast<int*>(take(4LL * zf.entries_max));
  ws.tiles = reinterpret_cast<int2*>(take(8LL * zf.ntiles_max));
  b.dvec = reinterpret_cast<float*>(take(4LL * zf.T * zf.Hq));
  b.dq_part = reinterpret_cast<float*>(take(4LL * zc.part_rows * zc.d));
  b.pack.cap = dkv_pack_cap(zf);
  b.pack.qp = reinterpret_cast<__nv_bfloat16*>(take(2LL * (b.pack.cap + 64) * zf.d));
  b.pack.gp = reinterpret_cast<__nv_bfloat16*>(take(2LL * (b.pack.cap + 64) * zf.d));
  b.pack.ld = reinterpret_cast<float2*>(take(8LL * (b.pack.cap + 64)));
  set_caps(zf, &ws);
  ws.cm_cap = ncm;
  if (w) *w = b;
  return c.off;
}

// Vector loads and cp.async copies read q, k, v and write out in 16-byte units.
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

moba_status run_prefix(const void* q, const void* k, const int32_t* cu, int32_t* idx,
                       const Sizes& z, const Workspace& ws, cudaStream_t st) {
  cudaError_t e = cudaMemsetAsync(ws.plan, 0, sizeof(DevPlan), st);
  if (e == cudaSuccess) e = launch_plan(cu, z, ws, st);
  if (e == cudaSuccess) e = launch_pool(k, z, ws, st);
  if (e == cudaSuccess)
    e = gate_tc_supported(z) ? launch_gate_tc(q, idx, z, ws, sm_count(), st)
                             : launch_gate(q, idx, z, ws, st);
  return cuda_status(e);
}

// Scratch of moba_gate_noalloc: one static device array per GPU that loads
// the library.  Host code must not use the symbol itself as a device address;
// its address on each device is looked up with that device current, once per
// CUDA context (a device reset or a new primary context in the same process
// gives the array a new address, so the cached one is keyed on the context).
constexpr size_t kStaticScratchBytes = MOBA_GATE_STATIC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;
__device__ __align__(256) unsigned char g_gate_scratch[kStaticScratchBytes];
std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};
const void* g_scratch_ctx[kMaxDevices] = {};

// The calling thread's current CUDA context (driver entry point looked up
// through the runtime, so the library needs no link against libcuda).
void* current_context() {
  typedef int (*GetCurrentFn)(void**);
  static GetCurrentFn fn = nullptr;
  static bool looked_up = false;
  if (!looked_up) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult qr;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &qr) == cudaSuccess &&
        qr == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<GetCurrentFn>(p);
    looked_up = true;
  }
  void* ctx = nullptr;
  if (fn && fn(&ctx) != 0) ctx = nullptr;
  return ctx;
}

moba_status static_scratch(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOBA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return MOBA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  // no current context yet (nothing has initialised the runtime on this
  // thread): the lookup below creates it, and the cache is keyed on it after
  const void* ctx = current_context();
  if (!g_scratch_addr[dev] || !ctx || ctx != g_scratch_ctx[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_gate_scratch) != cudaSuccess || !p) return MOBA_ERR_CUDA;
    g_scratch_addr[dev] = p;
    g_scratch_ctx[dev] = current_context();
  }
  *out = g_scratch_addr[dev];
  return MOBA_OK;
}

}  // namespace
}  // namespace moba

using namespace moba;

extern "C" {

const char* moba_status_string(moba_status s) {
  switch (s) {
    case MOBA_OK: return "MOBA_OK";
    case MOBA_ERR_INVALID_ARG: return "MOBA_ERR_INVALID_ARG";
    case MOBA_ERR_UNSUPPORTED: return "MOBA_ERR_UNSUPPORTED";
    case MOBA_ERR_WORKSPACE: return "MOBA_ERR_WORKSPACE";
    case MOBA_ERR_CUDA: return "MOBA_ERR_CUDA";
    case MOBA_ERR_TIMEOUT: return "MOBA_ERR_TIMEOUT";
    case MOBA_ERR_BAD_SEQLENS: return "MOBA_ERR_BAD_SEQLENS";
    case MOBA_ERR_BAD_SELECTION: return "MOBA_ERR_BAD_SELECTION";
    case MOBA_ERR_BOUNDS: return "MOBA_ERR_BOUNDS";
    case MOBA_ERR_CANARY: return "MOBA_ERR_CANARY";
  }
  return "MOBA_ERR_UNKNOWN";
}

size_t moba_workspace_size(int total_tokens, int n_seqs, int n_heads, int n_kv_heads, int head_dim,
                           int block_size, int topk, int chunk_tokens) {
  Sizes z;
  if (make_sizes(total_tokens, n_seqs, n_heads, n_kv_heads, head_dim, block_size, topk,
                 chunk_tokens, &z) != MOBA_OK)
    return 0;
  return (size_t)carve(z, nullptr, nullptr, nullptr);
}

moba_status moba_gate(const void* q, const void* k, const int32_t* cu_seqlens, int n_seqs,
                      int total_tokens, int n_heads, int n_kv_heads, int head_dim, int block_size,
                      int topk, int32_t* idx, void* workspace, size_t workspace_bytes,
                      void* stream) {
  Sizes z;
  moba_status s = make_sizes(total_tokens, n_seqs, n_heads, n_kv_heads, head_dim, block_size, topk,
                             0, &z);
  if (s != MOBA_OK) return s;
  if (!cu_seqlens || !idx) return MOBA_ERR_INVALID_ARG;
  if (total_tokens > 0 && (!q || !k)) return MOBA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || (reinterpret_cast<uintptr_t>(idx) & 3u))
    return MOBA_ERR_INVALID_ARG;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) % kAlign) != 0)
    return MOBA_ERR_WORKSPACE;
  long long gate_end = 0;
  carve(z, nullptr, nullptr, &gate_end);
  if ((long long)workspace_bytes < gate_end) return MOBA_ERR_WORKSPACE;
  Workspace ws;
  Guards g;
  carve(z, static_cast<char*>(workspace), &ws, nullptr, &g, gate_end);
  if (total_tokens == 0) return MOBA_OK;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (guards_begin(g, st) != cudaSuccess) return MOBA_ERR_CUDA;
  s = run_prefix(q, k, cu_seqlens, idx, z, ws, st);
  if (s != MOBA_OK) return s;
  return cuda_status(guards_end(g, ws.plan, st));
}

moba_status moba_gate_noalloc(const void* q, const void* k, const int32_t* cu_seqlens,
                              int n_seqs, int total_tokens, int n_heads, int n_kv_heads,
                              int head_dim, int block_size, int topk, int32_t* idx,
                              void* stream) {
  Sizes z;
  moba_status s = make_sizes(total_tokens, n_seqs, n_heads, n_kv_heads, head_dim, block_size, topk,
                             0, &z);
  if (s != MOBA_OK) return s;
  if (!cu_seqlens || !idx) return MOBA_ERR_INVALID_ARG;
  if (total_tokens > 0 && (!q || !k)) return MOBA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || (reinterpret_cast<uintptr_t>(idx) & 3u))
    return MOBA_ERR_INVALID_ARG;
  long long gate_end = 0;
  carve(z, nullptr, nullptr, &gate_end);
  if (gate_end > (long long)kStaticScratchBytes) return MOBA_ERR_WORKSPACE;
  void* scratch = nullptr;
  s = static_scratch(&scratch);
  if (s != MOBA_OK) return s;
  Workspace ws;
  Guards g;
  carve(z, static_cast<char*>(scratch), &ws, nullptr, &g, gate_end);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // an empty call still clears the error word, so moba_gate_noalloc_check
  // never reports an earlier call's error against this one
  if (total_tokens == 0) return cuda_status(cudaMemsetAsync(ws.plan, 0, sizeof(DevPlan), st));
  if (guards_begin(g, st) != cudaSuccess) return MOBA_ERR_CUDA;
  s = run_prefix(q, k, cu_seqlens, idx, z, ws, st);
  if (s != MOBA_OK) return s;
  return cuda_status(guards_end(g, ws.plan, st));
}

moba_status moba_gate_noalloc_check(void* stream) {
  void* scratch = nullptr;
  moba_status s = static_scratch(&scratch);
  if (s != MOBA_OK) return s;
  return moba_check(scratch, stream);
}

moba_status moba_forward_traced(const void* q, const void* k, const void* v,
                                const int32_t* cu_seqlens, int n_seqs, int total_tokens,
                                int n_heads, int n_kv_heads, int head_dim, int block_size, int topk,
                                float softmax_scale, void* out, float* lse, int32_t* idx_out,
                                int chunk_tokens, void* workspace, size_t workspace_bytes,
                                void* stream, void* const* stage_events, int n_stage_events) {
  Sizes z;
  moba_status s = make_sizes(total_tokens, n_seqs, n_heads, n_kv_heads, head_dim, block_size, topk,
                             chunk_tokens, &z);
  if (s != MOBA_OK) return s;
  if (!cu_seqlens) return MOBA_ERR_INVALID_ARG;
  if (total_tokens > 0 && (!q || !k || !v || !out || !lse)) return MOBA_ERR_INVALID_ARG;
  if (!(softmax_scale == softmax_scale)) return MOBA_ERR_INVALID_ARG;  // NaN
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) ||
      (reinterpret_cast<uintptr_t>(lse) & 3u) || (reinterpret_cast<uintptr_t>(idx_out) & 3u))
    return MOBA_ERR_INVALID_ARG;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) % kAlign) != 0)
    return MOBA_ERR_WORKSPACE;
  const long long need = carve(z, nullptr, nullptr, nullptr);
  if ((long long)workspace_bytes < need) return MOBA_ERR_WORKSPACE;
  Workspace ws;
  Guards g;
  carve(z, static_cast<char*>(workspace), &ws, nullptr, &g, need);
  if (total_tokens == 0) return MOBA_OK;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const float scale = softmax_scale > 0.f ? softmax_scale : 1.0f / sqrtf((float)head_dim);
  const float scale_log2 = scale * 1.4426950408889634f;
  int32_t* idx = idx_out ? idx_out : ws.idx;
  int ev = 0;
  auto mark = [&]() -> cudaError_t {
    cudaError_t r = cudaSuccess;
    if (stage_events && ev < n_stage_events && stage_events[ev])
      r = cudaEventRecord(static_cast<cudaEvent_t>(stage_events[ev]), st);
    ++ev;
    return r;
  };
  if (mark() != cudaSuccess) return MOBA_ERR_CUDA;
  if (guards_begin(g, st) != cudaSuccess) return MOBA_ERR_CUDA;
  s = run_prefix(q, k, cu_seqlens, idx, z, ws, st);
  if (s != MOBA_OK) return s;
  if (mark() != cudaSuccess) return MOBA_ERR_CUDA;
  const int nsm = sm_count();
  for (int t0 = 0; t0 < total_tokens; t0 += z.chunk) {
    const int t1 = t0 + z.chunk < total_tokens ? t0 + z.chunk : total_tokens;
    cudaError_t e = launch_sched(idx, z, ws, t0, t1, attn_unit_rows(), st);
    if (e == cudaSuccess) e = mark();
    if (e == cudaSuccess) e = launch_attn(q, k, v, z, ws, t0, t1, scale_log2, nsm, st);
    if (e == cudaSuccess) e = mark();
    if (e == cudaSuccess) e = launch_merge(idx, out, lse, z, ws, t0, t1, st);
    if (e == cudaSuccess) e = mark();
    if (e != cudaSuccess) return MOBA_ERR_CUDA;
  }
  return cuda_status(guards_end(g, ws.plan, st));
}

moba_status moba_forward(const void* q, const void* k, const void* v, const int32_t* cu_seqlens,
                         int n_seqs, int total_tokens, int n_heads, int n_kv_heads, int head_dim,
                         int block_size, int topk, float softmax_scale, void* out, float* lse,
                         int32_t* idx_out, int chunk_tokens, void* workspace,
                         size_t workspace_bytes, void* stream) {
  return moba_forward_traced(q, k, v, cu_seqlens, n_seqs, total_tokens, n_heads, n_kv_heads,
                             head_dim, block_size, topk, softmax_scale, out, lse, idx_out,
                             chunk_tokens, workspace, workspace_bytes, stream, nullptr, 0);
}

size_t moba_full_workspace_size(int total_tokens, int n_seqs, int n_heads, int n_kv_heads,
                                int head_dim) {
  Sizes z;
  if (make_sizes_full(total_tokens, n_seqs, n_heads, n_kv_heads, head_dim, &z) != MOBA_OK) return 0;
  return (size_t)carve_full(z, nullptr, nullptr);
}

moba_status moba_forward_full(const void* q, const void* k, const void* v,
                              const int32_t* cu_seqlens, int n_seqs, int total_tokens, int n_heads,
                              int n_kv_heads, int head_dim, float softmax_scale, void* out,
                              float* lse, void* workspace, size_t workspace_bytes, void* stream) {
  Sizes z;
  moba_status s = make_sizes_full(total_tokens, n_seqs, n_heads, n_kv_heads, head_dim, &z);
  if (s != MOBA_OK) return s;
  if (!cu_seqlens) return MOBA_ERR_INVALID_ARG;
  if (total_tokens > 0 && (!q || !k || !v || !out || !lse)) return MOBA_ERR_INVALID_ARG;
  if (!(softmax_scale == softmax_scale)) return MOBA_ERR_INVALID_ARG;  // NaN
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) ||
      (reinterpret_cast<uintptr_t>(lse) & 3u))
    return MOBA_ERR_INVALID_ARG;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) % kAlign) != 0)
    return MOBA_ERR_WORKSPACE;
  const long long need = carve_full(z, nullptr, nullptr);
  if ((long long)workspace_bytes < need) return MOBA_ERR_WORKSPACE;
  Workspace ws;
  Guards g;
  carve_full(z, static_cast<char*>(workspace), &ws, &g, need);
  if (total_tokens == 0) return MOBA_OK;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const float scale = softmax_scale > 0.f ? softmax_scale : 1.0f / sqrtf((float)head_dim);
  const float scale_log2 = scale * 1.4426950408889634f;
  cudaError_t e = guards_begin(g, st);
  if (e == cudaSuccess) e = cudaMemsetAsync(ws.plan, 0, sizeof(DevPlan), st);
  if (e == cudaSuccess) e = launch_plan(cu_seqlens, z, ws, st);
  ws.part_o = static_cast<__nv_bfloat16*>(out);
  ws.part_lse = lse;
  if (e == cudaSuccess) e = launch_attn_full(q, k, v, z, ws, scale_log2, sm_count(), st);
  if (e == cudaSuccess) e = guards_end(g, ws.plan, st);
  return cuda_status(e);
}

size_t moba_decode_workspace_size(int n_seqs, int max_len, int n_heads, int n_kv_heads,
                                  int head_dim, int block_size, int topk) {
  if (check_decode(n_seqs, max_len, n_heads, n_kv_heads, head_dim, block_size, topk) != MOBA_OK)
    return 0;
  return (size_t)carve_decode(n_seqs, n_heads, n_kv_heads, head_dim, block_size, topk, nullptr,
                              nullptr);
}

moba_status moba_decode_init(const void* k_cache, const int32_t* seqlens, int n_seqs, int max_len,
                             int n_kv_heads, int head_dim, int block_size, float* kbar,
                             void* workspace, size_t workspace_bytes, void* stream) {
  moba_status s = check_decode(n_seqs, max_len, n_kv_heads, n_kv_heads, head_dim, block_size, 1);
  if (s != MOBA_OK) return s;
  if (!k_cache || !seqlens || (!kbar && max_len >= block_size)) return MOBA_ERR_INVALID_ARG;
  if (!aligned16(k_cache) || !aligned16(kbar)) return MOBA_ERR_INVALID_ARG;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) % kAlign) != 0 ||
      workspace_bytes < sizeof(DevPlan))
    return MOBA_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  DevPlan* plan = static_cast<DevPlan*>(workspace);
  cudaError_t e = cudaMemsetAsync(plan, 0, sizeof(DevPlan), st);
  if (e == cudaSuccess)
    e = launch_decode_kbar(k_cache, seqlens, kbar, plan, n_seqs, max_len, n_kv_heads, head_dim,
                           block_size, false, st);
  return cuda_status(e);
}

moba_status moba_decode(const void* q, const void* k_cache, const void* v_cache,
                        const int32_t* seqlens, int n_seqs, int max_len, int n_heads,
                        int n_kv_heads, int head_dim, int block_size, int topk, float softmax_scale,
                        float* kbar, void* out, float* lse, int32_t* idx_out, void* workspace,
                        size_t workspace_bytes, void* stream) {
  moba_status s = check_decode(n_seqs, max_len, n_heads, n_kv_heads, head_dim, block_size, topk);
  if (s != MOBA_OK) return s;
  if (!q || !k_cache || !v_cache || !seqlens || !out || !lse) return MOBA_ERR_INVALID_ARG;
  if (!kbar && max_len >= block_size) return MOBA_ERR_INVALID_ARG;
  if (!(softmax_scale == softmax_scale)) return MOBA_ERR_INVALID_ARG;  // NaN
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out) ||
      !aligned16(kbar) || (reinterpret_cast<uintptr_t>(lse) & 3u) ||
      (reinterpret_cast<uintptr_t>(idx_out) & 3u))
    return MOBA_ERR_INVALID_ARG;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) % kAlign) != 0)
    return MOBA_ERR_WORKSPACE;
  const long long need = carve_decode(n_seqs, n_heads, n_kv_heads, head_dim, block_size, topk,
                                      nullptr, nullptr);
  if ((long long)workspace_bytes < need) return MOBA_ERR_WORKSPACE;
  DecodeWs ws;
  Guards g;
  carve_decode(n_seqs, n_heads, n_kv_heads, head_dim, block_size, topk,
               static_cast<char*>(workspace), &ws, &g, need);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const float scale = softmax_scale > 0.f ? softmax_scale : 1.0f / sqrtf((float)head_dim);
  cudaError_t e = cudaMemsetAsync(ws.plan, 0, (size_t)ws.zero_bytes, st);
  if (e == cudaSuccess) e = guards_begin(g, st);  // after the memset, which covers early guards
  if (e == cudaSuccess)
    e = launch_decode(q, k_cache, v_cache, seqlens, kbar, out, lse, idx_out ? idx_out : ws.idx,
                      ws.part_o, ws.part_lse, ws.row_done, ws.kb_part, ws.seq_done, ws.plan,
                      n_seqs, max_len, n_heads, n_kv_heads, head_dim, block_size, topk,
                      scale * 1.4426950408889634f, st);
  if (e == cudaSuccess) e = guards_end(g, ws.plan, st);
  return cuda_status(e);
}

// Sizes of the backward: zf with one pass over every token (bucket lists of
// the whole sequence set), zc with the dQ partials' query chunk.
moba_status make_sizes_bwd(int T, int n_seqs, int Hq, int Hkv, int d, int B, int topk, int chunk,
                           Sizes* zf, Sizes* zc) {
  moba_status s = make_sizes(T, n_seqs, Hq, Hkv, d, B, topk, 0, zf);
  if (s != MOBA_OK) return s;
  s = make_sizes(T, n_seqs, Hq, Hkv, d, B, topk, chunk, zc);
  if (s != MOBA_OK) return s;
  if (zf->entries_max >= (1LL << 31) || (long long)zc->part_rows * d >= (1LL << 40))
    return MOBA_ERR_UNSUPPORTED;
  return MOBA_OK;
}

size_t moba_backward_workspace_size(int total_tokens, int n_seqs, int n_heads, int n_kv_heads,
                                    int head_dim, int block_size, int topk, int chunk_tokens) {
  Sizes zf, zc;
  if (make_sizes_bwd(total_tokens, n_seqs, n_heads, n_kv_heads, head_dim, block_size, topk,
                     chunk_tokens, &zf, &zc) != MOBA_OK)
    return 0;
  return (size_t)carve_bwd(zf, zc, nullptr, nullptr);
}

moba_status moba_backward(const void* q, const void* k, const void* v, const void* out,
                          const float* lse, const void* dout, const int32_t* idx,
                          const int32_t* cu_seqlens, int n_seqs, int total_tokens, int n_heads,
                          int n_kv_heads, int head_dim, int block_size, int topk,
                          float softmax_scale, float* dq, float* dk, float* dv, int chunk_tokens,
                          void* workspace, size_t workspace_bytes, void* stream) {
  Sizes zf, zc;
  moba_status s = make_sizes_bwd(total_tokens, n_seqs, n_heads, n_kv_heads, head_dim, block_size,
                                 topk, chunk_tokens, &zf, &zc);
  if (s != MOBA_OK) return s;
  if (!cu_seqlens || !dq || !dk || !dv) return MOBA_ERR_INVALID_ARG;
  if (total_tokens > 0 && (!q || !k || !v || !out || !lse || !dout || !idx))
    return MOBA_ERR_INVALID_ARG;
  if (!(softmax_scale == softmax_scale)) return MOBA_ERR_INVALID_ARG;  // NaN
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(dout) ||
      (reinterpret_cast<uintptr_t>(lse) & 3u) || (reinterpret_cast<uintptr_t>(idx) & 3u) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
    return MOBA_ERR_INVALID_ARG;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) % kAlign) != 0)
    return MOBA_ERR_WORKSPACE;
  const long long need = carve_bwd(zf, zc, nullptr, nullptr);
  if ((long long)workspace_bytes < need) return MOBA_ERR_WORKSPACE;
  BwdWs b;
  Guards g;
  carve_bwd(zf, zc, static_cast<char*>(workspace), &b, &g, need);
  if (total_tokens == 0) return MOBA_OK;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const float scale = softmax_scale > 0.f ? softmax_scale : 1.0f / sqrtf((float)head_dim);
  const Workspace& ws = b.ws;
  const int nsm = sm_count();
  cudaError_t e = guards_begin(g, st);
  if (e == cudaSuccess) e = cudaMemsetAsync(ws.plan, 0, sizeof(DevPlan), st);
  if (e == cudaSuccess) e = launch_plan(cu_seqlens, zf, ws, st);
  if (e == cudaSuccess) e = launch_bwd_prep(out, dout, idx, cu_seqlens, zf, b.dvec, ws.plan, st);
  // dK, dV: bucket lists over every token, then one pass over the key tiles
  if (e == cudaSuccess) e = launch_sched(idx, zf, ws, 0, total_tokens, 128, st, /*stable=*/true);
  if (e == cudaSuccess)
    e = launch_backward_dkv(q, k, v, dout, lse, b.dvec, zf, ws, b.pack, dk, dv, scale, nsm, st);
  // dQ: per query chunk, partial slots and their sum
  for (int t0 = 0; e == cudaSuccess && t0 < total_tokens; t0 += zc.chunk) {
    const int t1 = t0 + zc.chunk < total_tokens ? t0 + zc.chunk : total_tokens;
    e = launch_sched(idx, zc, ws, t0, t1, 128, st);
    if (e == cudaSuccess)
      e = launch_backward_dq(q, k, v, dout, lse, b.dvec, zc, ws, b.dq_part, dq, t0, t1, scale, nsm,
                             st);
    if (e == cudaSuccess) e = launch_dq_merge(idx, b.dq_part, dq, zc, ws.plan, t0, t1, st);
  }
  if (e == cudaSuccess) e = guards_end(g, ws.plan, st);
  return cuda_status(e);
}

moba_status moba_debug_attention_wait_test(int enable) {
  set_attn_wait_test(enable);
  return MOBA_OK;
}

int moba_debug_build(void) {
#ifdef MOBA_DEBUG
  return 1;
#else
  return 0;
#endif
}

moba_status moba_debug_poison(int mode) {
#ifdef MOBA_DEBUG
  if (mode < 0 || mode > 2) return MOBA_ERR_INVALID_ARG;
  g_poison = mode;
  return MOBA_OK;
#else
  return mode == 0 ? MOBA_OK : MOBA_ERR_UNSUPPORTED;
#endif
}

moba_status moba_debug_error_info(const void* workspace, void* stream, int* info) {
  if (!workspace || !info) return MOBA_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return MOBA_ERR_CUDA;
  DevPlan p;
  if (cudaMemcpy(&p, workspace, sizeof(DevPlan), cudaMemcpyDeviceToHost) != cudaSuccess)
    return MOBA_ERR_CUDA;
  *info = p.err != 0 ? p.err_info : 0;
  return MOBA_OK;
}

moba_status moba_check(void* workspace, void* stream) {
  if (!workspace) return MOBA_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return MOBA_ERR_CUDA;
  DevPlan p;
  if (cudaMemcpy(&p, workspace, sizeof(DevPlan), cudaMemcpyDeviceToHost) != cudaSuccess)
    return MOBA_ERR_CUDA;
  if (p.err == kErrTimeout) return MOBA_ERR_TIMEOUT;
  if (p.err == kErrBadSeqlens) return MOBA_ERR_BAD_SEQLENS;
  if (p.err == kErrBadSelection) return MOBA_ERR_BAD_SELECTION;
  if (p.err == kErrBounds) return MOBA_ERR_BOUNDS;
  if (p.err == kErrCanary) return MOBA_ERR_CANARY;
  if (p.err != 0) return MOBA_ERR_CUDA;
  return MOBA_OK;
}

}  // extern "C"
