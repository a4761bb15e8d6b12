// Shared definitions of the MoBA sm_100a library: workspace layout, device
// plan, error word and small helpers.  Host and device code both include it.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>
#include <stddef.h>

namespace moba {

// Device error codes (same numbering as moba_status in moba.h).
enum : int {
  kOk = 0,
  kErrTimeout = 5,
  kErrBadSeqlens = 6,
  kErrBadSelection = 7,
  kErrBounds = 8,   // MOBA_DEBUG builds: an index failed its check (detail: the site)
  kErrCanary = 9,   // MOBA_DEBUG builds: a workspace guard was overwritten (detail: guard)
};

// Sites of the MOBA_DEBUG index checks (the error's detail word).
enum : int {
  kSiteAttnTile = 1,     // block attention: a tile's bucket / first entry
  kSiteAttnEntry = 2,    // block attention: a bucket entry (partial slot of a routed row)
  kSiteSchedEntry = 3,   // scheduler: a scatter position
  kSiteDkvBucket = 4,    // dK / dV: a unit's bucket and entry range
  kSiteDkvEntry = 5,     // dK / dV: a bucket entry (routed row)
  kSiteDqTile = 6,       // dQ: a tile's bucket / first entry
  kSiteDqEntry = 7,      // dQ: a bucket entry
  kSiteDecodeBlock = 8,  // decode: a selected block
};

// Rows of (query token, head) per attention tile of the gathered (past-block)
// path.  Every tile holds rows of ONE (block, kv head) bucket.
constexpr int kTileRows = 128;

// Number of row slices the pooling kernel splits one block into; the partial
// sums are reduced in a fixed order by a second kernel (deterministic means).
constexpr int kPoolSplit = 8;

// Device-resident plan written by plan_kernel (first bytes of the workspace).
struct DevPlan {
  int err;          // first error code raised on the device (0 = none)
  int err_info;     // free-form detail for the error (e.g. sequence index)
  int nblk_total;   // blocks over all sequences, short last blocks included
  int nfull_total;  // full blocks over all sequences
  int ntiles;       // gathered-attention tiles of the current chunk
  int pad[3];
};

// Pointers into the caller's workspace, carved on the host.
struct Workspace {
  DevPlan* plan;
  int* seq_blk_base;    // [n_seqs + 1] first global block of each sequence
  int* seq_full_base;   // [n_seqs + 1] first global full block of each sequence
  int* blk_start;       // [nblk_max] first token of the block
  int* blk_len;         // [nblk_max] tokens in the block (B, or less for a short last block)
  int* blk_j;           // [nblk_max] block index inside its sequence
  int* blk_fullbase;    // [nblk_max] seq_full_base of the block's sequence
  int* full_start;      // [nfull_max] first token of each full block
  // stable fill: full_nlater = blocks after the full block in its sequence,
  // full_cm = the sum of full_nlater over the full blocks before it
  int* full_nlater;     // [nfull_max]
  long long* full_cm;   // [nfull_max]
  int* cm;              // [cm_cap] stable fill: entries per (bucket, scheduler CTA), then run starts
  float* pool_part;     // [nfull_max, kPoolSplit, Hkv * d] partial key sums
  float* kbar;          // [nfull_max, Hkv, d] mean keys, fp32
  __nv_bfloat16* kbar_hi;  // [nfull_max, Hkv, d] bf16(kbar)
  __nv_bfloat16* kbar_lo;  // [nfull_max, Hkv, d] bf16(kbar - hi)
  int32_t* idx;         // [T, Hq, topk] gate output (when the caller gives none)
  int* bucket_count;    // [nbk_max + 1] past entries per (full block, kv head)
  int* bucket_off;      // [nbk_max + 1] exclusive scan of bucket_count
  int* bucket_cursor;   // [nbk_max] fill cursors
  int* tile_off;        // [nbk_max + 1] exclusive scan of tiles per bucket
  int* entries;         // [chunk * Hq * (topk - 1)] partial-slot ids grouped by bucket
  int2* tiles;          // [ntiles_max] (bucket, first entry) of each tile
  __nv_bfloat16* part_o;  // [chunk * Hq * topk, d] normalised partial outputs
  float* part_lse;        // [chunk * Hq * topk] partial log-sum-exp
  // capacities of the arrays above, for the MOBA_DEBUG index checks
  long long rows_cap;     // T * Hq rows of q, dout, out
  long long entries_cap;  // entries
  int nbk_cap;            // buckets (bucket_off has nbk_cap + 1)
  long long cm_cap;       // cm (0: no stable fill)
  int poison;             // MOBA_DEBUG builds: planted slip of moba_debug_poison (0: none)
};

struct Sizes {
  int T, n_seqs, Hq, Hkv, d, B, topk, chunk;
  int nblk_max, nfull_max, nbk_max, ntiles_max;
  long long entries_max, part_rows;
};

__host__ __device__ inline long long align_up(long long x, long long a) {
  return (x + a - 1) / a * a;
}

#ifdef __CUDACC__
__device__ __forceinline__ void raise_error(DevPlan* p, int code, int info) {
  if (atomicCAS(&p->err, 0, code) == 0) p->err_info = info;
}

// MOBA_INDEX_OK(plan, cond, site): in MOBA_DEBUG builds, tests an index read
// from the workspace against the buffer it addresses, records kErrBounds with
// the site on failure and yields the result, so that the caller replaces the
// index by a safe one (a skipped unit, a padding row, a dropped write) before
// any access.  Release builds compile the test out (it yields true).
#ifdef MOBA_DEBUG
__device__ __forceinline__ bool index_ok(const DevPlan* p, bool ok, int site) {
  if (!ok) raise_error(const_cast<DevPlan*>(p), kErrBounds, site);
  return ok;
}
#define MOBA_INDEX_OK(plan, cond, site) (::moba::index_ok((plan), (cond), (site)))
#else
#define MOBA_INDEX_OK(plan, cond, site) (true)
#endif
#endif

}  // namespace moba
