// internal.h -- declarations shared by the host runtime and the kernels of
// the indexer library (not part of the public C ABI).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace hwr {

// Device status bits kept in the first word of the workspace.
constexpr uint32_t kStatusWaitTimeout = 1u;
constexpr uint32_t kStatusOverflow = 2u;
constexpr uint32_t kStatusWitness = 4u;  // a seed threshold left a query fewer than min(K, visible) keys

// Candidate-buffer sets per CTA and epilogue group (the scoring kernel's
// kSets): blocks rotate through them while the row writers read finished ones.
constexpr int kCandSets = 3;

// Heads the pruning certificate keeps exactly (the first kPruneR of each query).
constexpr int kPruneR = 16;

// One query block of a launch over several documents (the segmented kernel):
// its rows in the batch, the visibility position of its first row within its
// document, and the document's keys.  Output indices are shifted by key0 (the
// document's first key row), which numbers them within the whole batch.
struct SegBlock {
  int64_t row0;    // first query row of the block
  int64_t pos0;    // position of row0 within its document (visibility)
  int64_t key0;    // the document's first key row
  int32_t rows;    // query rows of the block (at most the block size)
  int32_t n_keys;  // the document's keys (tokens or compressed keys)
};

// Arguments of the scoring + top-K kernel (one launch per indexer call).
struct ScoreParams {
  int64_t S;          // query rows
  int64_t n_keys;     // rows of the scored key matrix (tokens, compressed keys or pools)
  int64_t q_pos0;     // global position of query row 0
  int32_t ranged;     // 0: key i visible iff i <= g; 1: key j visible iff ratio*j + ratio - 1 <= g
  int32_t ratio;      // key span for ranged visibility
  int32_t out_ratio;  // 1, or the pool width: each selected pool expands to out_ratio positions + tail
  uint32_t out_ratio_inv;  // ceil(2^32 / out_ratio) when out_ratio > 1 (division-free pool expansion)
  int32_t ksel;       // keys (pools) to select per query
  int32_t width;      // row stride of out_idx / out_score
  int32_t n_blocks;   // query blocks
  int32_t cap;        // candidate-buffer entries per query
  const float* w;        // [S, H]
  const float* q_scale;  // [S, H] or null (FP8)
  const float* k_scale;  // [n_keys] or null (FP8)
  int32_t* out_idx;      // [S, width]
  int32_t* out_len;      // [S]
  float* out_score;      // [S, width] or null
  uint2* cand;           // candidate buffers: [grid][groups][queries per group][cap]
  uint32_t* status;      // device status word
  int32_t prune;               // 1: screen keys with the certificate before the full head sum
  const float* pq;             // [S][kPruneR + 2]: folded weights wt[0..r), Ceff, sum |w||q|
  const float* knorm;          // [n_keys]: |k_i| in the kernel's domain, rounded up
  unsigned long long* counters;  // [3]: pairs screened, bounded below the threshold, skipped
  int32_t splits;        // key-range splits per query block (1: each block is one work item)
  uint2* split_buf;      // splits > 1: [S][splits][ksel] top-K of each split, in key order
  int32_t* split_cnt;    // splits > 1: [S][splits] entries of each split
  uint32_t* split_kth;   // splits > 1: [S][splits] ordered score of each full split's K-th entry, else 0
  uint32_t* split_rth;   // splits > 1: [S][splits] ordered score of each split's r-th entry, r = ceil(K / splits)
                         // (0 when it has fewer than r)
  const uint32_t* seed_thr;  // [S] ordered-score threshold every query starts from, or null (0 for all)
  int64_t test_wait_ns;  // > 0: test hook, the MMA issuer waits this long on a barrier nothing arrives at
  const SegBlock* seg;   // segmented kernel: [n_blocks] query blocks, lightest first; else null
};

// Per-variant launch facts, filled by the kernel's translation unit.
struct ScoreVariant {
  const void* fn;         // kernel function
  const void* fn_split;   // the same with key ranges split across CTAs (ScoreParams::splits > 1)
  const void* fn_seg;     // the same over a table of query blocks of several documents (ScoreParams::seg)
  int queries_per_block;  // QB
  int queries_per_wg;     // queries owned by one epilogue warpgroup
  int groups;             // epilogue warpgroups per CTA
  int q_box_rows;         // rows of the q TMA box
  int box_elems;          // inner extent of every TMA box (128 bytes)
  int smem_bytes;         // dynamic shared memory
  int threads;
};

// Returns false when (H, D, fp8, prune) has no compiled variant.
bool score_variant(int H, int D, bool fp8, bool prune, ScoreVariant* out);

// Candidate-buffer capacity per query for a selection budget of ksel keys.
inline int candidate_capacity(int ksel, bool prune) {
  // the budget plus as much again for new candidates, and up to four times the
  // budget (eight without the pruning certificate) while that still fits the
  // register-resident selection (4,096): fewer cuts for small budgets.  With
  // pruning a smaller buffer fills, and so raises the running threshold the
  // certificate screens against, sooner on short rows.
  auto r128 = [](int x) { return ((x + 127) / 128) * 128; };
  int c = r128(2 * ksel);
  if (prune) {
    const int wide = r128(4 * ksel);
    if (wide <= 4096 && wide > c) c = wide;
  } else {
    const int wide = r128(8 * ksel) < 4096 ? r128(8 * ksel) : 4096;
    if (wide > c) c = wide;
  }
  return c < ksel + 256 ? r128(ksel + 256) : c;
}

cudaError_t launch_pool_keys(const void* k, int64_t n_pools, int D, const void* coef, int ratio, void* out,
                             cudaStream_t stream);
cudaError_t launch_prune_setup(const void* q, const float* w, const float* q_scale, bool fp8, int64_t S, int H,
                               int D, const void* keys, int64_t n_keys, float* pq, float* knorm,
                               cudaStream_t stream);
// Upper bound of key-range splits per query block (the merge keeps its
// per-split offsets in shared memory).
constexpr int kMaxSplits = 512;

// Visibility facts the merge needs to check a seeded run (seeded = 0: none).
struct MergeCheck {
  int32_t seeded;
  int32_t ranged;
  int32_t ratio;
  int64_t n_keys;
  uint32_t* status;
};

cudaError_t launch_merge_splits(int64_t S, int64_t q_pos0, int splits, int ksel, int width, int out_ratio,
                                const uint2* split_buf, const int32_t* split_cnt, const uint32_t* split_kth,
                                const uint32_t* split_rth, uint2* gather, int64_t gather_stride, int32_t* out_idx, int32_t* out_len,
                                float* out_score, const MergeCheck& check, cudaStream_t stream);

// Seed thresholds (witness.cu): thr[t] = the ksel-th largest lowered exact
// score over the distinct visible key rows that row t of `seeds` names.
struct WitnessParams {
  int64_t S;
  int64_t n_keys;       // rows of the scored key matrix
  int64_t q_pos0;
  int32_t H;
  int32_t ranged;       // visibility as in ScoreParams
  int32_t ratio;
  int32_t seed_div;     // seeds name key row e / seed_div (POOLED: token positions -> pools)
  int32_t ksel;
  int32_t fp8;
  int64_t n_seeds;      // seeds per row
  int64_t seed_stride;  // row stride of seeds
  const void* q;        // [S, H, D] (bf16 values or e4m3 codes)
  const float* w;       // [S, H]
  const float* q_scale; // [S, H] (FP8)
  const void* keys;     // [n_keys, D]: the scored key matrix (pools for POOLED)
  const float* k_scale; // [n_keys] (FP8)
  const int32_t* seeds; // [S, seed_stride]; -1 or any other invalid entry is ignored
  uint32_t* lowered;    // [S, n_seeds] scratch
  uint32_t* thr;        // [S] result
};
cudaError_t launch_witness(const WitnessParams& wp, int D, cudaStream_t stream);
cudaError_t launch_offset_indices(int32_t* idx, int64_t n, int32_t add, cudaStream_t stream);
cudaError_t launch_pair_regions(const int32_t* idx, const int32_t* len, int64_t n_pairs, int width,
                                int32_t* shared, int32_t* left, int32_t* right, int32_t* counts,
                                cudaStream_t stream);
cudaError_t launch_pair_overlap(const int32_t* idx, const int32_t* len, int64_t n_pairs, int width,
                                int32_t* out, cudaStream_t stream);

}  // namespace hwr
