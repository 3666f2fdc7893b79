/*
 * hwr_indexer.h -- C ABI of the B200 (sm_100a) DSA lightning indexer.
 *
 * The indexer scores, for every query t and every key i visible to it,
 *
 *     s[t,i] = sum_h  w[t,h] * max(0, q[t,h,:] . k[i,:])
 *
 * ("DoSA: Dots Sparse Attention", section 前置知识 / background: the indexer
 * score with ReLU and head weights of either sign), keeps the K best keys of
 * each query (ties: the higher score wins, then the lower key index; the same
 * page, section 研究动机 / motivation, asks for exact top-K under one tie
 * rule), and writes them sorted by key index with a valid length
 * ("Adjacent-Query KV-Index Overlap in 256K DSA Training", §1 and §3).
 *
 * Conventions for every entry point:
 *   - Pointers named q, k, w, *_scale, pool_coef, out_*, workspace are DEVICE
 *     pointers on the current CUDA device, owned by the caller; the library
 *     never frees or retains them.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Kernels are enqueued asynchronously on it; no call below
 *     synchronises unless it says so.
 *   - Argument errors are detected on the host before any launch and return a
 *     status other than INDEXER_OK; nothing is launched then.
 *   - The library allocates no device memory: scratch comes from the caller's
 *     workspace (see indexer_workspace_bytes), so every launch is shape-stable
 *     and can be replayed.
 *   - Rows are row-major with the last dimension contiguous.
 */
#ifndef HWR_INDEXER_H
#define HWR_INDEXER_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  INDEXER_OK = 0,
  INDEXER_EINVAL = 1,        /* a size, pointer or enum is out of range      */
  INDEXER_EWORKSPACE = 2,    /* workspace missing, misaligned or too small   */
  INDEXER_EUNSUPPORTED = 3,  /* valid problem outside the compiled variants  */
  INDEXER_ECUDA = 4,         /* a CUDA runtime / driver call failed          */
  INDEXER_EDEVICE = 5        /* the device is not sm_100 (B200 class)        */
} indexer_status;

/* Which keys a query at global position g may see.
 *   TOKEN:      token key i is visible iff i <= g ("Module 06 — DSA & KPool:
 *               Selective Retrieval", §3: position i sees j iff j <= i).
 *   COMPRESSED: key j summarises tokens m*j .. m*j+m-1 (m = `ratio`) and is
 *               visible iff m*j + m - 1 <= g (StreamIndex, arXiv 2605.02568,
 *               abstract: CSA keys compressed with m = 4; the completion rule
 *               is KPool §3's).
 *   POOLED:     k holds token keys; pool p is formed from tokens
 *               m*p .. m*p+m-1 as kp[p] = RNE_bf16(sum_j c[j] (*) k[m*p+j])
 *               (KPool §2: a channel-wise weighted representation of each
 *               complete pool), is visible iff m*p + m - 1 <= g, the best
 *               K/m pools are expanded to their m tokens, and the positions
 *               of the query's own incomplete pool (m*floor((g+1)/m) .. g,
 *               at most m-1) are appended as a tail (KPool §2). */
typedef enum {
  INDEXER_VIS_TOKEN = 0,
  INDEXER_VIS_COMPRESSED = 1,
  INDEXER_VIS_POOLED = 2
} indexer_visibility;

typedef enum {
  INDEXER_BF16 = 0,      /* q, k in bfloat16                                  */
  INDEXER_FP8_E4M3 = 1   /* q, k in FP8 e4m3 codes with FP32 per-row scales   */
} indexer_dtype;

typedef struct {
  int64_t S;          /* query rows                                           */
  int64_t T;          /* key rows: tokens (TOKEN, POOLED) or compressed keys  */
  int32_t H;          /* indexer heads (see D for the compiled pairs)         */
  int32_t D;          /* (H, D): BF16 (4,64) (8,128) (16,64) (32,128) (64,64) (64,128); FP8 (32,128) (64,128) */
  int64_t q_pos0;     /* global position of query row 0 (g = q_pos0 + t)      */
  int32_t visibility; /* indexer_visibility                                   */
  int32_t ratio;      /* m for COMPRESSED / POOLED (1..16); ignored for TOKEN */
  int32_t K;          /* budget in positions; POOLED selects K/ratio pools    */
  int32_t dtype;      /* indexer_dtype                                        */
  int32_t flags;      /* 0, INDEXER_FLAG_PRUNE (and the test hook below)     */
  int32_t reserved;   /* must be 0                                            */
} indexer_problem;

/* Lossless pruning ("DoSA: Dots Sparse Attention", 核心方法 / core method:
 * skip a key whose score upper bound U_i lies below a lower bound of the
 * K-th score, with the top-K unchanged).  The kernel keeps the first 16 heads
 * of every query exactly and folds each other head onto one of them:
 *   U_i = sum_{j<16} wt_j [q_j.k_i]_+ + Ceff |k_i|  >=  s_i,
 * wt_j = w_j + sum_{h->j} w_h beta_h,  Ceff = sum_h |w_h| |q_h - beta_h q_j|
 * plus an FP32 safety margin.  The lower bound is the running threshold of
 * the streaming selection, which after its first cut is the K-th score of a
 * subset of at least K visible keys (the same page's subset bound).  A key
 * is skipped only when U_i is below that threshold, so the result is
 * bit-identical to the run without the flag.  Needs H >= 32, D % 32 == 0,
 * D <= 128; adds two small set-up kernels and workspace. */
enum { INDEXER_FLAG_PRUNE = 1 };

/* Test hook for the kernel's failure path (not for production use).  With
 * this flag every CTA of the scoring kernel, right after issuing its first
 * tile's MMAs, waits on a barrier that nothing ever arrives at, for about one
 * millisecond.  The wait runs out, the kernel takes the same exit as after any
 * pipeline wait that gives up -- the other roles see the abort, in-flight
 * MMAs and tensor loads are awaited before TMEM is freed and the CTA exits --
 * and bit 0 of the status word is set (indexer_read_status).  The outputs are
 * not valid; the device stays usable for the next call.  (Bounded device waits
 * with an error status: no device fault, trap or endless loop is used.) */
enum { INDEXER_FLAG_TEST_WAIT_TIMEOUT = 1 << 30 };

/* Row width of out_idx / out_score: K, or K + ratio - 1 for POOLED (2,051 for
 * K = 2,048 and pools of 4; KPool §2, "size index buffers to 2,051").
 * Returns INDEXER_EINVAL for an invalid problem. */
indexer_status indexer_out_width(const indexer_problem* p, int32_t* width);

/* Bytes of device workspace indexer_topk needs for `p` on the CURRENT device
 * (it depends on the device's SM count).  The workspace must be 256-byte
 * aligned; its contents need no initialisation and are scratch between calls,
 * except the status words read by indexer_read_status. */
indexer_status indexer_workspace_bytes(const indexer_problem* p, size_t* bytes);

/* Split of one problem's query rows across n_parts devices (one process per
 * GPU, keys replicated on every device): writes bounds[0 .. n_parts] (HOST
 * array) with bounds[0] = 0, bounds[n_parts] = S, non-decreasing, every bound
 * a multiple of the compiled variant's query block (or S).  Part i is rows
 * [bounds[i], bounds[i+1]): an indexer problem of its own with S' = its row
 * count and q_pos0' = q_pos0 + bounds[i], reading rows bounds[i].. of q, w
 * and q_scale and writing the same rows of the outputs.  Rows are
 * independent, so the parts need no exchange; cuts are placed by visible
 * (query, key) pair count, not by row count, since under causal visibility
 * later rows see more keys: each part's pair count is within one query
 * block's pairs of an equal share.  Pure host computation (no device call);
 * INDEXER_EINVAL for an invalid problem, n_parts < 1 or > 4096, or a null
 * `bounds`. */
indexer_status indexer_partition_rows(const indexer_problem* p, int32_t n_parts, int64_t* bounds);

/* The indexer: scores, top-K and finalisation in one call.
 *   q         [S, H, D]  bf16, or e4m3 codes (uint8) for INDEXER_FP8_E4M3
 *   k         [T, D]     same storage as q
 *   w         [S, H]     float32 head weights (signed)
 *   q_scale   [S, H]     float32, FP8 only (else NULL): q value = code*scale
 *   k_scale   [T]        float32, FP8 only (else NULL): k value = code*scale
 *   pool_coef [ratio, D] bf16, POOLED only (else NULL): the c[j] of kp
 *   out_idx   [S, W]     int32, W = indexer_out_width: selected positions
 *                        ascending, then -1 padding
 *   out_len   [S]        int32 valid length of each row:
 *                        min(K, visible) (TOKEN, COMPRESSED),
 *                        ratio*min(K/ratio, pools) + tail (POOLED)
 *   out_score [S, W]     float32 or NULL: the score of each selected entry in
 *                        the same order (a pool's score for each of its
 *                        tokens), NaN for tail and padding slots
 *   workspace, workspace_bytes: scratch from the caller (see above)
 * TOKEN and POOLED require q_pos0 + S <= T (every query has its own token).
 * Asynchronous on `stream`; allocates nothing. */
indexer_status indexer_topk(const indexer_problem* p,
                            const void* q, const void* k, const float* w,
                            const float* q_scale, const float* k_scale,
                            const void* pool_coef,
                            int32_t* out_idx, int32_t* out_len, float* out_score,
                            void* workspace, size_t workspace_bytes,
                            void* stream);

/* indexer_topk for callers that cannot allocate device memory.  This entry
 * point has no counterpart in the source pages; it exists for code that must
 * not call cudaMalloc or any other allocator where it runs the indexer -- for
 * example inside an allocator or memory-pool hook, in a plugin whose host
 * framework owns every device allocation, or in a program that forbids
 * allocation after start-up.
 *   Same arguments and result as indexer_topk, minus the workspace: scratch
 *   comes from one fixed 64 MiB array in the library's device image, which
 *   every GPU that loads the library holds until the process exits.
 *   Problems whose indexer_workspace_bytes exceeds 64 MiB are rejected with
 *   INDEXER_EWORKSPACE before anything is launched (on a 148-SM B200 with
 *   H = 64 that allows budgets up to K = 3,520).
 *   The first call on each device looks up the array's device address (with
 *   that device current); make that first call before any stream capture.
 *   Nothing here allocates.  All calls share the one array and it keeps the
 *   previous call's contents (each call clears what must start at zero), so
 *   calls that may overlap on the GPU -- on different streams, or from
 *   different host threads -- race and corrupt each other's results;
 *   serialise them.  The device status word of a call (see indexer_read_status)
 *   is read with indexer_noalloc_read_status.  The array's device address is
 *   cached per device for the life of the process; after a cudaDeviceReset
 *   of that device the entry point must not be used again. */
indexer_status indexer_topk_noalloc(const indexer_problem* p,
                                    const void* q, const void* k, const float* w,
                                    const float* q_scale, const float* k_scale,
                                    const void* pool_coef,
                                    int32_t* out_idx, int32_t* out_len, float* out_score,
                                    void* stream);

/* indexer_read_status for indexer_topk_noalloc: synchronises `stream`, reads
 * and clears the status word kept at the start of the fixed scratch array
 * (the same bits as indexer_read_status).  Allocates nothing. */
indexer_status indexer_noalloc_read_status(int32_t* flags, void* stream);

/* indexer_topk on HOST buffers (page-locked for the copies to overlap):
 * q, k, w, q_scale, k_scale and pool_coef are host pointers with the layouts
 * of indexer_topk, and so are out_idx, out_len and out_score (NULL for none).
 * The keys (with their scales or pool coefficients) are copied to the
 * device once; the query rows then pass through it in chunks of a few
 * thousand rows, the copy of chunk c+1's rows and of chunk c-1's results
 * overlapping the indexer on chunk c.  Results equal indexer_topk's.
 *   `workspace` is device memory of indexer_host_workspace_bytes bytes
 *   (256-byte aligned): the indexer's workspace for one chunk first -- so
 *   indexer_read_status applies to it, over all chunks -- then the keys and
 *   two chunks of rows.
 *   Asynchronous with respect to the host: the work is ordered on `stream`
 *   (the copies run on two internal streams joined to it by events), and the
 *   host buffers must stay valid until `stream` has been synchronised.  No
 *   device memory is allocated; two streams and eight events are created and
 *   released per call.  Errors as indexer_topk, plus INDEXER_ECUDA when a
 *   copy or stream operation fails. */
indexer_status indexer_host_workspace_bytes(const indexer_problem* p, size_t* bytes);
indexer_status indexer_topk_host(const indexer_problem* p, const void* q, const void* k,
                                 const float* w, const float* q_scale,
                                 const float* k_scale, const void* pool_coef,
                                 int32_t* out_idx, int32_t* out_len, float* out_score,
                                 void* workspace, size_t workspace_bytes, void* stream);

/* indexer_topk starting from a seed threshold ("DoSA: Dots Sparse
 * Attention", 核心方法 / core method, first step: score at least K visible
 * seed keys exactly and take their K-th score as a lower bound tau of the
 * query's K-th score; 实验结果 / results: in decode the threshold comes from
 * keys selected at recent steps and cuts the selection work).
 *   seeds  [S, n_seeds] int32 DEVICE array: for each query row, key indices
 *          in the numbering of out_idx -- token positions for TOKEN and
 *          POOLED (a position names the pool that holds it), compressed-key
 *          indices for COMPRESSED.  The previous decode step's out_idx row is
 *          a typical seed row.  Entries that are negative or not visible to
 *          the query are ignored, and so is any entry naming a key at or below
 *          the largest visible key named earlier in its row (so rows in
 *          ascending order are used whole, and no key counts twice).
 * Each row's remaining seeds are scored exactly in FP32 on CUDA cores,
 * lowered by a margin that covers the difference to the tensor-core scores
 * (eps |k| sum_h |w_h||q_h| with eps = 2^-12 for BF16 and FP8, times
 * the key scale for FP8), and their K-th
 * largest (K/ratio-th for POOLED) becomes the query's starting threshold; with
 * fewer seeds than that the query starts from no threshold.  Keys below the
 * threshold never become candidates, which shortens the selection and, with
 * split key ranges, the merge; the result is identical to indexer_topk's.
 * A run in which some query kept fewer than min(K, visible) keys sets bit 2
 * of the status word (never expected: the margin was too small).  That is the
 * only way a too-small margin can show: a threshold above the true K-th score
 * leaves fewer than K keys at or above it, so no wrong row is full-length.
 *   workspace: indexer_witness_workspace_bytes bytes (the indexer's own
 * workspace, then the seed scores [S, n_seeds] and thresholds [S]).
 * n_seeds may be 0 (then nothing is seeded); INDEXER_EINVAL for n_seeds < 0
 * or > 2^20 or a null `seeds` with S, n_seeds > 0; INDEXER_EUNSUPPORTED for
 * H > 64 or D other than 64 and 128.  Scoring the seeds costs H*D multiply-
 * adds per seed on CUDA cores: meant for decode shapes (few rows). */
indexer_status indexer_witness_workspace_bytes(const indexer_problem* p, int64_t n_seeds,
                                               size_t* bytes);
indexer_status indexer_topk_witness(const indexer_problem* p, const void* q, const void* k,
                                    const float* w, const float* q_scale,
                                    const float* k_scale, const void* pool_coef,
                                    const int32_t* seeds, int64_t n_seeds,
                                    int32_t* out_idx, int32_t* out_len, float* out_score,
                                    void* workspace, size_t workspace_bytes, void* stream);

/* indexer_topk for a packed batch of documents ("Module 06 — DSA & KPool",
 * §3 and "Ship it": no token of one document may reach another document's
 * selection, and no pool may span a document boundary).  doc_bounds is a
 * HOST array of n_docs + 1 token positions, strictly rising: document d is
 * tokens [doc_bounds[d], doc_bounds[d+1]).  The query at global position g
 * sees only keys of the document holding g:
 *   TOKEN       tokens doc_start .. g;
 *   COMPRESSED  compressed keys of its document (every bound a multiple of
 *               the ratio; key j covers tokens ratio*j .. ratio*j+ratio-1);
 *   POOLED      the document's own pools, formed from its tokens starting at
 *               doc_start, then the document's incomplete tail.
 * Every query position must lie inside [doc_bounds[0], doc_bounds[n_docs]),
 * and doc_bounds[n_docs] within the keys.  Other arguments, output layout
 * (global positions, -1 padding, lengths) and errors as indexer_topk; the
 * workspace is indexer_docs_workspace_bytes bytes, and indexer_read_status
 * covers all documents.  A batch of many short token or compressed-key
 * documents (more query blocks than half the SMs, fewer than two per SM per
 * document on average; no INDEXER_FLAG_PRUNE) runs as ONE launch over a table
 * of every document's query blocks, copied into the workspace from host
 * memory; otherwise (pooled keys, pruning, long documents, a few queries)
 * each document runs as its own indexer call on `stream`. */
indexer_status indexer_docs_workspace_bytes(const indexer_problem* p, const int64_t* doc_bounds,
                                            int32_t n_docs, size_t* bytes);
indexer_status indexer_topk_docs(const indexer_problem* p, const void* q, const void* k,
                                 const float* w, const float* q_scale,
                                 const float* k_scale, const void* pool_coef,
                                 const int64_t* doc_bounds, int32_t n_docs,
                                 int32_t* out_idx, int32_t* out_len, float* out_score,
                                 void* workspace, size_t workspace_bytes, void* stream);

/* indexer_topk for a padded batch ("Module 06 — DSA & KPool", §3 and "Ship
 * it": the boundary lengths are checked with and without padding, and a
 * padding position must never reach a selection).  The batch holds n_seqs
 * sequences, each padded to `stride` rows: sequence b is query rows and token
 * keys b*stride .. b*stride + seq_lens[b] - 1, and the rest of its stride is
 * padding.  seq_lens is a HOST array (0 <= seq_lens[b] <= stride).
 *   p->S = n_seqs*stride query rows, p->q_pos0 = 0, p->T = n_seqs*stride
 *   token keys (TOKEN, POOLED) or n_seqs*stride/ratio compressed keys
 *   (COMPRESSED; stride a multiple of the ratio).
 * Inside a sequence everything is as for a sequence of its own, positions
 * counted from its first row (pools form from its first token, its own
 * incomplete tail is appended); output indices are rows of the padded key
 * array.  Padding query rows -- and rows that see no key -- get length 0,
 * indices -1 and scores NaN.  Workspace: indexer_padded_workspace_bytes
 * bytes; indexer_read_status covers every sequence.  Each sequence runs as
 * its own indexer call on `stream`.  Errors as indexer_topk, INDEXER_EINVAL
 * for sizes that do not fit the rules above. */
indexer_status indexer_padded_workspace_bytes(const indexer_problem* p, const int64_t* seq_lens,
                                              int32_t n_seqs, int64_t stride, size_t* bytes);
indexer_status indexer_topk_padded(const indexer_problem* p, const void* q, const void* k,
                                   const float* w, const float* q_scale,
                                   const float* k_scale, const void* pool_coef,
                                   const int64_t* seq_lens, int32_t n_seqs, int64_t stride,
                                   int32_t* out_idx, int32_t* out_len, float* out_score,
                                   void* workspace, size_t workspace_bytes, void* stream);

/* Pool formation alone (the first step of POOLED):
 *   kp[p, d] = RNE_bf16( exact sum_{j<ratio} c[j, d] * k[ratio*p + j, d] )
 * for p < T_tokens / ratio; k [T_tokens, D] bf16, pool_coef [ratio, D] bf16,
 * out_kp [T_tokens/ratio, D] bf16.  (KPool §2.) */
indexer_status indexer_pool_keys(const void* k, int64_t T_tokens, int32_t D,
                                 const void* pool_coef, int32_t ratio,
                                 void* out_kp, void* stream);

/* Exact shared-index count of the non-overlapping adjacent query pairs
 * (q0,q1), (q2,q3), ... ("Adjacent-Query KV-Index Overlap in 256K DSA
 * Training", §1; computed by batched binary search as in its §3):
 *   out_shared[p] = | idx[2p, :len[2p]]  ∩  idx[2p+1, :len[2p+1]] |
 * for p < S/2.  Each valid prefix must be strictly ascending (as indexer_topk
 * writes it).  idx [S, width] int32, len [S] int32, out_shared [S/2] int32. */
indexer_status indexer_pair_overlap(const int32_t* idx, const int32_t* len,
                                    int64_t S, int32_t width,
                                    int32_t* out_shared, void* stream);

/* The three index regions of the same pairs, the preprocessing of a
 * two-query cluster ("Adjacent-Query KV-Index Overlap in 256K DSA Training",
 * §6.1: indices both queries select, and those only the left or only the
 * right query selects; §6.4: fixed-capacity buffers with device-side counts,
 * so a captured CUDA graph keeps its shapes):
 *   shared[p] = A ∩ B,  left[p] = A \ B,  right[p] = B \ A,
 *   A = idx[2p, :len[2p]],  B = idx[2p+1, :len[2p+1]],
 * each in ascending KV order at the start of row p of its [S/2, width] int32
 * buffer, padded with -1; out_counts[3p + r] is the length of region r
 * (0 shared, 1 left, 2 right).  Valid prefixes must be strictly ascending (as
 * indexer_topk writes them).  All buffers are caller-owned device memory;
 * nothing is allocated and the host does not wait.  INDEXER_EINVAL for a
 * negative S or width or a null pointer (when S >= 2). */
indexer_status indexer_pair_regions(const int32_t* idx, const int32_t* len,
                                    int64_t S, int32_t width,
                                    int32_t* out_shared, int32_t* out_left,
                                    int32_t* out_right, int32_t* out_counts,
                                    void* stream);

/* Synchronises `stream`, then reads the device status word that indexer_topk
 * keeps in `workspace` (0 = no fault).  Bit 0: a pipeline wait in the kernel
 * gave up after its time limit (the result is not valid); bit 1: a candidate
 * buffer would have overflowed (never expected; the result is not valid);
 * bit 2: a seed threshold of indexer_topk_witness was above some query's
 * K-th score (never expected; that row may be short).
 * Also clears the word.  Host pointer `flags`. */
indexer_status indexer_read_status(void* workspace, int32_t* flags, void* stream);

/* Synchronises `stream`, then reads the pruning counters of the last
 * indexer_topk call that used `workspace` into counts[0..2] (host array):
 *   counts[0]  visible (query, key) pairs screened by the certificate,
 *   counts[1]  pairs whose bound was below the query's running threshold
 *              (the per-key pruning rate is counts[1] / counts[0]),
 *   counts[2]  pairs whose full head sum was skipped: all 32 keys of their
 *              warp were bounded out (the work actually saved).
 * All zero without INDEXER_FLAG_PRUNE. */
indexer_status indexer_read_prune_counters(void* workspace, uint64_t* counts, void* stream);

/* Human-readable name of a status code (static storage). */
const char* indexer_status_string(indexer_status s);

/* Version of this ABI (incremented on incompatible change). */
int32_t indexer_abi_version(void);

/* Identity of this build: "source_sha256=" and the SHA-256 of the sources and
 * compile flags it was built from (static storage). */
const char* indexer_build_info(void);

#ifdef __cplusplus
}
#endif

#endif /* HWR_INDEXER_H */
