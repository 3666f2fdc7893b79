// capi.cu -- host runtime behind include/hwr_indexer.h: argument checks,
// workspace carving, TMA descriptors and launches on the caller's stream.
// Nothing here allocates device memory or synchronises (except
// indexer_read_status, which says so).
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>
#include <vector>

#include "hwr_indexer.h"
#include "internal.h"

namespace hwr {
namespace {

constexpr size_t kStatusBytes = 256;
constexpr int kMaxDevices = 64;

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

bool get_encoder() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult qres;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &qres) == cudaSuccess &&
        qres == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  return g_encode != nullptr;
}

struct DeviceInfo {
  int sms = 0;
  bool sm100 = false;
};

DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mutex;

indexer_status device_info(DeviceInfo* out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return INDEXER_ECUDA;
  std::lock_guard<std::mutex> lock(g_dev_mutex);
  if (g_dev[dev].sms == 0) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return INDEXER_ECUDA;
    g_dev[dev].sms = sms;
    g_dev[dev].sm100 = (major == 10 && minor == 0);
  }
  *out = g_dev[dev];
  return INDEXER_OK;
}

// Everything derived from a validated problem.
struct Plan {
  ScoreVariant var;
  int64_t n_keys;    // rows scored: T, or T / ratio pools
  int32_t ksel;      // keys (pools) selected per query
  int32_t width;     // output row width
  int32_t out_ratio;
  int32_t ranged;
  int32_t n_blocks;
  int32_t grid;
  int32_t cap;
  size_t kp_bytes;   // pooled keys (POOLED only)
  size_t pq_bytes;   // per-query certificate terms (pruning only)
  size_t kn_bytes;   // key norms (pruning only)
  bool prune;
  size_t cand_bytes;
  int32_t splits;          // key-range splits per query block (1: none)
  size_t split_bytes;      // per-split top-K lists
  int64_t gather_stride;   // entries per query of the merge's gathered list (a multiple of 128)
  size_t gather_bytes;
  size_t split_cnt_bytes;  // per-split list lengths, K-th and r-th scores
  size_t ws_bytes;
};

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

indexer_status make_plan(const indexer_problem* p, bool need_device, Plan* pl) {
  if (!p) return INDEXER_EINVAL;
  if (p->S < 0 || p->T < 1 || p->q_pos0 < 0 || p->K < 1 ||
      (p->flags & ~(INDEXER_FLAG_PRUNE | INDEXER_FLAG_TEST_WAIT_TIMEOUT)) != 0 ||
      p->reserved != 0)
    return INDEXER_EINVAL;
  if (p->visibility < INDEXER_VIS_TOKEN || p->visibility > INDEXER_VIS_POOLED) return INDEXER_EINVAL;
  if (p->dtype != INDEXER_BF16 && p->dtype != INDEXER_FP8_E4M3) return INDEXER_EINVAL;
  if (p->S > (int64_t(1) << 31) / 64 || p->T > (int64_t(1) << 30) || p->q_pos0 > (int64_t(1) << 40))
    return INDEXER_EUNSUPPORTED;
  const bool token = p->visibility == INDEXER_VIS_TOKEN;
  const int ratio = token ? 1 : p->ratio;
  if (!token && (ratio < 1 || ratio > 16)) return INDEXER_EINVAL;
  if (p->visibility != INDEXER_VIS_COMPRESSED && p->q_pos0 + p->S > p->T) return INDEXER_EINVAL;
  if (p->visibility == INDEXER_VIS_POOLED) {
    if (p->K % ratio != 0) return INDEXER_EINVAL;
    if (p->dtype != INDEXER_BF16) return INDEXER_EUNSUPPORTED;
  }
  if (!score_variant(p->H, p->D, p->dtype == INDEXER_FP8_E4M3, (p->flags & INDEXER_FLAG_PRUNE) != 0, &pl->var))
    return INDEXER_EUNSUPPORTED;
  pl->n_keys = p->visibility == INDEXER_VIS_POOLED ? p->T / ratio : p->T;
  pl->ksel = p->visibility == INDEXER_VIS_POOLED ? p->K / ratio : p->K;
  if (pl->ksel > (1 << 20)) return INDEXER_EUNSUPPORTED;
  pl->width = p->visibility == INDEXER_VIS_POOLED ? p->K + ratio - 1 : p->K;
  pl->out_ratio = p->visibility == INDEXER_VIS_POOLED ? ratio : 1;
  pl->ranged = token ? 0 : 1;
  const int64_t nb = (p->S + pl->var.queries_per_block - 1) / pl->var.queries_per_block;
  pl->n_blocks = static_cast<int32_t>(nb);
  pl->cap = candidate_capacity(pl->ksel, (p->flags & INDEXER_FLAG_PRUNE) != 0);
  pl->grid = 0;
  pl->cand_bytes = 0;
  pl->splits = 1;
  pl->split_bytes = 0;
  pl->gather_stride = 0;
  pl->gather_bytes = 0;
  pl->split_cnt_bytes = 0;
  if (need_device) {
    DeviceInfo di;
    const indexer_status st = device_info(&di);
    if (st != INDEXER_OK) return st;
    // Fewer query blocks than half the SMs (decode-like shapes): cut each
    // block's key tiles into consecutive ranges of at least 16 tiles, one CTA
    // each, so that every SM has work; a merge step joins the ranges.
    if (nb > 0 && nb * 2 <= di.sms) {
      const int64_t g_last = p->q_pos0 + p->S - 1;
      int64_t nvis = pl->ranged ? (g_last + 1) / ratio : g_last + 1;
      if (nvis > pl->n_keys) nvis = pl->n_keys;
      int64_t s = di.sms / nb;
      const int64_t by_tiles = (nvis + 127) / 128 / 16;
      if (s > by_tiles) s = by_tiles;
      if (s > kMaxSplits) s = kMaxSplits;
      if (s >= 2) pl->splits = static_cast<int32_t>(s);
    }
    const int64_t items = nb * pl->splits;
    pl->grid = static_cast<int32_t>(items < di.sms ? items : di.sms);
    // kCandSets sets: a finished block's buffers are read by the row writers
    // while the next blocks fill the other sets
    pl->cand_bytes = static_cast<size_t>(pl->grid) * kCandSets * pl->var.groups * pl->var.queries_per_wg *
                     static_cast<size_t>(pl->cap) * sizeof(uint2);
    if (pl->splits > 1) {
      pl->split_bytes = align256(static_cast<size_t>(p->S) * pl->splits * pl->ksel * sizeof(uint2));
      // the selection reads entries in pairs: a padded stride keeps those reads
      // inside the query's own region
      pl->gather_stride = (static_cast<int64_t>(pl->splits) * pl->ksel + 127) / 128 * 128;
      pl->gather_bytes = align256(static_cast<size_t>(p->S) * pl->gather_stride * sizeof(uint2));
      pl->split_cnt_bytes = 3 * align256(static_cast<size_t>(p->S) * pl->splits * sizeof(int32_t));
    }
  }
  pl->kp_bytes = p->visibility == INDEXER_VIS_POOLED
                     ? align256(static_cast<size_t>(pl->n_keys) * p->D * 2)
                     : 0;
  pl->prune = (p->flags & INDEXER_FLAG_PRUNE) != 0;
  if (pl->prune && (p->H < 2 * kPruneR || p->D % 32 != 0 || p->D > 128)) return INDEXER_EUNSUPPORTED;
  pl->pq_bytes = pl->prune ? align256(static_cast<size_t>(p->S) * (kPruneR + 2) * sizeof(float)) : 0;
  pl->kn_bytes = pl->prune ? align256(static_cast<size_t>(pl->n_keys) * sizeof(float)) : 0;
  pl->ws_bytes = kStatusBytes + pl->kp_bytes + pl->pq_bytes + pl->kn_bytes + align256(pl->cand_bytes) +
                 pl->split_bytes + pl->gather_bytes + pl->split_cnt_bytes;
  return INDEXER_OK;
}

bool encode_2d(CUtensorMap* tm, const void* base, bool fp8, int64_t rows, int D, int box_rows) {
  const int elem = fp8 ? 1 : 2;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(D) * elem};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(128 / elem), static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  const CUresult r = g_encode(tm, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                              const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

}  // namespace
}  // namespace hwr

using namespace hwr;

extern "C" {

int32_t indexer_abi_version(void) { return 1; }

const char* indexer_status_string(indexer_status s) {
  switch (s) {
    case INDEXER_OK: return "ok";
    case INDEXER_EINVAL: return "invalid argument";
    case INDEXER_EWORKSPACE: return "workspace missing, misaligned or too small";
    case INDEXER_EUNSUPPORTED: return "problem outside the compiled variants";
    case INDEXER_ECUDA: return "CUDA call failed";
    case INDEXER_EDEVICE: return "device is not sm_100 (B200 class)";
  }
  return "unknown status";
}

indexer_status indexer_out_width(const indexer_problem* p, int32_t* width) {
  Plan pl;
  const indexer_status st = make_plan(p, false, &pl);
  if (st != INDEXER_OK) return st;
  if (!width) return INDEXER_EINVAL;
  *width = pl.width;
  return INDEXER_OK;
}

indexer_status indexer_workspace_bytes(const indexer_problem* p, size_t* bytes) {
  Plan pl;
  const indexer_status st = make_plan(p, true, &pl);
  if (st != INDEXER_OK) return st;
  if (!bytes) return INDEXER_EINVAL;
  *bytes = pl.ws_bytes;
  return INDEXER_OK;
}

indexer_status indexer_partition_rows(const indexer_problem* p, int32_t n_parts, int64_t* bounds) {
  Plan pl;
  const indexer_status st = make_plan(p, false, &pl);
  if (st != INDEXER_OK) return st;
  if (!bounds || n_parts < 1 || n_parts > 4096) return INDEXER_EINVAL;
  // visible keys (pools) of row t; rows are independent problems, and the
  // scoring work of a row is its visible count
  const int64_t ratio = pl.ranged ? p->ratio : 1;
  auto visible = [&](int64_t t) -> int64_t {
    const int64_t g = p->q_pos0 + t;
    const int64_t n = pl.ranged ? (g + 1) / ratio : g + 1;
    return n < pl.n_keys ? n : pl.n_keys;
  };
  const int64_t qb = pl.var.queries_per_block;
  const int64_t n_blocks = (p->S + qb - 1) / qb;
  int64_t total = 0;
  for (int64_t t = 0; t < p->S; ++t) total += visible(t);
  // cut i goes to the query-block boundary whose pair prefix is nearest to
  // i * total / n_parts (each part then differs from an equal share by at
  // most one block's pairs)
  bounds[0] = 0;
  int64_t blk = 0, prefix = 0;  // pairs of rows [0, blk * qb)
  for (int32_t i = 1; i < n_parts; ++i) {
    const long double target = static_cast<long double>(total) * i / n_parts;
    while (blk < n_blocks) {
      int64_t bp = 0;
      const int64_t r1 = (blk + 1) * qb < p->S ? (blk + 1) * qb : p->S;
      for (int64_t t = blk * qb; t < r1; ++t) bp += visible(t);
      // advance while the boundary after this block is nearer the target
      if (static_cast<long double>(prefix) + bp / 2.0L > target) break;
      prefix += bp;
      ++blk;
    }
    const int64_t r = blk * qb < p->S ? blk * qb : p->S;
    bounds[i] = r > bounds[i - 1] ? r : bounds[i - 1];
  }
  bounds[n_parts] = p->S;
  return INDEXER_OK;
}

}  // extern "C"

namespace hwr {
namespace {

// Seeds of indexer_topk_witness: [S, n] key rows per query, and the scratch
// after the indexer's own workspace.
struct Seeds {
  const int32_t* idx;
  int64_t n;
  uint32_t* lowered;  // [S, n]
  uint32_t* thr;      // [S]
};

size_t witness_extra_bytes(int64_t S, int64_t n_seeds) {
  return align256(static_cast<size_t>(S) * n_seeds * sizeof(uint32_t)) + align256(static_cast<size_t>(S) * 4);
}

// indexer_topk; reset_status = false leaves the device status word as it is
// (the host pipeline resets it once and runs one call per chunk of rows).
// With seeds, every query starts from the seed threshold.
indexer_status run_topk(const indexer_problem* p, const void* q, const void* k, const float* w,
                        const float* q_scale, const float* k_scale, const void* pool_coef, int32_t* out_idx,
                        int32_t* out_len, float* out_score, void* workspace, size_t workspace_bytes,
                        void* stream_, bool reset_status, const Seeds* seeds = nullptr) {
  Plan pl;
  indexer_status st = make_plan(p, true, &pl);
  if (st != INDEXER_OK) return st;
  DeviceInfo di;
  st = device_info(&di);
  if (st != INDEXER_OK) return st;
  if (!di.sm100) return INDEXER_EDEVICE;
  const bool fp8 = p->dtype == INDEXER_FP8_E4M3;
  const bool pooled = p->visibility == INDEXER_VIS_POOLED;
  if (p->S > 0 && (!q || !w || !out_idx || !out_len)) return INDEXER_EINVAL;
  if (!k || !aligned(k, 16) || (q && !aligned(q, 16))) return INDEXER_EINVAL;
  if (fp8 && (!q_scale || !k_scale)) return INDEXER_EINVAL;
  if (pooled && !pool_coef) return INDEXER_EINVAL;
  if (!workspace || !aligned(workspace, 256)) return INDEXER_EWORKSPACE;
  if (workspace_bytes < pl.ws_bytes) return INDEXER_EWORKSPACE;
  if (!get_encoder()) return INDEXER_ECUDA;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);

  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint32_t* status = reinterpret_cast<uint32_t*>(ws);
  void* kp = ws + kStatusBytes;
  float* pq = reinterpret_cast<float*>(ws + kStatusBytes + pl.kp_bytes);
  float* knorm = reinterpret_cast<float*>(ws + kStatusBytes + pl.kp_bytes + pl.pq_bytes);
  uint2* cand = reinterpret_cast<uint2*>(ws + kStatusBytes + pl.kp_bytes + pl.pq_bytes + pl.kn_bytes);
  uint8_t* split_base = reinterpret_cast<uint8_t*>(cand) + align256(pl.cand_bytes);
  uint2* split_buf = reinterpret_cast<uint2*>(split_base);
  uint2* split_gather = reinterpret_cast<uint2*>(split_base + pl.split_bytes);
  int32_t* split_cnt = reinterpret_cast<int32_t*>(split_base + pl.split_bytes + pl.gather_bytes);
  uint32_t* split_kth =
      reinterpret_cast<uint32_t*>(split_base + pl.split_bytes + pl.gather_bytes + pl.split_cnt_bytes / 3);
  uint32_t* split_rth =
      reinterpret_cast<uint32_t*>(split_base + pl.split_bytes + pl.gather_bytes + 2 * (pl.split_cnt_bytes / 3));
  // status word and the three pruning counters (bytes 0, 8, 16, 24) start at zero
  if (reset_status && cudaMemsetAsync(status, 0, 32, stream) != cudaSuccess) return INDEXER_ECUDA;
  if (p->S == 0) return INDEXER_OK;

  const void* keys = k;
  if (pooled) {
    if (launch_pool_keys(k, pl.n_keys, p->D, pool_coef, p->ratio, kp, stream) != cudaSuccess)
      return INDEXER_ECUDA;
    keys = kp;
  }

  CUtensorMap tm_q, tm_k;
  if (!encode_2d(&tm_q, q, fp8, p->S * p->H, p->D, pl.var.q_box_rows)) return INDEXER_ECUDA;
  // With no complete pool (a sequence shorter than one pool) no key tile is
  // ever loaded; the map still needs a non-empty extent.
  if (!encode_2d(&tm_k, keys, fp8, pl.n_keys > 0 ? pl.n_keys : 1, p->D, 128)) return INDEXER_ECUDA;

  ScoreParams sp;
  sp.S = p->S;
  sp.n_keys = pl.n_keys;
  sp.q_pos0 = p->q_pos0;
  sp.ranged = pl.ranged;
  sp.ratio = pl.ranged ? p->ratio : 1;
  sp.out_ratio = pl.out_ratio;
  sp.out_ratio_inv = pl.out_ratio > 1 ? 0xFFFFFFFFu / static_cast<uint32_t>(pl.out_ratio) + 1u : 0u;
  sp.ksel = pl.ksel;
  sp.width = pl.width;
  sp.n_blocks = pl.n_blocks;
  sp.cap = pl.cap;
  sp.w = w;
  sp.q_scale = q_scale;
  sp.k_scale = k_scale;
  sp.out_idx = out_idx;
  sp.out_len = out_len;
  sp.out_score = out_score;
  sp.cand = cand;
  sp.status = status;
  sp.prune = pl.prune ? 1 : 0;
  sp.pq = pq;
  sp.knorm = knorm;
  sp.counters = reinterpret_cast<unsigned long long*>(ws + 8);
  sp.splits = pl.splits;
  sp.split_buf = split_buf;
  sp.split_cnt = split_cnt;
  sp.split_kth = split_kth;
  sp.split_rth = split_rth;
  sp.seed_thr = nullptr;
  sp.test_wait_ns = (p->flags & INDEXER_FLAG_TEST_WAIT_TIMEOUT) ? 1000000 : 0;
  sp.seg = nullptr;
  if (seeds) {
    WitnessParams wp;
    wp.S = p->S;
    wp.n_keys = pl.n_keys;
    wp.q_pos0 = p->q_pos0;
    wp.H = p->H;
    wp.ranged = pl.ranged;
    wp.ratio = sp.ratio;
    wp.seed_div = pl.out_ratio;
    wp.ksel = pl.ksel;
    wp.fp8 = fp8 ? 1 : 0;
    wp.n_seeds = seeds->n;
    wp.seed_stride = seeds->n;
    wp.q = q;
    wp.w = w;
    wp.q_scale = q_scale;
    wp.keys = keys;
    wp.k_scale = k_scale;
    wp.seeds = seeds->idx;
    wp.lowered = seeds->lowered;
    wp.thr = seeds->thr;
    if (launch_witness(wp, p->D, stream) != cudaSuccess) return INDEXER_ECUDA;
    sp.seed_thr = seeds->thr;
  }
  if (pl.prune && launch_prune_setup(q, w, q_scale, fp8, p->S, p->H, p->D, keys, pl.n_keys, pq, knorm,
                                     stream) != cudaSuccess)
    return INDEXER_ECUDA;

  const void* fn = pl.splits > 1 ? pl.var.fn_split : pl.var.fn;
  if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, pl.var.smem_bytes) != cudaSuccess)
    return INDEXER_ECUDA;
  void* args[] = {&tm_q, &tm_k, &sp};
  if (cudaLaunchKernel(fn, dim3(pl.grid), dim3(pl.var.threads), args, pl.var.smem_bytes, stream) != cudaSuccess)
    return INDEXER_ECUDA;
  if (pl.splits > 1 &&
      launch_merge_splits(p->S, p->q_pos0, pl.splits, pl.ksel, pl.width, pl.out_ratio, split_buf, split_cnt,
                          split_kth, split_rth, split_gather, pl.gather_stride, out_idx, out_len, out_score,
                          MergeCheck{seeds ? 1 : 0, pl.ranged, sp.ratio, pl.n_keys, status}, stream) != cudaSuccess)
    return INDEXER_ECUDA;
  return INDEXER_OK;
}

}  // namespace
}  // namespace hwr

extern "C" {

indexer_status indexer_topk(const indexer_problem* p, const void* q, const void* k, const float* w,
                            const float* q_scale, const float* k_scale, const void* pool_coef, int32_t* out_idx,
                            int32_t* out_len, float* out_score, void* workspace, size_t workspace_bytes,
                            void* stream) {
  return hwr::run_topk(p, q, k, w, q_scale, k_scale, pool_coef, out_idx, out_len, out_score, workspace,
                       workspace_bytes, stream, true);
}

indexer_status indexer_witness_workspace_bytes(const indexer_problem* p, int64_t n_seeds, size_t* bytes) {
  Plan pl;
  const indexer_status st = make_plan(p, true, &pl);
  if (st != INDEXER_OK) return st;
  if (!bytes || n_seeds < 0 || n_seeds > (int64_t(1) << 20)) return INDEXER_EINVAL;
  *bytes = pl.ws_bytes + hwr::witness_extra_bytes(p->S, n_seeds);
  return INDEXER_OK;
}

indexer_status indexer_topk_witness(const indexer_problem* p, const void* q, const void* k, const float* w,
                                    const float* q_scale, const float* k_scale, const void* pool_coef,
                                    const int32_t* seeds, int64_t n_seeds, int32_t* out_idx, int32_t* out_len,
                                    float* out_score, void* workspace, size_t workspace_bytes, void* stream) {
  Plan pl;
  indexer_status st = make_plan(p, true, &pl);
  if (st != INDEXER_OK) return st;
  if (n_seeds < 0 || n_seeds > (int64_t(1) << 20) || (p->S > 0 && n_seeds > 0 && !seeds))
    return INDEXER_EINVAL;
  if (p->H > 64 || (p->D != 64 && p->D != 128)) return INDEXER_EUNSUPPORTED;
  if (!workspace || workspace_bytes < pl.ws_bytes + hwr::witness_extra_bytes(p->S, n_seeds))
    return INDEXER_EWORKSPACE;
  uint8_t* extra = static_cast<uint8_t*>(workspace) + pl.ws_bytes;
  const hwr::Seeds sd{seeds, n_seeds, reinterpret_cast<uint32_t*>(extra),
                      reinterpret_cast<uint32_t*>(extra + align256(static_cast<size_t>(p->S) * n_seeds * 4))};
  return hwr::run_topk(p, q, k, w, q_scale, k_scale, pool_coef, out_idx, out_len, out_score, workspace,
                       workspace_bytes, stream, true, &sd);
}

indexer_status indexer_pool_keys(const void* k, int64_t T_tokens, int32_t D, const void* pool_coef,
                                 int32_t ratio, void* out_kp, void* stream) {
  if (!k || !pool_coef || !out_kp || T_tokens < 0 || D < 1 || D > 4096 || ratio < 1 || ratio > 16)
    return INDEXER_EINVAL;
  if (launch_pool_keys(k, T_tokens / ratio, D, pool_coef, ratio, out_kp, static_cast<cudaStream_t>(stream)) !=
      cudaSuccess)
    return INDEXER_ECUDA;
  return INDEXER_OK;
}

indexer_status indexer_pair_overlap(const int32_t* idx, const int32_t* len, int64_t S, int32_t width,
                                    int32_t* out_shared, void* stream) {
  if (S < 0 || width < 0) return INDEXER_EINVAL;
  if (S / 2 == 0) return INDEXER_OK;
  if (!idx || !len || !out_shared) return INDEXER_EINVAL;
  if (launch_pair_overlap(idx, len, S / 2, width, out_shared, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return INDEXER_ECUDA;
  return INDEXER_OK;
}

indexer_status indexer_pair_regions(const int32_t* idx, const int32_t* len, int64_t S, int32_t width,
                                    int32_t* out_shared, int32_t* out_left, int32_t* out_right,
                                    int32_t* out_counts, void* stream) {
  if (S < 0 || width < 0) return INDEXER_EINVAL;
  if (S / 2 == 0) return INDEXER_OK;
  if (!idx || !len || !out_shared || !out_left || !out_right || !out_counts) return INDEXER_EINVAL;
  if (launch_pair_regions(idx, len, S / 2, width, out_shared, out_left, out_right, out_counts,
                          static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return INDEXER_ECUDA;
  return INDEXER_OK;
}

indexer_status indexer_read_prune_counters(void* workspace, uint64_t* counts, void* stream) {
  if (!workspace || !counts) return INDEXER_EINVAL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  unsigned long long v[3] = {0, 0, 0};
  if (cudaMemcpyAsync(v, static_cast<uint8_t*>(workspace) + 8, sizeof(v), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return INDEXER_ECUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return INDEXER_ECUDA;
  for (int i = 0; i < 3; ++i) counts[i] = v[i];
  return INDEXER_OK;
}

indexer_status indexer_read_status(void* workspace, int32_t* flags, void* stream) {
  if (!workspace || !flags) return INDEXER_EINVAL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t v = 0;
  if (cudaMemcpyAsync(&v, workspace, sizeof(v), cudaMemcpyDeviceToHost, s) != cudaSuccess) return INDEXER_ECUDA;
  if (cudaMemsetAsync(workspace, 0, sizeof(uint32_t), s) != cudaSuccess) return INDEXER_ECUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return INDEXER_ECUDA;
  *flags = static_cast<int32_t>(v);
  return INDEXER_OK;
}

}  // extern "C"

// ------------------------------------------------------------------------
// indexer_topk on host buffers: keys copied once, query rows streamed through
// the device in chunks so that the copies overlap the indexer.
// ------------------------------------------------------------------------
namespace hwr {
namespace {

struct HostLayout {
  int64_t chunk;         // query rows per chunk
  int64_t n_chunks;
  size_t elem;           // bytes per q / k element
  size_t q_row, w_row;   // bytes of one query row of q, and of w (and of q_scale)
  int32_t width;
  size_t topk_ws;        // indexer workspace for one chunk (first, so its status word is at offset 0)
  size_t off_k, off_ks, off_pc, off_slot;
  size_t slot;           // bytes of one chunk slot: q, w, q_scale, idx, len, score rows
  size_t s_w, s_qs, s_idx, s_len, s_sc;  // offsets inside a slot
  size_t total;
};

indexer_problem chunk_problem(const indexer_problem* p, int64_t first, int64_t rows) {
  indexer_problem c = *p;
  c.S = rows;
  c.q_pos0 = p->q_pos0 + first;
  return c;
}

indexer_status host_layout(const indexer_problem* p, HostLayout* L) {
  if (!p || p->S < 0) return INDEXER_EINVAL;
  // about sixteen chunks (a short first copy before the pipeline fills), each
  // large enough to fill the GPU on its own
  const int64_t target = (p->S + 15) / 16;
  int64_t chunk = target < 4096 ? 4096 : (target + 127) / 128 * 128;
  if (chunk > p->S) chunk = p->S > 0 ? p->S : 1;
  L->chunk = chunk;
  L->n_chunks = p->S > 0 ? (p->S + chunk - 1) / chunk : 0;
  L->elem = p->dtype == INDEXER_FP8_E4M3 ? 1 : 2;
  L->q_row = static_cast<size_t>(p->H) * p->D * L->elem;
  L->w_row = static_cast<size_t>(p->H) * sizeof(float);
  int32_t width = 0;
  indexer_status st = indexer_out_width(p, &width);
  if (st != INDEXER_OK) return st;
  L->width = width;
  // every full chunk has the same shape; a shorter last chunk can plan
  // differently (split key ranges), so both are sized
  size_t ws = 0;
  const int64_t last = L->n_chunks > 0 ? (L->n_chunks - 1) * chunk : 0;
  for (int64_t first : {int64_t(0), last}) {
    const int64_t rows = p->S - first < chunk ? p->S - first : chunk;
    const indexer_problem c = chunk_problem(p, first, rows > 0 ? rows : 0);
    size_t b = 0;
    st = indexer_workspace_bytes(&c, &b);
    if (st != INDEXER_OK) return st;
    ws = b > ws ? b : ws;
  }
  L->topk_ws = align256(ws);
  const bool fp8 = p->dtype == INDEXER_FP8_E4M3;
  const bool pooled = p->visibility == INDEXER_VIS_POOLED;
  L->off_k = L->topk_ws;
  L->off_ks = L->off_k + align256(static_cast<size_t>(p->T) * p->D * L->elem);
  L->off_pc = L->off_ks + (fp8 ? align256(static_cast<size_t>(p->T) * sizeof(float)) : 0);
  L->off_slot = L->off_pc + (pooled ? align256(static_cast<size_t>(p->ratio) * p->D * 2) : 0);
  const size_t c = static_cast<size_t>(chunk);
  L->s_w = align256(c * L->q_row);
  L->s_qs = L->s_w + align256(c * L->w_row);
  L->s_idx = L->s_qs + (fp8 ? align256(c * L->w_row) : 0);
  L->s_len = L->s_idx + align256(c * width * sizeof(int32_t));
  L->s_sc = L->s_len + align256(c * sizeof(int32_t));
  L->slot = L->s_sc + align256(c * width * sizeof(float));
  L->total = L->off_slot + 2 * L->slot;
  return INDEXER_OK;
}

}  // namespace
}  // namespace hwr

extern "C" {

indexer_status indexer_host_workspace_bytes(const indexer_problem* p, size_t* bytes) {
  HostLayout L;
  const indexer_status st = host_layout(p, &L);
  if (st != INDEXER_OK) return st;
  if (!bytes) return INDEXER_EINVAL;
  *bytes = L.total;
  return INDEXER_OK;
}

indexer_status indexer_topk_host(const indexer_problem* p, const void* q, const void* k, const float* w,
                                 const float* q_scale, const float* k_scale, const void* pool_coef,
                                 int32_t* out_idx, int32_t* out_len, float* out_score, void* workspace,
                                 size_t workspace_bytes, void* stream_) {
  HostLayout L;
  indexer_status st = host_layout(p, &L);
  if (st != INDEXER_OK) return st;
  const bool fp8 = p->dtype == INDEXER_FP8_E4M3;
  const bool pooled = p->visibility == INDEXER_VIS_POOLED;
  if (!k || (p->S > 0 && (!q || !w || !out_idx || !out_len))) return INDEXER_EINVAL;
  if (fp8 && (!q_scale || !k_scale)) return INDEXER_EINVAL;
  if (pooled && !pool_coef) return INDEXER_EINVAL;
  if (!workspace || !aligned(workspace, 256)) return INDEXER_EWORKSPACE;
  if (workspace_bytes < L.total) return INDEXER_EWORKSPACE;
  cudaStream_t sc = static_cast<cudaStream_t>(stream_);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  // the status word and counters start at zero once for all chunks
  if (cudaMemsetAsync(ws, 0, 32, sc) != cudaSuccess) return INDEXER_ECUDA;
  if (p->S == 0) return INDEXER_OK;

  // copies run on two streams of their own; events order them with the
  // compute stream: a slot is refilled only after the indexer call that read
  // it, and its results are overwritten only after they have been copied out
  cudaStream_t sh = nullptr, sd = nullptr;
  cudaEvent_t ev[8] = {};
  auto cleanup = [&]() {
    for (cudaEvent_t& e : ev)
      if (e) cudaEventDestroy(e);
    if (sh) cudaStreamDestroy(sh);
    if (sd) cudaStreamDestroy(sd);
  };
  if (cudaStreamCreateWithFlags(&sh, cudaStreamNonBlocking) != cudaSuccess ||
      cudaStreamCreateWithFlags(&sd, cudaStreamNonBlocking) != cudaSuccess) {
    cleanup();
    return INDEXER_ECUDA;
  }
  for (cudaEvent_t& e : ev)
    if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) {
      cleanup();
      return INDEXER_ECUDA;
    }
  cudaEvent_t ev_start = ev[0], ev_keys = ev[1];
  cudaEvent_t ev_in[2] = {ev[2], ev[3]}, ev_done[2] = {ev[4], ev[5]}, ev_out[2] = {ev[6], ev[7]};
  bool ok = true;
  auto chk = [&](cudaError_t e) { ok = ok && e == cudaSuccess; };
  // earlier work on the compute stream may still use the workspace
  chk(cudaEventRecord(ev_start, sc));
  chk(cudaStreamWaitEvent(sh, ev_start, 0));
  chk(cudaStreamWaitEvent(sd, ev_start, 0));
  chk(cudaMemcpyAsync(ws + L.off_k, k, static_cast<size_t>(p->T) * p->D * L.elem, cudaMemcpyHostToDevice, sh));
  if (fp8)
    chk(cudaMemcpyAsync(ws + L.off_ks, k_scale, static_cast<size_t>(p->T) * sizeof(float), cudaMemcpyHostToDevice,
                        sh));
  if (pooled)
    chk(cudaMemcpyAsync(ws + L.off_pc, pool_coef, static_cast<size_t>(p->ratio) * p->D * 2, cudaMemcpyHostToDevice,
                        sh));
  chk(cudaEventRecord(ev_keys, sh));
  chk(cudaStreamWaitEvent(sc, ev_keys, 0));
  for (int64_t c = 0; ok && c < L.n_chunks; ++c) {
    const int si = static_cast<int>(c & 1);
    uint8_t* slot = ws + L.off_slot + si * L.slot;
    const int64_t first = c * L.chunk;
    const int64_t rows = p->S - first < L.chunk ? p->S - first : L.chunk;
    // inputs of chunk c into slot si, once the call of chunk c - 2 is done with it
    if (c >= 2) chk(cudaStreamWaitEvent(sh, ev_done[si], 0));
    chk(cudaMemcpyAsync(slot, static_cast<const uint8_t*>(q) + first * L.q_row, rows * L.q_row,
                        cudaMemcpyHostToDevice, sh));
    chk(cudaMemcpyAsync(slot + L.s_w, w + first * p->H, rows * L.w_row, cudaMemcpyHostToDevice, sh));
    if (fp8)
      chk(cudaMemcpyAsync(slot + L.s_qs, q_scale + first * p->H, rows * L.w_row, cudaMemcpyHostToDevice, sh));
    chk(cudaEventRecord(ev_in[si], sh));
    // the indexer on chunk c, once its inputs are in and the results of
    // chunk c - 2 have left slot si
    chk(cudaStreamWaitEvent(sc, ev_in[si], 0));
    if (c >= 2) chk(cudaStreamWaitEvent(sc, ev_out[si], 0));
    if (!ok) break;
    const indexer_problem cp = chunk_problem(p, first, rows);
    st = run_topk(&cp, slot, ws + L.off_k, reinterpret_cast<const float*>(slot + L.s_w),
                  fp8 ? reinterpret_cast<const float*>(slot + L.s_qs) : nullptr,
                  fp8 ? reinterpret_cast<const float*>(ws + L.off_ks) : nullptr, pooled ? ws + L.off_pc : nullptr,
                  reinterpret_cast<int32_t*>(slot + L.s_idx), reinterpret_cast<int32_t*>(slot + L.s_len),
                  out_score ? reinterpret_cast<float*>(slot + L.s_sc) : nullptr, ws, L.topk_ws, sc, false);
    if (st != INDEXER_OK) break;
    chk(cudaEventRecord(ev_done[si], sc));
    // results of chunk c to the host
    chk(cudaStreamWaitEvent(sd, ev_done[si], 0));
    chk(cudaMemcpyAsync(out_idx + first * L.width, slot + L.s_idx, rows * L.width * sizeof(int32_t),
                        cudaMemcpyDeviceToHost, sd));
    chk(cudaMemcpyAsync(out_len + first, slot + L.s_len, rows * sizeof(int32_t), cudaMemcpyDeviceToHost, sd));
    if (out_score)
      chk(cudaMemcpyAsync(out_score + first * L.width, slot + L.s_sc, rows * L.width * sizeof(float),
                          cudaMemcpyDeviceToHost, sd));
    chk(cudaEventRecord(ev_out[si], sd));
  }
  // the compute stream ends after the last copies out (the caller synchronises it)
  chk(cudaEventRecord(ev_out[0], sd));
  chk(cudaStreamWaitEvent(sc, ev_out[0], 0));
  cleanup();
  if (st != INDEXER_OK) return st;
  return ok ? INDEXER_OK : INDEXER_ECUDA;
}

}  // extern "C"

// ------------------------------------------------------------------------
// Packed-document batches: each document is its own indexer problem.
// ------------------------------------------------------------------------
namespace hwr {
namespace {

// Document d of a packed batch as an indexer problem on its own: its query
// rows [r0, r0 + sub.S), its keys from key number key0, positions relative to
// its first token.  `shift` turns its output indices into global ones.
struct DocPart {
  indexer_problem sub;
  int64_t r0;
  int64_t key0;
  int32_t shift;
};

indexer_status doc_part(const indexer_problem* p, const int64_t* b, int32_t d, DocPart* out, bool* empty) {
  const bool compressed = p->visibility == INDEXER_VIS_COMPRESSED;
  const int64_t ratio = p->visibility == INDEXER_VIS_TOKEN ? 1 : p->ratio;
  const int64_t lo = b[d], hi = b[d + 1];
  int64_t r0 = lo - p->q_pos0, r1 = hi - p->q_pos0;
  if (r0 < 0) r0 = 0;
  if (r1 > p->S) r1 = p->S;
  *empty = r1 <= r0;
  out->sub = *p;
  out->sub.S = *empty ? 0 : r1 - r0;
  out->sub.q_pos0 = p->q_pos0 + r0 - lo;
  out->sub.T = compressed ? (hi - lo) / ratio : hi - lo;
  out->r0 = r0;
  out->key0 = compressed ? lo / ratio : lo;
  // token keys and pooled positions shift by the document's first token;
  // compressed keys by its first compressed key
  const int64_t shift = compressed ? lo / ratio : lo;
  if (shift > INT32_MAX) return INDEXER_EUNSUPPORTED;
  out->shift = static_cast<int32_t>(shift);
  return INDEXER_OK;
}

// Packed documents of token or compressed keys, without the pruning
// certificate and the test hook, run as one launch of the segmented kernel
// (every document's query blocks in one table) when the batch has more query
// blocks than half the SMs but its documents average fewer than two blocks
// per SM.  Fewer blocks in all (a few queries at the end of long documents)
// keep one launch per document, which can split each block's keys over
// several CTAs; long documents keep it too, since each launch then fills
// the GPU (measured: 64 documents of 4,096 tokens 19.9 ms in 64 launches,
// 21.9 ms in one; 1,024 of 256 tokens 25.2 ms against 6.6 ms).
indexer_status docs_fold(const indexer_problem* p, const int64_t* b, int32_t n_docs, bool* fold);

// The segmented launch of a packed batch: the whole problem's plan with one
// range per block and a grid over the table's blocks, the block table sorted
// by key tiles, lightest first (the kernel deals blocks out heaviest first),
// and the workspace (status block, candidate buffers, table).
struct SegPlan {
  Plan pl;
  std::vector<SegBlock> blocks;
  size_t cand_off, table_off, ws_bytes;
};

indexer_status seg_plan(const indexer_problem* p, const int64_t* b, int32_t n_docs, SegPlan* sp) {
  indexer_status st = make_plan(p, true, &sp->pl);
  if (st != INDEXER_OK) return st;
  Plan& pl = sp->pl;
  DeviceInfo di;
  st = device_info(&di);
  if (st != INDEXER_OK) return st;
  const int64_t qb = pl.var.queries_per_block;
  const int64_t ratio = pl.ranged ? p->ratio : 1;
  sp->blocks.clear();
  for (int32_t d = 0; d < n_docs; ++d) {
    DocPart part;
    bool empty = false;
    st = doc_part(p, b, d, &part, &empty);
    if (st != INDEXER_OK) return st;
    if (empty) continue;
    if (part.sub.T > INT32_MAX || part.key0 > INT32_MAX) return INDEXER_EUNSUPPORTED;
    for (int64_t r = 0; r < part.sub.S; r += qb) {
      SegBlock blk;
      blk.row0 = part.r0 + r;
      blk.pos0 = part.sub.q_pos0 + r;
      blk.key0 = part.key0;
      blk.rows = static_cast<int32_t>(part.sub.S - r < qb ? part.sub.S - r : qb);
      blk.n_keys = static_cast<int32_t>(part.sub.T);
      sp->blocks.push_back(blk);
    }
  }
  if (sp->blocks.size() > static_cast<size_t>(INT32_MAX)) return INDEXER_EUNSUPPORTED;
  auto tiles = [&](const SegBlock& blk) {
    const int64_t g = blk.pos0 + blk.rows - 1;
    int64_t n = pl.ranged ? (g + 1) / ratio : g + 1;
    if (n > blk.n_keys) n = blk.n_keys;
    return (n + 127) / 128;
  };
  std::stable_sort(sp->blocks.begin(), sp->blocks.end(),
                   [&](const SegBlock& x, const SegBlock& y) { return tiles(x) < tiles(y); });
  const int64_t nb = static_cast<int64_t>(sp->blocks.size());
  pl.n_blocks = static_cast<int32_t>(nb);
  pl.splits = 1;
  pl.split_bytes = pl.gather_bytes = pl.split_cnt_bytes = 0;
  pl.gather_stride = 0;
  pl.grid = static_cast<int32_t>(nb < di.sms ? nb : di.sms);
  pl.cand_bytes = static_cast<size_t>(pl.grid) * kCandSets * pl.var.groups * pl.var.queries_per_wg *
                  static_cast<size_t>(pl.cap) * sizeof(uint2);
  sp->cand_off = kStatusBytes;
  sp->table_off = sp->cand_off + align256(pl.cand_bytes);
  sp->ws_bytes = sp->table_off + align256(sp->blocks.size() * sizeof(SegBlock));
  return INDEXER_OK;
}

// The segmented launch itself: the block table copied into the workspace
// (a small copy from host memory, staged by the driver), then one launch
// over every document's blocks.  Output indices carry each document's key
// offset, so no separate shift pass runs.
indexer_status run_seg(const indexer_problem* p, const int64_t* b, int32_t n_docs, const void* q, const void* k,
                       const float* w, const float* q_scale, const float* k_scale, int32_t* out_idx,
                       int32_t* out_len, float* out_score, void* workspace, size_t workspace_bytes,
                       cudaStream_t stream) {
  SegPlan sp;
  indexer_status st = seg_plan(p, b, n_docs, &sp);
  if (st != INDEXER_OK) return st;
  const Plan& pl = sp.pl;
  DeviceInfo di;
  st = device_info(&di);
  if (st != INDEXER_OK) return st;
  if (!di.sm100) return INDEXER_EDEVICE;
  if (!pl.var.fn_seg) return INDEXER_EUNSUPPORTED;
  const bool fp8 = p->dtype == INDEXER_FP8_E4M3;
  if (!k || !aligned(k, 16) || (q && !aligned(q, 16))) return INDEXER_EINVAL;
  if (workspace_bytes < sp.ws_bytes) return INDEXER_EWORKSPACE;
  if (!get_encoder()) return INDEXER_ECUDA;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  if (cudaMemsetAsync(ws, 0, 32, stream) != cudaSuccess) return INDEXER_ECUDA;
  if (p->S == 0 || sp.blocks.empty()) return INDEXER_OK;
  SegBlock* table = reinterpret_cast<SegBlock*>(ws + sp.table_off);
  if (cudaMemcpyAsync(table, sp.blocks.data(), sp.blocks.size() * sizeof(SegBlock), cudaMemcpyHostToDevice,
                      stream) != cudaSuccess)
    return INDEXER_ECUDA;
  CUtensorMap tm_q, tm_k;
  if (!encode_2d(&tm_q, q, fp8, p->S * p->H, p->D, pl.var.q_box_rows)) return INDEXER_ECUDA;
  if (!encode_2d(&tm_k, k, fp8, pl.n_keys > 0 ? pl.n_keys : 1, p->D, 128)) return INDEXER_ECUDA;
  ScoreParams prm{};
  prm.S = p->S;
  prm.n_keys = pl.n_keys;
  prm.q_pos0 = p->q_pos0;
  prm.ranged = pl.ranged;
  prm.ratio = pl.ranged ? p->ratio : 1;
  prm.out_ratio = 1;
  prm.out_ratio_inv = 0u;
  prm.ksel = pl.ksel;
  prm.width = pl.width;
  prm.n_blocks = pl.n_blocks;
  prm.cap = pl.cap;
  prm.w = w;
  prm.q_scale = q_scale;
  prm.k_scale = k_scale;
  prm.out_idx = out_idx;
  prm.out_len = out_len;
  prm.out_score = out_score;
  prm.cand = reinterpret_cast<uint2*>(ws + sp.cand_off);
  prm.status = reinterpret_cast<uint32_t*>(ws);
  prm.prune = 0;
  prm.pq = nullptr;
  prm.knorm = nullptr;
  prm.counters = reinterpret_cast<unsigned long long*>(ws + 8);
  prm.splits = 1;
  prm.split_buf = nullptr;
  prm.split_cnt = nullptr;
  prm.split_kth = nullptr;
  prm.split_rth = nullptr;
  prm.seed_thr = nullptr;
  prm.test_wait_ns = 0;
  prm.seg = table;
  if (cudaFuncSetAttribute(pl.var.fn_seg, cudaFuncAttributeMaxDynamicSharedMemorySize, pl.var.smem_bytes) !=
      cudaSuccess)
    return INDEXER_ECUDA;
  void* args[] = {&tm_q, &tm_k, &prm};
  if (cudaLaunchKernel(pl.var.fn_seg, dim3(pl.grid), dim3(pl.var.threads), args, pl.var.smem_bytes, stream) !=
      cudaSuccess)
    return INDEXER_ECUDA;
  return INDEXER_OK;
}

indexer_status docs_fold(const indexer_problem* p, const int64_t* b, int32_t n_docs, bool* fold) {
  *fold = false;
  if (p->visibility == INDEXER_VIS_POOLED || (p->flags & (INDEXER_FLAG_PRUNE | INDEXER_FLAG_TEST_WAIT_TIMEOUT)) != 0)
    return INDEXER_OK;
  Plan pl;
  indexer_status st = make_plan(p, false, &pl);
  if (st != INDEXER_OK) return st;
  DeviceInfo di;
  st = device_info(&di);
  if (st != INDEXER_OK) return st;
  const int64_t qb = pl.var.queries_per_block;
  int64_t nb = 0, docs = 0;
  for (int32_t d = 0; d < n_docs; ++d) {
    DocPart part;
    bool empty = false;
    st = doc_part(p, b, d, &part, &empty);
    if (st != INDEXER_OK) return st;
    if (!empty) {
      nb += (part.sub.S + qb - 1) / qb;
      ++docs;
    }
  }
  *fold = nb * 2 > di.sms && nb < docs * 2 * di.sms;
  return INDEXER_OK;
}

// Bounds must rise strictly, cover every query position, stay within the
// keys, and (compressed keys) start documents on a whole compressed key.
indexer_status check_docs(const indexer_problem* p, const int64_t* b, int32_t n_docs) {
  if (!p || !b || n_docs < 1) return INDEXER_EINVAL;
  const bool compressed = p->visibility == INDEXER_VIS_COMPRESSED;
  const int64_t ratio = p->visibility == INDEXER_VIS_TOKEN ? 1 : p->ratio;
  if (ratio < 1) return INDEXER_EINVAL;
  if (b[0] < 0) return INDEXER_EINVAL;
  for (int32_t d = 0; d < n_docs; ++d) {
    if (b[d + 1] <= b[d]) return INDEXER_EINVAL;
    if (compressed && (b[d] % ratio != 0 || b[d + 1] % ratio != 0)) return INDEXER_EINVAL;
  }
  const int64_t key_tokens = compressed ? p->T * ratio : p->T;
  if (b[n_docs] > key_tokens) return INDEXER_EINVAL;
  if (p->S > 0 && (p->q_pos0 < b[0] || p->q_pos0 + p->S > b[n_docs])) return INDEXER_EINVAL;
  return INDEXER_OK;
}

}  // namespace
}  // namespace hwr

extern "C" {

indexer_status indexer_docs_workspace_bytes(const indexer_problem* p, const int64_t* doc_bounds, int32_t n_docs,
                                            size_t* bytes) {
  indexer_status st = check_docs(p, doc_bounds, n_docs);
  if (st != INDEXER_OK) return st;
  if (!bytes) return INDEXER_EINVAL;
  bool fold = false;
  st = hwr::docs_fold(p, doc_bounds, n_docs, &fold);
  if (st != INDEXER_OK) return st;
  if (fold) {
    hwr::SegPlan sp;
    st = hwr::seg_plan(p, doc_bounds, n_docs, &sp);
    if (st != INDEXER_OK) return st;
    *bytes = sp.ws_bytes;
    return INDEXER_OK;
  }
  size_t most = 0;
  for (int32_t d = 0; d < n_docs; ++d) {
    DocPart part;
    bool empty = false;
    st = doc_part(p, doc_bounds, d, &part, &empty);
    if (st != INDEXER_OK) return st;
    if (empty) continue;
    size_t b = 0;
    st = indexer_workspace_bytes(&part.sub, &b);
    if (st != INDEXER_OK) return st;
    most = b > most ? b : most;
  }
  *bytes = most > 256 ? most : 256;
  return INDEXER_OK;
}

}  // extern "C"

namespace hwr {
namespace {

// Sequence b of a padded batch as an indexer problem of its own: rows
// [b*stride, b*stride + len), positions from 0, keys from its first row.
// `empty` when it has no query row or (compressed keys) no complete key.
indexer_status seq_part(const indexer_problem* p, const int64_t* lens, int64_t stride, int32_t b, DocPart* out,
                        bool* empty) {
  const bool compressed = p->visibility == INDEXER_VIS_COMPRESSED;
  const int64_t ratio = p->visibility == INDEXER_VIS_TOKEN ? 1 : p->ratio;
  out->sub = *p;
  out->sub.S = lens[b];
  out->sub.q_pos0 = 0;
  out->sub.T = compressed ? lens[b] / ratio : lens[b];
  out->r0 = b * stride;
  out->key0 = compressed ? b * stride / ratio : b * stride;
  if (out->key0 > INT32_MAX) return INDEXER_EUNSUPPORTED;
  out->shift = static_cast<int32_t>(out->key0);
  *empty = out->sub.S == 0 || out->sub.T == 0;
  return INDEXER_OK;
}

// S and T cover every padded row, q_pos0 is 0, lengths fit their stride, and
// (compressed keys) the stride is a whole number of compressed keys.
indexer_status check_padded(const indexer_problem* p, const int64_t* lens, int32_t n_seqs, int64_t stride) {
  if (!p || !lens || n_seqs < 1 || stride < 1) return INDEXER_EINVAL;
  const bool compressed = p->visibility == INDEXER_VIS_COMPRESSED;
  const int64_t ratio = p->visibility == INDEXER_VIS_TOKEN ? 1 : p->ratio;
  if (ratio < 1 || (compressed && stride % ratio != 0)) return INDEXER_EINVAL;
  if (p->q_pos0 != 0 || p->S != n_seqs * stride) return INDEXER_EINVAL;
  if (p->T != (compressed ? n_seqs * stride / ratio : n_seqs * stride)) return INDEXER_EINVAL;
  for (int32_t b = 0; b < n_seqs; ++b)
    if (lens[b] < 0 || lens[b] > stride) return INDEXER_EINVAL;
  return INDEXER_OK;
}

}  // namespace
}  // namespace hwr

extern "C" {

indexer_status indexer_padded_workspace_bytes(const indexer_problem* p, const int64_t* seq_lens, int32_t n_seqs,
                                              int64_t stride, size_t* bytes) {
  indexer_status st = check_padded(p, seq_lens, n_seqs, stride);
  if (st != INDEXER_OK) return st;
  if (!bytes) return INDEXER_EINVAL;
  size_t most = 0;
  for (int32_t b = 0; b < n_seqs; ++b) {
    DocPart part;
    bool empty = false;
    st = seq_part(p, seq_lens, stride, b, &part, &empty);
    if (st != INDEXER_OK) return st;
    if (empty) continue;
    size_t need = 0;
    st = indexer_workspace_bytes(&part.sub, &need);
    if (st != INDEXER_OK) return st;
    most = need > most ? need : most;
  }
  *bytes = most > 256 ? most : 256;
  return INDEXER_OK;
}

indexer_status indexer_topk_padded(const indexer_problem* p, const void* q, const void* k, const float* w,
                                   const float* q_scale, const float* k_scale, const void* pool_coef,
                                   const int64_t* seq_lens, int32_t n_seqs, int64_t stride, int32_t* out_idx,
                                   int32_t* out_len, float* out_score, void* workspace, size_t workspace_bytes,
                                   void* stream) {
  indexer_status st = check_padded(p, seq_lens, n_seqs, stride);
  if (st != INDEXER_OK) return st;
  if (!q || !k || !w || !out_idx || !out_len) return INDEXER_EINVAL;
  if (p->dtype == INDEXER_FP8_E4M3 && (!q_scale || !k_scale)) return INDEXER_EINVAL;
  if (p->visibility == INDEXER_VIS_POOLED && !pool_coef) return INDEXER_EINVAL;
  size_t need = 0;
  st = indexer_padded_workspace_bytes(p, seq_lens, n_seqs, stride, &need);
  if (st != INDEXER_OK) return st;
  if (!workspace || !aligned(workspace, 256)) return INDEXER_EWORKSPACE;
  if (workspace_bytes < need) return INDEXER_EWORKSPACE;
  const size_t elem = p->dtype == INDEXER_FP8_E4M3 ? 1 : 2;
  int32_t width = 0;
  st = indexer_out_width(p, &width);
  if (st != INDEXER_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // the status word and counters start at zero once for all sequences
  if (cudaMemsetAsync(workspace, 0, 32, s) != cudaSuccess) return INDEXER_ECUDA;
  const size_t q_row = static_cast<size_t>(p->H) * p->D * elem;
  for (int32_t b = 0; b < n_seqs; ++b) {
    DocPart part;
    bool empty = false;
    st = seq_part(p, seq_lens, stride, b, &part, &empty);
    if (st != INDEXER_OK) return st;
    // rows that select nothing: the sequence's padding, and every row of a
    // sequence without a visible key (length 0, indices -1, scores NaN)
    const int64_t first_empty = empty ? part.r0 : part.r0 + part.sub.S;
    const int64_t n_empty = part.r0 + stride - first_empty;
    if (n_empty > 0) {
      if (cudaMemsetAsync(out_idx + first_empty * width, 0xFF, n_empty * width * sizeof(int32_t), s) != cudaSuccess ||
          cudaMemsetAsync(out_len + first_empty, 0, n_empty * sizeof(int32_t), s) != cudaSuccess ||
          (out_score && cudaMemsetAsync(out_score + first_empty * width, 0xFF, n_empty * width * sizeof(float), s) !=
                            cudaSuccess))
        return INDEXER_ECUDA;
    }
    if (empty) continue;
    const int64_t r0 = part.r0;
    st = run_topk(&part.sub, static_cast<const uint8_t*>(q) + r0 * q_row,
                  static_cast<const uint8_t*>(k) + part.key0 * static_cast<int64_t>(p->D) * elem, w + r0 * p->H,
                  q_scale ? q_scale + r0 * p->H : nullptr, k_scale ? k_scale + part.key0 : nullptr, pool_coef,
                  out_idx + r0 * width, out_len + r0, out_score ? out_score + r0 * width : nullptr, workspace,
                  workspace_bytes, stream, false);
    if (st != INDEXER_OK) return st;
    if (part.shift != 0 &&
        launch_offset_indices(out_idx + r0 * width, part.sub.S * width, part.shift, s) != cudaSuccess)
      return INDEXER_ECUDA;
  }
  return INDEXER_OK;
}

indexer_status indexer_topk_docs(const indexer_problem* p, const void* q, const void* k, const float* w,
                                 const float* q_scale, const float* k_scale, const void* pool_coef,
                                 const int64_t* doc_bounds, int32_t n_docs, int32_t* out_idx, int32_t* out_len,
                                 float* out_score, void* workspace, size_t workspace_bytes, void* stream) {
  indexer_status st = check_docs(p, doc_bounds, n_docs);
  if (st != INDEXER_OK) return st;
  // pointers are checked here: per document they are offset before use
  if (!k || (p->S > 0 && (!q || !w || !out_idx || !out_len))) return INDEXER_EINVAL;
  if (p->dtype == INDEXER_FP8_E4M3 && (!q_scale || !k_scale)) return INDEXER_EINVAL;
  if (p->visibility == INDEXER_VIS_POOLED && !pool_coef) return INDEXER_EINVAL;
  size_t need = 0;
  st = indexer_docs_workspace_bytes(p, doc_bounds, n_docs, &need);
  if (st != INDEXER_OK) return st;
  if (!workspace || !aligned(workspace, 256)) return INDEXER_EWORKSPACE;
  if (workspace_bytes < need) return INDEXER_EWORKSPACE;
  bool fold = false;
  st = hwr::docs_fold(p, doc_bounds, n_docs, &fold);
  if (st != INDEXER_OK) return st;
  if (fold)
    return hwr::run_seg(p, doc_bounds, n_docs, q, k, w, q_scale, k_scale, out_idx, out_len, out_score, workspace,
                        workspace_bytes, static_cast<cudaStream_t>(stream));
  const bool fp8 = p->dtype == INDEXER_FP8_E4M3;
  const size_t elem = fp8 ? 1 : 2;
  int32_t width = 0;
  st = indexer_out_width(p, &width);
  if (st != INDEXER_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // the status word and counters start at zero once for all documents
  if (cudaMemsetAsync(workspace, 0, 32, s) != cudaSuccess) return INDEXER_ECUDA;
  for (int32_t d = 0; d < n_docs; ++d) {
    DocPart part;
    bool empty = false;
    st = doc_part(p, doc_bounds, d, &part, &empty);
    if (st != INDEXER_OK) return st;
    if (empty) continue;
    const int64_t r0 = part.r0;
    const size_t q_row = static_cast<size_t>(p->H) * p->D * elem;
    st = run_topk(&part.sub, q ? static_cast<const uint8_t*>(q) + r0 * q_row : nullptr,
                  static_cast<const uint8_t*>(k) + part.key0 * static_cast<int64_t>(p->D) * elem,
                  w ? w + r0 * p->H : nullptr, q_scale ? q_scale + r0 * p->H : nullptr,
                  k_scale ? k_scale + part.key0 : nullptr, pool_coef, out_idx + r0 * width, out_len + r0,
                  out_score ? out_score + r0 * width : nullptr, workspace, workspace_bytes, stream, false);
    if (st != INDEXER_OK) return st;
    if (launch_offset_indices(out_idx + r0 * width, part.sub.S * width, part.shift, s) != cudaSuccess)
      return INDEXER_ECUDA;
  }
  return INDEXER_OK;
}

}  // extern "C"
