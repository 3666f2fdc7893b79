// merge_splits.cu -- the second step of a split key range (decode-like
// shapes: a few query blocks against many keys).  The scoring kernel then
// cuts each query block's key tiles into consecutive ranges, one CTA each,
// and every range leaves the exact top-K of its own keys, in key order.  The
// top-K of a query over all its keys is the top-K of the union of those lists
// (a key outside its range's top-K has K better keys in that range alone), so
// this kernel concatenates the lists in range order -- which is key order --
// and runs the same exact selection and output step as the single-range path.
// A range that kept K entries also bounds the answer: the final K-th score is
// at least that range's K-th score, so while concatenating, every entry below
// the largest such bound is dropped (an entry equal to it is kept, for ties)
// ("DoSA: Dots Sparse Attention", 前置知识: top-K by score, ties to the lower
// KV index; "Adjacent-Query KV-Index Overlap in 256K DSA Training", §3: rows
// in KV order with a valid length; "Module 06 — DSA & KPool", §2: each pool
// expands to its tokens, then the incomplete tail).
#include "score_topk.cuh"

namespace hwr {

struct MergeParams {
  int64_t S;            // query rows
  int64_t q_pos0;       // global position of query row 0
  int32_t splits;       // ranges per query block
  int32_t ksel;         // keys (pools) per query
  int32_t width;        // row stride of out_idx / out_score
  int32_t out_ratio;    // pool width (1 for token and compressed keys)
  const uint2* split_buf;   // [S][splits][ksel]
  const int32_t* split_cnt; // [S][splits]
  const uint32_t* split_kth; // [S][splits]: ordered K-th score of a full range, else 0
  uint2* gather;            // [S][gather_stride] scratch
  int64_t gather_stride;    // >= splits * ksel, a multiple of 128
  int32_t* out_idx;
  int32_t* out_len;
  float* out_score;
};

// One CTA of 128 threads (one warpgroup) per query row.
__global__ void __launch_bounds__(kBM) merge_splits_kernel(const MergeParams mp) {
  __shared__ uint32_t hist[kHistBins];
  __shared__ WgState<1> st;
  __shared__ uint32_t bound_s;
  const int etid = threadIdx.x;
  const int lane = etid & 31;
  constexpr int bar_id = 1;
  for (int64_t t = blockIdx.x; t < mp.S; t += gridDim.x) {
    const int32_t* cnt = mp.split_cnt + t * mp.splits;
    const uint32_t* kth = mp.split_kth + t * mp.splits;
    // the largest K-th score of a full range
    uint32_t bound = 0u;
    for (int sp = etid; sp < mp.splits; sp += kBM) bound = max(bound, kth[sp]);
    bound = warp_max_u32(bound);
    if (etid == 0) bound_s = 0u;
    named_bar(bar_id, kBM);
    if (lane == 0) atomicMax(&bound_s, bound);
    named_bar(bar_id, kBM);
    bound = bound_s;
    // concatenate the lists in range order, keeping entries >= bound
    uint2* buf = mp.gather + static_cast<size_t>(t) * mp.gather_stride;
    const Cut keep_from{bound, 0xFFFFFFFFu};  // keeps ordered scores >= bound
    int n = 0;
    for (int sp = 0; sp < mp.splits; ++sp) {
      const uint2* src = mp.split_buf + (static_cast<size_t>(t) * mp.splits + sp) * mp.ksel;
      n += wg_compact(src, cnt[sp], keep_from, bound == 0u, &st.cwc[0][0], etid, bar_id,
                      [&](int pos, uint2 e) { buf[n + pos] = e; });
    }
    named_bar(bar_id, kBM);  // the gathered list is visible to the group

    const bool all = n <= mp.ksel;
    int32_t* orow = mp.out_idx + t * mp.width;
    float* srow = mp.out_score ? mp.out_score + t * mp.width : nullptr;
    const int m = mp.out_ratio;
    auto emit = [&](int pos, uint32_t k, uint32_t ix) {
      const float sc = key_to_float(k);
      for (int rr = 0; rr < m; ++rr) {
        orow[pos * m + rr] = static_cast<int32_t>(ix) * m + rr;
        if (srow) srow[pos * m + rr] = sc;
      }
    };
    int kept;
    if (n <= kRegCap) {
      RegBuf rb;
      rb_load(rb, buf, n, etid);
      RegCut c{0u, 0xFFFFFFFFu, false, n};
      if (!all) c = rb_cut(rb, n, static_cast<uint32_t>(mp.ksel), false, 0, hist, st.red, etid, bar_id);
      kept = rb_compact(rb, n, c, all, st.scan, etid, bar_id, emit);
    } else {
      Cut cut{0u, 0xFFFFFFFFu};
      if (!all) cut = wg_topk_cut(buf, n, static_cast<uint32_t>(mp.ksel), hist, st.red, etid, bar_id);
      kept = wg_compact(buf, n, cut, all, &st.cwc[0][0], etid, bar_id,
                        [&](int pos, uint2 e) { emit(pos, e.x, e.y); });
    }
    int len = kept * m;
    if (m > 1) {
      const int64_t g = mp.q_pos0 + t;
      const int tail = static_cast<int>((g + 1) % m);
      const int64_t first = g + 1 - tail;
      for (int i = etid; i < tail; i += kBM) {
        orow[len + i] = static_cast<int32_t>(first + i);
        if (srow) srow[len + i] = __uint_as_float(0x7FC00000u);
      }
      len += tail;
    }
    for (int i = len + etid; i < mp.width; i += kBM) {
      orow[i] = -1;
      if (srow) srow[i] = __uint_as_float(0x7FC00000u);
    }
    if (etid == 0) mp.out_len[t] = len;
    named_bar(bar_id, kBM);  // the selection scratch is reused by the next row
  }
}

cudaError_t launch_merge_splits(int64_t S, int64_t q_pos0, int splits, int ksel, int width, int out_ratio,
                                const uint2* split_buf, const int32_t* split_cnt, const uint32_t* split_kth,
                                uint2* gather, int64_t gather_stride, int32_t* out_idx, int32_t* out_len,
                                float* out_score, cudaStream_t stream) {
  if (S == 0) return cudaSuccess;
  if (splits > kMaxSplits) return cudaErrorInvalidValue;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const MergeParams mp{S, q_pos0, splits, ksel, width, out_ratio, split_buf, split_cnt, split_kth,
                       gather, gather_stride, out_idx, out_len, out_score};
  int64_t blocks = S < static_cast<int64_t>(sms) * 8 ? S : static_cast<int64_t>(sms) * 8;
  merge_splits_kernel<<<static_cast<unsigned>(blocks), kBM, 0, stream>>>(mp);
  return cudaGetLastError();
}

}  // namespace hwr
