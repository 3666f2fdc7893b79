// merge_splits.cu -- the second step of a split key range (decode-like
// shapes: a few query blocks against many keys).  The scoring kernel then
// cuts each query block's key tiles into consecutive ranges, one CTA each,
// and every range leaves the exact top-K of its own keys, in key order.  The
// top-K of a query over all its keys is the top-K of the union of those lists
// (a key outside its range's top-K has K better keys in that range alone), so
// this kernel concatenates the lists in range order -- which is key order --
// and runs the same exact selection and output step as the single-range path.
// The ranges also bound the answer from below, so that the concatenation can
// drop every entry under the bound (an entry equal to it is kept, for ties):
//   * a range that kept K entries has K entries at or above its K-th score;
//   * with r = ceil(K / splits), if every range has r entries at or above its
//     r-th score v_sp, then splits * r >= K entries are at or above min v_sp.
// Either way the final K-th score is at least the bound, which for splits of
// similar keys lies close to it, so the selection runs on about K entries
// ("DoSA: Dots Sparse Attention", 前置知识: top-K by score, ties to the lower
// KV index; "Adjacent-Query KV-Index Overlap in 256K DSA Training", §3: rows
// in KV order with a valid length; "Module 06 — DSA & KPool", §2: each pool
// expands to its tokens, then the incomplete tail).
#include "score_topk.cuh"

namespace hwr {

// The merge's lists reach splits x K entries per query (75,776 for 37 ranges
// of 2,048), far above the register-resident selection's 4,096, so its passes
// over global memory keep kU loads per thread in flight: each pass costs
// n / (128 kU) load round trips instead of n / 128.
constexpr int kU = 8;

// f(e) for every entry of buf[0, n), kU entries per thread per step.
template <class F>
__device__ __forceinline__ void m_for_each(const uint2* __restrict__ buf, int n, int etid, F f) {
  for (int i0 = etid; i0 < n; i0 += kBM * kU) {
    uint2 e[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int i = i0 + u * kBM;
      e[u] = i < n ? buf[i] : make_uint2(0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < kU; ++u)
      if (i0 + u * kBM < n) f(e[u]);
  }
}

// rank-th largest (1-based) of f(e) over buf[0, n) -- f(e) = e.x (ordered
// score) or ~e.y (so that the largest is the lowest index) -- counting only
// entries with e.x == fval when `filt`; `total` = entries passing the filter.
// MSB-first radix select, 10-bit digits below the bits every entry shares.
__device__ SelResult m_radix_select(const uint2* __restrict__ buf, int n, uint32_t rank, bool idx_field, bool filt,
                                    uint32_t fval, uint32_t total, uint32_t* hist, uint32_t* red, int etid,
                                    int bar_id) {
  const int lane = etid & 31, wq = etid >> 5;
  uint32_t mx = 0u, mn = 0xFFFFFFFFu;
  m_for_each(buf, n, etid, [&](uint2 e) {
    if (!filt || e.x == fval) {
      const uint32_t f = idx_field ? ~e.y : e.x;
      mx = max(mx, f);
      mn = min(mn, f);
    }
  });
  mx = warp_max_u32(mx);
  mn = warp_min_u32(mn);
  if (lane == 0) {
    red[wq] = mx;
    red[4 + wq] = mn;
  }
  named_bar(bar_id, kBM);
  mx = max(max(red[0], red[1]), max(red[2], red[3]));
  mn = min(min(red[4], red[5]), min(red[6], red[7]));
  named_bar(bar_id, kBM);
  if (mx == mn) return {mx, 0u, total};
  int lo = 32 - __clz(mx ^ mn);
  uint32_t prefix = lo >= 32 ? 0u : (mx >> lo) << lo;
  uint32_t rem = rank, above = 0u, eq = 0u;
  while (lo > 0) {
    const int width = lo < kDigitBits ? lo : kDigitBits;
    const int shift = lo - width;
    const int nb = 1 << width;
    for (int i = etid; i < nb; i += kBM) hist[i] = 0u;
    named_bar(bar_id, kBM);
    m_for_each(buf, n, etid, [&](uint2 e) {
      if (filt && e.x != fval) return;
      const uint32_t f = idx_field ? ~e.y : e.x;
      if (lo < 32 && (f >> lo) != (prefix >> lo)) return;
      atomicAdd(&hist[(f >> shift) & static_cast<uint32_t>(nb - 1)], 1u);
    });
    named_bar(bar_id, kBM);
    // thread etid owns bins [b0, b1); ranks count from the top bin down
    const int per = nb >= kBM ? nb / kBM : 1;
    const int b0 = etid * per;
    const int b1 = min(b0 + per, nb);
    uint32_t local = 0u;
    for (int b = b0; b < b1; ++b) local += hist[b];
    uint32_t incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t t = __shfl_down_sync(kFullMask, incl, o);
      if (lane + o < 32) incl += t;
    }
    if (lane == 0) red[wq] = incl;
    named_bar(bar_id, kBM);
    uint32_t higher = 0u;
    for (int w2 = wq + 1; w2 < 4; ++w2) higher += red[w2];
    const uint32_t excl = incl - local + higher;
    if (local > 0u && excl < rem && rem <= excl + local) {
      uint32_t acc = excl;
      for (int b = b1 - 1; b >= b0; --b) {
        const uint32_t h = hist[b];
        if (acc + h >= rem) {
          red[8] = static_cast<uint32_t>(b);
          red[9] = acc;
          red[10] = h;
          break;
        }
        acc += h;
      }
    }
    named_bar(bar_id, kBM);
    rem -= red[9];
    above += red[9];
    eq = red[10];
    prefix |= red[8] << shift;
    lo = shift;
    named_bar(bar_id, kBM);
  }
  return {prefix, above, eq};
}

// Exact top-`ksel` of buf[0, n) under (higher ordered score, then lower index).
__device__ Cut m_topk_cut(const uint2* __restrict__ buf, int n, uint32_t ksel, uint32_t* hist, uint32_t* red,
                          int etid, int bar_id) {
  const SelResult s1 =
      m_radix_select(buf, n, ksel, false, false, 0u, static_cast<uint32_t>(n), hist, red, etid, bar_id);
  const uint32_t need = ksel - s1.above;
  if (need >= s1.eq) return {s1.v, 0xFFFFFFFFu};
  const SelResult s2 = m_radix_select(buf, n, need, true, true, s1.v, s1.eq, hist, red, etid, bar_id);
  return {s1.v, ~s2.v};
}

// emit(pos, e) for every entry of buf[0, n) that the cut keeps (all of them
// when keep_all), pos counting kept entries in buffer order.  Warp w takes
// the w-th quarter of the buffer: it counts its kept entries, one exchange
// gives each warp its first position, and it emits in order.  Returns the
// number kept.  buf must not be written by emit.
template <class Emit>
__device__ int m_compact(const uint2* __restrict__ buf, int n, Cut c, bool keep_all, int32_t* cwc, int etid,
                         int bar_id, Emit emit) {
  const int lane = etid & 31, wq = etid >> 5;
  const int qn = (n + 3) / 4;
  const int q0 = min(wq * qn, n), q1 = min(q0 + qn, n);
  auto keep_of = [&](uint2 e) { return keep_all || e.x > c.v || (e.x == c.v && e.y <= c.icut); };
  int cnt = 0;
  for (int b = q0; b < q1; b += 32 * kU) {
    uint2 e[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int i = b + u * 32 + lane;
      e[u] = i < q1 ? buf[i] : make_uint2(0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < kU; ++u) cnt += __popc(__ballot_sync(kFullMask, b + u * 32 + lane < q1 && keep_of(e[u])));
  }
  if (lane == 0) cwc[wq] = cnt;
  named_bar(bar_id, kBM);
  int pos = 0, total = 0;
#pragma unroll
  for (int w2 = 0; w2 < 4; ++w2) {
    total += cwc[w2];
    pos += w2 < wq ? cwc[w2] : 0;
  }
  const uint32_t lt = (1u << lane) - 1u;
  for (int b = q0; b < q1; b += 32 * kU) {
    uint2 e[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int i = b + u * 32 + lane;
      e[u] = i < q1 ? buf[i] : make_uint2(0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const bool keep = b + u * 32 + lane < q1 && keep_of(e[u]);
      const uint32_t bal = __ballot_sync(kFullMask, keep);
      if (keep) emit(pos + __popc(bal & lt), e[u]);
      pos += __popc(bal);
    }
  }
  named_bar(bar_id, kBM);  // cwc is reused by the next call
  return total;
}

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
  const uint32_t* split_rth; // [S][splits]: ordered r-th score of a range, else 0
  uint2* gather;            // [S][gather_stride] scratch
  int64_t gather_stride;    // >= splits * ksel, a multiple of 128
  int32_t* out_idx;
  int32_t* out_len;
  float* out_score;
  MergeCheck check;
};

// One CTA of 128 threads (one warpgroup) per query row.
__global__ void __launch_bounds__(kBM) merge_splits_kernel(const MergeParams mp) {
  __shared__ uint32_t hist[kHistBins];
  __shared__ WgState<1> st;
  __shared__ uint32_t bound_s[2];
  __shared__ int32_t off_s[kMaxSplits + 1];  // start of each range's list in the gathered row
  __shared__ int32_t wsum_s[kBM / 32];
  const int etid = threadIdx.x;
  const int lane = etid & 31;
  constexpr int bar_id = 1;
  // after a wait timeout in the scoring kernel the per-range lists are not
  // valid (the result is reported invalid through the status word): read none
  if (*reinterpret_cast<volatile const uint32_t*>(mp.check.status) & kStatusWaitTimeout) return;
  for (int64_t t = blockIdx.x; t < mp.S; t += gridDim.x) {
    const int32_t* cnt = mp.split_cnt + t * mp.splits;
    const uint32_t* kth = mp.split_kth + t * mp.splits;
    const uint32_t* rth = mp.split_rth + t * mp.splits;
    // the largest K-th score of a full range, and the smallest r-th score
    uint32_t b1 = 0u, b2 = 0xFFFFFFFFu;
    for (int sp = etid; sp < mp.splits; sp += kBM) {
      b1 = max(b1, kth[sp]);
      b2 = min(b2, rth[sp]);
    }
    b1 = warp_max_u32(b1);
    b2 = warp_min_u32(b2);
    if (etid == 0) {
      bound_s[0] = 0u;
      bound_s[1] = 0xFFFFFFFFu;
    }
    named_bar(bar_id, kBM);
    if (lane == 0) {
      atomicMax(&bound_s[0], b1);
      atomicMin(&bound_s[1], b2);
    }
    named_bar(bar_id, kBM);
    const uint32_t bound = max(bound_s[0], bound_s[1]);
    // offsets of the lists: thread etid owns ranges 4 etid .. 4 etid + 3
    // (splits <= 512 = 4 x 128), exclusive scan over the group
    int32_t c4[4], local = 0;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int sp = 4 * etid + u;
      c4[u] = sp < mp.splits ? min(max(cnt[sp], 0), mp.ksel) : 0;
      local += c4[u];
    }
    int32_t incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t v = __shfl_up_sync(kFullMask, incl, o);
      if (lane >= o) incl += v;
    }
    if (lane == 31) wsum_s[etid >> 5] = incl;
    named_bar(bar_id, kBM);
    int32_t run = incl - local;
    for (int w2 = 0; w2 < (etid >> 5); ++w2) run += wsum_s[w2];
    const int32_t total = wsum_s[0] + wsum_s[1] + wsum_s[2] + wsum_s[3];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int sp = 4 * etid + u;
      if (sp < mp.splits) off_s[sp] = run;
      run += c4[u];
    }
    named_bar(bar_id, kBM);
    // concatenate the lists in range order (key order).  Short lists (a seed
    // threshold leaves about K entries in all), or lists with no bound to
    // filter by, are copied whole, one warp per range, with no barrier
    // between ranges; long ones keep only entries >= bound, range by range
    uint2* buf = mp.gather + static_cast<size_t>(t) * mp.gather_stride;
    int n = 0;
    if (total <= kRegCap || bound == 0u) {
      const int wq = etid >> 5;
      for (int sp = wq; sp < mp.splits; sp += kBM / 32) {
        const uint2* src = mp.split_buf + (static_cast<size_t>(t) * mp.splits + sp) * mp.ksel;
        const int c = cnt[sp], o = off_s[sp];
        for (int i = lane; i < c; i += 32) buf[o + i] = src[i];
      }
      n = total;
    } else {
      const Cut keep_from{bound, 0xFFFFFFFFu};  // keeps ordered scores >= bound
      for (int sp = 0; sp < mp.splits; ++sp) {
        const uint2* src = mp.split_buf + (static_cast<size_t>(t) * mp.splits + sp) * mp.ksel;
        n += m_compact(src, cnt[sp], keep_from, bound == 0u, &st.cwc[0][0], etid, bar_id,
                       [&](int pos, uint2 e) { buf[n + pos] = e; });
      }
    }
    named_bar(bar_id, kBM);  // the gathered list is visible to the group

    const bool all = n <= mp.ksel;
    int32_t* orow = mp.out_idx + t * mp.width;
    float* srow = mp.out_score ? mp.out_score + t * mp.width : nullptr;
    const int m = mp.out_ratio;
    const uint32_t minv = m > 1 ? 0xFFFFFFFFu / static_cast<uint32_t>(m) + 1u : 0u;
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
      // hist is scratch from here on: pooled entries expand through it
      kept = rb_compact_steps(rb, n, c, all, st.scan, etid, bar_id,
                              [&](bool keep, int pos, uint32_t k, uint32_t ix, int first, int count) {
                                if (m == 1) {
                                  if (keep) emit(pos, k, ix);
                                } else {
                                  emit_expanded(keep, pos, k, ix, first, count, m, minv, orow, srow,
                                                hist + (etid >> 5) * 64, lane);
                                }
                              });
    } else {
      Cut cut{0u, 0xFFFFFFFFu};
      if (!all) cut = m_topk_cut(buf, n, static_cast<uint32_t>(mp.ksel), hist, st.red, etid, bar_id);
      kept = m_compact(buf, n, cut, all, &st.cwc[0][0], etid, bar_id,
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
    if (etid == 0) {
      mp.out_len[t] = len;
      if (mp.check.seeded) {
        // with a seed threshold at least min(K, visible) keys must pass it
        const int64_t g = mp.q_pos0 + t;
        int64_t nvis = mp.check.ranged ? (g + 1) / mp.check.ratio : g + 1;
        if (nvis > mp.check.n_keys) nvis = mp.check.n_keys;
        if (kept < min(static_cast<int64_t>(mp.ksel), nvis)) atomicOr(mp.check.status, kStatusWitness);
      }
    }
    named_bar(bar_id, kBM);  // the selection scratch is reused by the next row
  }
}

cudaError_t launch_merge_splits(int64_t S, int64_t q_pos0, int splits, int ksel, int width, int out_ratio,
                                const uint2* split_buf, const int32_t* split_cnt, const uint32_t* split_kth,
                                const uint32_t* split_rth, uint2* gather, int64_t gather_stride, int32_t* out_idx, int32_t* out_len,
                                float* out_score, const MergeCheck& check, cudaStream_t stream) {
  if (S == 0) return cudaSuccess;
  if (splits > kMaxSplits) return cudaErrorInvalidValue;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const MergeParams mp{S, q_pos0, splits, ksel, width, out_ratio, split_buf, split_cnt, split_kth, split_rth,
                       gather, gather_stride, out_idx, out_len, out_score, check};
  int64_t blocks = S < static_cast<int64_t>(sms) * 8 ? S : static_cast<int64_t>(sms) * 8;
  merge_splits_kernel<<<static_cast<unsigned>(blocks), kBM, 0, stream>>>(mp);
  return cudaGetLastError();
}

}  // namespace hwr
