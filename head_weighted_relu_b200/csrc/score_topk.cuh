// score_topk.cu -- the indexer's hot path on sm_100a: tcgen05 scoring with the
// ReLU / signed head weights / visibility mask fused into the TMEM epilogue,
// and a streaming exact top-K per query.  Scores are never written to HBM.
//
// Method ("DoSA: Dots Sparse Attention", section 前置知识 / background):
//   s[t,i] = sum_h w[t,h] * max(0, q[t,h,:] . k[i,:])
// for every key i visible to query t, then the K best keys of each query
// (higher score first, then lower key index), emitted in key order with a
// valid length ("Adjacent-Query KV-Index Overlap in 256K DSA Training", §3).
// StreamIndex (arXiv 2605.02568, abstract) streams keys through a chunked
// partition-merge top-K instead of materialising scores; this kernel streams
// keys in ascending order and merges into a running selection.
//
// One persistent CTA per SM, 20 warps, one query block (the queries of one
// accumulator: 4 for 64 heads, 8 for 32, ...) at a time:
//   warp 0      TMA producer: the block's q rows once, then key tiles of 128
//               rows through a ring of shared-memory stages;
//   warp 1      MMA issuer: key tile n goes to accumulator n % NACC (two
//               at N = 256, four at N = 128: as many as TMEM's columns hold),
//               acc[key, (query, head)] = k_tile . q_block^T
//               (M = 128 keys = TMEM lanes, N = queries x heads <= 256 columns,
//               K = D), tcgen05.mma with FP32 accumulation in TMEM, so the
//               next tile's product overlaps the epilogue of this one;
//   warps 2, 3  row writers (bf16 single-range instances): they write the
//               output rows of a finished block from its candidate buffers
//               and final cuts while the epilogue goes on with the next
//               block (buffers rotate through kSets sets);
//   warps 4..19 four epilogue warpgroups, each owning a quarter of the
//               columns (whole queries).  A warpgroup keeps its queries' head
//               weights in registers for the whole block, so the head sum
//               reads nothing but TMEM: 16-column loads, double-buffered, and
//               one packed FMA per pair of heads.  Each thread owns one key
//               (one TMEM lane) and, for every query of its group, reduces
//               sum_h w[t,h] * max(acc, 0), applies the visibility mask, and
//               appends (ordered score, key) pairs that beat the query's
//               running threshold to a per-query candidate buffer in global
//               memory -- in key order, so the buffer is always sorted by key
//               index.  A buffer about to overflow is cut back toward its
//               top-K by a warpgroup radix select, which raises the threshold
//               (bf16: groups whose buffers fill cut together, in rounds).
//               After the block's last tile the same select gives the final
//               top-K, written in key order by the row writers (or by the
//               group itself: FP8 and split key ranges).
//
// Instances: SPLIT cuts each block's key tiles into ranges merged afterwards
// (decode-like shapes); SEG takes its query blocks from a table spanning the
// documents of a packed batch (each block's rows, visibility origin and
// keys), so that many short documents run as one launch.
//
// Keys arrive in ascending index order, so once a buffer holds the top-K of
// the keys seen so far with K-th entry (v, i), a later key (index > i) can
// only enter the final top-K with a score strictly above v: the threshold is
// exact for the tie rule, and every candidate the final select sees is kept
// or rejected exactly as a full sort of the score row would.
#pragma once

#include <cstddef>

#include "internal.h"
#include "ptx.cuh"

namespace hwr {

// 20 warps: warpgroup 0 = TMA producer, MMA issuer and two row writers;
// warpgroups 1..4 = epilogue.  Registers at launch: 640 x 96 = 61,440.
// Warpgroup 0 drops to 32 per thread and the epilogue takes 112:
// 128 x 32 + 512 x 112 = 61,440 (per SMSP: 32*32 + 4*112*32 = 15,360 <= 16,384).
constexpr int kThreads = 640;
constexpr int kRegsControl = 32;
constexpr int kRegsEpilogue = 112;
constexpr int kEpiGroups = 4;
constexpr int kBM = 128;                         // keys per tile = MMA M = TMEM lanes
constexpr int kDigitBits = 10;                   // radix digit width
constexpr int kHistBins = 1 << kDigitBits;
constexpr int kSmemLimit = 232448;               // 227 KB opt-in shared memory per CTA
constexpr uint64_t kWaitLimitNs = 4000000000ull; // give up a pipeline wait after 4 s
// Candidate-buffer sets: a block's buffers are read by the row writers while
// the groups fill the next sets (block r uses set r % kSets).
constexpr int kSets = kCandSets;
// Final hand-off: what the writer warps do with one query's candidate buffer.
constexpr uint32_t kJobSkip = 0;   // no such query row (past the last)
constexpr uint32_t kJobAll = 1;    // every entry is kept (at most K of them)
constexpr uint32_t kJobCut = 2;    // keep e.x > v, or e.x == v and e.y <= icut

template <int NQ>
struct WgState {
  uint32_t thr[NQ];      // a candidate is appended iff its ordered score >= thr
  int32_t cnt[2][NQ];    // candidates held, double-buffered by tile parity
  int32_t nvis[NQ];      // keys visible to each query of the group
  int4 wc[2][NQ];        // per-warp pass counts (x..w = warps 0..3), double-buffered by tile parity
  uint32_t red[24];      // reduction scratch (of the second half-group team: red2)
  uint32_t red2[24];
  int32_t cwc[2][4];     // per-warp counts during compaction (double-buffered)
  int32_t scan[4];       // per-warp totals of a register-resident compaction
  // pruning: folded weights of the kept heads, then Ceff (read as float4)
  alignas(16) float pq[NQ][kPruneR + 4];
};
static_assert(offsetof(WgState<1>, pq) % 16 == 0 && offsetof(WgState<2>, pq) % 16 == 0 &&
                  offsetof(WgState<8>, pq) % 16 == 0 && sizeof(WgState<1>) % 16 == 0,
              "pruning weights are read as float4");

template <int STAGES>
struct Barriers {
  uint64_t kfull[STAGES];
  uint64_t kempty[STAGES];
  uint64_t qfull, qempty;
  uint64_t accfull[4], accempty[4];
  uint64_t mma_done;
  uint64_t never;      // test hook: a barrier nothing arrives at
  uint32_t tmem_slot;
  int abort;
  int tmem_busy;       // MMAs may still write TMEM: leave it allocated
  int cut_round;       // raised by a group whose buffer filled: others cut too
  int seen[4];         // the cut round each epilogue group has taken part in
  // Final hand-off (single-range kernel): candidate buffers rotate through
  // kSets sets by the CTA's block count; a group posts its block's cuts to
  // set s and arrives on fin_full[s] (4 arrivals), the two writer warps write
  // the output rows and arrive on fin_free[s] (2 arrivals) once they are done
  // with the set's buffers.
  uint64_t fin_full[kSets], fin_free[kSets];
  uint4 jobs[kSets][4][8];   // [set][group][query]: n, v, icut, mode (kJob*)
  uint32_t fstage[2][64];    // per writer warp: kept pools of one step (pool expansion)
};

template <int H, int D, bool FP8>
struct Cfg {
  static constexpr int ELEM = FP8 ? 1 : 2;
  static constexpr int ROW_BYTES = D * ELEM;
  static constexpr int NBOX = ROW_BYTES / 128;          // 128-byte swizzle boxes per row
  static constexpr int BOX_ELEMS = 128 / ELEM;
  static constexpr int KSTEPS = ROW_BYTES / 32;          // MMA K steps of 32 bytes
  static constexpr int NQA = (256 / H) < 32 ? (256 / H) : 32;  // queries per accumulator = per block
  static constexpr int QB = NQA;                         // queries per block
  static constexpr int BN = NQA * H;                     // accumulator columns = MMA N
  static constexpr int CW = BN / 4;                      // columns (query, head) per epilogue warpgroup
  static constexpr int NQW = CW / H;                     // queries per epilogue warpgroup
  static constexpr int NCH = CW / 16;                    // 16-column TMEM loads per warpgroup and tile
  // Columns whose head weights are read from shared memory each tile; the
  // rest stay in registers for the whole block.  Measured per variant: the
  // bf16 one-query groups run fastest with every weight in registers, the FP8
  // and two-query groups with 16 in registers (register pressure elsewhere).
  static constexpr bool WREG = NQW <= 2;
  static constexpr int WSM_COLS = !WREG ? CW : ((!FP8 && NQW == 1) ? 0 : 48);
  static constexpr int CHAINS = FP8 ? 1 : 2;             // packed partial sums per query (FP8: fewest registers)
  static constexpr int Q_ACC_BYTES = BN * ROW_BYTES;
  static constexpr int Q_BYTES = Q_ACC_BYTES;
  static constexpr int K_STAGE_BYTES = kBM * ROW_BYTES;
  // accumulators: as many as TMEM's 512 columns hold (2 at N = 256, 4 at
  // N = 128); key tile n goes to accumulator n % NACC
  static constexpr int NACC = 512 / BN;
  static constexpr int TMEM_COLS = NACC * BN;
  static constexpr int SMALL_BYTES =
      kHistBins * 4 * kEpiGroups + BN * 4 + kEpiGroups * (int)sizeof(WgState<NQW>);
  static constexpr int AVAIL = kSmemLimit - 1024 - Q_BYTES - SMALL_BYTES - (int)sizeof(Barriers<8>);
  static constexpr int STAGES_RAW = AVAIL / K_STAGE_BYTES;
  static constexpr int STAGES = STAGES_RAW > 6 ? 6 : STAGES_RAW;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = Q_BYTES;
  static constexpr int OFF_HIST = OFF_K + STAGES * K_STAGE_BYTES;
  static constexpr int OFF_W = OFF_HIST + kHistBins * 4 * kEpiGroups;
  static constexpr int OFF_ST = OFF_W + BN * 4;
  static constexpr int OFF_BAR = OFF_ST + kEpiGroups * (int)sizeof(WgState<NQW>);
  static constexpr int SMEM_BYTES = 1024 + OFF_BAR + (int)sizeof(Barriers<STAGES>);
  static constexpr uint32_t IDESC = FP8 ? idesc_e4m3<kBM, BN>() : idesc_bf16<kBM, BN>();
  static_assert(H % 4 == 0 && H <= 64, "heads");
  static_assert(ROW_BYTES % 128 == 0, "row must be whole 128-byte swizzle rows");
  static_assert(BN % 128 == 0 && BN >= 128 && BN <= 256, "accumulator width");
  static_assert(CW % 16 == 0 && CW % H == 0 && H % 2 == 0, "whole queries per group, 16-column loads");
  static_assert(STAGES >= 2, "shared memory too small for a 2-stage key ring");
  static_assert(SMEM_BYTES <= kSmemLimit, "shared memory");
  static_assert(OFF_K % 1024 == 0 && K_STAGE_BYTES % 1024 == 0 && Q_ACC_BYTES % 1024 == 0, "swizzle alignment");
  static_assert(OFF_BAR % 16 == 0 && OFF_ST % 16 == 0 && OFF_W % 16 == 0, "alignment");
  static_assert(NQW <= 8, "final hand-off slots");
};

__device__ __forceinline__ int32_t n_visible(const ScoreParams& p, int64_t g) {
  const int64_t n = p.ranged ? (g + 1) / p.ratio : g + 1;
  return static_cast<int32_t>(n < p.n_keys ? n : p.n_keys);
}
// the same against a document's own key count
__device__ __forceinline__ int32_t n_visible_in(const ScoreParams& p, int64_t g, int32_t n_keys) {
  const int64_t n = p.ranged ? (g + 1) / p.ratio : g + 1;
  return static_cast<int32_t>(n < n_keys ? n : n_keys);
}

// Where query block b sits: its first row, the visibility position of that
// row, the first key row of its keys, its row count and its key count.  A
// single problem's blocks are QB consecutive rows over all keys; the
// segmented kernel reads them from its block table.
struct BlockGeom {
  int64_t row0, pos0, key0;
  int32_t rows, n_keys;
};
template <int QB, bool SEG>
__device__ __forceinline__ BlockGeom geom_of(const ScoreParams& p, int b) {
  if constexpr (SEG) {
    const SegBlock sb = p.seg[b];
    return {sb.row0, sb.pos0, sb.key0, sb.rows, sb.n_keys};
  } else {
    const int64_t row0 = static_cast<int64_t>(b) * QB;
    const int64_t left = p.S - row0;
    return {row0, p.q_pos0 + row0, 0, static_cast<int32_t>(left < QB ? left : QB), static_cast<int32_t>(p.n_keys)};
  }
}

// Heaviest query blocks first (they see the most keys), dealt to the CTAs in
// a snake order so that per-CTA work evens out.  -1 once this CTA is done.
__device__ __forceinline__ int block_of(int round, int cta, int grid, int n_blocks) {
  const int item = round * grid + ((round & 1) ? (grid - 1 - cta) : cta);
  return item < n_blocks ? n_blocks - 1 - item : -1;
}

template <int QB, bool SEG>
__device__ __forceinline__ int tiles_of_block(const ScoreParams& p, int b) {
  const BlockGeom g = geom_of<QB, SEG>(p, b);
  const int32_t n = n_visible_in(p, g.pos0 + g.rows - 1, g.n_keys);
  return (n + kBM - 1) / kBM;
}

// A CTA's work item: query block b, key tiles [j0, j1) of it, split index sp.
// With few query blocks (decode-like shapes) each block's key tiles are cut
// into p.splits consecutive ranges, each its own item; the per-split top-K
// lists are merged afterwards.  b < 0 once this CTA is done.
struct Item {
  int b, j0, j1, sp;
};
template <int QB, bool SPLIT, bool SEG = false>
__device__ __forceinline__ Item item_of(const ScoreParams& p, int round, int cta, int grid) {
  if constexpr (!SPLIT) {
    const int b = block_of(round, cta, grid, p.n_blocks);
    return {b, 0, b < 0 ? 0 : tiles_of_block<QB, SEG>(p, b), 0};
  }
  const int it = block_of(round, cta, grid, p.n_blocks * p.splits);
  if (it < 0) return {-1, 0, 0, 0};
  const int b = it / p.splits;
  const int sp = it - b * p.splits;
  const int nt = tiles_of_block<QB, false>(p, b);
  const int per = (nt + p.splits - 1) / p.splits;
  const int j0 = min(sp * per, nt);
  return {b, j0, min(j0 + per, nt), sp};
}

// 2 * max(x, 0) for two accumulator columns, computed as x + |x| with one
// packed add (exact: 2x for x >= 0, +0 otherwise).  The head weights are
// staged halved (also exact), so w/2 * (x + |x|) rounds exactly like
// w * max(x, 0).
__device__ __forceinline__ float2 relu2x2(uint32_t b0, uint32_t b1) {
  const float2 x = make_float2(__uint_as_float(b0), __uint_as_float(b1));
  return __fadd2_rn(x, make_float2(fabsf(x.x), fabsf(x.y)));
}

// Adds one 16-column TMEM chunk of the group's columns into the packed partial
// sums: column col0 + k holds query (col0 + k) / H, head (col0 + k) % H.  Each
// pair of heads goes through one packed FMA with the pair's halved weights
// (wget(col) returns them as a float2); pair p of a query feeds chain
// p % CHAINS.  Every index is a compile-time constant once the callers'
// loops are unrolled, so the sums and register-held weights stay in registers.
template <int H, int NQW, int CHAINS, class WGet>
__device__ __forceinline__ void chunk_fma(const uint32_t (&r)[16], int col0, WGet wget,
                                          float2 (&acc)[NQW][CHAINS]) {
#pragma unroll
  for (int k = 0; k < 16; k += 2) {
    const int col = col0 + k;
    const int qi = col / H;
    const int ch = ((col % H) >> 1) % CHAINS;
    acc[qi][ch] = __ffma2_rn(wget(col), relu2x2(r[k], r[k + 1]), acc[qi][ch]);
  }
}

// The score from a query's partial sums, added in a fixed tree.
template <int CHAINS>
__device__ __forceinline__ float chain_total(const float2 (&a)[CHAINS]) {
  if constexpr (CHAINS == 4)
    return ((a[0].x + a[0].y) + (a[1].x + a[1].y)) + ((a[2].x + a[2].y) + (a[3].x + a[3].y));
  else if constexpr (CHAINS == 2)
    return (a[0].x + a[0].y) + (a[1].x + a[1].y);
  else
    return a[0].x + a[0].y;
}

// Upper bound of a key's score from the first kPruneR heads of a query
// ("DoSA: Dots Sparse Attention", 核心方法): U = sum_{j<16} wt_j max(acc_j, 0) +
// Ceff |k|, widened by a few roundings; r holds the query's first 16 columns.
template <bool FP8>
__device__ __forceinline__ float prune_bound(const uint32_t (&r)[16], const float* wt, float ks, float kn) {
  float2 u0 = make_float2(0.f, 0.f), u1 = make_float2(0.f, 0.f);
#pragma unroll
  for (int h = 0; h < kPruneR; h += 4) {
    const float4 wv = *reinterpret_cast<const float4*>(wt + h);
    u0 = __ffma2_rn(make_float2(wv.x, wv.y), relu2x2(r[h], r[h + 1]), u0);
    u1 = __ffma2_rn(make_float2(wv.z, wv.w), relu2x2(r[h + 2], r[h + 3]), u1);
  }
  float u = (u0.x + u0.y) + (u1.x + u1.y);
  u = fmaf(wt[kPruneR], kn, u);
  u += fabsf(u) * 0x1p-20f;
  if (FP8) {
    u *= ks;
    u += fabsf(u) * 0x1p-20f;
  }
  return __fadd_rn(u, 0.f);  // -0 -> +0, as for scores
}

// ------------------------------------------------------------------------
// Warpgroup-cooperative selection over a candidate buffer (128 threads).
// ------------------------------------------------------------------------
struct SelResult {
  uint32_t v;      // the rank-th largest value
  uint32_t above;  // entries (passing the filter) with a larger value
  uint32_t eq;     // entries equal to v
};

// rank-th largest (1-based) of f(e) over buf[0, n), where f(e) = e.x (ordered
// score) or ~e.y (so that the largest is the lowest index), counting only the
// entries with e.x == fval when `filt`.  `total` = entries passing the filter.
// MSB-first radix select with 11-bit digits, starting below the bits that all
// entries share.
__device__ inline SelResult wg_radix_select(const uint2* buf, int n, uint32_t rank, bool idx_field, bool filt,
                                     uint32_t fval, uint32_t total, uint32_t* hist, uint32_t* red,
                                     int etid, int bar_id) {
  const int lane = etid & 31, wq = etid >> 5;
  uint32_t mx = 0u, mn = 0xFFFFFFFFu;
  for (int i = etid; i < n; i += kBM) {
    const uint2 e = buf[i];
    if (!filt || e.x == fval) {
      const uint32_t f = idx_field ? ~e.y : e.x;
      mx = max(mx, f);
      mn = min(mn, f);
    }
  }
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
  int lo = 32 - __clz(mx ^ mn);  // bits [lo, 32) are shared by every entry
  uint32_t prefix = lo >= 32 ? 0u : (mx >> lo) << lo;
  uint32_t rem = rank, above = 0u, eq = 0u;
  while (lo > 0) {
    const int width = lo < kDigitBits ? lo : kDigitBits;
    const int shift = lo - width;
    const int nb = 1 << width;
    for (int i = etid; i < nb; i += kBM) hist[i] = 0u;
    named_bar(bar_id, kBM);
    for (int i = etid; i < n; i += kBM) {
      const uint2 e = buf[i];
      if (filt && e.x != fval) continue;
      const uint32_t f = idx_field ? ~e.y : e.x;
      if (lo < 32 && (f >> lo) != (prefix >> lo)) continue;
      atomicAdd(&hist[(f >> shift) & static_cast<uint32_t>(nb - 1)], 1u);
    }
    named_bar(bar_id, kBM);
    // thread etid owns bins [b0, b1); ranks count from the top bin down
    const int per = nb >= kBM ? nb / kBM : 1;
    const int b0 = etid * per;
    const int b1 = min(b0 + per, nb);
    uint32_t local = 0u;
    for (int b = b0; b < b1; ++b) local += hist[b];
    uint32_t incl = local;  // sum over lanes >= this lane
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t t = __shfl_down_sync(kFullMask, incl, o);
      if (lane + o < 32) incl += t;
    }
    if (lane == 0) red[wq] = incl;
    named_bar(bar_id, kBM);
    uint32_t higher = 0u;
    for (int w2 = wq + 1; w2 < 4; ++w2) higher += red[w2];
    const uint32_t excl = incl - local + higher;  // entries in bins owned by higher threads
    if (local > 0u && excl < rem && rem <= excl + local) {
      uint32_t acc = excl;
      for (int b = b1 - 1; b >= b0; --b) {
        const uint32_t h = hist[b];
        if (acc + h >= rem) {
          red[8] = static_cast<uint32_t>(b);
          red[9] = acc;  // entries above digit b in this pass
          red[10] = h;
          break;
        }
        acc += h;
      }
    }
    named_bar(bar_id, kBM);
    const uint32_t d = red[8];
    rem -= red[9];
    above += red[9];
    eq = red[10];
    prefix |= d << shift;
    lo = shift;
    named_bar(bar_id, kBM);
  }
  return {prefix, above, eq};
}

// Entries to keep: e.x > v, or e.x == v and e.y <= icut.
struct Cut {
  uint32_t v;
  uint32_t icut;
};

// Exact top-`ksel` of buf[0, n) under (higher ordered score, then lower index).
__device__ inline Cut wg_topk_cut(const uint2* buf, int n, uint32_t ksel, uint32_t* hist, uint32_t* red, int etid,
                           int bar_id) {
  const SelResult s1 = wg_radix_select(buf, n, ksel, false, false, 0u, static_cast<uint32_t>(n), hist, red,
                                       etid, bar_id);
  const uint32_t need = ksel - s1.above;  // entries equal to v that make the cut
  if (need >= s1.eq) return {s1.v, 0xFFFFFFFFu};
  // the need-th lowest index among the entries tied at v
  const SelResult s2 = wg_radix_select(buf, n, need, true, true, s1.v, s1.eq, hist, red, etid, bar_id);
  return {s1.v, ~s2.v};
}

// Streams buf[0, n) in order and calls emit(pos, e) for every kept entry, pos
// counting kept entries in buffer order.  In place (emit writing buf[pos]) is
// safe: pos never exceeds the entry's own index and reads of a chunk finish
// before its writes.  Returns the number kept.
template <class Emit>
__device__ int wg_compact(const uint2* buf, int n, Cut c, bool keep_all, int32_t* cwc, int etid, int bar_id,
                          Emit emit) {
  const int lane = etid & 31, wq = etid >> 5;
  int running = 0, par = 0;
  for (int base = 0; base < n; base += kBM) {
    const int i = base + etid;
    uint2 e = make_uint2(0u, 0u);
    bool keep = false;
    if (i < n) {
      e = buf[i];
      keep = keep_all || e.x > c.v || (e.x == c.v && e.y <= c.icut);
    }
    const uint32_t bal = __ballot_sync(kFullMask, keep);
    if (lane == 0) cwc[par * 4 + wq] = __popc(bal);
    named_bar(bar_id, kBM);
    int prior = 0, tot = 0;
#pragma unroll
    for (int w2 = 0; w2 < 4; ++w2) {
      const int cc = cwc[par * 4 + w2];
      tot += cc;
      prior += (w2 < wq) ? cc : 0;
    }
    if (keep) emit(running + prior + __popc(bal & ((1u << lane) - 1u)), e);
    running += tot;
    par ^= 1;
  }
  named_bar(bar_id, kBM);
  return running;
}

// ------------------------------------------------------------------------
// Register-resident selection: the warpgroup holds the whole candidate
// buffer in registers.  Entry e lives in warp e / 1024, register
// (e % 1024) / 32, lane e % 32, so each register step of a warp covers 32
// consecutive entries: loading the buffer and writing kept entries back (or
// out) are coalesced 256-byte accesses, and order-preserving compaction needs
// one ballot per step and one exchange of per-warp counts.  Used whenever the
// buffer fits (capacity <= 4,096 entries, i.e. budgets up to 2,048).
// ------------------------------------------------------------------------
constexpr int kRegEntries = 32;
// A selection runs on a team of NW warps (4: a whole epilogue group; 2: half
// a group, each half selecting for one of the group's two queries) with
// NW * 32 threads, a histogram of team_bins<NW>() bins in shared memory and
// radix digits of at most team_digit_bits<NW>() bits.
template <int NW>
__host__ __device__ constexpr int team_bins() { return NW == 4 ? kHistBins : kHistBins / 2; }
template <int NW>
__host__ __device__ constexpr int team_digit_bits() { return NW == 4 ? kDigitBits : kDigitBits - 1; }
constexpr int kRegCap = kRegEntries * kBM;
constexpr int kWarpEntries = kRegEntries * 32;   // entries held by one warp

struct RegBuf {
  uint32_t key[kRegEntries];
  uint32_t idx[kRegEntries];
};

// Register r of this thread holds buffer position (etid / 32) * 1024 +
// 32 r + etid % 32; it is valid iff 32 r < rb_room(n, etid).
__device__ __forceinline__ int rb_room(int n, int etid) {
  return n - (etid >> 5) * kWarpEntries - (etid & 31);
}

__device__ __forceinline__ void rb_load(RegBuf& b, const uint2* buf, int n, int etid) {
  const int room = rb_room(n, etid);
  const uint2* src = buf + (etid >> 5) * kWarpEntries + (etid & 31);
#pragma unroll
  for (int r = 0; r < kRegEntries; ++r) {
    uint2 v = make_uint2(0u, 0u);
    if (32 * r < room) v = src[32 * r];
    b.key[r] = v.x;
    b.idx[r] = v.y;
  }
}

// The value ranked: the ordered score, or ~index (so that larger = lower index).
__device__ __forceinline__ uint32_t rb_field(const RegBuf& b, int r, bool idx_field) {
  return idx_field ? ~b.idx[r] : b.key[r];
}

// Largest and smallest ranked value over the valid entries (only those whose
// ordered score equals fval when `filt`).  The next pass's barriers order the
// reuse of `red`.
template <int NW = 4>
__device__ inline void rb_maxmin(const RegBuf& b, int n, bool idx_field, bool filt, uint32_t fval, uint32_t& mx,
                          uint32_t& mn, uint32_t* red, int etid, int bar_id) {
  const int lane = etid & 31, wq = etid >> 5;
  mx = 0u;
  mn = 0xFFFFFFFFu;
  const int room = rb_room(n, etid);
#pragma unroll
  for (int r = 0; r < kRegEntries; ++r) {
    // branch-free: every condition is a predicate, every update a select
    const bool ok = (32 * r < room) & (!filt | (b.key[r] == fval));
    const uint32_t f = rb_field(b, r, idx_field);
    mx = max(mx, ok ? f : 0u);
    mn = min(mn, ok ? f : 0xFFFFFFFFu);
  }
  mx = warp_max_u32(mx);
  mn = warp_min_u32(mn);
  if (lane == 0) {
    red[wq] = mx;
    red[4 + wq] = mn;
  }
  named_bar(bar_id, NW * 32);
  mx = red[0];
  mn = red[4];
#pragma unroll
  for (int w2 = 1; w2 < NW; ++w2) {
    mx = max(mx, red[w2]);
    mn = min(mn, red[4 + w2]);
  }
}

struct Digit {
  uint32_t d;      // the digit holding the rank-th largest
  uint32_t above;  // entries in higher digits (this pass)
  uint32_t cnt;    // entries in digit d
};

// One radix pass over the valid entries whose ranked value f lies in
// [base, base + 2^(shift + width)): digit (f - base) >> shift, 2^width bins,
// counted from the top.  Digits are offsets from a base rather than bit
// fields of f, so a range of values that straddles a power of two (where all
// exponent bits of the ordered score change) still spreads over the bins.
// hist[0, 2^width) must be zero on entry and is zero again on return.  Every
// thread adds its entries to the histogram; warp 0 then finds the digit:
// lane L sums bins [L*per, L*per+per) (rotated so that the lanes read
// distinct banks), a suffix scan over the lanes finds the lane holding the
// rank-th largest, a second scan over that lane's bins finds the digit, and
// the warp clears the bins.  Two barriers.
template <int NW>
__device__ inline Digit rb_find_digit(int nb, uint32_t rank, uint32_t* hist, uint32_t* red, int etid, int bar_id);

// (entries above `top` are left out: they lie in higher bins of an earlier
// pass)
template <int NW = 4>
__device__ inline Digit rb_pass(const RegBuf& b, int n, bool idx_field, bool filt, uint32_t fval, uint32_t base,
                         int shift, int width, uint32_t rank, uint32_t* hist, uint32_t* red, int etid, int bar_id,
                         uint32_t top = 0xFFFFFFFFu) {
  const int nb = 1 << width;
  const unsigned long long span = 1ull << (shift + width);
  const int room = rb_room(n, etid);
#pragma unroll
  for (int r = 0; r < kRegEntries; ++r) {
    const uint32_t f = rb_field(b, r, idx_field);
    // branch-free: every condition is a predicate
    const bool ok = (32 * r < room) & (!filt | (b.key[r] == fval)) & (f >= base) &
                    (static_cast<unsigned long long>(f - base) < span) & (f <= top);
    if (ok) atomicAdd(&hist[(f - base) >> shift], 1u);
  }
  return rb_find_digit<NW>(nb, rank, hist, red, etid, bar_id);
}

// The digit of a filled histogram (2^width = nb bins, counted from the top)
// that holds the rank-th largest entry; clears the bins.  Two barriers.
template <int NW>
__device__ inline Digit rb_find_digit(int nb, uint32_t rank, uint32_t* hist, uint32_t* red, int etid, int bar_id) {
  const int lane = etid & 31, wq = etid >> 5;
  named_bar(bar_id, NW * 32);
  if (wq == 0) {
    const int per = nb >= 32 ? nb >> 5 : 1;   // bins per lane (a power of two)
    const int owners = nb >= 32 ? 32 : nb;
    uint32_t local = 0u;
    if (lane < owners)
      for (int k = 0; k < per; ++k) local += hist[lane * per + ((k + lane) & (per - 1))];
    uint32_t incl = local;  // entries in bins of lanes >= this lane
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t t = __shfl_down_sync(kFullMask, incl, o);
      if (lane + o < 32) incl += t;
    }
    const uint32_t excl = incl - local;
    const int ls = max(__ffs(__ballot_sync(kFullMask, lane < owners && excl < rank && rank <= incl)) - 1, 0);
    const uint32_t above = __shfl_sync(kFullMask, excl, ls);
    // inside lane ls's bins: lane j takes bin ls * per + j
    const uint32_t h = lane < per ? hist[ls * per + lane] : 0u;
    uint32_t inc2 = h;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t t = __shfl_down_sync(kFullMask, inc2, o);
      if (lane + o < 32) inc2 += t;
    }
    const uint32_t ex2 = inc2 - h;
    if (lane < per && above + ex2 < rank && rank <= above + inc2) {
      red[8] = static_cast<uint32_t>(ls * per + lane);
      red[9] = above + ex2;
      red[10] = h;
    }
    __syncwarp();
    for (int i = lane; i < nb; i += 32) hist[i] = 0u;
  }
  named_bar(bar_id, NW * 32);
  return Digit{red[8], red[9], red[10]};
}

// A cut of a buffer to its top `ksel`: keep key >= v when `ge`, otherwise keep
// key > v, or key == v and index <= icut.  `kept` = entries the cut keeps.
struct RegCut {
  uint32_t v;
  uint32_t icut;
  bool ge;
  int kept;
};

// Entries at most this many in the bin that holds the ksel-th largest are
// sorted in one warp instead of further radix passes.
constexpr int kSmallSel = 64;

// Sorts 64 keys held as v[j] = element 32 j + lane into descending order
// (bitonic network; pairs at distance 32 sit in the same lane).
__device__ __forceinline__ void warp_sort64_desc(unsigned long long (&v)[2], int lane) {
#pragma unroll
  for (int k = 2; k <= 64; k <<= 1) {
#pragma unroll
    for (int s = k >> 1; s > 0; s >>= 1) {
      unsigned long long nv[2];
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int i = j * 32 + lane;
        const unsigned long long other = s == 32 ? v[j ^ 1] : __shfl_xor_sync(kFullMask, v[j], s);
        // in a block sorted descending the lower index of a pair takes the larger
        const bool take_max = ((i & s) == 0) == ((i & k) == 0);
        nv[j] = take_max ? (v[j] > other ? v[j] : other) : (v[j] < other ? v[j] : other);
      }
      v[0] = nv[0];
      v[1] = nv[1];
    }
  }
}

// The cut when the remaining candidates -- the entries whose ordered score
// lies in [base, base + span) -- number at most kSmallSel: they are
// gathered into shared memory (hist[512, 640), free after the passes), warp
// 0 sorts them by (ordered score desc, index asc) and the rank-th of them
// gives v and the index cut.  red[12] counts the gathered entries (cleared by
// the caller before its first barrier).
template <int NW = 4>
__device__ inline RegCut rb_small_select(const RegBuf& b, int n, uint32_t base, unsigned long long span,
                                         uint32_t rank, uint32_t ksel, uint32_t* hist, uint32_t* red, int etid,
                                         int bar_id) {
  const int lane = etid & 31, wq = etid >> 5;
  const int room = rb_room(n, etid);
  // the upper half of the team's histogram (zero after the passes) holds the
  // gathered entries: 64 x 8 bytes fit in 256 of its words
  uint2* list = reinterpret_cast<uint2*>(hist + team_bins<NW>() / 2);
#pragma unroll
  for (int r = 0; r < kRegEntries; ++r) {
    const uint32_t k = b.key[r];
    const bool in = (32 * r < room) & (k >= base) & (static_cast<unsigned long long>(k - base) < span);
    if (in) list[atomicAdd(&red[12], 1u)] = make_uint2(k, b.idx[r]);
  }
  named_bar(bar_id, NW * 32);
  if (wq == 0) {
    const uint32_t m = red[12];
    unsigned long long v[2];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const uint32_t i = j * 32 + lane;
      // (score, ~index): larger is better; unused slots sort last
      v[j] = i < m ? (static_cast<unsigned long long>(list[i].x) << 32) | (~list[i].y) : 0ull;
    }
    warp_sort64_desc(v, lane);
    const uint32_t at = rank - 1;  // 0-based position of the rank-th best
    const unsigned long long w = __shfl_sync(kFullMask, at < 32 ? v[0] : v[1], at & 31);
    if (lane == 0) {
      red[8] = static_cast<uint32_t>(w >> 32);
      red[9] = ~static_cast<uint32_t>(w);
    }
  }
  named_bar(bar_id, NW * 32);
  return {red[8], red[9], false, static_cast<int>(ksel)};
}

// Bin of an entry in a first pass linear in the score value: 1,024 bins over
// [fmn, fmn + 1024 / scale].  Rounded subtraction, multiplication by a
// positive scale and truncation are each monotone, so a higher bin holds only
// strictly higher scores and equal scores share a bin.
template <int NW = 4>
__device__ __forceinline__ uint32_t score_bin(uint32_t key, float fmn, float scale) {
  return min(static_cast<uint32_t>(team_bins<NW>() - 1), __float2uint_rz((key_to_float(key) - fmn) * scale));
}

// First pass over score values: the bin holding the rank-th largest entry.
template <int NW = 4>
__device__ inline Digit rb_fpass(const RegBuf& b, int n, float fmn, float scale, uint32_t rank, uint32_t* hist,
                                 uint32_t* red, int etid, int bar_id) {
  const int room = rb_room(n, etid);
#pragma unroll
  for (int r = 0; r < kRegEntries; ++r)
    if (32 * r < room) atomicAdd(&hist[score_bin<NW>(b.key[r], fmn, scale)], 1u);
  return rb_find_digit<NW>(team_bins<NW>(), rank, hist, red, etid, bar_id);
}

// Smallest and largest ordered score among the entries of first-pass bin d
// (the bin is not empty).  One barrier; `red` is reused by the next phase
// only after its own barrier.
template <int NW = 4>
__device__ inline void rb_bin_range(const RegBuf& b, int n, float fmn, float scale, uint32_t d, uint32_t& lo,
                                    uint32_t& hi, uint32_t* red, int etid, int bar_id) {
  const int lane = etid & 31, wq = etid >> 5;
  const int room = rb_room(n, etid);
  uint32_t mx = 0u, mn = 0xFFFFFFFFu;
#pragma unroll
  for (int r = 0; r < kRegEntries; ++r) {
    const uint32_t k = b.key[r];
    const bool in = (32 * r < room) & (score_bin<NW>(k, fmn, scale) == d);
    mx = max(mx, in ? k : 0u);
    mn = min(mn, in ? k : 0xFFFFFFFFu);
  }
  mx = warp_max_u32(mx);
  mn = warp_min_u32(mn);
  if (lane == 0) {
    red[16 + wq] = mx;
    red[20 + wq] = mn;
  }
  named_bar(bar_id, NW * 32);
  hi = red[16];
  lo = red[20];
#pragma unroll
  for (int w2 = 1; w2 < NW; ++w2) {
    hi = max(hi, red[16 + w2]);
    lo = min(lo, red[20 + w2]);
  }
}

// Radix select of the ksel-th largest (ordered score, then lowest index).
// The first pass puts the scores into 1,024 bins linear in their value (a
// pass on the bits of the ordered score would put most of a score
// distribution into the few bins of one or two binary exponents); later
// passes of up to 10 bits walk down the ordered scores of the bin holding
// the ksel-th entry.  With `approx`, stops after the first pass if keeping
// everything from that bin up keeps at most `room` entries: a safe lower
// bound for a running threshold.  Once the bin holding the ksel-th entry has
// at most kSmallSel entries, they are sorted in one warp (rb_small_select)
// instead of further passes.
template <int NW = 4>
__device__ inline RegCut rb_cut(const RegBuf& b, int n, uint32_t ksel, bool approx, int room, uint32_t* hist,
                         uint32_t* red, int etid, int bar_id) {
  constexpr int kBins = team_bins<NW>();
  constexpr int kBits = team_digit_bits<NW>();
  uint32_t mx, mn;
  // the passes keep the histogram zero between them; the barrier of the
  // max / min below orders this clearing (and of the gather counter) before
  // the first pass
  for (int i = etid; i < kBins; i += NW * 32) hist[i] = 0u;
  if (etid == 0) red[12] = 0u;
  rb_maxmin<NW>(b, n, false, false, 0u, mx, mn, red, etid, bar_id);
  uint32_t base = mn, above = 0u, cnt = static_cast<uint32_t>(n), rank = ksel;
  if (mx != mn) {
    const float fmn = key_to_float(mn);
    float scale = static_cast<float>(kBins) / (key_to_float(mx) - fmn);
    if (!(scale < 1.0e30f)) scale = 0.f;  // a span too narrow for float bins: one bin, passes below
    const Digit d0 = rb_fpass<NW>(b, n, fmn, scale, rank, hist, red, etid, bar_id);
    above += d0.above;
    rank -= d0.above;
    cnt = d0.cnt;
    uint32_t lo, hi;
    rb_bin_range<NW>(b, n, fmn, scale, d0.d, lo, hi, red, etid, bar_id);
    // every entry of a higher bin scores above hi, every entry of a lower
    // one below lo: [lo, hi] holds exactly the bin's entries
    if (approx && static_cast<int>(above + cnt) <= room) return {lo, 0u, true, static_cast<int>(above + cnt)};
    if (cnt <= static_cast<uint32_t>(kSmallSel))
      return rb_small_select<NW>(b, n, lo, static_cast<unsigned long long>(hi - lo) + 1ull, rank, ksel, hist, red,
                                 etid, bar_id);
    base = lo;
    if (hi != lo) {
      int shift = 32 - __clz(hi - lo);  // bits of the bin's span of ordered scores
      while (shift > 0) {
        const int width = shift < kBits ? shift : kBits;
        shift -= width;
        const Digit dg = rb_pass<NW>(b, n, false, false, 0u, base, shift, width, rank, hist, red, etid, bar_id, hi);
        base += dg.d << shift;
        above += dg.above;
        rank -= dg.above;
        cnt = dg.cnt;
        if (cnt <= static_cast<uint32_t>(kSmallSel)) {
          const unsigned long long digit_span = 1ull << shift;
          const unsigned long long to_hi = static_cast<unsigned long long>(hi - base) + 1ull;
          return rb_small_select<NW>(b, n, base, digit_span < to_hi ? digit_span : to_hi, rank, ksel, hist, red,
                                     etid, bar_id);
        }
      }
    }
  }
  // base is now v, the ksel-th largest ordered score; `rank` of the `cnt`
  // entries tied at v make the cut
  if (rank >= cnt) return {base, 0xFFFFFFFFu, false, static_cast<int>(above + cnt)};
  if (cnt <= static_cast<uint32_t>(kSmallSel))
    return rb_small_select<NW>(b, n, base, 1ull, rank, ksel, hist, red, etid, bar_id);
  // many ties at v: the rank-th largest ~index among them, by the same passes
  const uint32_t v = base;
  uint32_t imx, imn;
  rb_maxmin<NW>(b, n, true, true, v, imx, imn, red, etid, bar_id);
  uint32_t ibase = imn;
  if (imx != imn) {
    int shift = 32 - __clz(imx - imn);
    while (shift > 0) {
      const int width = shift < kBits ? shift : kBits;
      shift -= width;
      const Digit dg = rb_pass<NW>(b, n, true, true, v, ibase, shift, width, rank, hist, red, etid, bar_id);
      ibase += dg.d << shift;
      rank -= dg.above;
    }
  }
  return {v, ~ibase, false, static_cast<int>(ksel)};
}

// Order-preserving compaction of the register buffer; returns the number
// kept.  Each warp counts its kept entries (one ballot per register step),
// the counts are exchanged once, and a second ballot pass gives every kept
// entry its position pos (counting kept entries in buffer, i.e. key, order).
// The kept entries of one warp step land on consecutive positions
// [first, first + count), so writes are coalesced.  step(keep, pos, key,
// idx, first, count) is called by every lane of the warp for every register
// step (keep: this lane's entry is kept), so it may use warp-collective
// operations.  All reads are from registers: writing back into the same
// buffer is safe.
template <class Step>
__device__ int rb_compact_steps(const RegBuf& b, int n, const RegCut& c, bool keep_all, int32_t* red_i, int etid,
                                int bar_id, Step step) {
  const int lane = etid & 31, wq = etid >> 5;
  const uint32_t lt = (1u << lane) - 1u;
  const int room = rb_room(n, etid);
  // keep: key > v, or key == v and index <= icut (a `ge` cut keeps every
  // index at v), as one branch-free predicate
  const uint32_t icut = (keep_all || c.ge) ? 0xFFFFFFFFu : c.icut;
  const uint32_t v = keep_all ? 0u : c.v;
  auto keep_of = [&](int r) -> bool {
    const uint32_t k = b.key[r];
    return (32 * r < room) & ((k > v) | ((k == v) & (b.idx[r] <= icut)));
  };
  int mine = 0;  // kept entries of this warp
#pragma unroll
  for (int r = 0; r < kRegEntries; ++r) mine += __popc(__ballot_sync(kFullMask, keep_of(r)));
  if (lane == 0) red_i[wq] = mine;
  named_bar(bar_id, kBM);
  int pos = 0, total = 0;
#pragma unroll
  for (int w2 = 0; w2 < 4; ++w2) {
    const int t = red_i[w2];
    total += t;
    pos += (w2 < wq) ? t : 0;
  }
#pragma unroll
  for (int r = 0; r < kRegEntries; ++r) {
    const bool k = keep_of(r);
    const uint32_t bal = __ballot_sync(kFullMask, k);
    if (bal != 0u) step(k, pos + __popc(bal & lt), b.key[r], b.idx[r], pos, __popc(bal));
    pos += __popc(bal);
  }
  named_bar(bar_id, kBM);
  return total;
}

// rb_compact_steps with emit(pos, key, idx) called for each kept entry.
template <class Emit>
__device__ int rb_compact(const RegBuf& b, int n, const RegCut& c, bool keep_all, int32_t* red_i, int etid,
                          int bar_id, Emit emit) {
  return rb_compact_steps(b, n, c, keep_all, red_i, etid, bar_id,
                          [&](bool keep, int pos, uint32_t k, uint32_t ix, int, int) {
                            if (keep) emit(pos, k, ix);
                          });
}

// One compaction step's kept pools, each expanded to its m token positions
// ("Module 06 — DSA & KPool", §2), written with consecutive lanes on
// consecutive output slots: the step's pools go to slots [first * m,
// (first + count) * m).  Called by every lane of the warp; `stage` is 64
// words of this warp's shared-memory scratch.  srow (optional) gets each
// pool's score for each of its tokens.  minv = ceil(2^32 / m): j / m is
// umulhi(j, minv) for every j < count * m (j * m < 2^32).
__device__ __forceinline__ void emit_expanded(bool keep, int pos, uint32_t key, uint32_t ix, int first, int count,
                                              int m, uint32_t minv, int32_t* orow, float* srow, uint32_t* stage,
                                              int lane) {
  if (keep) {
    stage[pos - first] = ix;
    stage[32 + pos - first] = key;
  }
  __syncwarp();
  for (int j = lane; j < count * m; j += 32) {
    const int e = static_cast<int>(__umulhi(static_cast<uint32_t>(j), minv));
    __stcs(&orow[first * m + j], static_cast<int32_t>(stage[e]) * m + (j - e * m));
    if (srow) srow[first * m + j] = key_to_float(stage[32 + e]);
  }
  __syncwarp();
}

// The output row of query t, written by one warp from the query's candidate
// buffer (entries in key order) and the cut its group computed (`job`): the
// kept keys in key order ("Adjacent-Query KV-Index Overlap in 256K DSA
// Training", §3), each pool expanded to its token positions and the
// incomplete pool's positions appended ("Module 06 — DSA & KPool", §2), then
// -1 padding and the valid length.  Entries are read two warp-steps at a time
// so that two loads are in flight.  `stage` is 64 words of this warp's
// shared memory.  g is the row's visibility position, n_keys its keys, and
// `shift` is added to every key index (a document's first key row in a
// segmented launch, else 0; pooled rows always have 0).
__device__ inline void warp_write_row(const uint2* buf, uint4 job, const ScoreParams& p, int64_t t, int64_t g,
                                      int32_t n_keys, int32_t shift, uint32_t* stage, int lane) {
  const int n = static_cast<int>(job.x);
  const bool all = job.w == kJobAll;
  const uint32_t v = all ? 0u : job.y;
  const uint32_t icut = all ? 0xFFFFFFFFu : job.z;
  const int m = p.out_ratio;
  int32_t* orow = p.out_idx + t * p.width;
  float* srow = p.out_score ? p.out_score + t * p.width : nullptr;
  const uint32_t lt = (1u << lane) - 1u;
  int kept = 0;
  for (int i0 = 0; i0 < n; i0 += 2 * 32) {
    uint2 e[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int i = i0 + u * 32 + lane;
      e[u] = i < n ? buf[i] : make_uint2(0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int i = i0 + u * 32 + lane;
      const bool keep = (i < n) & ((e[u].x > v) | ((e[u].x == v) & (e[u].y <= icut)));
      const uint32_t bal = __ballot_sync(kFullMask, keep);
      const int pos = kept + __popc(bal & lt);
      if (m == 1) {
        if (keep) {
          __stcs(&orow[pos], static_cast<int32_t>(e[u].y) + shift);
          if (srow) srow[pos] = key_to_float(e[u].x);
        }
      } else if (bal != 0u) {
        emit_expanded(keep, pos, e[u].x, e[u].y, kept, __popc(bal), m, p.out_ratio_inv, orow, srow, stage, lane);
      }
      kept += __popc(bal);
    }
  }
  int len = kept * m;
  if (m > 1) {
    const int tail = static_cast<int>((g + 1) % m);
    const int64_t first = g + 1 - tail;
    for (int i = lane; i < tail; i += 32) {
      __stcs(&orow[len + i], static_cast<int32_t>(first + i));
      if (srow) srow[len + i] = __uint_as_float(0x7FC00000u);
    }
    len += tail;
  }
  for (int i = len + lane; i < p.width; i += 32) {
    __stcs(&orow[i], -1);
    if (srow) srow[i] = __uint_as_float(0x7FC00000u);
  }
  if (lane == 0) {
    p.out_len[t] = len;
    // with a seed threshold at least min(K, visible) keys must pass it
    if (p.seed_thr != nullptr && kept < min(p.ksel, n_visible_in(p, g, n_keys))) atomicOr(p.status, kStatusWitness);
  }
}

// ------------------------------------------------------------------------
// The kernel.
// ------------------------------------------------------------------------
template <int H, int D, bool FP8, bool PRUNE, bool SPLIT, bool SEG = false>
__global__ void __launch_bounds__(kThreads, 1)
    score_topk_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const ScoreParams p) {
  using C = Cfg<H, D, FP8>;
  constexpr int NQW = C::NQW;
  constexpr int BN = C::BN;
  constexpr int QB = C::QB;
  constexpr int STAGES = C::STAGES;
  // the pruning screen needs registers of its own: keep 48 columns' weights in
  // shared memory there
  constexpr int kWsm = (PRUNE && C::WREG) ? 48 : C::WSM_COLS;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint32_t* hist_base = reinterpret_cast<uint32_t*>(smem + C::OFF_HIST);
  float* wsm_base = reinterpret_cast<float*>(smem + C::OFF_W);
  WgState<NQW>* states = reinterpret_cast<WgState<NQW>*>(smem + C::OFF_ST);
  Barriers<STAGES>* bars = reinterpret_cast<Barriers<STAGES>*>(smem + C::OFF_BAR);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&bars->kfull[s], 1);
      mbar_init(&bars->kempty[s], 1);
    }
    mbar_init(&bars->qfull, 1);
    mbar_init(&bars->qempty, 1);
    for (int a = 0; a < 4; ++a) {
      mbar_init(&bars->accfull[a], 1);
      mbar_init(&bars->accempty[a], 16);  // one arrival per epilogue warp
    }
    mbar_init(&bars->mma_done, 1);
    mbar_init(&bars->never, 1);
    for (int f = 0; f < kSets; ++f) {
      mbar_init(&bars->fin_full[f], kEpiGroups);  // one arrival per epilogue group
      mbar_init(&bars->fin_free[f], 2);           // one per writer warp
    }
    bars->abort = 0;
    bars->tmem_busy = 0;
    bars->cut_round = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = bars->tmem_slot;
  volatile int* abort_flag = &bars->abort;

  // The two register classes never rejoin: each branch ends in the same named
  // barrier (id 15, all threads), after which warp 1 frees TMEM.
  constexpr int kExitBar = 15;
  if (warp < 4) {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsControl));
  uint32_t n_kloads_done = 0, n_qloads_done = 0;  // loads the producer issued
  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_k);
      // q rows are read once; key tiles are read by every CTA: keep the keys
      // (and the candidate buffers) in L2 ahead of the q stream
      const uint64_t pol_q = l2_policy_evict_first();
      const uint64_t pol_k = l2_policy_evict_last();
      int stage = 0;
      uint32_t kph = 0, qe_ph = 0;
      bool first = true, ok = true;
      // loads issued so far: key tiles (stage of each follows from the count)
      // and q blocks; after an abort the last ones may still be landing
      uint32_t n_kloads = 0, n_qloads = 0;
      for (int r = 0; ok; ++r) {
        const Item it = item_of<QB, SPLIT, SEG>(p, r, blockIdx.x, gridDim.x);
        const int b = it.b;
        if (b < 0) break;
        if (it.j1 == it.j0) continue;
        if (!first) {
          ok = mbar_wait(&bars->qempty, qe_ph, abort_flag, kWaitLimitNs);
          qe_ph ^= 1;
          if (!ok) break;
        }
        first = false;
        ++n_qloads;
        // the block's q rows (a segmented launch: rows of one document, the
        // box's rows past them are scored and never used) and its keys
        const BlockGeom bg = geom_of<QB, SEG>(p, b);
        const int32_t q_row = static_cast<int32_t>(bg.row0 * H);
        const int32_t k_row0 = static_cast<int32_t>(bg.key0);
        mbar_arrive_expect_tx(&bars->qfull, C::Q_BYTES);
#pragma unroll
        for (int bx = 0; bx < C::NBOX; ++bx)
          tma_load_2d_hint(smem + C::OFF_Q + bx * BN * 128, &tm_q, bx * C::BOX_ELEMS, q_row, &bars->qfull, pol_q);
        for (int j = it.j0; j < it.j1; ++j) {
          ok = mbar_wait(&bars->kempty[stage], kph ^ 1u, abort_flag, kWaitLimitNs);
          if (!ok) break;
          ++n_kloads;
          mbar_arrive_expect_tx(&bars->kfull[stage], C::K_STAGE_BYTES);
#pragma unroll
          for (int bx = 0; bx < C::NBOX; ++bx)
            tma_load_2d_hint(smem + C::OFF_K + stage * C::K_STAGE_BYTES + bx * kBM * 128, &tm_k, bx * C::BOX_ELEMS,
                             k_row0 + j * kBM, &bars->kfull[stage], pol_k);
          if (++stage == STAGES) {
            stage = 0;
            kph ^= 1u;
          }
        }
      }
      if (!ok) {
        atomicOr(p.status, kStatusWaitTimeout);
        bars->abort = 1;
      }
      n_kloads_done = n_kloads;
      n_qloads_done = n_qloads;
    }
  } else if (warp == 1) {
    // -------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t q_base = smem_u32(smem + C::OFF_Q);
      const uint32_t k_base = smem_u32(smem + C::OFF_K);
      int stage = 0;
      uint32_t kph = 0, qf_ph = 0;
      uint32_t ae_ph[4] = {0u, 0u, 0u, 0u};
      uint32_t tcount = 0;  // tiles issued so far; tile n goes to accumulator n % NACC
      bool ok = true;
      for (int r = 0; ok; ++r) {
        const Item it = item_of<QB, SPLIT, SEG>(p, r, blockIdx.x, gridDim.x);
        if (it.b < 0) break;
        const int nt = it.j1 - it.j0;
        if (nt == 0) continue;
        ok = mbar_wait(&bars->qfull, qf_ph, abort_flag, kWaitLimitNs);
        qf_ph ^= 1u;
        if (!ok) break;
        for (int j = 0; j < nt && ok; ++j) {
          ok = mbar_wait(&bars->kfull[stage], kph, abort_flag, kWaitLimitNs);
          if (!ok) break;
          tc_fence_after();
          const uint32_t kst = k_base + stage * C::K_STAGE_BYTES;
          const int a = static_cast<int>(tcount % C::NACC);
          ok = mbar_wait(&bars->accempty[a], ae_ph[a] ^ 1u, abort_flag, kWaitLimitNs);
          ae_ph[a] ^= 1u;
          if (!ok) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < C::KSTEPS; ++kk) {
            const uint64_t adesc = sw128_desc(kst + (kk >> 2) * (kBM * 128) + (kk & 3) * 32);
            const uint64_t bdesc = sw128_desc(q_base + (kk >> 2) * (BN * 128) + (kk & 3) * 32);
            if constexpr (FP8)
              tc_mma_e4m3(tmem_base + a * BN, adesc, bdesc, C::IDESC, kk > 0 ? 1u : 0u);
            else
              tc_mma_bf16(tmem_base + a * BN, adesc, bdesc, C::IDESC, kk > 0 ? 1u : 0u);
          }
          tc_commit(&bars->accfull[a]);
          tc_commit(&bars->kempty[stage]);
          if (p.test_wait_ns > 0 && tcount == 0) {
            // test hook: a wait that runs out with an MMA in flight, so that
            // the whole timeout path below runs
            ok = mbar_wait(&bars->never, 0u, abort_flag, static_cast<uint64_t>(p.test_wait_ns));
          }
          ++tcount;
          if (++stage == STAGES) {
            stage = 0;
            kph ^= 1u;
          }
          if (!ok) break;
        }
        if (!ok) break;
        tc_commit(&bars->qempty);
      }
      if (!ok) {
        atomicOr(p.status, kStatusWaitTimeout);
        bars->abort = 1;
      }
      // every MMA issued by this thread has completed before TMEM is freed:
      // this wait ignores the abort flag (an MMA in flight always completes)
      // and only a time limit ends it; if that ever runs out, TMEM stays
      // allocated rather than being freed under a running MMA
      tc_commit(&bars->mma_done);
      if (!mbar_wait(&bars->mma_done, 0u, nullptr, kWaitLimitNs)) {
        atomicOr(p.status, kStatusWaitTimeout);
        bars->tmem_busy = 1;
      }
    }
  } else if constexpr (!SPLIT && !FP8) {
    // ---------------------------------------------------- output-row writers
    // Warps 2 and 3 write the output rows of each finished query block while
    // the epilogue groups go on with the next block: a group hands over its
    // queries' candidate buffers (one of kSets sets) with their final cuts.
    const int ww = warp - 2;
    for (int r = 0;; ++r) {
      const Item it = item_of<QB, SPLIT, SEG>(p, r, blockIdx.x, gridDim.x);
      if (it.b < 0) break;
      const BlockGeom bg = geom_of<QB, SEG>(p, it.b);
      const int set = r % kSets;
      bool ok = mbar_wait(&bars->fin_full[set], static_cast<uint32_t>(r / kSets) & 1u, abort_flag, kWaitLimitNs);
      if (!__any_sync(kFullMask, ok)) {
        if (lane == 0) {
          atomicOr(p.status, kStatusWaitTimeout);
          bars->abort = 1;
        }
        break;
      }
      for (int jb = ww; jb < kEpiGroups * NQW; jb += 2) {
        const int g = jb / NQW, qi = jb - g * NQW;
        const uint4 job = bars->jobs[set][g][qi];
        if (job.w == kJobSkip) continue;
        const int local = g * NQW + qi;  // row within the block
        const uint2* buf = p.cand + ((static_cast<size_t>(blockIdx.x) * kSets + set) * kEpiGroups + g) * NQW *
                                        static_cast<size_t>(p.cap) +
                           qi * static_cast<size_t>(p.cap);
        warp_write_row(buf, job, p, bg.row0 + local, bg.pos0 + local, bg.n_keys, static_cast<int32_t>(bg.key0),
                       bars->fstage[ww], lane);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->fin_free[set]);
    }
  }
  __syncwarp();  // lane 0 of warps 0 and 1 rejoins its warp before the aligned barrier
  tc_fence_before();
  named_bar(kExitBar, kThreads);
  tc_fence_after();
  if (warp == 1 && !*reinterpret_cast<volatile int*>(&bars->tmem_busy)) tmem_dealloc(tmem_base, C::TMEM_COLS);
  if (warp == 0 && lane == 0 && *abort_flag) {
    // After an abort the consumers may have left loads unconsumed: wait (time
    // limit only) until every load that can still be in flight has landed, so
    // that none writes into shared memory after the CTA has exited.  Key load
    // L went to stage L % STAGES in phase L / STAGES; only the last STAGES can
    // be pending, and no later phase of their stages was started.
    const uint32_t first_pending = n_kloads_done > STAGES ? n_kloads_done - STAGES : 0u;
    for (uint32_t L = first_pending; L < n_kloads_done; ++L)
      mbar_wait(&bars->kfull[L % STAGES], (L / STAGES) & 1u, nullptr, kWaitLimitNs);
    if (n_qloads_done > 0) mbar_wait(&bars->qfull, (n_qloads_done - 1) & 1u, nullptr, kWaitLimitNs);
  }
  } else {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsEpilogue));
  {
    // ------------------------------------------------------ epilogue warpgroups
    const int eg = (warp - 4) >> 2;    // epilogue group 0..3
    const int wq = warp & 3;           // TMEM lane quarter accessible to this warp
    const int etid = wq * 32 + lane;   // key row within the tile == order within the group
    const int bar_id = 1 + eg;
    WgState<NQW>* st = states + eg;
    float* wsm = wsm_base + eg * C::CW;
    uint32_t* hist = hist_base + eg * kHistBins;
    // the group's columns eg*CW .. eg*CW+CW-1 of either accumulator hold its
    // NQW queries (all H heads of each)
    const uint32_t tbase = tmem_base + (static_cast<uint32_t>(wq * 32) << 16) + static_cast<uint32_t>(eg * C::CW);
    uint32_t af_bits = 0u;  // phase parity of accumulator a's full barrier in bit a
    // Cut rounds.  While one group cuts a buffer, the other groups soon stall
    // (every group drains every tile), so a group whose buffer fills raises
    // the CTA's round counter and the others, seeing it at their next tile,
    // cut their fuller buffers at the same time: the cuts overlap instead of
    // stalling the tensor core one after another.
    // (bf16 variants; the FP8 ones keep the plain per-group cuts, which
    // measured faster there)
    constexpr bool kRounds = !FP8;
    // The single-range bf16 kernels hand each finished block's output rows to
    // the writer warps (warps 2 and 3) and go on with the next block; the
    // split-range kernel writes its per-range lists itself, and the FP8 kernel
    // (long rows, few blocks, the most register-bound epilogue) its rows.
    constexpr bool kDefer = !SPLIT && !FP8;
    volatile int* cut_round = &bars->cut_round;
    volatile int* seen = &bars->seen[eg];
    uint32_t tcount = 0;    // tiles drained so far; tile n sits in accumulator n % NACC
    int par = 0;
    bool failed = false;
    unsigned long long n_screened = 0ull, n_bounded = 0ull, n_skipped = 0ull;  // pruning counters (lane 0)
    for (int r = 0; !failed; ++r) {
      const Item it = item_of<QB, SPLIT, SEG>(p, r, blockIdx.x, gridDim.x);
      const int b = it.b;
      if (b < 0) break;
      const int nt = it.j1;
      // the block's rows [row0, t_end), their visibility origin and keys
      const BlockGeom bg = geom_of<QB, SEG>(p, b);
      const int64_t tq0 = bg.row0 + eg * NQW;
      const int64_t t_end = SEG ? bg.row0 + bg.rows : p.S;
      const int64_t pos_shift = SEG ? bg.pos0 - bg.row0 : p.q_pos0;  // visibility position = t + pos_shift
      const int64_t kcap = SEG ? bg.n_keys : p.n_keys;
      const float* ksc = FP8 ? p.k_scale + (SEG ? bg.key0 : 0) : nullptr;
      const int32_t out_shift = SEG ? static_cast<int32_t>(bg.key0) : 0;
      const int set = r % kSets;  // candidate-buffer set of this block
      uint2* cand = p.cand + ((static_cast<size_t>(blockIdx.x) * kSets + set) * kEpiGroups + eg) * NQW *
                                 static_cast<size_t>(p.cap);
      bool free_ok = true;
      if (kDefer && r >= kSets) {
        // the writer warps are done with this set's buffers (block r - kSets)
        free_ok = mbar_wait(&bars->fin_free[set], static_cast<uint32_t>(r / kSets - 1) & 1u, abort_flag,
                            kWaitLimitNs);
        free_ok = __any_sync(kFullMask, free_ok);
      }
      // the previous block is completely done with the state
      if (named_bar_or(bar_id, kBM, !free_ok)) {
        failed = true;
        break;
      }
      for (int i = etid; i < C::CW; i += kBM) {
        const int64_t t = tq0 + i / H;
        float v = 0.f;
        if (t < t_end) {
          v = p.w[t * H + (i % H)];
          if constexpr (FP8) v *= p.q_scale[t * H + (i % H)];
        }
        wsm[i] = 0.5f * v;  // halved: the ReLU is computed doubled (relu2)
      }
      if constexpr (PRUNE) {
        for (int i = etid; i < NQW * (kPruneR + 2); i += kBM) {
          const int qi = i / (kPruneR + 2), c = i % (kPruneR + 2);
          const int64_t t = tq0 + qi;
          const float v = t < t_end ? p.pq[t * (kPruneR + 2) + c] : 0.f;
          st->pq[qi][c] = c < kPruneR ? 0.5f * v : v;  // kept-head weights halved, as for relu2
        }
      }
      if (kRounds && etid == 0) *seen = *cut_round;
      if (etid < NQW) {
        const int64_t t = tq0 + etid;
        st->nvis[etid] = t < t_end ? n_visible_in(p, t + pos_shift, static_cast<int32_t>(kcap)) : 0;
        st->cnt[par][etid] = 0;
        // a seed threshold, when given, is a lower bound of the K-th score
        st->thr[etid] = (p.seed_thr != nullptr && t < t_end) ? p.seed_thr[t] : 0u;
      }
      named_bar(bar_id, kBM);

      // Tiles run in a tight loop that leaves when a candidate buffer is about
      // to overflow or the block's tiles are done; the selection steps (cut of
      // the full buffers, or the final top-K of every query) follow it, so the
      // per-tile path carries none of their code.
      int j = it.j0;
      while (true) {
        // the group's head weights, in registers for the whole tile loop when
        // they fit (reloaded after a cut, which needs the registers)
        float wr[C::CW > kWsm ? C::CW - kWsm : 4];
        if constexpr (C::CW > kWsm) {
#pragma unroll
          for (int i = 0; i < C::CW - kWsm; i += 4) {
            const float4 v = *reinterpret_cast<const float4*>(wsm + kWsm + i);
            wr[i] = v.x;
            wr[i + 1] = v.y;
            wr[i + 2] = v.z;
            wr[i + 3] = v.w;
          }
        }
        auto wget = [&](int col) -> float2 {
          if constexpr (kWsm < C::CW) {
            if (col >= kWsm) return make_float2(wr[col - kWsm], wr[col - kWsm + 1]);
          }
          return *reinterpret_cast<const float2*>(wsm + col);
        };
        // per-query state that only the selection steps change, in registers
        // for the tile loop: candidates held, threshold, visible keys
        int held[NQW];
        uint32_t thr_r[NQW];
        int32_t nvis_r[NQW];
#pragma unroll
        for (int qi = 0; qi < NQW; ++qi) {
          held[qi] = st->cnt[par][qi];
          thr_r[qi] = st->thr[qi];
          nvis_r[qi] = st->nvis[qi];
        }
        bool any_full = false, join = false;
        // per-key values of the next tile (FP8 key scale, pruning key norm),
        // loaded one tile ahead so that their latency hides behind the wait
        // for the accumulator and the head sums
        float ks_next = 1.f, kn_next = 0.f;
        {
          const int32_t key = j * kBM + etid;
          if constexpr (FP8) ks_next = (j < nt && key < kcap) ? ksc[key] : 0.f;
          if constexpr (PRUNE) kn_next = (j < nt && key < kcap) ? p.knorm[key] : 0.f;
        }
        for (; j < nt; ++j) {
          const int a = static_cast<int>(tcount % C::NACC);
          ++tcount;
          const int32_t key = j * kBM + etid;
          const float ks = ks_next, kn = kn_next;
          if (FP8 || PRUNE) {
            const int32_t key1 = key + kBM;
            const bool more = j + 1 < nt && key1 < kcap;
            if constexpr (FP8) ks_next = more ? ksc[key1] : 0.f;
            if constexpr (PRUNE) kn_next = more ? p.knorm[key1] : 0.f;
          }
          // every lane polls (no divergent branch around the wait); the phase
          // is complete for all once any lane has seen it complete
          bool ok = mbar_wait(&bars->accfull[a], (af_bits >> a) & 1u, abort_flag, kWaitLimitNs);
          ok = __any_sync(kFullMask, ok);
          af_bits ^= 1u << a;
          float s[NQW];
#pragma unroll
          for (int qi = 0; qi < NQW; ++qi) s[qi] = 0.f;
          if (ok) {
            tc_fence_after();
            const uint32_t tb = tbase + static_cast<uint32_t>(a * BN);
            float2 acc[NQW][C::CHAINS];
#pragma unroll
            for (int qi = 0; qi < NQW; ++qi)
#pragma unroll
              for (int c = 0; c < C::CHAINS; ++c) acc[qi][c] = make_float2(0.f, 0.f);
            if constexpr (PRUNE && H >= 2 * kPruneR) {  // the host rejects pruning for fewer heads
              // per query: bound from its first 16 heads; the rest of its
              // columns are read only if some key of the warp may pass
              bool skip[NQW];
#pragma unroll
              for (int qi = 0; qi < NQW; ++qi) {
                constexpr int CPQ = H / 16;  // chunks per query
                uint32_t ra[16];
                tmem_ld_x16(tb + qi * H, ra);
                tmem_wait_ld(ra);
                const float u = prune_bound<FP8>(ra, st->pq[qi], ks, kn);
                const bool vis = key < st->nvis[qi];
                const bool sk = !vis || ordered_key(u) < st->thr[qi];
                const uint32_t vb = __ballot_sync(kFullMask, vis);
                const uint32_t bb = __ballot_sync(kFullMask, vis && sk);
                skip[qi] = __all_sync(kFullMask, sk);
                if (lane == 0) {
                  n_screened += static_cast<unsigned long long>(__popc(vb));
                  n_bounded += static_cast<unsigned long long>(__popc(bb));
                  if (skip[qi]) n_skipped += static_cast<unsigned long long>(__popc(vb));
                }
                if (skip[qi]) continue;
                chunk_fma<H, NQW, C::CHAINS>(ra, qi * H, wget, acc);
#pragma unroll
                for (int c = 1; c < CPQ; ++c) {
                  tmem_ld_x16(tb + qi * H + c * 16, ra);
                  tmem_wait_ld(ra);
                  chunk_fma<H, NQW, C::CHAINS>(ra, qi * H + c * 16, wget, acc);
                }
              }
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(&bars->accempty[a]);
#pragma unroll
              for (int qi = 0; qi < NQW; ++qi) s[qi] = skip[qi] ? -3.0e38f : chain_total<C::CHAINS>(acc[qi]);
            } else {
              // two chunk buffers: chunk c + 1 is on its way from TMEM while
              // chunk c is summed
              uint32_t ra[2][16];
              tmem_ld_x16(tb, ra[0]);
              tmem_wait_ld(ra[0]);
#pragma unroll
              for (int c = 0; c < C::NCH; ++c) {
                if (c + 1 < C::NCH) tmem_ld_x16(tb + (c + 1) * 16, ra[(c + 1) & 1]);
                chunk_fma<H, NQW, C::CHAINS>(ra[c & 1], c * 16, wget, acc);
                if (c + 1 < C::NCH) {
                  tmem_wait_ld(ra[(c + 1) & 1]);
                  if (c + 2 == C::NCH) {
                    // everything this warp needs from TMEM is in registers:
                    // hand the accumulator back before the last chunk's sums
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&bars->accempty[a]);
                  }
                }
              }
#pragma unroll
              for (int qi = 0; qi < NQW; ++qi) s[qi] = chain_total<C::CHAINS>(acc[qi]);
            }
          }
          if constexpr (FP8) {
#pragma unroll
            for (int qi = 0; qi < NQW; ++qi) s[qi] *= ks;
          }
          // pass flags and per-warp counts
          uint32_t okeys[NQW], bals[NQW];
#pragma unroll
          for (int qi = 0; qi < NQW; ++qi) {
            okeys[qi] = ordered_key(__fadd_rn(s[qi], 0.f));
            const bool pass = ok && key < nvis_r[qi] && okeys[qi] >= thr_r[qi];
            bals[qi] = __ballot_sync(kFullMask, pass);
            if (lane == 0) reinterpret_cast<int32_t*>(&st->wc[par][qi])[wq] = __popc(bals[qi]);
          }
          // one barrier for two votes: a failed wait (every thread of the
          // failing warp but etid 1, so at least 31) and a new cut round
          // (etid 1 alone)
          if constexpr (kRounds) {
            const bool vote = etid == 1 ? (*cut_round != *seen) : !ok;
            const uint32_t votes = named_bar_popc(bar_id, kBM, vote);
            if (votes > 1u) {
              failed = true;
              break;
            }
            join = votes == 1u;
          } else {
            if (named_bar_or(bar_id, kBM, !ok)) {
              failed = true;
              break;
            }
          }
          // ordered append: position = held + earlier warps + earlier lanes.  No
          // barrier follows: every thread knows the new counts, and the per-warp
          // counts read here are double-buffered by tile parity.
          const uint32_t lt_mask = (1u << lane) - 1u;
#pragma unroll
          for (int qi = 0; qi < NQW; ++qi) {
            const uint32_t bal = bals[qi];
            const int4 wc = st->wc[par][qi];
            const int tot = wc.x + wc.y + wc.z + wc.w;
            const int prior = (wq > 0 ? wc.x : 0) + (wq > 1 ? wc.y : 0) + (wq > 2 ? wc.z : 0);
            if ((bal >> lane) & 1u) {
              const int pos = held[qi] + prior + __popc(bal & lt_mask);
              cand[qi * static_cast<size_t>(p.cap) + pos] = make_uint2(okeys[qi], static_cast<uint32_t>(key));
            }
            held[qi] += tot;
          }
          par ^= 1;
#pragma unroll
          for (int qi = 0; qi < NQW; ++qi) any_full |= held[qi] > p.cap - kBM;
          if (any_full || join) {
            ++j;
            break;
          }
        }
        if (failed) break;
#pragma unroll
        for (int qi = 0; qi < NQW; ++qi)
          if (etid == qi) st->cnt[par][qi] = held[qi];
        // a cut round: this group's own buffer is full, or another group's
        // round is joined; otherwise the block's tiles are done and the final
        // top-K of each query is written
        const bool fin = !(any_full || join);
        if (kRounds && !fin && etid == 0) {
          if (any_full) atomicAdd(const_cast<int*>(cut_round), 1);
          *seen = *cut_round;
        }
        named_bar(bar_id, kBM);  // every append and count of the last tile is visible to the group
        // buffers fuller than this are cut in a round: every full one (held >
        // cap - kBM >= cut_min) and those of the joining groups that are well
        // on their way
        const int cut_min = kRounds ? (p.cap + p.ksel) / 2 : p.cap - kBM;
        // Two queries per group and both buffers within two warps' registers
        // (2,048 entries): warps 0-1 and 2-3 select for query 0 and query 1
        // at once, each on half of the group's histogram, instead of the
        // whole group selecting for one query after the other.
        bool halves_done = false;
        if constexpr (kDefer && NQW == 2) {
          const int n0 = st->cnt[par][0], n1 = st->cnt[par][1];
          if (fin && n0 <= kRegCap / 2 && n1 <= kRegCap / 2) {
            const int h = wq >> 1;
            const int qi = h;
            const int tid = etid - h * 64;
            const int n = h ? n1 : n0;
            const int64_t t = tq0 + qi;
            uint4 job = make_uint4(static_cast<uint32_t>(n), 0u, 0xFFFFFFFFu, t < t_end ? kJobAll : kJobSkip);
            if (t < t_end && n > p.ksel) {
              RegBuf rb;
              rb_load(rb, cand + qi * static_cast<size_t>(p.cap), n, tid);
              const RegCut c = rb_cut<2>(rb, n, static_cast<uint32_t>(p.ksel), false, 0, hist + h * (kHistBins / 2),
                                         h ? st->red2 : st->red, tid, 5 + 2 * eg + h);
              job = make_uint4(static_cast<uint32_t>(n), c.v, c.icut, kJobCut);
            }
            if (tid == 0) bars->jobs[set][eg][qi] = job;
            named_bar(bar_id, kBM);
            halves_done = true;
          }
        }
#pragma unroll 1
        for (int qi = 0; qi < (halves_done ? 0 : NQW); ++qi) {
          const int n = st->cnt[par][qi];
          const int64_t t = tq0 + qi;
          if (kDefer && fin && etid == 0 && t >= t_end) bars->jobs[set][eg][qi] = make_uint4(0u, 0u, 0u, kJobSkip);
          if (fin ? t >= t_end : n <= cut_min) continue;
          if (!fin) {
            uint2* buf = cand + qi * static_cast<size_t>(p.cap);
            int kept;
            uint32_t thr;
            if (n <= kRegCap) {
              RegBuf rb;
              rb_load(rb, buf, n, etid);
              const RegCut c = rb_cut(rb, n, static_cast<uint32_t>(p.ksel), true, p.cap - 2 * kBM, hist,
                                      st->red, etid, bar_id);
              kept = rb_compact(rb, n, c, false, st->scan, etid, bar_id,
                                [&](int pos, uint32_t k, uint32_t ix) { buf[pos] = make_uint2(k, ix); });
              thr = c.ge ? c.v : (c.v == 0xFFFFFFFFu ? c.v : c.v + 1u);
            } else {
              const Cut cut = wg_topk_cut(buf, n, static_cast<uint32_t>(p.ksel), hist, st->red, etid, bar_id);
              kept = wg_compact(buf, n, cut, false, &st->cwc[0][0], etid, bar_id,
                                [&](int pos, uint2 e) { buf[pos] = e; });
              thr = cut.v == 0xFFFFFFFFu ? cut.v : cut.v + 1u;
            }
            if (etid == 0) {
              st->cnt[par][qi] = kept;
              st->thr[qi] = thr;
            }
          } else if constexpr (kDefer) {
            // the cut only: the writer warps write the row
            uint2* buf = cand + qi * static_cast<size_t>(p.cap);
            uint4 job = make_uint4(static_cast<uint32_t>(n), 0u, 0xFFFFFFFFu, kJobAll);
            if (n > p.ksel) {
              if (n <= kRegCap) {
                RegBuf rb;
                rb_load(rb, buf, n, etid);
                const RegCut c = rb_cut(rb, n, static_cast<uint32_t>(p.ksel), false, 0, hist, st->red, etid, bar_id);
                job = make_uint4(static_cast<uint32_t>(n), c.v, c.icut, kJobCut);
              } else {
                const Cut c = wg_topk_cut(buf, n, static_cast<uint32_t>(p.ksel), hist, st->red, etid, bar_id);
                job = make_uint4(static_cast<uint32_t>(n), c.v, c.icut, kJobCut);
              }
            }
            if (etid == 0) bars->jobs[set][eg][qi] = job;
          } else {
            uint2* buf = cand + qi * static_cast<size_t>(p.cap);
            const bool all = n <= p.ksel;
            int32_t* orow = p.out_idx + t * p.width;
            float* srow = p.out_score ? p.out_score + t * p.width : nullptr;
            const int m = p.out_ratio;
            const uint32_t minv = p.out_ratio_inv;
            // with split key ranges this is one split's top-K, kept as
            // (ordered score, key) pairs in key order for the merge
            uint2* srow_split = nullptr;
            if constexpr (SPLIT) srow_split = p.split_buf + (static_cast<size_t>(t) * p.splits + it.sp) * p.ksel;
            auto emit = [&](int pos, uint32_t k, uint32_t ix) {
              if constexpr (SPLIT) {
                srow_split[pos] = make_uint2(k, ix);
                return;
              }
              const float sc = key_to_float(k);
              if (m == 1) {
                __stcs(&orow[pos], static_cast<int32_t>(ix) + out_shift);
                if (srow) srow[pos] = sc;
              } else {
                for (int rr = 0; rr < m; ++rr) {
                  __stcs(&orow[pos * m + rr], static_cast<int32_t>(ix) * m + rr);
                  if (srow) srow[pos * m + rr] = sc;
                }
              }
            };
            // the same, by warp steps: pooled entries expand with coalesced writes
            auto step = [&](bool keep, int pos, uint32_t k, uint32_t ix, int first, int count) {
              if (SPLIT || m == 1) {
                if (keep) emit(pos, k, ix);
              } else {
                emit_expanded(keep, pos, k, ix, first, count, m, minv, orow, srow, hist + (etid >> 5) * 64,
                              etid & 31);
              }
            };
            int kept;
            [[maybe_unused]] uint32_t kth = 0u;  // ordered score of the K-th entry kept (0: fewer than K)
            [[maybe_unused]] uint32_t rth = 0u;  // split ranges: ordered score of the r-th entry (0: fewer)
            if (n <= kRegCap) {
              RegBuf rb;
              rb_load(rb, buf, n, etid);
              RegCut c{0u, 0xFFFFFFFFu, false, n};
              if (!all) c = rb_cut(rb, n, static_cast<uint32_t>(p.ksel), false, 0, hist, st->red, etid, bar_id);
              // hist is scratch from here on (rb_cut clears it before use)
              kept = rb_compact_steps(rb, n, c, all, st->scan, etid, bar_id, step);
              if constexpr (SPLIT) {
                kth = all ? 0u : c.v;
                // the r-th largest score of the range, r = ceil(K / splits)
                const int r = (p.ksel + p.splits - 1) / p.splits;
                if (n >= r)
                  rth = rb_cut(rb, n, static_cast<uint32_t>(r), false, 0, hist, st->red, etid, bar_id).v;
              }
            } else {
              Cut cut{0u, 0xFFFFFFFFu};
              if (!all) cut = wg_topk_cut(buf, n, static_cast<uint32_t>(p.ksel), hist, st->red, etid, bar_id);
              if constexpr (SPLIT) {
                kth = all ? 0u : cut.v;
                const int r = (p.ksel + p.splits - 1) / p.splits;
                if (n >= r)
                  rth = wg_radix_select(buf, n, static_cast<uint32_t>(r), false, false, 0u,
                                        static_cast<uint32_t>(n), hist, st->red, etid, bar_id).v;
              }
              kept = wg_compact(buf, n, cut, all, &st->cwc[0][0], etid, bar_id,
                                [&](int pos, uint2 e) { emit(pos, e.x, e.y); });
            }
            if constexpr (SPLIT) {
              if (etid == 0) {
                p.split_cnt[t * p.splits + it.sp] = kept;
                p.split_kth[t * p.splits + it.sp] = kth;
                p.split_rth[t * p.splits + it.sp] = rth;
              }
              named_bar(bar_id, kBM);
              continue;
            }
            int len = kept * m;
            if (m > 1) {
              const int64_t g = t + pos_shift;
              const int tail = static_cast<int>((g + 1) % m);
              const int64_t first = g + 1 - tail;
              for (int i = etid; i < tail; i += kBM) {
                __stcs(&orow[len + i], static_cast<int32_t>(first + i));
                if (srow) srow[len + i] = __uint_as_float(0x7FC00000u);
              }
              len += tail;
            }
            for (int i = len + etid; i < p.width; i += kBM) {
              __stcs(&orow[i], -1);
              if (srow) srow[i] = __uint_as_float(0x7FC00000u);
            }
            if (etid == 0) {
              p.out_len[t] = len;
              // with a seed threshold at least min(K, visible) keys must pass it
              if (p.seed_thr != nullptr && kept < min(p.ksel, st->nvis[qi])) atomicOr(p.status, kStatusWitness);
            }
          }
          named_bar(bar_id, kBM);
        }
        if (fin) {
          // every cut of the block is posted (and the last tile's appends are
          // visible to the group): hand the block to the writer warps
          if (kDefer && etid == 0) mbar_arrive(&bars->fin_full[set]);
          break;
        }
      }
    }
    if (failed && etid == 0) {
      atomicOr(p.status, kStatusWaitTimeout);
      bars->abort = 1;
    }
    if (PRUNE && lane == 0) {
      atomicAdd(&p.counters[0], n_screened);
      atomicAdd(&p.counters[1], n_bounded);
      atomicAdd(&p.counters[2], n_skipped);
    }
  }
  tc_fence_before();
  named_bar(kExitBar, kThreads);
  }
}


// Launch facts of one compiled variant.
template <int H, int D, bool FP8, bool PRUNE>
void fill_variant(ScoreVariant* v) {
  using C = Cfg<H, D, FP8>;
  v->fn = reinterpret_cast<const void*>(&score_topk_kernel<H, D, FP8, PRUNE, false>);
  v->fn_split = reinterpret_cast<const void*>(&score_topk_kernel<H, D, FP8, PRUNE, true>);
  // the segmented instance serves packed documents without the pruning
  // certificate (whose key norms are numbered over a single problem's keys)
  if constexpr (!PRUNE)
    v->fn_seg = reinterpret_cast<const void*>(&score_topk_kernel<H, D, FP8, false, false, true>);
  else
    v->fn_seg = nullptr;
  v->queries_per_block = C::QB;
  v->queries_per_wg = C::NQW;
  v->groups = kEpiGroups;
  v->q_box_rows = C::BN;
  v->box_elems = C::BOX_ELEMS;
  v->smem_bytes = C::SMEM_BYTES;
  v->threads = kThreads;
}

}  // namespace hwr
