// aux_kernels.cu -- the small steps around the scoring kernel:
//   * pool formation for pooled indexing ("Module 06 — DSA & KPool:
//     Selective Retrieval", §2: a channel-wise weighted representation of each
//     complete pool of 4 tokens), and
//   * exact shared-index counts of adjacent query pairs ("Adjacent-Query
//     KV-Index Overlap in 256K DSA Training", §1 pairs (q0,q1),(q2,q3),...;
//     §3 exact intersections by batched binary search), and
//   * the shared / left-only / right-only index regions of those pairs (same
//     page, §6.1 and §6.4: q-cluster preprocessing into fixed-capacity
//     buffers with device-side counts).
#include <cuda_bf16.h>

#include "internal.h"
#include "ptx.cuh"

namespace hwr {

__device__ __forceinline__ double bf16_bits_to_double(uint16_t b) {
  return static_cast<double>(__uint_as_float(static_cast<uint32_t>(b) << 16));
}

// binary64 -> bfloat16 with round-to-nearest-even in one step.
__device__ __forceinline__ uint16_t cvt_rn_bf16_f64(double x) {
  uint16_t r;
  asm("cvt.rn.bf16.f64 %0, %1;" : "=h"(r) : "d"(x));
  return r;
}

// Exact summation and rounding of pool keys.  Each product of two bfloat16
// values is exact in binary64, so the sum of a pool's products is an exact
// rational that a binary64 running sum may round (for example 2^60 + 1 - 2^60
// - 1 or 259*2^52 - 2^-60).  When every addition is exact the running sum is
// rounded directly; otherwise the sum is kept as a nonoverlapping expansion
// (Shewchuk, "Adaptive Precision Floating-Point Arithmetic and Fast Robust
// Geometric Predicates", 1997: TwoSum and Grow-Expansion), whose sign is the
// sign of its largest nonzero component, and the bfloat16 rounding is decided
// by exact comparisons with the midpoints next to a near candidate.

constexpr int kMaxPoolRatio = 16;
constexpr int kExpMax = kMaxPoolRatio + 1;   // products, plus one midpoint

__device__ __forceinline__ void two_sum(double a, double b, double& s, double& err) {
  s = __dadd_rn(a, b);
  const double bb = __dsub_rn(s, a);
  err = __dadd_rn(__dsub_rn(a, __dsub_rn(s, bb)), __dsub_rn(b, bb));
}

// e[0, n) nonoverlapping, increasing magnitude (zeros allowed) -> the same
// for e + b, one component longer.
__device__ __forceinline__ void grow_expansion(double (&e)[kExpMax], int& n, double b) {
  double q = b;
#pragma unroll
  for (int i = 0; i < kExpMax; ++i) {
    if (i < n) {
      double h;
      two_sum(q, e[i], q, h);
      e[i] = h;
    }
  }
#pragma unroll
  for (int i = 0; i < kExpMax; ++i)
    if (i == n) e[i] = q;
  ++n;
}

// Sign (-1, 0, 1) of the exact value of a nonoverlapping expansion: the sign
// of its largest nonzero component, which is the last one.
__device__ __forceinline__ int expansion_sign(const double (&e)[kExpMax], int n) {
  int sg = 0;
#pragma unroll
  for (int i = 0; i < kExpMax; ++i)
    if (i < n && e[i] != 0.0) sg = e[i] > 0.0 ? 1 : -1;
  return sg;
}

// Sign of (value of e[0, n)) - m, exactly.
__device__ __forceinline__ int compare_expansion(const double (&e)[kExpMax], int n, double m) {
  double f[kExpMax];
#pragma unroll
  for (int i = 0; i < kExpMax; ++i) f[i] = e[i];
  int nf = n;
  grow_expansion(f, nf, -m);
  return expansion_sign(f, nf);
}

// Value of a non-negative bfloat16 pattern; the infinity pattern 0x7F80
// stands for 2^128, where round-to-nearest overflows.
__device__ __forceinline__ double bf16_pattern_value(uint32_t pat) {
  return pat >= 0x7F80u ? 0x1p128 : bf16_bits_to_double(static_cast<uint16_t>(pat));
}

// Round the exact value of e[0, n) (nonzero) to bfloat16, nearest-even.
__device__ uint16_t round_expansion_to_bf16(double (&e)[kExpMax], int n) {
  const int sg = expansion_sign(e, n);
  double approx = 0.0;  // within a few binary64 ulps of the magnitude
#pragma unroll
  for (int i = 0; i < kExpMax; ++i) {
    if (i < n) {
      if (sg < 0) e[i] = -e[i];
      approx = __dadd_rn(approx, e[i]);
    }
  }
  // the candidate is the exact answer or one of its neighbours
  uint32_t pat = cvt_rn_bf16_f64(approx) & 0x7FFFu;
  if (pat > 0x7F80u) pat = 0x7F80u;
  const double v = bf16_pattern_value(pat);
  if (pat < 0x7F80u) {
    const double up_mid = 0.5 * (v + bf16_pattern_value(pat + 1));
    const int c = compare_expansion(e, n, up_mid);
    if (c > 0 || (c == 0 && (pat & 1u))) return static_cast<uint16_t>((sg < 0 ? 0x8000u : 0u) | (pat + 1));
  }
  if (pat > 0) {
    const double lo_mid = 0.5 * (bf16_pattern_value(pat - 1) + v);
    const int c = compare_expansion(e, n, lo_mid);
    if (c < 0 || (c == 0 && (pat & 1u))) return static_cast<uint16_t>((sg < 0 ? 0x8000u : 0u) | (pat - 1));
  }
  return static_cast<uint16_t>((sg < 0 ? 0x8000u : 0u) | pat);
}

// kp[p, d] = RNE_bf16( sum_j c[j, d] * k[ratio*p + j, d] ), the sum exact.
// Inputs are finite; ratio <= kMaxPoolRatio.
__global__ void pool_keys_kernel(const uint16_t* __restrict__ k, const uint16_t* __restrict__ coef, int ratio,
                                 int64_t n_pools, int D, uint16_t* __restrict__ out) {
  const int64_t n = n_pools * D;
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < n;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t pool = e / D;
    const int d = static_cast<int>(e - pool * D);
    double sum = 0.0;
    bool exact = true;
    for (int j = 0; j < ratio; ++j) {
      const double prod = bf16_bits_to_double(coef[j * D + d]) * bf16_bits_to_double(k[(pool * ratio + j) * D + d]);
      if (j == 0) {
        sum = prod;
      } else {
        double err;
        two_sum(sum, prod, sum, err);
        exact = exact && err == 0.0;
      }
    }
    if (exact) {
      out[e] = cvt_rn_bf16_f64(sum);  // the running sum is the exact sum (signed zero included)
      continue;
    }
    double ex[kExpMax] = {};
    int m = 0;
    for (int j = 0; j < ratio; ++j)
      grow_expansion(ex, m, bf16_bits_to_double(coef[j * D + d]) * bf16_bits_to_double(k[(pool * ratio + j) * D + d]));
    out[e] = expansion_sign(ex, m) == 0 ? static_cast<uint16_t>(0) : round_expansion_to_bf16(ex, m);
  }
}

cudaError_t launch_pool_keys(const void* k, int64_t n_pools, int D, const void* coef, int ratio, void* out,
                             cudaStream_t stream) {
  const int64_t n = n_pools * D;
  if (n == 0) return cudaSuccess;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int threads = 256;
  int64_t blocks = (n + threads - 1) / threads;
  if (blocks > static_cast<int64_t>(sms) * 8) blocks = static_cast<int64_t>(sms) * 8;
  pool_keys_kernel<<<static_cast<unsigned>(blocks), threads, 0, stream>>>(
      static_cast<const uint16_t*>(k), static_cast<const uint16_t*>(coef), ratio, n_pools, D,
      static_cast<uint16_t*>(out));
  return cudaGetLastError();
}

// One warp per pair: each lane takes entries of A and binary-searches B.
// Rows up to this width are searched in shared memory (one row per warp at a
// time): a search step then costs a shared-memory access instead of an L2
// round trip.  2,304 covers budgets of 2,048 and the pooled 2,051 slots.
constexpr int kPairSmemRow = 2304;
constexpr int kPairWarps = 4;

// Copies row[0, n) to the warp's shared-memory slot and returns it, or returns
// the row itself when it is wider than the slot.
__device__ __forceinline__ const int32_t* stage_row(const int32_t* __restrict__ row, int n, int32_t* slot,
                                                    int lane) {
  if (n > kPairSmemRow) return row;
#pragma unroll 4
  for (int i = lane; i < n; i += 32) slot[i] = row[i];
  __syncwarp();
  return slot;
}

// Entries per lane and step in the pair kernels: four loads and four
// searches in flight hide the load latency.
constexpr int kPairILP = 4;

// hit[u] = the strictly ascending row b[0, lb) holds x[u].  The four searches
// advance together (binary lifting: pos counts the entries below x), so their
// shared-memory reads overlap.
__device__ __forceinline__ void rows_hold(const int32_t* __restrict__ b, int lb, const int32_t (&x)[kPairILP],
                                          bool (&hit)[kPairILP]) {
  int pos[kPairILP];
#pragma unroll
  for (int u = 0; u < kPairILP; ++u) pos[u] = 0;
  for (int step = lb > 0 ? (1 << (31 - __clz(lb))) : 0; step > 0; step >>= 1) {
#pragma unroll
    for (int u = 0; u < kPairILP; ++u) {
      const int c = pos[u] + step;
      if (c <= lb && b[c - 1] < x[u]) pos[u] = c;
    }
  }
#pragma unroll
  for (int u = 0; u < kPairILP; ++u) hit[u] = pos[u] < lb && b[pos[u]] == x[u];
}

__global__ void pair_overlap_kernel(const int32_t* __restrict__ idx, const int32_t* __restrict__ len,
                                    int64_t n_pairs, int width, int32_t* __restrict__ out) {
  __shared__ int32_t rows_s[kPairWarps][kPairSmemRow];
  const int lane = threadIdx.x & 31;
  int32_t* slot = rows_s[threadIdx.x >> 5];
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t pr = blockIdx.x * static_cast<int64_t>(blockDim.x >> 5) + (threadIdx.x >> 5); pr < n_pairs;
       pr += warps) {
    const int32_t* a = idx + (2 * pr) * width;
    const int32_t* b = idx + (2 * pr + 1) * width;
    const int la = min(max(len[2 * pr], 0), width);
    const int lb = min(max(len[2 * pr + 1], 0), width);
    const int32_t* bs = stage_row(b, lb, slot, lane);
    int count = 0;
    for (int base = 0; base < la; base += 32 * kPairILP) {
      int32_t x[kPairILP];
#pragma unroll
      for (int u = 0; u < kPairILP; ++u) {
        const int i = base + u * 32 + lane;
        x[u] = i < la ? a[i] : 0;
      }
      bool hit[kPairILP];
      rows_hold(bs, lb, x, hit);
#pragma unroll
      for (int u = 0; u < kPairILP; ++u) count += (base + u * 32 + lane < la && hit[u]) ? 1 : 0;
    }
    count = warp_sum_i32(count);
    if (lane == 0) out[pr] = count;
    __syncwarp();  // the slot is restaged for the next pair
  }
}

// One warp per pair.  The rows are ascending, so taking a row's entries in
// order keeps every region ascending: the warp tests 32 consecutive entries
// against the other row and writes each region's members at the region's
// running length plus their ballot rank.
__global__ void pair_regions_kernel(const int32_t* __restrict__ idx, const int32_t* __restrict__ len,
                                    int64_t n_pairs, int width, int32_t* __restrict__ shared,
                                    int32_t* __restrict__ left, int32_t* __restrict__ right,
                                    int32_t* __restrict__ counts) {
  __shared__ int32_t rows_s[kPairWarps][kPairSmemRow];
  const int lane = threadIdx.x & 31;
  const uint32_t lt = (1u << lane) - 1u;
  int32_t* slot = rows_s[threadIdx.x >> 5];
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t pr = blockIdx.x * static_cast<int64_t>(blockDim.x >> 5) + (threadIdx.x >> 5); pr < n_pairs;
       pr += warps) {
    const int32_t* a = idx + (2 * pr) * width;
    const int32_t* b = idx + (2 * pr + 1) * width;
    const int la = min(max(len[2 * pr], 0), width);
    const int lb = min(max(len[2 * pr + 1], 0), width);
    const int32_t* bs = stage_row(b, lb, slot, lane);
    int32_t* so = shared + pr * width;
    int32_t* lo = left + pr * width;
    int32_t* ro = right + pr * width;
    int ns = 0, nl = 0, nr = 0;
    for (int base = 0; base < la; base += 32 * kPairILP) {
      int32_t x[kPairILP];
      bool both[kPairILP];
#pragma unroll
      for (int u = 0; u < kPairILP; ++u) {
        const int i = base + u * 32 + lane;
        x[u] = i < la ? a[i] : 0;
      }
      rows_hold(bs, lb, x, both);
#pragma unroll
      for (int u = 0; u < kPairILP; ++u) both[u] = both[u] && base + u * 32 + lane < la;
#pragma unroll
      for (int u = 0; u < kPairILP; ++u) {  // groups of 32 in row order keep each region ascending
        const bool in = base + u * 32 + lane < la;
        const uint32_t bsh = __ballot_sync(kFullMask, both[u]);
        const uint32_t bl = __ballot_sync(kFullMask, in && !both[u]);
        if (both[u]) so[ns + __popc(bsh & lt)] = x[u];
        if (in && !both[u]) lo[nl + __popc(bl & lt)] = x[u];
        ns += __popc(bsh);
        nl += __popc(bl);
      }
    }
    __syncwarp();  // every lane is done with the staged right row
    const int32_t* as = stage_row(a, la, slot, lane);
    for (int base = 0; base < lb; base += 32 * kPairILP) {
      int32_t x[kPairILP];
      bool only[kPairILP];
#pragma unroll
      for (int u = 0; u < kPairILP; ++u) {
        const int i = base + u * 32 + lane;
        x[u] = i < lb ? b[i] : 0;
      }
      rows_hold(as, la, x, only);
#pragma unroll
      for (int u = 0; u < kPairILP; ++u) only[u] = !only[u] && base + u * 32 + lane < lb;
#pragma unroll
      for (int u = 0; u < kPairILP; ++u) {
        const uint32_t br = __ballot_sync(kFullMask, only[u]);
        if (only[u]) ro[nr + __popc(br & lt)] = x[u];
        nr += __popc(br);
      }
    }
    for (int i = ns + lane; i < width; i += 32) so[i] = -1;
    for (int i = nl + lane; i < width; i += 32) lo[i] = -1;
    for (int i = nr + lane; i < width; i += 32) ro[i] = -1;
    if (lane == 0) {
      counts[3 * pr] = ns;
      counts[3 * pr + 1] = nl;
      counts[3 * pr + 2] = nr;
    }
    __syncwarp();  // the slot is restaged for the next pair
  }
}

cudaError_t launch_pair_regions(const int32_t* idx, const int32_t* len, int64_t n_pairs, int width,
                                int32_t* shared, int32_t* left, int32_t* right, int32_t* counts,
                                cudaStream_t stream) {
  if (n_pairs == 0) return cudaSuccess;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int threads = 32 * kPairWarps;  // one pair per warp at a time
  int64_t blocks = (n_pairs + kPairWarps - 1) / kPairWarps;
  if (blocks > static_cast<int64_t>(sms) * 16) blocks = static_cast<int64_t>(sms) * 16;
  pair_regions_kernel<<<static_cast<unsigned>(blocks), threads, 0, stream>>>(idx, len, n_pairs, width, shared,
                                                                            left, right, counts);
  return cudaGetLastError();
}

// Adds `add` to every valid index (>= 0) of n consecutive output entries: a
// document's rows are computed with document-relative key numbers and then
// shifted to global positions.
__global__ void offset_indices_kernel(int32_t* __restrict__ idx, int64_t n, int32_t add) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int32_t v = idx[i];
    if (v >= 0) idx[i] = v + add;
  }
}

cudaError_t launch_offset_indices(int32_t* idx, int64_t n, int32_t add, cudaStream_t stream) {
  if (n == 0 || add == 0) return cudaSuccess;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int64_t blocks = (n + 255) / 256;
  if (blocks > static_cast<int64_t>(sms) * 8) blocks = static_cast<int64_t>(sms) * 8;
  offset_indices_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(idx, n, add);
  return cudaGetLastError();
}

cudaError_t launch_pair_overlap(const int32_t* idx, const int32_t* len, int64_t n_pairs, int width,
                                int32_t* out, cudaStream_t stream) {
  if (n_pairs == 0) return cudaSuccess;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int threads = 32 * kPairWarps;  // one pair per warp at a time
  int64_t blocks = (n_pairs + kPairWarps - 1) / kPairWarps;
  if (blocks > static_cast<int64_t>(sms) * 16) blocks = static_cast<int64_t>(sms) * 16;
  pair_overlap_kernel<<<static_cast<unsigned>(blocks), threads, 0, stream>>>(idx, len, n_pairs, width, out);
  return cudaGetLastError();
}

}  // namespace hwr
