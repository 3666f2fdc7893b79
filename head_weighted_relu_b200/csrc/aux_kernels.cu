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

// Round hi + lo (|lo| at most half an ulp of hi, the pair an error-free sum)
// to bfloat16, nearest-even.  Rounding hi alone is right unless hi sits exactly
// halfway between two bfloat16 values; then the sign of lo decides.
__device__ __forceinline__ uint16_t round_pair_to_bf16(double hi, double lo) {
  if (lo != 0.0 && hi != 0.0) {
    int e;
    frexp(hi, &e);                          // |hi| = f * 2^e, 0.5 <= f < 1
    const int qexp = max(e - 8, -133);      // bfloat16 spacing at |hi|: 2^qexp
    const double halves = ldexp(hi, 1 - qexp);  // hi in units of half a spacing (exact)
    const double r = rint(halves);
    if (r == halves && fmod(fabs(r), 2.0) == 1.0) {  // exactly halfway
      const double half = ldexp(1.0, qexp - 1);
      return cvt_rn_bf16_f64(lo > 0.0 ? hi + half : hi - half);
    }
  }
  return cvt_rn_bf16_f64(hi);
}

// kp[p, d] = RNE_bf16( sum_j c[j, d] * k[ratio*p + j, d] ), the sum exact:
// each product of two bfloat16 values is exact in binary64 and the running
// sum is kept as an unevaluated pair (hi, lo) with Knuth's TwoSum.
__global__ void pool_keys_kernel(const uint16_t* __restrict__ k, const uint16_t* __restrict__ coef, int ratio,
                                 int64_t n_pools, int D, uint16_t* __restrict__ out) {
  const int64_t n = n_pools * D;
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < n;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t pool = e / D;
    const int d = static_cast<int>(e - pool * D);
    double hi = 0.0, lo = 0.0;
    for (int j = 0; j < ratio; ++j) {
      const double prod = bf16_bits_to_double(coef[j * D + d]) * bf16_bits_to_double(k[(pool * ratio + j) * D + d]);
      const double s = __dadd_rn(hi, prod);
      const double bb = __dsub_rn(s, hi);
      const double err = __dadd_rn(__dsub_rn(hi, __dsub_rn(s, bb)), __dsub_rn(prod, bb));
      hi = s;
      lo = __dadd_rn(lo, err);
    }
    // fold lo into hi once more so that |lo| is below half an ulp of hi
    const double s = __dadd_rn(hi, lo);
    const double bb = __dsub_rn(s, hi);
    const double err = __dadd_rn(__dsub_rn(hi, __dsub_rn(s, bb)), __dsub_rn(lo, bb));
    out[e] = round_pair_to_bf16(s, err);
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
__global__ void pair_overlap_kernel(const int32_t* __restrict__ idx, const int32_t* __restrict__ len,
                                    int64_t n_pairs, int width, int32_t* __restrict__ out) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t pr = blockIdx.x * static_cast<int64_t>(blockDim.x >> 5) + (threadIdx.x >> 5); pr < n_pairs;
       pr += warps) {
    const int32_t* a = idx + (2 * pr) * width;
    const int32_t* b = idx + (2 * pr + 1) * width;
    const int la = min(max(len[2 * pr], 0), width);
    const int lb = min(max(len[2 * pr + 1], 0), width);
    int count = 0;
    for (int i = lane; i < la; i += 32) {
      const int32_t x = a[i];
      int lo = 0, hi = lb;
      while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (b[mid] < x)
          lo = mid + 1;
        else
          hi = mid;
      }
      count += (lo < lb && b[lo] == x) ? 1 : 0;
    }
    count = warp_sum_i32(count);
    if (lane == 0) out[pr] = count;
  }
}

// True when the strictly ascending row b[0, lb) holds x (binary search).
__device__ __forceinline__ bool row_holds(const int32_t* __restrict__ b, int lb, int32_t x) {
  int lo = 0, hi = lb;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (b[mid] < x)
      lo = mid + 1;
    else
      hi = mid;
  }
  return lo < lb && b[lo] == x;
}

// One warp per pair.  The rows are ascending, so taking a row's entries in
// order keeps every region ascending: the warp tests 32 consecutive entries
// against the other row and writes each region's members at the region's
// running length plus their ballot rank.
__global__ void pair_regions_kernel(const int32_t* __restrict__ idx, const int32_t* __restrict__ len,
                                    int64_t n_pairs, int width, int32_t* __restrict__ shared,
                                    int32_t* __restrict__ left, int32_t* __restrict__ right,
                                    int32_t* __restrict__ counts) {
  const int lane = threadIdx.x & 31;
  const uint32_t lt = (1u << lane) - 1u;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t pr = blockIdx.x * static_cast<int64_t>(blockDim.x >> 5) + (threadIdx.x >> 5); pr < n_pairs;
       pr += warps) {
    const int32_t* a = idx + (2 * pr) * width;
    const int32_t* b = idx + (2 * pr + 1) * width;
    const int la = min(max(len[2 * pr], 0), width);
    const int lb = min(max(len[2 * pr + 1], 0), width);
    int32_t* so = shared + pr * width;
    int32_t* lo = left + pr * width;
    int32_t* ro = right + pr * width;
    int ns = 0, nl = 0, nr = 0;
    for (int base = 0; base < la; base += 32) {
      const int i = base + lane;
      const bool in = i < la;
      const int32_t x = in ? a[i] : 0;
      const bool both = in && row_holds(b, lb, x);
      const uint32_t bs = __ballot_sync(kFullMask, both);
      const uint32_t bl = __ballot_sync(kFullMask, in && !both);
      if (both) so[ns + __popc(bs & lt)] = x;
      if (in && !both) lo[nl + __popc(bl & lt)] = x;
      ns += __popc(bs);
      nl += __popc(bl);
    }
    for (int base = 0; base < lb; base += 32) {
      const int i = base + lane;
      const bool only = i < lb && !row_holds(a, la, b[i]);
      const uint32_t br = __ballot_sync(kFullMask, only);
      if (only) ro[nr + __popc(br & lt)] = b[i];
      nr += __popc(br);
    }
    for (int i = ns + lane; i < width; i += 32) so[i] = -1;
    for (int i = nl + lane; i < width; i += 32) lo[i] = -1;
    for (int i = nr + lane; i < width; i += 32) ro[i] = -1;
    if (lane == 0) {
      counts[3 * pr] = ns;
      counts[3 * pr + 1] = nl;
      counts[3 * pr + 2] = nr;
    }
  }
}

cudaError_t launch_pair_regions(const int32_t* idx, const int32_t* len, int64_t n_pairs, int width,
                                int32_t* shared, int32_t* left, int32_t* right, int32_t* counts,
                                cudaStream_t stream) {
  if (n_pairs == 0) return cudaSuccess;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int threads = 256;  // 8 pairs per block
  int64_t blocks = (n_pairs + 7) / 8;
  if (blocks > static_cast<int64_t>(sms) * 16) blocks = static_cast<int64_t>(sms) * 16;
  pair_regions_kernel<<<static_cast<unsigned>(blocks), threads, 0, stream>>>(idx, len, n_pairs, width, shared,
                                                                            left, right, counts);
  return cudaGetLastError();
}

cudaError_t launch_pair_overlap(const int32_t* idx, const int32_t* len, int64_t n_pairs, int width,
                                int32_t* out, cudaStream_t stream) {
  if (n_pairs == 0) return cudaSuccess;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int threads = 256;  // 8 pairs per block
  int64_t blocks = (n_pairs + 7) / 8;
  if (blocks > static_cast<int64_t>(sms) * 16) blocks = static_cast<int64_t>(sms) * 16;
  pair_overlap_kernel<<<static_cast<unsigned>(blocks), threads, 0, stream>>>(idx, len, n_pairs, width, out);
  return cudaGetLastError();
}

}  // namespace hwr
