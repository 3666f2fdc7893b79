// witness.cu -- a lower bound of every query's K-th score from seed keys.
//
// "DoSA: Dots Sparse Attention", 核心方法 (core method, first step): score a
// set of at least K visible keys exactly and take the K-th largest of those
// scores as tau; since tau_K(seeds) <= tau_K(all visible keys), a key scoring
// below tau can never be selected (核心创新, first point).  The same page's
// decode result (实验结果) gets its speed-up from a threshold kept across
// decode steps, i.e. seeds taken from keys selected recently.
//
// Here the seeds are given per query row (e.g. the previous step's output
// row) and scored on CUDA cores in FP32, in an order that differs from the
// tensor-core accumulation of the scoring kernel.  Each seed's score is
// therefore lowered by a margin that covers both roundings,
//   eps * |k| * sum_h |w_h| |q_h|   (times the key scale for FP8).
// Each dot product over D = 128 exact products carries at most about
// D * 2^-24 = 2^-17 of |q_h| |k| in FP32 on either side, the head sums far
// less.  The tensor-core scores, measured against FP64 on inputs whose
// products all have one sign (the largest accumulation error relative to the
// norms), stay within 2^-23 of |k| sum_h |w_h| |q_h| for BF16 and for FP8
// (kind::f8f6f4) alike, so eps = 2^-12 leaves a wide factor for both.  The
// threshold is the K-th largest lowered score over the row's distinct visible
// seeds, so at least K keys score at or above it in the scoring kernel and
// the exact top-K is unchanged.  A margin that fell short could only put the
// threshold above the true K-th score, which leaves fewer than K keys at or
// above it: the row comes out short, and the kernels check for exactly that
// and raise a status bit.  No failure is silent.
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "internal.h"
#include "ptx.cuh"

namespace hwr {
namespace {

constexpr int kSeedThreads = 128;  // seeds scored per CTA, one per thread
constexpr int kSelThreads = 256;
constexpr int kSelSmem = 8192;     // seed rows up to this length are selected in shared memory
constexpr int kMaxHD = 64 * 128;   // largest H * D staged in shared memory

// Converts n (a multiple of 16 for FP8, of 8 for bf16) consecutive elements
// starting at element i0 of a 16-byte aligned row to float, 16 bytes per load.
template <int N>
__device__ __forceinline__ void load_row(const void* base, bool fp8, size_t i0, float (&out)[N]) {
  if (fp8) {
    const uint4* src = reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(base) + i0);
#pragma unroll
    for (int c = 0; c < N / 16; ++c) {
      const uint4 v = src[c];
      const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int b = 0; b < 16; ++b) {
        __nv_fp8_e4m3 e;
        e.__x = static_cast<uint8_t>(wv[b >> 2] >> (8 * (b & 3)));
        out[16 * c + b] = static_cast<float>(e);
      }
    }
  } else {
    const uint4* src = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(base) + i0);
#pragma unroll
    for (int c = 0; c < N / 8; ++c) {
      const uint4 v = src[c];
      const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        out[8 * c + 2 * b] = __uint_as_float(wv[b] << 16);
        out[8 * c + 2 * b + 1] = __uint_as_float(wv[b] & 0xFFFF0000u);
      }
    }
  }
}

// n visible keys (rows of the scored matrix) for the query at position g.
__device__ __forceinline__ int64_t visible(const WitnessParams& wp, int64_t g) {
  const int64_t n = wp.ranged ? (g + 1) / wp.ratio : g + 1;
  return n < wp.n_keys ? n : wp.n_keys;
}

// Key row named by a seed entry, or -1: POOLED seeds are token positions
// (an output row of the indexer) and name the pool holding them.
__device__ __forceinline__ int64_t seed_row(const WitnessParams& wp, int32_t e, int64_t g) {
  if (e < 0) return -1;
  const int64_t r = wp.seed_div > 1 ? e / wp.seed_div : e;
  return r < visible(wp, g) ? r : -1;
}

// grid (ceil(n_seeds / 128), rows): thread j of CTA (x, .) scores seed
// x * 128 + j of each of its query rows t and writes the lowered score as an
// ordered key, or 0 (below every score) for a seed that names no visible key.
template <int D>
__global__ void __launch_bounds__(kSeedThreads) witness_scores_kernel(const WitnessParams wp) {
  __shared__ __align__(16) float qs[kMaxHD];
  __shared__ float ws[64];
  __shared__ float qn[64];
  const int H = wp.H;
  const int lane = threadIdx.x & 31, wq = threadIdx.x >> 5;
  const int64_t j = static_cast<int64_t>(blockIdx.x) * kSeedThreads + threadIdx.x;
  for (int64_t t = blockIdx.y; t < wp.S; t += gridDim.y) {
    const int64_t g = wp.q_pos0 + t;
    // the query's H * D values, 16 per thread and step (16-byte loads)
    for (int i = 16 * threadIdx.x; i < H * D; i += 16 * kSeedThreads) {
      float v[16];
      load_row<16>(wp.q, wp.fp8, static_cast<size_t>(t) * H * D + i, v);
#pragma unroll
      for (int u = 0; u < 16; ++u) qs[i + u] = v[u];
    }
    if (threadIdx.x < H) {
      float wv = wp.w[t * H + threadIdx.x];
      if (wp.fp8) wv *= wp.q_scale[t * H + threadIdx.x];
      ws[threadIdx.x] = wv;
    }
    __syncthreads();
    // |w_h| |q_h| per head, each norm rounded up a little (one warp per head)
    for (int h = wq; h < H; h += kSeedThreads / 32) {
      float n2 = 0.f;
      for (int d = lane; d < D; d += 32) n2 = fmaf(qs[h * D + d], qs[h * D + d], n2);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) n2 += __shfl_xor_sync(kFullMask, n2, o);
      if (lane == 0) qn[h] = fabsf(ws[h]) * (sqrtf(n2) * (1.0f + 0x1p-18f));
    }
    __syncthreads();
    if (j < wp.n_seeds) {
      const int64_t r = seed_row(wp, wp.seeds[t * wp.seed_stride + j], g);
      uint32_t out = 0u;
      if (r >= 0) {
        float amp = 0.f;  // sum_h |w_h| |q_h|
        for (int h = 0; h < H; ++h) amp += qn[h];
        float kr[D];
        load_row<D>(wp.keys, wp.fp8, static_cast<size_t>(r) * D, kr);
        float kn2 = 0.f;
#pragma unroll
        for (int d = 0; d < D; ++d) kn2 = fmaf(kr[d], kr[d], kn2);
        float s = 0.f;
        for (int h = 0; h < H; ++h) {
          const float4* qh = reinterpret_cast<const float4*>(qs + h * D);
          float x0 = 0.f, x1 = 0.f, x2 = 0.f, x3 = 0.f;  // four independent chains
          // 32 dims at a time: eight shared-memory loads in flight, then their
          // 32 multiply-adds
#pragma unroll
          for (int blk = 0; blk < D / 32; ++blk) {
            float4 v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) v[u] = qh[8 * blk + u];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              const int d = 32 * blk + 4 * u;
              x0 = fmaf(v[u].x, kr[d], x0);
              x1 = fmaf(v[u].y, kr[d + 1], x1);
              x2 = fmaf(v[u].z, kr[d + 2], x2);
              x3 = fmaf(v[u].w, kr[d + 3], x3);
            }
          }
          s = fmaf(ws[h], fmaxf((x0 + x1) + (x2 + x3), 0.f), s);
        }
        float margin = 0x1p-12f * (sqrtf(kn2) * (1.0f + 0x1p-18f)) * amp;
        if (wp.fp8) {
          const float ks = wp.k_scale[r];
          s *= ks;
          margin *= ks;
        }
        const float lo = s - margin;
        out = ordered_key(__fadd_rn(lo - fabsf(lo) * 0x1p-20f, 0.f));
      }
      wp.lowered[t * wp.n_seeds + j] = out;
    }
    __syncthreads();  // qs, ws and qn are rewritten for the next row
  }
}

// One CTA per query row (grid-stride): keeps only the first entry of each
// key row among the seeds (a later entry naming a row at or below the
// largest row already seen is dropped, so every kept row is distinct), then
// writes the ksel-th largest lowered score -- 0, which lets every key pass,
// when fewer than ksel distinct visible seeds remain.
__global__ void __launch_bounds__(kSelThreads) witness_select_kernel(const WitnessParams wp) {
  __shared__ uint32_t hist[256];
  __shared__ uint32_t row_s[kSelSmem];  // the row's lowered scores, when they fit
  __shared__ int64_t wmax[kSelThreads / 32];
  __shared__ uint32_t pick[2];
  const int lane = threadIdx.x & 31, wq = threadIdx.x >> 5;
  for (int64_t t = blockIdx.x; t < wp.S; t += gridDim.x) {
    const int64_t g = wp.q_pos0 + t;
    uint32_t* row = wp.lowered + t * wp.n_seeds;
    if (wp.n_seeds <= kSelSmem) {
      for (int64_t j = threadIdx.x; j < wp.n_seeds; j += kSelThreads) row_s[j] = row[j];
      row = row_s;  // every pass below reads and writes shared memory
      __syncthreads();
    }
    // 1. distinct rows: exclusive running maximum of the seed rows
    int64_t carry = -1;
    for (int64_t base = 0; base < wp.n_seeds; base += kSelThreads) {
      const int64_t j = base + threadIdx.x;
      int64_t r = -1;
      if (j < wp.n_seeds && row[j] != 0u) r = seed_row(wp, wp.seeds[t * wp.seed_stride + j], g);
      int64_t incl = r;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int64_t v = __shfl_up_sync(kFullMask, incl, o);
        if (lane >= o) incl = max(incl, v);
      }
      if (lane == 31) wmax[wq] = incl;
      __syncthreads();
      int64_t before = carry;
      for (int w2 = 0; w2 < wq; ++w2) before = max(before, wmax[w2]);
      int64_t excl = __shfl_up_sync(kFullMask, incl, 1);
      if (lane > 0) before = max(before, excl);
      if (j < wp.n_seeds && r >= 0 && r <= before) row[j] = 0u;
      int64_t total = carry;
      for (int w2 = 0; w2 < kSelThreads / 32; ++w2) total = max(total, wmax[w2]);
      __syncthreads();
      carry = total;
    }
    __syncthreads();
    // 2. ksel-th largest of the row (zeros included), 8 bits per pass
    uint32_t prefix = 0u, rank = static_cast<uint32_t>(wp.ksel);
    const bool enough = wp.n_seeds >= wp.ksel;
    for (int shift = 24; shift >= 0 && enough; shift -= 8) {
      hist[threadIdx.x] = 0u;
      __syncthreads();
      for (int64_t j = threadIdx.x; j < wp.n_seeds; j += kSelThreads) {
        const uint32_t v = row[j];
        if (shift == 24 || (v >> (shift + 8)) == (prefix >> (shift + 8))) atomicAdd(&hist[(v >> shift) & 255u], 1u);
      }
      __syncthreads();
      if (wq == 0) {
        // lane l owns bins 255 - 8l down to 248 - 8l; counts above a lane's
        // bins come from a warp scan of the per-lane sums
        uint32_t mine = 0u;
#pragma unroll
        for (int i = 0; i < 8; ++i) mine += hist[255 - 8 * lane - i];
        uint32_t incl = mine;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t v = __shfl_up_sync(kFullMask, incl, o);
          if (lane >= o) incl += v;
        }
        const uint32_t above = incl - mine;
        if (above < rank && rank <= incl) {  // exactly one lane
          uint32_t acc = above;
          int b = 255 - 8 * lane;
          for (int i = 0; i < 7; ++i, --b) {
            if (acc + hist[b] >= rank) break;
            acc += hist[b];
          }
          pick[0] = static_cast<uint32_t>(b);
          pick[1] = acc;
        }
      }
      __syncthreads();
      prefix |= pick[0] << shift;
      rank -= pick[1];
      __syncthreads();
    }
    if (threadIdx.x == 0) wp.thr[t] = enough ? prefix : 0u;
    __syncthreads();
  }
}

}  // namespace

cudaError_t launch_witness(const WitnessParams& wp, int D, cudaStream_t stream) {
  if (wp.S == 0) return cudaSuccess;
  if (wp.H > 64 || wp.H * D > kMaxHD || (D != 64 && D != 128)) return cudaErrorInvalidValue;
  if (wp.n_seeds > 0) {
    const int64_t rows = wp.S < 65535 ? wp.S : 65535;
    const dim3 grid(static_cast<unsigned>((wp.n_seeds + kSeedThreads - 1) / kSeedThreads),
                    static_cast<unsigned>(rows));
    if (D == 128)
      witness_scores_kernel<128><<<grid, kSeedThreads, 0, stream>>>(wp);
    else
      witness_scores_kernel<64><<<grid, kSeedThreads, 0, stream>>>(wp);
  }
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t blocks = wp.S < static_cast<int64_t>(sms) * 8 ? wp.S : static_cast<int64_t>(sms) * 8;
  witness_select_kernel<<<static_cast<unsigned>(blocks), kSelThreads, 0, stream>>>(wp);
  return cudaGetLastError();
}

}  // namespace hwr
