// prune.cu -- set-up of the lossless pruning stage.
//
// "DoSA: Dots Sparse Attention", 核心方法 / 方法步骤详情 (core method): a key
// is skipped when a cheap upper bound U_i of its score lies below a lower
// bound of the query's K-th score; the result must equal unpruned top-K.
// Here the scoring kernel keeps the first kPruneR heads of every query exactly
// and folds each other head h onto an anchor j among them, with
// beta = [q_h.q_j]_+ / |q_j|^2 and d_h = q_h - beta q_j:
//   w_h > 0:  w_h [q_h.k]_+ <= w_h beta [q_j.k]_+ + w_h |d_h| |k|
//   w_h < 0:  w_h [q_h.k]_+ <= w_h beta [q_j.k]_+ + |w_h| |d_h| |k|
// (ReLU subadditivity, positive homogeneity and Cauchy-Schwarz, the same
// page's background section), so
//   U_i = sum_{j < r} wt_j [a_j]_+ + Ceff |k_i|,
//   wt_j = w_j + sum_{h -> j} w_h beta_h,  Ceff = sum_h |w_h| |d_h| + margin.
// Everything is in the kernel's own domain: for FP8, q and k are the e4m3
// codes the MMA multiplies, w already carries the q scale, and the key scale
// multiplies U after the sum exactly as it multiplies the score.
//
// The residual allowance is the smaller of two bounds of
//   R = sum_h [x_h . k]_+,   x_h = w_h d_h   (both signs of w_h),
// the per-head one E_P |k| = sum_h |x_h| |k|, and the same page's joint one
// (技术新颖性, second point), which uses how the residuals align:
//   R = 1/2 ((sum_h x_h) . k + sum_h |x_h . k|)
//     <= 1/2 (|sum_h x_h| + sqrt(sum_{h,l} |x_h . x_l|)) |k| = E_joint |k|,
// since sum_h |x_h . k| = (sum_h s_h x_h) . k for signs s_h, and
// |sum_h s_h x_h|^2 <= sum_{h,l} |x_h . x_l|.  E_joint <= E_P always; for
// nearly orthogonal residuals it is about sqrt(#heads) times smaller.
//
// The margin covers the MMA's accumulation error and the FP32 rounding of
// both the score and U: 2^-11 * |k| * sum_h |w_h| |q_h|.
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "internal.h"
#include "ptx.cuh"

namespace hwr {

__device__ __forceinline__ float load_q_elem(const void* q, bool fp8, size_t i) {
  if (fp8) {
    __nv_fp8_e4m3 v;
    v.__x = static_cast<const uint8_t*>(q)[i];
    return static_cast<float>(v);
  }
  return __uint_as_float(static_cast<uint32_t>(static_cast<const uint16_t*>(q)[i]) << 16);
}

__device__ __forceinline__ float warp_sum_f32(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kFullMask, v, o);
  return v;
}

// Slightly enlarges a non-negative float so that it bounds the exact value the
// FP32 computation approximated (relative 2^-18 covers a few roundings).
__device__ __forceinline__ float round_up_pos(float x) { return x * (1.0f + 0x1p-18f) + 0x1p-100f; }

// One warp (the whole block) per query row t: out[t] = {wt[0..r), Ceff,
// sum |w||q|}.  Requires D % 32 == 0 and D <= 128 (four values per lane),
// H <= 64.  Dot products between heads run one per lane over rows staged in
// shared memory (a padded row stride keeps lanes on different rows off each
// other's banks), so a query's set-up is a few long independent chains
// rather than one warp reduction per pair -- it is on the critical path of
// decode-like shapes, which have a handful of query rows.
constexpr int kRow = 129;  // padded row stride (floats)

// sum_d a[d] b[d] over D dims of two shared-memory rows, four chains.
__device__ __forceinline__ float row_dot(const float* a, const float* b, int D) {
  float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
  for (int d = 0; d < D; d += 4) {
    s0 = fmaf(a[d], b[d], s0);
    s1 = fmaf(a[d + 1], b[d + 1], s1);
    s2 = fmaf(a[d + 2], b[d + 2], s2);
    s3 = fmaf(a[d + 3], b[d + 3], s3);
  }
  return (s0 + s1) + (s2 + s3);
}

__global__ void __launch_bounds__(32) prune_prep_kernel(const void* __restrict__ q, const float* __restrict__ w,
                                                        const float* __restrict__ q_scale, bool fp8, int64_t S,
                                                        int H, int D, float* __restrict__ out) {
  const int lane = threadIdx.x & 31;
  __shared__ float wt[kPruneR];
  __shared__ float nk_s[kPruneR];
  __shared__ float qk[kPruneR][kRow];        // kept heads
  __shared__ float qv[kRow];                 // the omitted head being folded
  __shared__ float xs[64 - kPruneR][kRow];   // x_h = w_h d_h, row h - kPruneR
  const int per = D / 32;  // values per lane
  for (int64_t t = blockIdx.x; t < S; t += gridDim.x) {
    const size_t qbase = static_cast<size_t>(t) * H * D;
    // kept heads in registers (head j, dims lane + 32 m) and in shared memory
    float kept[kPruneR][4];
    float wsum = 0.f;  // sum_h |w_h| |q_h|, rounded up
#pragma unroll
    for (int j = 0; j < kPruneR; ++j) {
      float ss = 0.f;
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        kept[j][m] = m < per ? load_q_elem(q, fp8, qbase + static_cast<size_t>(j) * D + lane + 32 * m) : 0.f;
        ss = fmaf(kept[j][m], kept[j][m], ss);
        if (m < per) qk[j][lane + 32 * m] = kept[j][m];
      }
      const float nj = round_up_pos(sqrtf(warp_sum_f32(ss)));
      float wj = w[t * H + j];
      if (fp8) wj *= q_scale[t * H + j];
      if (lane == 0) {
        wt[j] = wj;
        nk_s[j] = nj;
      }
      wsum += fabsf(wj) * nj;
    }
    __syncwarp();
    float C = 0.f;
    float xsum[4] = {0.f, 0.f, 0.f, 0.f};  // sum_h x_h (this lane's dims)
    float gdiag = 0.f;                     // this lane's part of sum_h |x_h|^2
    for (int h = kPruneR; h < H; ++h) {
      float v[4];
      float ss = 0.f;
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        v[m] = m < per ? load_q_elem(q, fp8, qbase + static_cast<size_t>(h) * D + lane + 32 * m) : 0.f;
        ss = fmaf(v[m], v[m], ss);
        if (m < per) qv[lane + 32 * m] = v[m];
      }
      __syncwarp();
      const float nh = round_up_pos(sqrtf(warp_sum_f32(ss)));
      float wh = w[t * H + h];
      if (fp8) wh *= q_scale[t * H + h];
      wsum += fabsf(wh) * nh;
      // anchor: the kept head with the largest positive projection (lane j
      // computes q_h . q_j; ties go to the lower j)
      float dd = 0.f, proj = -1.f;
      if (lane < kPruneR) {
        dd = row_dot(qv, qk[lane], D);
        proj = (dd > 0.f && nk_s[lane] > 0.f) ? dd / nk_s[lane] : -1.f;
      }
      int best = lane < kPruneR ? lane : kPruneR;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float p2 = __shfl_xor_sync(kFullMask, proj, o);
        const int b2 = __shfl_xor_sync(kFullMask, best, o);
        if (p2 > proj || (p2 == proj && b2 < best)) {
          proj = p2;
          best = b2;
        }
      }
      const float best_dot = __shfl_sync(kFullMask, dd, best & 31);
      if (proj <= 0.f) best = -1;
      float beta = 0.f, nd = nh;
      float d[4];
#pragma unroll
      for (int m = 0; m < 4; ++m) d[m] = v[m];
      if (best >= 0) {
        // any beta >= 0 gives a valid bound once |d| is measured for that beta
        const float nj = nk_s[best];
        const float nj2 = nj * nj;
        beta = best_dot / nj2;
        float ds = 0.f;
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          d[m] = m < per ? fmaf(-beta, qk[best][lane + 32 * m], v[m]) : 0.f;
          ds = fmaf(d[m], d[m], ds);
        }
        nd = round_up_pos(sqrtf(warp_sum_f32(ds)));
        // the FP32 residual d differs from q_h - beta q_j by at most one
        // rounding per component
        nd += 0x1p-20f * (nh + beta * nj);
        if (lane == 0) wt[best] += wh * beta;
      }
      C += fabsf(wh) * nd;
      // x_h = w_h d_h (the FP32 residual; the joint bound's slack below covers
      // its rounding)
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const float x = m < per ? wh * d[m] : 0.f;
        xsum[m] += x;
        gdiag = fmaf(x, x, gdiag);
        if (m < per) xs[h - kPruneR][lane + 32 * m] = x;
      }
      __syncwarp();
    }
    // off-diagonal Gram terms: lane l of round h takes the pairs (h, l + 32 i)
    float goff = 0.f;
    const int nx = H - kPruneR;
    for (int h = 1; h < nx; ++h)
      for (int l = lane; l < h; l += 32) goff += 2.f * fabsf(row_dot(xs[h], xs[l], D));
    const float G = warp_sum_f32(gdiag) + warp_sum_f32(goff);
    float sx = 0.f;
#pragma unroll
    for (int m = 0; m < 4; ++m) sx = fmaf(xsum[m], xsum[m], sx);
    sx = warp_sum_f32(sx);
    // FP32 slack of the joint bound: the Gram sum and |sum x| carry relative
    // errors of about D * 2^-24 of (sum |x_h|)^2 and sum |x_h|, and x_h
    // itself differs from w_h (q_h - beta q_j) by 2^-20-relative amounts;
    // 2^-7 * C (about 0.8% of the per-head bound) covers all of them
    const float joint = round_up_pos(0.5f * (sqrtf(sx) + sqrtf(G))) + 0x1p-7f * C;
    const float resid = fminf(round_up_pos(C), joint);
    const float ceff = round_up_pos(resid + 0x1p-11f * wsum);
    float* o = out + static_cast<size_t>(t) * (kPruneR + 2);
    __syncwarp();
    if (lane < kPruneR) o[lane] = wt[lane];
    if (lane == 0) {
      o[kPruneR] = ceff;
      o[kPruneR + 1] = wsum;
    }
    __syncwarp();
  }
}

// norms[i] = |k_i| (kernel domain: bf16 values or e4m3 codes), rounded up.
__global__ void key_norms_kernel(const void* __restrict__ k, bool fp8, int64_t n, int D, float* __restrict__ norms) {
  const int lane = threadIdx.x & 31;
  const int warps = blockDim.x >> 5;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(warps) + (threadIdx.x >> 5); i < n;
       i += static_cast<int64_t>(gridDim.x) * warps) {
    float ss = 0.f;
    for (int d = lane; d < D; d += 32) {
      const float x = load_q_elem(k, fp8, static_cast<size_t>(i) * D + d);
      ss = fmaf(x, x, ss);
    }
    ss = warp_sum_f32(ss);
    if (lane == 0) norms[i] = round_up_pos(sqrtf(ss));
  }
}

cudaError_t launch_prune_setup(const void* q, const float* w, const float* q_scale, bool fp8, int64_t S, int H,
                               int D, const void* keys, int64_t n_keys, float* pq, float* knorm,
                               cudaStream_t stream) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int threads = 256;  // 8 warps
  if (S > 0) {
    int64_t blocks = S;  // one warp per query row
    if (blocks > static_cast<int64_t>(sms) * 32) blocks = static_cast<int64_t>(sms) * 32;
    prune_prep_kernel<<<static_cast<unsigned>(blocks), 32, 0, stream>>>(q, w, q_scale, fp8, S, H, D, pq);
  }
  if (n_keys > 0) {
    int64_t blocks = (n_keys + 7) / 8;
    if (blocks > static_cast<int64_t>(sms) * 16) blocks = static_cast<int64_t>(sms) * 16;
    key_norms_kernel<<<static_cast<unsigned>(blocks), threads, 0, stream>>>(keys, fp8, n_keys, D, knorm);
  }
  return cudaGetLastError();
}

}  // namespace hwr
