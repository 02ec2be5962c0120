// Spatial-repetition detection of CalibAtt ("Accelerating Text-to-Video
// Generation with Calibrated Sparse Attention", paper note, Key Designs 3):
// for every frame f and spatial row rho of a head, the cosine similarity of
// the row-flattened attention of the row's W queries and of its nearest
// anchor row's W queries (same columns), over all N keys:
//   sim(f, rho) = sum_w <P[(f,rho,w)], P[(f,a,w)]>
//                 / sqrt(sum_w |P[(f,rho,w)]|^2 * sum_w |P[(f,a,w)]|^2),
// then the per-head mean over prompts, frames and rows against a threshold.
// Pass 1 (energy.cu, row_lse_kernel) gives each query's log2-sum-exp, so
// P_ij = 2^(s_ij log2 e - lse2_i) is available key by key without storing P.
// Calibration work on CUDA cores in float32, fixed reduction orders: repeated
// calls give bitwise identical scores.  (bf16 inputs take the tensor-core
// pass of attn_tc.cu instead, which leaves per-query sums for
// similarity_from_sums_kernel below.)
#include "internal.h"

#include <cuda_bf16.h>
#include <math.h>

namespace calibatt {
namespace {

constexpr int kKeysPerStage = 32;
constexpr int kCols = 64;               // columns w per pass of a CTA
constexpr int kThreads = 4 * kCols;     // (w, query of the row | of the anchor, half of D)

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

// One CTA per (frame * rows + rho, head, batch).  Thread t works on column
// w = w0 + t/4: lanes with (t/2) & 1 == 0 hold the query (f, rho, w), the
// others the anchor query (f, a, w); t & 1 selects half of D.  Each key's
// probability pair meets through a lane shuffle.
template <typename T, int HD>
__global__ void __launch_bounds__(kThreads) spatial_sim_kernel(const __grid_constant__ RepetitionParams p) {
  __shared__ float sK[kKeysPerStage][HD];
  __shared__ float red[3][kThreads / 4];
  __shared__ float acc[3];
  const int tid = threadIdx.x;
  const int half = tid & 1, role = (tid >> 1) & 1, wl = tid >> 2;
  constexpr int kE = HD / 2;
  const int fr = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int f = fr / p.rows, rho = fr % p.rows, a = p.nearest[rho];
  const int64_t bh = static_cast<int64_t>(b) * p.sb + static_cast<int64_t>(h) * p.sh;
  const T* q = static_cast<const T*>(p.q) + bh;
  const T* k = static_cast<const T*>(p.k) + bh;
  const float* lse = p.lse + (static_cast<int64_t>(b) * p.heads + h) * p.seq_len;
  if (tid < 3) acc[tid] = 0.f;
  for (int w0 = 0; w0 < p.cols; w0 += kCols) {
    const int w = w0 + wl;
    const bool valid = w < p.cols;
    const int i = (f * p.rows + (role ? a : rho)) * p.cols + (valid ? w : 0);
    float qr[kE];
#pragma unroll
    for (int e = 0; e < kE; ++e) qr[e] = to_f32(q[static_cast<int64_t>(i) * p.sn + 2 * e + half]);
    const float l2 = lse[i];
    float dot = 0.f, sq = 0.f;
    for (int k0 = 0; k0 < p.seq_len; k0 += kKeysPerStage) {
      __syncthreads();
      for (int idx = tid; idx < kKeysPerStage * HD; idx += kThreads) {
        const int kk = idx / HD, d = idx % HD;
        sK[kk][d] = (k0 + kk < p.seq_len) ? to_f32(k[static_cast<int64_t>(k0 + kk) * p.sn + d]) : 0.f;
      }
      __syncthreads();
#pragma unroll 4
      for (int kk = 0; kk < kKeysPerStage; ++kk) {
        float part = 0.f;
#pragma unroll
        for (int e = 0; e < kE; ++e) part = fmaf(qr[e], sK[kk][2 * e + half], part);
        part += __shfl_xor_sync(0xFFFFFFFFu, part, 1);
        const float pr = (k0 + kk < p.seq_len) ? exp2f(part * p.scale_log2 - l2) : 0.f;
        const float other = __shfl_xor_sync(0xFFFFFFFFu, pr, 2);
        dot = fmaf(pr, other, dot);
        sq = fmaf(pr, pr, sq);
      }
    }
    // Column sums in a fixed order: lane (w, role 0, half 0) holds the row's
    // products and squares, lane (w, role 1, half 0) the anchor's squares.
    if (half == 0) {
      if (role == 0) {
        red[0][wl] = valid ? dot : 0.f;
        red[1][wl] = valid ? sq : 0.f;
      } else {
        red[2][wl] = valid ? sq : 0.f;
      }
    }
    __syncthreads();
    for (int stride = kCols / 2; stride > 0; stride >>= 1) {
      if (tid < stride) {
        red[0][tid] += red[0][tid + stride];
        red[1][tid] += red[1][tid + stride];
        red[2][tid] += red[2][tid + stride];
      }
      __syncthreads();
    }
    if (tid < 3) acc[tid] += red[tid][0];
    __syncthreads();
  }
  if (tid == 0) {
    const float den = sqrtf(acc[1]) * sqrtf(acc[2]);
    p.sim[((static_cast<int64_t>(b) * p.heads + h) * p.frames + f) * p.rows + rho] =
        den > 0.f ? acc[0] / den : 0.f;
  }
}

// One CTA per head: the mean over prompts and rows in double, in a fixed
// order, and the strict "exceeds" of the threshold.
constexpr int kFlagThreads = 256;
__global__ void __launch_bounds__(kFlagThreads) repetition_flags_kernel(const float* __restrict__ sim,
                                                                        int32_t n_prompts, int32_t n_heads,
                                                                        int32_t per_head, float threshold,
                                                                        float* __restrict__ mean,
                                                                        uint8_t* __restrict__ flags) {
  __shared__ double red[kFlagThreads];
  const int h = blockIdx.x;
  double s = 0.0;
  const int64_t n = static_cast<int64_t>(n_prompts) * per_head;
  for (int64_t idx = threadIdx.x; idx < n; idx += kFlagThreads) {
    const int64_t pr = idx / per_head, r = idx % per_head;
    s += static_cast<double>(sim[(pr * n_heads + h) * static_cast<int64_t>(per_head) + r]);
  }
  red[threadIdx.x] = s;
  __syncthreads();
  for (int stride = kFlagThreads / 2; stride > 0; stride >>= 1) {
    if (threadIdx.x < stride) red[threadIdx.x] += red[threadIdx.x + stride];
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    const double m = red[0] / static_cast<double>(n);
    if (mean) mean[h] = static_cast<float>(m);
    flags[h] = m > static_cast<double>(threshold) ? 1 : 0;
  }
}

// The rows' similarities from the tensor-core pass's per-query sums: one
// thread per (batch, head, frame, row) adds its cols queries' three sums in
// column order.
__global__ void similarity_from_sums_kernel(const float* __restrict__ sums, int64_t plane, int32_t bh_count,
                                            int32_t seq_len, int32_t frames, int32_t rows, int32_t cols,
                                            float* __restrict__ sim) {
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t total = static_cast<int64_t>(bh_count) * frames * rows;
  if (idx >= total) return;
  const int64_t bh = idx / (static_cast<int64_t>(frames) * rows);
  const int64_t fr = idx % (static_cast<int64_t>(frames) * rows);
  const float* ab = sums + bh * seq_len + fr * cols;
  float dot = 0.f, na = 0.f, nb = 0.f;
  for (int w = 0; w < cols; ++w) {
    dot += ab[w];
    na += ab[plane + w];
    nb += ab[2 * plane + w];
  }
  const float den = sqrtf(na) * sqrtf(nb);
  sim[idx] = den > 0.f ? dot / den : 0.f;
}

}  // namespace

cudaError_t launch_similarity_from_sums(const float* sums, int64_t plane, int32_t bh_count, int32_t seq_len,
                                        int32_t frames, int32_t rows, int32_t cols, float* sim, cudaStream_t s) {
  const int64_t total = static_cast<int64_t>(bh_count) * frames * rows;
  if (total == 0) return cudaSuccess;
  similarity_from_sums_kernel<<<static_cast<unsigned>((total + 255) / 256), 256, 0, s>>>(
      sums, plane, bh_count, seq_len, frames, rows, cols, sim);
  return cudaGetLastError();
}

cudaError_t launch_spatial_similarity(const RepetitionParams& p, int head_dim, int dtype, cudaStream_t s) {
  dim3 g(p.frames * p.rows, p.heads, p.batch);
  if (head_dim == 64) {
    if (dtype == 1) spatial_sim_kernel<float, 64><<<g, kThreads, 0, s>>>(p);
    else spatial_sim_kernel<__nv_bfloat16, 64><<<g, kThreads, 0, s>>>(p);
  } else if (head_dim == 128) {
    if (dtype == 1) spatial_sim_kernel<float, 128><<<g, kThreads, 0, s>>>(p);
    else spatial_sim_kernel<__nv_bfloat16, 128><<<g, kThreads, 0, s>>>(p);
  } else {
    return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_repetition_flags(const float* sim, int32_t n_prompts, int32_t n_heads, int32_t per_head,
                                    float threshold, float* mean, uint8_t* flags, cudaStream_t s) {
  if (n_heads == 0) return cudaSuccess;
  repetition_flags_kernel<<<n_heads, kFlagThreads, 0, s>>>(sim, n_prompts, n_heads, per_head, threshold, mean,
                                                           flags);
  return cudaGetLastError();
}

}  // namespace calibatt
