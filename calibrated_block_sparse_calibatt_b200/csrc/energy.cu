// Offline calibration kernels of CalibAtt ("Accelerating Text-to-Video
// Generation with Calibrated Sparse Attention", paper note, Key Designs 1-2):
//   block_energy   E_{r,c} = (1/|I_r|) sum_{i in I_r} sum_{j in J_c} P_ij (Eq. (5)),
//                  from the dense post-softmax attention without storing P;
//   select_blocks  shortest energy-descending prefix with mass >= tau;
//   aggregate      M = 1[count / |D| >= rho] (Eq. (8)-(9)).
// The energy is two passes over Q K^T on CUDA cores in float32: pass 1 finds
// each query's log-sum-exp over all keys, pass 2 recomputes the scores of one
// (query block, key block) tile, sums exp(s - lse) and reduces over the
// block's valid queries in a fixed order, so results are bitwise repeatable.
#include "internal.h"

#include <cuda_bf16.h>
#include <math.h>

namespace calibatt {
namespace {

constexpr int kKeysPerStage = 32;
inline unsigned ceil_blocks(int n, int b) { return static_cast<unsigned>((n + b - 1) / b); }
constexpr int kKeysPerChunk = 8;  // keys scored per register chunk

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

// Pass 1: lse2[b, h, i] = log2 sum_j 2^(s_ij * log2 e) over valid keys j.
template <typename T, int HD, int BLK>
__global__ void __launch_bounds__(2 * BLK) row_lse_kernel(const __grid_constant__ EnergyParams p) {
  __shared__ float sK[kKeysPerStage][HD];
  const int tid = threadIdx.x, row = tid >> 1, half = tid & 1;
  constexpr int kE = HD / 2;
  const int r = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int64_t bh = static_cast<int64_t>(b) * p.sb + static_cast<int64_t>(h) * p.sh;
  const T* q = static_cast<const T*>(p.q) + bh;
  const T* k = static_cast<const T*>(p.k) + bh;
  const int i = r * BLK + row;
  float qr[kE];
#pragma unroll
  for (int e = 0; e < kE; ++e) qr[e] = i < p.seq_len ? to_f32(q[static_cast<int64_t>(i) * p.sn + 2 * e + half]) : 0.f;
  float m = -INFINITY, l = 0.f;
  for (int k0 = 0; k0 < p.seq_len; k0 += kKeysPerStage) {
    __syncthreads();
    for (int idx = tid; idx < kKeysPerStage * HD; idx += 2 * BLK) {
      const int kk = idx / HD, d = idx % HD;
      sK[kk][d] = (k0 + kk < p.seq_len) ? to_f32(k[static_cast<int64_t>(k0 + kk) * p.sn + d]) : 0.f;
    }
    __syncthreads();
#pragma unroll 1
    for (int g = 0; g < kKeysPerStage; g += kKeysPerChunk) {
      float sc[kKeysPerChunk];
      float mx = -INFINITY;
#pragma unroll
      for (int kk = 0; kk < kKeysPerChunk; ++kk) {
        float part = 0.f;
#pragma unroll
        for (int e = 0; e < kE; ++e) part = fmaf(qr[e], sK[g + kk][2 * e + half], part);
        part += __shfl_xor_sync(0xFFFFFFFFu, part, 1);
        sc[kk] = (k0 + g + kk < p.seq_len) ? part * p.scale_log2 : -INFINITY;
        mx = fmaxf(mx, sc[kk]);
      }
      const float m_new = fmaxf(m, mx);
      if (m_new == -INFINITY) continue;
      l *= exp2f(m - m_new);
#pragma unroll
      for (int kk = 0; kk < kKeysPerChunk; ++kk) l += exp2f(sc[kk] - m_new);
      m = m_new;
    }
  }
  if (i < p.seq_len && half == 0)
    p.lse[(static_cast<int64_t>(b) * p.heads + h) * p.seq_len + i] = m + log2f(l);
}

// Pass 2: one CTA per (key block c, query block r, batch*head).
template <typename T, int HD, int BLK>
__global__ void __launch_bounds__(2 * BLK) block_energy_kernel(const __grid_constant__ EnergyParams p) {
  __shared__ float sK[kKeysPerStage][HD];
  __shared__ float red[BLK];
  const int tid = threadIdx.x, row = tid >> 1, half = tid & 1;
  constexpr int kE = HD / 2;
  const int c = blockIdx.x, r = blockIdx.y;
  const int b = blockIdx.z / p.heads, h = blockIdx.z % p.heads;
  const int64_t bh = static_cast<int64_t>(b) * p.sb + static_cast<int64_t>(h) * p.sh;
  const T* q = static_cast<const T*>(p.q) + bh;
  const T* k = static_cast<const T*>(p.k) + bh;
  const int i = r * BLK + row;
  const bool valid_row = i < p.seq_len;
  float qr[kE];
#pragma unroll
  for (int e = 0; e < kE; ++e) qr[e] = valid_row ? to_f32(q[static_cast<int64_t>(i) * p.sn + 2 * e + half]) : 0.f;
  const float lse2 = valid_row ? p.lse[(static_cast<int64_t>(b) * p.heads + h) * p.seq_len + i] : 0.f;
  float sum = 0.f;
  for (int k0 = c * BLK; k0 < c * BLK + BLK; k0 += kKeysPerStage) {
    __syncthreads();
    for (int idx = tid; idx < kKeysPerStage * HD; idx += 2 * BLK) {
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
      if (k0 + kk < p.seq_len) sum += exp2f(part * p.scale_log2 - lse2);
    }
  }
  if (half == 0) red[row] = valid_row ? sum : 0.f;
  __syncthreads();
  // Fixed-order tree reduction over the block's rows.
  for (int stride = BLK / 2; stride > 0; stride >>= 1) {
    if (tid < stride) red[tid] += red[tid + stride];
    __syncthreads();
  }
  if (tid == 0) {
    const int valid = min(BLK, p.seq_len - r * BLK);
    p.energy[((static_cast<int64_t>(b) * p.heads + h) * p.nb + r) * p.nb + c] = red[0] / static_cast<float>(valid);
  }
}

template <typename T, int HD, int BLK>
cudaError_t launch_energy_t(const EnergyParams& p, cudaStream_t s) {
  dim3 g1(p.nb, p.heads, p.batch);
  row_lse_kernel<T, HD, BLK><<<g1, 2 * BLK, 0, s>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  dim3 g2(p.nb, p.nb, p.batch * p.heads);
  block_energy_kernel<T, HD, BLK><<<g2, 2 * BLK, 0, s>>>(p);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_energy_dt(const EnergyParams& p, int head_dim, int block, cudaStream_t s) {
  if (head_dim == 64 && block == 64) return launch_energy_t<T, 64, 64>(p, s);
  if (head_dim == 64 && block == 128) return launch_energy_t<T, 64, 128>(p, s);
  if (head_dim == 128 && block == 64) return launch_energy_t<T, 128, 64>(p, s);
  if (head_dim == 128 && block == 128) return launch_energy_t<T, 128, 128>(p, s);
  return cudaErrorInvalidValue;
}

constexpr int kSelectThreads = 256;

// One CTA per row of energies.  rank(c) = number of blocks ordered before c
// (higher energy, or equal energy and lower index); the prefix sum runs in
// float64 in rank order on one thread, exactly as the selection rule reads.
__global__ void __launch_bounds__(kSelectThreads) select_blocks_kernel(const float* __restrict__ energy,
                                                                       int nk, float tau, uint8_t* mask,
                                                                       int32_t* count_accum) {
  extern __shared__ float sm[];
  float* e = sm;
  float* sorted = sm + nk;
  int* rank = reinterpret_cast<int*>(sm + 2 * nk);
  __shared__ int kstar;
  const int64_t row = blockIdx.x;
  const float* er = energy + row * nk;
  for (int c = threadIdx.x; c < nk; c += kSelectThreads) e[c] = er[c];
  __syncthreads();
  for (int c = threadIdx.x; c < nk; c += kSelectThreads) {
    const float ec = e[c];
    int rk = 0;
    for (int c2 = 0; c2 < nk; ++c2) {
      const float e2 = e[c2];
      rk += (e2 > ec) || (e2 == ec && c2 < c);
    }
    rank[c] = rk;
    sorted[rk] = ec;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const double t = static_cast<double>(tau);
    double cum = 0.0;
    int ks = nk;
    for (int i = 0; i < nk; ++i) {
      cum += static_cast<double>(sorted[i]);
      if (cum >= t) {
        ks = i + 1;
        break;
      }
    }
    kstar = ks;
  }
  __syncthreads();
  for (int c = threadIdx.x; c < nk; c += kSelectThreads) {
    const uint8_t keep = rank[c] < kstar ? 1 : 0;
    mask[row * nk + c] = keep;
    if (count_accum) count_accum[row * nk + c] += keep;
  }
}

__global__ void aggregate_kernel(const int32_t* __restrict__ counts, int64_t n, int32_t n_prompts,
                                 float rho, uint8_t* mask) {
  const double d = static_cast<double>(n_prompts), r = static_cast<double>(rho);
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    mask[i] = (static_cast<double>(counts[i]) / d >= r) ? 1 : 0;
}

}  // namespace

// Pass 1 alone (also the first pass of the spatial-repetition score):
// lse2[b, h, i] for every query, 128 queries per CTA.
cudaError_t launch_row_lse(const EnergyParams& p, int head_dim, int dtype, cudaStream_t s) {
  dim3 g(ceil_blocks(p.seq_len, 128), p.heads, p.batch);
  if (head_dim == 64) {
    if (dtype == 1) row_lse_kernel<float, 64, 128><<<g, 256, 0, s>>>(p);
    else row_lse_kernel<__nv_bfloat16, 64, 128><<<g, 256, 0, s>>>(p);
  } else if (head_dim == 128) {
    if (dtype == 1) row_lse_kernel<float, 128, 128><<<g, 256, 0, s>>>(p);
    else row_lse_kernel<__nv_bfloat16, 128, 128><<<g, 256, 0, s>>>(p);
  } else {
    return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_block_energy(const EnergyParams& p, int head_dim, int block, int dtype,
                                cudaStream_t s) {
  if (dtype == 1) return launch_energy_dt<float>(p, head_dim, block, s);
  return launch_energy_dt<__nv_bfloat16>(p, head_dim, block, s);
}

cudaError_t launch_select_blocks(const float* energy, int64_t n_rows, int32_t nk, float tau,
                                 uint8_t* mask, int32_t* count_accum, cudaStream_t s) {
  if (n_rows <= 0) return cudaSuccess;
  const size_t smem = static_cast<size_t>(nk) * 12;
  select_blocks_kernel<<<static_cast<unsigned>(n_rows), kSelectThreads, smem, s>>>(energy, nk, tau, mask,
                                                                                   count_accum);
  return cudaGetLastError();
}

cudaError_t launch_aggregate(const int32_t* counts, int64_t n, int32_t n_prompts, float rho,
                             uint8_t* mask, cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  const int threads = 256;
  const int64_t blocks = (n + threads - 1) / threads;
  aggregate_kernel<<<static_cast<unsigned>(blocks < 4096 ? blocks : 4096), threads, 0, s>>>(counts, n,
                                                                                          n_prompts, rho, mask);
  return cudaGetLastError();
}

}  // namespace calibatt
