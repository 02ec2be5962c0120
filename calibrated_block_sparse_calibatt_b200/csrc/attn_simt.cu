// CUDA-core attention for CalibAtt: the float32 path (and the 64-token-block
// path), block-sparse or anchor-row with broadcast.
//
// Same definition as the tensor-core kernel ("Accelerating Text-to-Video
// Generation with Calibrated Sparse Attention", paper note, Key Designs 3-4),
// evaluated with float32 products and float32 online softmax so that float32
// inputs meet a 1e-4 error bound; tensor cores offer no float32 mode that
// precise.  One CTA per (batch, head, query tile of BLK rows); two threads per
// query row split the head dimension (even / odd elements); keys are staged
// through shared memory 32 at a time.
#include "internal.h"

#include <cuda_bf16.h>
#include <math.h>

namespace calibatt {
namespace {

constexpr int kKeysPerStage = 32;
constexpr int kKeysPerChunk = 8;  // keys scored per register chunk

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
__device__ __forceinline__ void store_val(float* p, float x) { *p = x; }
__device__ __forceinline__ void store_val(__nv_bfloat16* p, float x) { *p = __float2bfloat16_rn(x); }

template <typename T, int HD, int BLK, bool ANCHOR>
__global__ void __launch_bounds__(2 * BLK) simt_attn_kernel(const __grid_constant__ SimtParams p) {
  __shared__ float sK[kKeysPerStage][HD];
  __shared__ float sV[kKeysPerStage][HD];
  const int tid = threadIdx.x;
  const int row = tid >> 1, half = tid & 1;
  constexpr int kE = HD / 2;
  if (!ANCHOR && p.sched.csr_gate) {
    // caller-held lists that the check before this launch found invalid
    __shared__ int skip;
    if (tid == 0) skip = p.status != nullptr && csr_violation_recorded(p.status);
    __syncthreads();
    if (skip) return;
  }

  // ---- which tile
  int b, h, tile, n;
  const uint16_t* cols = nullptr;
  if (ANCHOR) {
    const int per_batch = p.anc.n_heads * p.anc.tiles_per_head;
    b = blockIdx.x / per_batch;
    const int r = blockIdx.x % per_batch;
    h = p.anc.head_ids[r / p.anc.tiles_per_head];
    tile = r % p.anc.tiles_per_head;
    n = p.nb;
  } else {
    const int per_batch = p.n_heads * p.sched.nq;
    b = blockIdx.x / per_batch;
    const int r = blockIdx.x % per_batch;
    h = p.head_ids[r / p.sched.nq];
    tile = r % p.sched.nq;
    const int32_t* rp = p.sched.row_ptr + static_cast<int64_t>(h) * (p.sched.nq + 1);
    n = rp[tile + 1] - rp[tile];
    cols = p.sched.col + p.sched.col_base[h] + rp[tile];
  }
  const int64_t bh = static_cast<int64_t>(b) * p.sb + static_cast<int64_t>(h) * p.sh;
  const T* q = static_cast<const T*>(p.q) + bh;
  const T* k = static_cast<const T*>(p.k) + bh;
  const T* v = static_cast<const T*>(p.v) + bh;

  // ---- this row's query
  int64_t q_token = -1;
  int anchor_f = 0, anchor_w = 0, lo = 0, n_dst = 0;
  if (ANCHOR) {
    const int pq = tile * BLK + row;
    if (pq < p.anc.anchor_tokens) {
      const int per_frame = p.anc.n_anchors * p.anc.cols;
      anchor_f = pq / per_frame;
      const int rem = pq % per_frame;
      const int a = rem / p.anc.cols;
      anchor_w = rem % p.anc.cols;
      q_token = (static_cast<int64_t>(anchor_f) * p.anc.rows + p.anc.anchor_row[a]) * p.anc.cols + anchor_w;
      lo = p.anc.group_lo[a];
      n_dst = p.anc.group_hi[a] - lo + 1;
    }
  } else {
    const int token = tile * BLK + row;
    if (token < p.seq_len) {
      q_token = token;
      n_dst = 1;
    }
  }
  float qr[kE], acc[kE];
#pragma unroll
  for (int e = 0; e < kE; ++e) {
    qr[e] = q_token >= 0 ? to_f32(q[q_token * p.sn + 2 * e + half]) : 0.f;
    acc[e] = 0.f;
  }

  float m = -INFINITY, l = 0.f;
  const float sl2 = p.scale_log2;
  for (int j = 0; j < n; ++j) {
    const int c = ANCHOR ? j : static_cast<int>(cols[j]);
    if (c >= p.nb) {
      // a block index outside the key range (device lists the host never
      // checked): record it and skip the block rather than read past N
      if (tid == 0 && p.status) atomicCAS(p.status, 0, 1 | (22 << 8));
      continue;
    }
    for (int k0 = c * BLK; k0 < c * BLK + BLK; k0 += kKeysPerStage) {
      __syncthreads();
      for (int idx = tid; idx < kKeysPerStage * HD; idx += 2 * BLK) {
        const int kk = idx / HD, d = idx % HD;
        const int key = k0 + kk;
        float kv = 0.f, vv = 0.f;
        if (key < p.seq_len) {
          kv = to_f32(k[static_cast<int64_t>(key) * p.sn + d]);
          vv = to_f32(v[static_cast<int64_t>(key) * p.sn + d]);
        }
        sK[kk][d] = kv;
        sV[kk][d] = vv;
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
          sc[kk] = (k0 + g + kk < p.seq_len) ? part * sl2 : -INFINITY;
          mx = fmaxf(mx, sc[kk]);
        }
        const float m_new = fmaxf(m, mx);
        if (m_new == -INFINITY) continue;
        const float corr = exp2f(m - m_new);
        l *= corr;
#pragma unroll
        for (int e = 0; e < kE; ++e) acc[e] *= corr;
#pragma unroll
        for (int kk = 0; kk < kKeysPerChunk; ++kk) {
          const float pj = exp2f(sc[kk] - m_new);
          l += pj;
#pragma unroll
          for (int e = 0; e < kE; ++e) acc[e] = fmaf(pj, sV[g + kk][2 * e + half], acc[e]);
        }
        m = m_new;
      }
    }
  }

  const float inv_l = l > 0.f ? 1.f / l : 0.f;
  T* o = static_cast<T*>(p.o) + bh;
  for (int d = 0; d < n_dst; ++d) {
    const int64_t token = ANCHOR
        ? (static_cast<int64_t>(anchor_f) * p.anc.rows + lo + d) * p.anc.cols + anchor_w
        : q_token;
#pragma unroll
    for (int e = 0; e < kE; ++e) store_val(o + token * p.sn + 2 * e + half, acc[e] * inv_l);
  }
  if (!ANCHOR && p.lse != nullptr && q_token >= 0 && half == 0) {
    p.lse[(static_cast<int64_t>(b) * p.heads + h) * p.seq_len + q_token] =
        l > 0.f ? (m + log2f(l)) * 0.69314718055994531f : -INFINITY;
  }
}

template <typename T, int HD, int BLK>
cudaError_t launch_t(const SimtParams& p, bool anchor, int n_items, cudaStream_t s) {
  if (anchor)
    simt_attn_kernel<T, HD, BLK, true><<<n_items, 2 * BLK, 0, s>>>(p);
  else
    simt_attn_kernel<T, HD, BLK, false><<<n_items, 2 * BLK, 0, s>>>(p);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_dt(const SimtParams& p, int head_dim, int block, bool anchor, int n_items,
                      cudaStream_t s) {
  if (head_dim == 64 && block == 64) return launch_t<T, 64, 64>(p, anchor, n_items, s);
  if (head_dim == 64 && block == 128) return launch_t<T, 64, 128>(p, anchor, n_items, s);
  if (head_dim == 128 && block == 64) return launch_t<T, 128, 64>(p, anchor, n_items, s);
  if (head_dim == 128 && block == 128) return launch_t<T, 128, 128>(p, anchor, n_items, s);
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_simt_attn(const SimtParams& p, int head_dim, int block, int dtype, bool anchor,
                             int n_items, cudaStream_t s) {
  if (n_items <= 0) return cudaSuccess;
  if (dtype == 1) return launch_dt<float>(p, head_dim, block, anchor, n_items, s);
  return launch_dt<__nv_bfloat16>(p, head_dim, block, anchor, n_items, s);
}

}  // namespace calibatt
