// Device-side check of skip lists the host never reads: the direct-CSR
// attention call takes its lists in device memory, so they are checked on
// the device, ahead of the attention kernel on the same stream.
#include "internal.h"

namespace calibatt {
namespace {

// One warp per (listed head, query block): the head's row pointers start at
// 0 and do not decrease, a row holds at most nq blocks, and its block
// indices are strictly ascending in [0, nq).  The first violation is recorded
// in the status word; nothing else is written.
__global__ void csr_check_kernel(const __grid_constant__ CsrCheckParams p) {
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= static_cast<int64_t>(p.n_heads) * p.nq) return;
  const int h = p.head_ids[warp / p.nq];
  const int r = static_cast<int>(warp % p.nq);
  const int32_t* rp = p.row_ptr + static_cast<int64_t>(h) * (p.nq + 1);
  const int32_t lo = rp[r], hi = rp[r + 1];
  bool bad = lo < 0 || (r == 0 && lo != 0) || hi < lo || hi - lo > p.nq;
  if (!bad) {
    const uint16_t* c = p.col + p.col_base[h] + lo;
    for (int i = lane; i < hi - lo; i += 32) {
      const int x = c[i];
      bad = bad || x >= p.nq || (i > 0 && c[i - 1] >= x);
    }
  }
  if (__any_sync(0xFFFFFFFFu, bad) && lane == 0) atomicCAS(p.status, 0, 1 | (23 << 8));
}

}  // namespace

cudaError_t launch_csr_check(const CsrCheckParams& p, cudaStream_t s) {
  const int64_t warps = static_cast<int64_t>(p.n_heads) * p.nq;
  if (warps == 0) return cudaSuccess;
  const int threads = 256;
  const int64_t blocks = (warps * 32 + threads - 1) / threads;
  csr_check_kernel<<<static_cast<unsigned>(blocks), threads, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace calibatt
