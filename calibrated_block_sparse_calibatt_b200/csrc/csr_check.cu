// Device-side check of skip lists and schedules the host never reads: the
// direct-CSR attention call takes them in device memory, so they are checked
// on the device, ahead of the attention kernel on the same stream.  A
// violation is recorded in the status word, and the attention kernels of that
// call (and of every later direct-CSR call until the word is read and
// cleared) then return before reading any list.
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
  if (__any_sync(0xFFFFFFFFu, bad) && lane == 0) atomicCAS(p.status, 0, 1 | (kCodeListViolation << 8));
}

// The persistent schedule the tensor-core kernel walks: cta_ptr starts at 0,
// does not decrease and ends at n_heads * nq (so every CTA's item range lies
// inside items), and every item names a listed head and a query block < nq.
// Grid-stride over max(items, grid + 1) entries.
__global__ void schedule_check_kernel(const __grid_constant__ CsrCheckParams p) {
  const int64_t n_items = static_cast<int64_t>(p.n_heads) * p.nq;
  const int64_t n = n_items > p.grid + 1 ? n_items : p.grid + 1;
  bool bad = false;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    if (i < n_items) {
      const uint32_t w = p.items[i];
      const int h = static_cast<int>(w >> 16), tile = static_cast<int>(w & 0xFFFFu);
      bool listed = false;
      for (int x = 0; x < p.n_heads; ++x) listed = listed || p.head_ids[x] == h;
      bad = bad || !listed || tile >= p.nq;
    }
    if (i <= p.grid) {
      const int32_t c = p.cta_ptr[i];
      bad = bad || (i == 0 && c != 0) || (i == p.grid && c != n_items) || c < 0 || c > n_items ||
            (i < p.grid && p.cta_ptr[i + 1] < c);
    }
  }
  if (bad) atomicCAS(p.status, 0, 1 | (kCodeScheduleViolation << 8));
}

}  // namespace

cudaError_t launch_csr_check(const CsrCheckParams& p, cudaStream_t s) {
  const int64_t warps = static_cast<int64_t>(p.n_heads) * p.nq;
  if (warps == 0) return cudaSuccess;
  const int threads = 256;
  const int64_t blocks = (warps * 32 + threads - 1) / threads;
  csr_check_kernel<<<static_cast<unsigned>(blocks), threads, 0, s>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || p.items == nullptr) return e;
  schedule_check_kernel<<<64, 256, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace calibatt
