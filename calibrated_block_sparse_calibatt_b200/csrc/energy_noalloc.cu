// calibatt_block_energy_noalloc: the block-energy call for callers that may
// not allocate device memory.
//
// Some callers cannot call cudaMalloc, or any routine that allocates, when
// they compute block energies:
//   - a serving process that reserved all device memory at start-up for
//     weights and caches, where a further allocation would fail or fragment
//     the reservation;
//   - a host runtime that owns the device allocator and forbids plug-in code
//     from going around it;
//   - embedded integrations whose host side is not permitted to call the
//     CUDA memory-management API at all.
// Such callers still own the inputs and the energy output.  The only scratch
// the energy computation needs (one float32 row log-sum-exp per query row)
// comes from a fixed array compiled into this library instead of a
// caller-provided workspace.
//
// Costs and rules of that array:
//   - Every GPU that loads the library holds it (kMaxRows floats, 4 MiB)
//     until the process exits.
//   - All calls share it.  Two calls whose work overlaps on the GPU (on
//     different streams, or from different threads without ordering) race on
//     it and give undefined energies; order them on one stream.
//   - It keeps the previous call's contents.  No clearing is needed: the first
//     pass writes every row it covers before the second pass reads it.
//   - The first call on each device looks up the array's device address
//     (cudaGetSymbolAddress, with that device current).  Make that first call
//     before capturing any stream.
#include "calibatt.h"
#include "internal.h"

#include <mutex>

namespace {

// Row log-sum-exp scratch: batch * heads * seq_len floats at most.
constexpr size_t kMaxRows = size_t(1) << 20;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) float g_energy_scratch[kMaxRows];

// Per-device address of the array, looked up on the first call that runs on
// that device.  Only a successful lookup is kept: a failed one (a sticky error
// left by earlier work, or a call made during stream capture) is retried on
// the next call instead of failing every later call on that device.
void* g_scratch_ptr[kMaxDevices] = {};
std::mutex g_scratch_mu;

// Device address of the scratch array on the current device, or an error.  In
// host code the array's name is only a host-side stand-in; a kernel must be
// given this address instead.
cudaError_t scratch_on_current_device(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_energy_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" calibatt_status calibatt_block_energy_noalloc(const void* q, const void* k,
                                                        const calibatt_shape* shape, int32_t block,
                                                        float softmax_scale, float* energy,
                                                        void* stream) {
  size_t need = 0;
  calibatt_status st = calibatt_block_energy_workspace_size(shape, &need);  // validates shape
  if (st != CALIBATT_OK) return st;
  if (need > sizeof(float) * kMaxRows) {
    calibatt::set_last_error(
        "block energy without allocation: batch*heads*seq_len = %zu rows exceeds the built-in "
        "scratch of %zu rows; use calibatt_block_energy with a caller-provided workspace",
        need / sizeof(float), kMaxRows);
    return CALIBATT_ERR_INVALID_ARG;
  }
  void* scratch = nullptr;
  const cudaError_t e = scratch_on_current_device(&scratch);
  if (e != cudaSuccess) {
    cudaGetLastError();
    calibatt::set_last_error("block energy without allocation: scratch address lookup failed: %s",
                             cudaGetErrorString(e));
    return CALIBATT_ERR_CUDA;
  }
  return calibatt_block_energy(q, k, shape, block, softmax_scale, energy, scratch,
                               sizeof(float) * kMaxRows, stream);
}
