// tp_block_forward_noalloc: a block decode step whose scratch lives in a
// fixed-size array inside this library, for callers that cannot allocate
// device memory (see include/tp_block.h).
//
// The array is a file-scope __device__ variable, so every GPU that loads this
// library reserves TP_NOALLOC_SCRATCH_BYTES for it until the process exits. In
// host code the array's name is only a host-side stand-in: its device address
// is obtained with cudaGetSymbolAddress, with the device current, and passed to
// the kernels like any other workspace pointer. tp_block_noalloc_error reads
// the kernels' error word back from it.
#include <mutex>

#include "kernels.cuh"

namespace tp {
namespace {

__device__ __align__(256) uint8_t g_block_scratch[TP_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
void* g_scratch_addr[kMaxDevices];  // device address of g_block_scratch, per device
std::mutex g_scratch_mu;

// Device address of the scratch array on the current device. Looked up on the
// first call made with that device current, and again on every call made
// outside stream capture, so that a call after a device reset (which loads the
// module again, at a new address) does not use a stale pointer; a call under
// capture uses the address of the last call outside it.
int scratch_address(void** out, cudaStream_t stream) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return TP_ECUDA;
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(stream, &cap) != cudaSuccess) return TP_ECUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_addr[dev] || cap == cudaStreamCaptureStatusNone) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_block_scratch) != cudaSuccess || !p) return TP_ECUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return TP_OK;
}

}  // namespace
}  // namespace tp

using namespace tp;

extern "C" int tp_block_forward_noalloc(const tp_dims* dims, int n_slices, int partition,
                                        int sync_quant, const tp_block_weights* w, float* x,
                                        void* k_cache, void* v_cache, const int32_t* pos,
                                        int batch, tp_stream stream) {
  size_t need = 0;
  int rc = tp_block_workspace_bytes(dims, n_slices, partition, sync_quant, &need);
  if (rc) return rc;
  if (need > (size_t)TP_NOALLOC_SCRATCH_BYTES) return TP_ESCRATCH;
  rc = device_check();
  if (rc) return rc;
  void* scratch = nullptr;
  rc = scratch_address(&scratch, (cudaStream_t)stream);
  if (rc) return rc;
  return block_forward_on_workspace(dims, n_slices, partition, sync_quant, w, scratch,
                                    (size_t)TP_NOALLOC_SCRATCH_BYTES, x, k_cache, v_cache, pos,
                                    batch, (cudaStream_t)stream);
}

// The kernels' error word of the last tp_block_forward_noalloc on this device:
// the int at byte 0 of the array (every block workspace starts with it), copied
// to host memory on `stream`. No allocation.
extern "C" int tp_block_noalloc_error(int* err, tp_stream stream) {
  if (!err) return TP_EINVAL;
  int rc = device_check();
  if (rc) return rc;
  if (cudaMemcpyFromSymbolAsync(err, g_block_scratch, sizeof(int), 0, cudaMemcpyDeviceToHost,
                                (cudaStream_t)stream) != cudaSuccess)
    return TP_ECUDA;
  return TP_OK;
}
