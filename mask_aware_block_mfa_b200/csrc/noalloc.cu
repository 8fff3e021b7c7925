// mfa_fwd_noalloc: the attention forward pass for callers that cannot
// allocate device memory.
//
// Who needs it: code that runs where it does not own the GPU allocator, such as
// a plugin or extension inside a host application that hands out device memory
// only for the tensors it passes in, or code that must not allocate between
// two points of a larger pipeline. The regular path needs one caller-owned
// buffer for the tile map (mfa_tile_map_bytes); this path keeps that map and
// the forward pass's work counters in a fixed array the library itself holds
// in device memory.
//
// The array is a file-scope __device__ variable of MFA_NOALLOC_SCRATCH_BYTES.
// Every GPU on which the library's kernels are loaded holds one copy until the
// process exits. Host code cannot use the variable's name as a device address,
// so the address is looked up with cudaGetSymbolAddress, with the call's device
// current: on the first call on each device, and again on every later call
// made while the stream is not capturing (after a cudaDeviceReset the module is
// loaded anew and the array may sit elsewhere). A call on a capturing stream
// uses the address the last lookup on that device found.
// All calls on a device share the one array: calls that overlap on the GPU
// race with each other and must be ordered by the caller (one stream, or
// events between streams).
#include <cstdint>
#include <mutex>

#include <cuda_runtime.h>

#include "mfa.h"
#include "mfa_internal.h"

namespace mfa {
namespace {

constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_noalloc_scratch[MFA_NOALLOC_SCRATCH_BYTES];

std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of the current device's copy of the scratch array (nullptr
// if the lookup fails or no address is known while `stream` is capturing).
void* device_scratch(cudaStream_t stream) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(stream, &cap) != cudaSuccess) return nullptr;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (cap == cudaStreamCaptureStatusNone || !g_scratch_addr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr) return nullptr;
    g_scratch_addr[dev] = ptr;
  }
  return g_scratch_addr[dev];
}

}  // namespace
}  // namespace mfa

extern "C" mfa_status mfa_fwd_noalloc(const mfa_tensor* q, const mfa_tensor* k, const mfa_tensor* v,
                                      const mfa_mask_desc* mask, int32_t block_q, int32_t block_k,
                                      const mfa_tensor* out, float* lse, uint32_t* dev_err, void* stream) {
  using namespace mfa;
  mfa_status st = check_mask(mask);
  if (st != MFA_OK) return st;
  const size_t need = mfa_tile_map_bytes(mask->B, mask->Hm, mask->Nq, mask->Nk, block_q, block_k);
  if (need == 0) return MFA_ERR_UNSUPPORTED;                    // block sizes other than 64 / 128
  if (need > MFA_NOALLOC_SCRATCH_BYTES) return MFA_ERR_UNSUPPORTED;  // the map does not fit the array
  // Everything mfa_fwd would reject is rejected here, before the map build
  // launches anything or touches the shared array.
  if ((st = check_fwd_args(q, k, v, mask, nullptr, out, lse, block_q)) != MFA_OK) return st;
  void* buf = device_scratch(static_cast<cudaStream_t>(stream));
  if (!buf) return MFA_ERR_CUDA;
  mfa_tile_map map;
  st = mfa_tile_map_init(&map, buf, MFA_NOALLOC_SCRATCH_BYTES, mask->B, mask->Hm, mask->Nq, mask->Nk, block_q,
                         block_k);
  if (st != MFA_OK) return st;
  // The build clears the error word and the work counters left by earlier
  // calls and rewrites every array of the map.
  st = mfa_build_tile_map(mask, &map, stream);
  if (st != MFA_OK) return st;
  mfa_mask_desc d = *mask;
  d.map = &map;
  st = mfa_fwd(q, k, v, &d, out, lse, stream);
  if (st != MFA_OK) return st;
  if (dev_err && cudaMemcpyAsync(dev_err, map.err, sizeof(uint32_t), cudaMemcpyDeviceToDevice,
                                 static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return MFA_ERR_CUDA;
  return MFA_OK;
}
