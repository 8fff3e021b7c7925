// Host entry points of libmfa.so that launch nothing: version, status names,
// tile-map sizing and carving, and reading back the device error word.
#include <cuda_runtime.h>

#include "mfa.h"
#include "mfa_internal.h"

extern "C" int32_t mfa_abi_version(void) { return MFA_ABI_VERSION; }

extern "C" const char* mfa_status_string(mfa_status s) {
  switch (s) {
    case MFA_OK: return "ok";
    case MFA_ERR_INVALID_ARG: return "invalid argument";
    case MFA_ERR_UNSUPPORTED: return "unsupported combination";
    case MFA_ERR_SHAPE_MISMATCH: return "shape mismatch";
    case MFA_ERR_CUDA: return "CUDA runtime error";
    case MFA_ERR_DEVICE: return "device-side error recorded";
  }
  return "unknown status";
}

extern "C" size_t mfa_tile_map_bytes(int32_t B, int32_t Hm, int32_t Nq, int32_t Nk,
                                     int32_t block_q, int32_t block_k) {
  mfa::MapLayout L;
  if (!mfa::map_layout(B, Hm, Nq, Nk, block_q, block_k, &L)) return 0;
  return L.total;
}

extern "C" mfa_status mfa_tile_map_init(mfa_tile_map* map, void* device_buf, size_t bytes,
                                        int32_t B, int32_t Hm, int32_t Nq, int32_t Nk,
                                        int32_t block_q, int32_t block_k) {
  if (!map || !device_buf) return MFA_ERR_INVALID_ARG;
  mfa::MapLayout L;
  if (B <= 0 || Hm <= 0 || Nq < 0 || Nk < 0) return MFA_ERR_INVALID_ARG;
  if (!mfa::map_layout(B, Hm, Nq, Nk, block_q, block_k, &L)) return MFA_ERR_UNSUPPORTED;
  if (bytes < L.total) return MFA_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(device_buf) % 256 != 0) return MFA_ERR_INVALID_ARG;
  char* base = static_cast<char*>(device_buf);
  map->B = B; map->Hm = Hm; map->Nq = Nq; map->Nk = Nk;
  map->block_q = block_q; map->block_k = block_k;
  map->nqt = static_cast<int32_t>(mfa::cdiv64(Nq, block_q));
  map->nkt = static_cast<int32_t>(mfa::cdiv64(Nk, block_k));
  map->kind = -1;
  map->reserved = 0;
  map->kminmax = reinterpret_cast<int32_t*>(base + L.kminmax);
  map->tile_class = reinterpret_cast<uint8_t*>(base + L.tile_class);
  map->tile_list = reinterpret_cast<int32_t*>(base + L.tile_list);
  map->tile_count = reinterpret_cast<int32_t*>(base + L.tile_count);
  map->order = reinterpret_cast<int32_t*>(base + L.order);
  map->err = reinterpret_cast<uint32_t*>(base + L.err);
  return MFA_OK;
}

extern "C" mfa_status mfa_get_device_status(const mfa_tile_map* map, void* stream, uint32_t* err_bits) {
  if (!map || !map->err) return MFA_ERR_INVALID_ARG;
  uint32_t host = 0;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(&host, map->err, sizeof(host), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return MFA_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return MFA_ERR_CUDA;
  if (err_bits) *err_bits = host;
  return host ? MFA_ERR_DEVICE : MFA_OK;
}
