// Host-side helpers shared by the translation units of libmfa.so.
#pragma once

#include <atomic>
#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include "mfa.h"

namespace mfa {

constexpr int kSelBlock = 64;
constexpr int kMaxSelK = 256;

inline int64_t cdiv64(int64_t a, int64_t b) { return (a + b - 1) / b; }
inline size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// The driver's cuTensorMapEncodeTiled (through the runtime, so the library
// does not link libcuda), looked up on first use; nullptr if unavailable.
inline PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static std::atomic<void*> cached{nullptr};
  void* fn = cached.load(std::memory_order_acquire);
  if (!fn) {
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !fn)
      return nullptr;
    cached.store(fn, std::memory_order_release);
  }
  return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
}

// Streaming multiprocessors of the current device (0 on error).
inline int device_sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return n;
}

// A kernel's dynamic shared-memory limit is a per-device attribute:
// cudaFuncSetAttribute sets it for the current device only. `done` holds
// one bit per device (0..63) on which it is already set, so that a process
// driving several GPUs sets it once on each.
inline bool ensure_smem_attr(const void* func, int bytes, std::atomic<uint64_t>& done) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  const uint64_t bit = (dev >= 0 && dev < 64) ? (uint64_t{1} << dev) : 0;
  if (bit != 0 && (done.load(std::memory_order_acquire) & bit) != 0) return true;
  if (cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess) return false;
  done.fetch_or(bit, std::memory_order_acq_rel);
  return true;
}

// Byte offsets of the tile map's arrays inside its device buffer.
struct MapLayout {
  size_t kminmax, tile_class, tile_list, tile_count, order, err, total;
};

inline bool map_layout(int32_t B, int32_t Hm, int32_t Nq, int32_t Nk, int32_t bq, int32_t bk,
                       MapLayout* L) {
  if (B <= 0 || Hm <= 0 || Nq < 0 || Nk < 0) return false;
  if ((bq != 64 && bq != 128) || (bk != 64 && bk != 128)) return false;
  const size_t nqt = static_cast<size_t>(cdiv64(Nq, bq));
  const size_t nkt = static_cast<size_t>(cdiv64(Nk, bk));
  const size_t bh = static_cast<size_t>(B) * static_cast<size_t>(Hm);
  size_t off = 0;
  L->kminmax = off;    off = align256(off + bh * nkt * 8 * sizeof(int32_t));
  L->tile_class = off; off = align256(off + bh * nqt * nkt);
  L->tile_list = off;  off = align256(off + bh * nqt * nkt * sizeof(int32_t));
  L->tile_count = off; off = align256(off + bh * nqt * sizeof(int32_t));
  L->order = off;      off = align256(off + bh * nqt * sizeof(int32_t));
  L->err = off;        off = align256(off + 4 * sizeof(uint32_t));  // error word + 2 scheduling words
  L->total = off;
  return true;
}

// Mask fields a kernel needs, passed by value.
struct MaskArgs {
  int32_t kind, B, Hm, Nq, Nk, sel_k;
  const int32_t *lts, *lte, *uts, *ute;
  int32_t pre, nxt;  // band parameters clamped to +-(Nq + Nk + 1): same mask, no overflow
  const int32_t* sel;
};

inline int32_t clamp_band(int64_t x, int64_t lim) {
  if (x > lim) return static_cast<int32_t>(lim);
  if (x < -lim) return static_cast<int32_t>(-lim);
  return static_cast<int32_t>(x);
}

inline MaskArgs mask_args(const mfa_mask_desc* d) {
  MaskArgs m;
  m.kind = d->kind; m.B = d->B; m.Hm = d->Hm; m.Nq = d->Nq; m.Nk = d->Nk; m.sel_k = d->sel_k;
  const bool lt = d->lts && d->lte, ut = d->uts && d->ute;
  m.lts = lt ? d->lts : nullptr; m.lte = lt ? d->lte : nullptr;
  m.uts = ut ? d->uts : nullptr; m.ute = ut ? d->ute : nullptr;
  const int64_t lim = static_cast<int64_t>(d->Nq) + d->Nk + 1;
  m.pre = clamp_band(d->pre_tokens, lim);
  m.nxt = clamp_band(d->next_tokens, lim);
  m.sel = d->sel;
  return m;
}

// Host validation of a mask description (no device access).
inline mfa_status check_mask(const mfa_mask_desc* d) {
  if (!d) return MFA_ERR_INVALID_ARG;
  if (d->B <= 0 || d->Hm <= 0 || d->Nq < 0 || d->Nk < 0) return MFA_ERR_INVALID_ARG;
  if (static_cast<int64_t>(d->Nq) + d->Nk >= (int64_t(1) << 30)) return MFA_ERR_UNSUPPORTED;
  switch (d->kind) {
    case MFA_MASK_COLWISE: return MFA_OK;
    case MFA_MASK_BAND: return MFA_OK;
    case MFA_MASK_BLOCKSEL:
      if (!d->sel || d->sel_k <= 0) return MFA_ERR_INVALID_ARG;
      if (d->sel_block != kSelBlock || d->sel_k > kMaxSelK) return MFA_ERR_UNSUPPORTED;
      return MFA_OK;
    default: return MFA_ERR_INVALID_ARG;
  }
}

inline mfa_status check_map_matches(const mfa_mask_desc* d, const mfa_tile_map* m) {
  if (!m || !m->kminmax || !m->tile_class || !m->tile_list || !m->tile_count || !m->order || !m->err)
    return MFA_ERR_INVALID_ARG;
  if (m->B != d->B || m->Hm != d->Hm || m->Nq != d->Nq || m->Nk != d->Nk) return MFA_ERR_SHAPE_MISMATCH;
  MapLayout L;
  if (!map_layout(m->B, m->Hm, m->Nq, m->Nk, m->block_q, m->block_k, &L)) return MFA_ERR_INVALID_ARG;
  if (m->nqt != cdiv64(m->Nq, m->block_q) || m->nkt != cdiv64(m->Nk, m->block_k))
    return MFA_ERR_SHAPE_MISMATCH;
  return MFA_OK;
}

// Every host-side check mfa_fwd / mfa_fwd_bias make on their arguments except
// those on the tile map itself, for a map with `block_q`-row tiles (bias may
// be NULL). MFA_OK when the forward pass can run.
mfa_status check_fwd_args(const mfa_tensor* q, const mfa_tensor* k, const mfa_tensor* v, const mfa_mask_desc* mask,
                          const mfa_bias* bias, const mfa_tensor* out, const float* lse, int32_t block_q);

// fp32 inputs: the same tile map walked by an fp32 CUDA-core kernel
// (fwd_f32_simt.cu). Arguments are already validated by mfa_fwd.
mfa_status launch_fwd_f32(const mfa_tensor* q, const mfa_tensor* k, const mfa_tensor* v, const mfa_mask_desc* mask,
                          const mfa_tile_map* map, const mfa_tensor* out, float* lse, cudaStream_t s);

}  // namespace mfa
