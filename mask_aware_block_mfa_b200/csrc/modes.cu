// mfa_mask_from_sparse_mode: the Ascend sparse modes (Ascend CANN "sparseMode
// introduction" page, one paragraph per mode) as the library's compact mask
// descriptions.
//
// Band-type modes are a band with shifted tokens (host only). The prefix and
// varlen modes become column-wise row intervals: every key column j masks the
// query rows outside one visible interval [v0, v1), which is the two masked
// intervals UT = [0, v0) and LT = [v1, Nq) of FlashMask's format. One thread
// per (batch, key column) writes them.
#include <climits>
#include <cstdint>
#include <cuda_runtime.h>

#include "mfa.h"

namespace mfa {
namespace {

__device__ __forceinline__ int64_t clamp64(int64_t x, int64_t lo, int64_t hi) { return x < lo ? lo : (x > hi ? hi : x); }

// Sequence s spans queries [q_end(s-1), q_end(s)) and keys [k_end(s-1), k_end(s)),
// ends clamped to the shape (the caller's ends do not decrease).
struct Seqs {
  const int64_t* q;
  const int64_t* k;
  int n, Nq, Nk;
  __device__ int64_t qe(int s) const { return s < 0 ? 0 : clamp64(q[s], 0, Nq); }
  __device__ int64_t ke(int s) const { return s < 0 ? 0 : clamp64(k[s], 0, Nk); }
  __device__ bool nonempty(int s) const { return qe(s) > qe(s - 1) && ke(s) > ke(s - 1); }
};

__global__ void k_sparse_mode_colwise(int mode, int Nq, int Nk, int64_t pre, int64_t nxt,
                                      const int64_t* __restrict__ prefix, const int64_t* __restrict__ seq_q,
                                      const int64_t* __restrict__ seq_kv, int n_seq, int32_t* __restrict__ lts,
                                      int32_t* __restrict__ lte, int32_t* __restrict__ uts,
                                      int32_t* __restrict__ ute) {
  const int b = blockIdx.y;
  const int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t d = static_cast<int64_t>(Nk) - Nq;
  int64_t v0 = 0, v1 = Nq;  // visible query rows of column j
  if (mode == 5 || mode == 6) {
    if (j >= clamp64(prefix[b], 0, Nk)) v0 = clamp64(j - d, 0, Nq);  // rightDownCausal: masked rows i < j - d
  } else {
    // Modes 7 / 8: the band sequence is the last (7) or first (8) non-empty one.
    const Seqs sq{seq_q, seq_kv, n_seq, Nq, Nk};
    __shared__ int s_band;
    if (threadIdx.x == 0) s_band = mode == 7 ? -1 : INT_MAX;
    __syncthreads();
    for (int s = threadIdx.x; s < n_seq; s += blockDim.x) {
      if (!sq.nonempty(s)) continue;
      if (mode == 7) atomicMax(&s_band, s);
      else atomicMin(&s_band, s);
    }
    __syncthreads();
    const int band = s_band;
    if (j >= Nk) return;
    // The sequence holding key j: the first s with k_end(s) > j.
    int lo = 0, hi = n_seq;
    while (lo < hi) {
      const int mid = (lo + hi) / 2;
      if (sq.ke(mid) > j) hi = mid;
      else lo = mid + 1;
    }
    const int s = lo;
    if (s >= n_seq || !(j >= sq.ke(s - 1))) {
      v0 = v1 = 0;  // past the last sequence: masked for every query
    } else {
      const int64_t q0 = sq.qe(s - 1), q1 = q0 > sq.qe(s) ? q0 : sq.qe(s);
      const int64_t k0 = sq.ke(s - 1);
      const int64_t lq = q1 - q0, lk = sq.ke(s) - k0, lj = j - k0;
      if (s == band) {
        // -pre <= lj - li - (lk - lq) <= nxt
        v0 = q0 + clamp64(lj - (lk - lq) - nxt, 0, lq);
        v1 = q0 + clamp64(lj - (lk - lq) + pre + 1, 0, lq);
      } else if (mode == 7) {
        v0 = q0 + clamp64(lj - (lk - lq), 0, lq);  // rightDownCausal in the sequence
        v1 = q1;
      } else {
        v0 = q0 + clamp64(lj, 0, lq);  // leftUpCausal in the sequence
        v1 = q1;
      }
      if (v1 < v0) v1 = v0;
    }
  }
  if (j >= Nk) return;
  const size_t idx = static_cast<size_t>(b) * Nk + j;
  uts[idx] = 0;
  ute[idx] = static_cast<int32_t>(v0);
  lts[idx] = static_cast<int32_t>(v1 < Nq ? v1 : Nq);
  lte[idx] = Nq;
}

}  // namespace
}  // namespace mfa

extern "C" mfa_status mfa_mask_from_sparse_mode(const mfa_sparse_mode* sm, int32_t B, int32_t Nq, int32_t Nk,
                                                int32_t* lts, int32_t* lte, int32_t* uts, int32_t* ute,
                                                mfa_mask_desc* out, void* stream) {
  using namespace mfa;
  if (!sm || !out || B < 0 || B > 65535 || Nq < 0 || Nk < 0) return MFA_ERR_INVALID_ARG;
  const int mode = sm->mode;
  if (mode == 1 || mode < 0 || mode > 8) return MFA_ERR_UNSUPPORTED;
  mfa_mask_desc d{};
  d.B = B;
  d.Hm = 1;
  d.Nq = Nq;
  d.Nk = Nk;
  d.map = nullptr;
  const int64_t shift = static_cast<int64_t>(Nk) - Nq;
  const int64_t all = static_cast<int64_t>(Nq) + Nk;  // more than any |j - i|
  if (mode == 0 || mode == 2 || mode == 3 || mode == 4) {
    d.kind = MFA_MASK_BAND;
    if (mode == 0) {
      d.pre_tokens = sm->pre_tokens;
      d.next_tokens = sm->next_tokens;
    } else if (mode == 2) {
      d.pre_tokens = all;
      d.next_tokens = 0;
    } else if (mode == 3) {
      d.pre_tokens = all;
      d.next_tokens = shift;
    } else {
      d.pre_tokens = sm->pre_tokens - shift;
      d.next_tokens = sm->next_tokens + shift;
    }
    *out = d;
    return MFA_OK;
  }
  if (!lts || !lte || !uts || !ute) return MFA_ERR_INVALID_ARG;
  if ((mode == 5 || mode == 6) && !sm->prefix && B > 0) return MFA_ERR_INVALID_ARG;
  if ((mode == 7 || mode == 8) && (B != 1 || sm->n_seq < 1 || !sm->seq_q || !sm->seq_kv)) return MFA_ERR_INVALID_ARG;
  d.kind = MFA_MASK_COLWISE;
  d.lts = lts;
  d.lte = lte;
  d.uts = uts;
  d.ute = ute;
  if (B > 0 && Nk > 0) {
    constexpr int kThreads = 256;
    const dim3 grid((Nk + kThreads - 1) / kThreads, B);
    // Tokens beyond +-(Nq + Nk + 1) act like that bound (no |j - i| reaches it).
    const int64_t pre = sm->pre_tokens < -all - 1 ? -all - 1 : (sm->pre_tokens > all + 1 ? all + 1 : sm->pre_tokens);
    const int64_t nxt =
        sm->next_tokens < -all - 1 ? -all - 1 : (sm->next_tokens > all + 1 ? all + 1 : sm->next_tokens);
    k_sparse_mode_colwise<<<grid, kThreads, 0, static_cast<cudaStream_t>(stream)>>>(
        mode, Nq, Nk, pre, nxt, sm->prefix, sm->seq_q, sm->seq_kv, sm->n_seq, lts, lte, uts, ute);
    if (cudaGetLastError() != cudaSuccess) return MFA_ERR_CUDA;
  }
  *out = d;
  return MFA_OK;
}
