// mfa_build_tile_map: reduce a compact mask description to the per-tile
// SKIP / FULL / PARTIAL map and the compacted per-query-tile key-tile lists.
//
// Binary Block Masking ("Efficiently Dispatching Flash Attention For Partially
// Filled Attention Masks", abstract) classifies tiles so that fully masked
// tiles are skipped and fully visible ones run without the element mask. The
// classification here works from per-key-tile minima and maxima of the
// column-wise row intervals (FlashMask's O(N) description), so the map costs
// O(N) reads plus O(nqt * nkt) integer work, never an N x N mask.
//
// Two launches on the caller's stream:
//   k_tile_minmax    grid (nkt, B*Hm), block BK: per k-tile min/max of the
//                    (normalised) bounds; validates them.
//   k_tile_classify  grid (nqt, B*Hm), block 256: class of every (qt, kt),
//                    ordered compaction of the non-SKIP kt, count; the block
//                    that finishes last (a counter in err[3]) then sorts the
//                    q-tiles by count, largest first (the forward pass's work
//                    order), which saves a third launch per build.
#include <climits>
#include <cuda_runtime.h>

#include "mfa.h"
#include "mfa_internal.h"
#include "order.cuh"

namespace mfa {
namespace {

constexpr int kSkip = 0, kFull = 1, kPartial = 2;

__device__ __forceinline__ int clampi(long long x, int lo, int hi) {
  return static_cast<int>(x < lo ? lo : (x > hi ? hi : x));
}

__device__ __forceinline__ int warp_min(int v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = min(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ int warp_max(int v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Column j's four bounds (lts, lte, uts, ute); an empty interval becomes
// (Nq, 0). Out-of-range bounds flag MFA_DEVERR_BOUNDS and are clamped.
__device__ __forceinline__ void column_bounds(const MaskArgs& m, int bh, int j, int (&c)[4],
                                              uint32_t* err) {
  const int Nq = m.Nq;
  if (m.kind == MFA_MASK_BAND) {
    c[0] = clampi(static_cast<long long>(j) + m.pre + 1, 0, Nq);  // LT = [j + pre + 1, Nq)
    c[1] = Nq;
    c[2] = 0;                                                       // UT = [0, j - next)
    c[3] = clampi(static_cast<long long>(j) - m.nxt, 0, Nq);
  } else {
    const size_t idx = static_cast<size_t>(bh) * m.Nk + j;
    c[0] = m.lts ? m.lts[idx] : 0;
    c[1] = m.lte ? m.lte[idx] : 0;
    c[2] = m.uts ? m.uts[idx] : 0;
    c[3] = m.ute ? m.ute[idx] : 0;
    bool bad = false;
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      if (c[a] < 0 || c[a] > Nq) {
        bad = true;
        c[a] = c[a] < 0 ? 0 : Nq;
      }
    }
    if (bad) atomicOr(err, MFA_DEVERR_BOUNDS);
  }
#pragma unroll
  for (int a = 0; a < 4; a += 2) {
    if (c[a] >= c[a + 1]) {
      c[a] = Nq;
      c[a + 1] = 0;
    }
  }
}

__global__ void k_tile_minmax(MaskArgs m, int BK, int nkt, int32_t* __restrict__ kmm,
                              uint32_t* __restrict__ err) {
  const int kt = blockIdx.x, bh = blockIdx.y, t = threadIdx.x;
  int32_t* out = kmm + (static_cast<size_t>(bh) * nkt + kt) * 8;
  if (m.kind == MFA_MASK_BLOCKSEL) {
    if (t < 8) out[t] = 0;
    return;
  }
  const int j = kt * BK + t;
  int mn[4], mx[4];
  if (j < m.Nk) {
    int c[4];
    column_bounds(m, bh, j, c, err);
#pragma unroll
    for (int a = 0; a < 4; ++a) mn[a] = mx[a] = c[a];
  } else {
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      mn[a] = INT_MAX;
      mx[a] = INT_MIN;
    }
  }
  __shared__ int s_mn[4][4], s_mx[4][4];  // [warp][bound], BK <= 128
  const int w = t >> 5, lane = t & 31;
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    const int a_mn = warp_min(mn[a]), a_mx = warp_max(mx[a]);
    if (lane == 0) {
      s_mn[w][a] = a_mn;
      s_mx[w][a] = a_mx;
    }
  }
  __syncthreads();
  if (t < 8) {
    const int a = t >> 1;
    const bool want_max = t & 1;
    int r = want_max ? INT_MIN : INT_MAX;
    for (int ww = 0; ww < (BK + 31) / 32; ++ww) r = want_max ? max(r, s_mx[ww][a]) : min(r, s_mn[ww][a]);
    out[t] = r;
  }
}

// Exclusive block-wide prefix count of `flag` over 256 threads; returns the
// prefix and writes the block total to *total.
__device__ __forceinline__ int block_scan256(bool flag, int* s_warp, int* total) {
  const int t = threadIdx.x, w = t >> 5, lane = t & 31;
  const unsigned bal = __ballot_sync(0xffffffffu, flag);
  const int in_warp = __popc(bal & ((1u << lane) - 1u));
  if (lane == 0) s_warp[w] = __popc(bal);
  __syncthreads();
  int before = 0, sum = 0;
#pragma unroll
  for (int ww = 0; ww < 8; ++ww) {
    const int c = s_warp[ww];
    if (ww < w) before += c;
    sum += c;
  }
  *total = sum;
  __syncthreads();  // s_warp is reused by the next chunk
  return before + in_warp;
}

__global__ void __launch_bounds__(256) k_tile_classify(MaskArgs m, int BQ, int BK, int nqt, int nkt,
                                                       const int32_t* __restrict__ kmm,
                                                       uint8_t* __restrict__ cls,
                                                       int32_t* __restrict__ list,
                                                       int32_t* __restrict__ count,
                                                       int32_t* __restrict__ order,
                                                       uint32_t* __restrict__ err) {
  extern __shared__ int s_sel[];  // BLOCKSEL: [BQ/64][sel_k]; then the order histogram
  __shared__ int s_warp[8];
  const int qt = blockIdx.x, bh = blockIdx.y, t = threadIdx.x;
  const size_t e = static_cast<size_t>(bh) * nqt + qt;
  const int r0 = qt * BQ, r1 = min(r0 + BQ, m.Nq);
  const int nqs = (m.Nq + kSelBlock - 1) / kSelBlock, nks = (m.Nk + kSelBlock - 1) / kSelBlock;
  const int qs_per = BQ / kSelBlock, ks_per = BK / kSelBlock;

  if (m.kind == MFA_MASK_BLOCKSEL) {
    for (int i = t; i < qs_per * m.sel_k; i += blockDim.x) {
      const int qsl = i / m.sel_k, slot = i % m.sel_k;
      const int qs = qt * qs_per + qsl;
      int v = -1;
      if (qs < nqs) {
        v = m.sel[(static_cast<size_t>(bh) * nqs + qs) * m.sel_k + slot];
        if (v < -1 || v >= nks) {
          atomicOr(err, MFA_DEVERR_SEL);
          v = -1;
        }
      }
      s_sel[i] = v;
    }
    __syncthreads();
  }

  int running = 0;
  for (int base = 0; base < nkt; base += 256) {
    const int kt = base + t;
    int c = kSkip;
    if (kt < nkt) {
      if (m.kind == MFA_MASK_BLOCKSEL) {
        bool all_empty = true, all_full = true;
        int bits = 0;
        for (int qsl = 0; qsl < qs_per; ++qsl) {
          const int qs = qt * qs_per + qsl;
          if (qs >= nqs) continue;
          for (int ksl = 0; ksl < ks_per; ++ksl) {
            const int ks = kt * ks_per + ksl;
            if (ks >= nks) continue;
            bool listed = false;
            for (int s = 0; s < m.sel_k; ++s) listed |= (s_sel[qsl * m.sel_k + s] == ks);
            if (!listed || ks > qs) {
              all_full = false;
            } else {
              all_empty = false;
              if (ks == qs) all_full = false;
              bits |= 1 << (4 + 2 * qsl + ksl);
            }
          }
        }
        c = (all_empty ? kSkip : (all_full ? kFull : kPartial)) | bits;
      } else {
        const int32_t* mm = kmm + (static_cast<size_t>(bh) * nkt + kt) * 8;
        const int lts_min = mm[0], lts_max = mm[1], lte_min = mm[2], lte_max = mm[3];
        const int uts_min = mm[4], uts_max = mm[5], ute_min = mm[6], ute_max = mm[7];
        const bool lt_covers = lts_max <= r0 && lte_min >= r1;
        const bool ut_covers = uts_max <= r0 && ute_min >= r1;
        if (lt_covers || ut_covers) {
          c = kSkip;
        } else {
          const bool lt_clear = lts_min >= r1 || lte_max <= r0;
          const bool ut_clear = uts_min >= r1 || ute_max <= r0;
          c = (lt_clear && ut_clear) ? kFull : kPartial;
        }
      }
      cls[e * nkt + kt] = static_cast<uint8_t>(c);
    }
    const bool keep = kt < nkt && (c & 3) != kSkip;
    int total;
    const int pos = block_scan256(keep, s_warp, &total);
    if (keep) list[e * nkt + running + pos] = kt;
    running += total;
  }
  if (t == 0) count[e] = running;
  for (int kt = running + t; kt < nkt; kt += 256) list[e * nkt + kt] = -1;

  // The last block to finish (counter err[3], cleared with the error word at
  // the start of the build) sorts the q-tiles; the fences order every block's
  // count before its increment and the increments before the last block's
  // reads.
  __shared__ bool s_last;
  if (t == 0) {
    __threadfence();
    const uint32_t n_blocks = gridDim.x * gridDim.y;
    s_last = atomicAdd(&err[3], 1u) == n_blocks - 1;
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  order_by_count_desc(count, static_cast<int>(gridDim.y) * nqt, nkt, order, s_sel);
  if (t == 0) err[3] = 0;
}

}  // namespace
}  // namespace mfa

extern "C" mfa_status mfa_build_tile_map(const mfa_mask_desc* mask, mfa_tile_map* map, void* stream) {
  using namespace mfa;
  mfa_status st = check_mask(mask);
  if (st != MFA_OK) return st;
  st = check_map_matches(mask, map);
  if (st != MFA_OK) return st;
  if (mask->kind == MFA_MASK_BLOCKSEL &&
      static_cast<size_t>(map->block_q / kSelBlock) * mask->sel_k * sizeof(int) > 48 * 1024)
    return MFA_ERR_UNSUPPORTED;
  if (static_cast<size_t>(map->nkt + 1) * sizeof(int) > 200 * 1024) return MFA_ERR_UNSUPPORTED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const MaskArgs m = mask_args(mask);
  map->kind = mask->kind;
  if (cudaMemsetAsync(map->err, 0, 4 * sizeof(uint32_t), s) != cudaSuccess) return MFA_ERR_CUDA;
  const int BH = mask->B * mask->Hm;
  if (map->nkt > 0) {
    k_tile_minmax<<<dim3(map->nkt, BH), map->block_k, 0, s>>>(m, map->block_k, map->nkt, map->kminmax,
                                                               map->err);
  }
  if (map->nqt > 0) {
    const size_t sel_smem =
        mask->kind == MFA_MASK_BLOCKSEL ? static_cast<size_t>(map->block_q / kSelBlock) * mask->sel_k * sizeof(int) : 0;
    const size_t ord_smem = static_cast<size_t>(map->nkt + 1) * sizeof(int);
    const size_t smem = sel_smem > ord_smem ? sel_smem : ord_smem;
    if (smem > 48 * 1024 &&
        cudaFuncSetAttribute(k_tile_classify, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
      return MFA_ERR_CUDA;
    k_tile_classify<<<dim3(map->nqt, BH), 256, smem, s>>>(m, map->block_q, map->block_k, map->nqt, map->nkt,
                                                           map->kminmax, map->tile_class, map->tile_list,
                                                           map->tile_count, map->order, map->err);
  }
  return cudaGetLastError() == cudaSuccess ? MFA_OK : MFA_ERR_CUDA;
}
