// mfa_decode: selected-key attention for a few query rows (decode) on sm_100a.
//
// Each (batch b, key/value head g, query row i) has a list of 64-key blocks
// ("vulkan : selected-key flash attention for QSA block selection", overview
// and kernel description): -1 entries are skipped, a block listed twice counts
// once, and the list is shared by the G query heads of head g. Query row i
// sits at position i + Nk - Nq and sees only keys at or before it (the forward
// pass's block-selection rule when Nq == Nk). The work is a gather of whole
// 64-key K/V blocks, so it is bound by HBM, not by the tensor cores: with G
// query rows per block there is little to multiply, and the CUDA cores keep up
// with the memory (for D = 256, G = 4 a 64 KB block takes ~2,850 cycles of an
// SM's share of HBM and ~1,000 FMA cycles).
//
// Split-K, as in the pull request: a list is cut into n_split parts handled by
// different CTAs; each writes an unnormalised partial (m, l, o), and a second
// kernel combines them. An empty part writes m = -FLT_MAX, not -inf, so the
// combination never evaluates exp(-inf - -inf).
//
// CTA = (part, query row, batch x key/value head), 256 threads (8 warps).
//   1. The list is deduplicated in shared memory (first occurrence kept,
//      entries outside [-1, ceil(Nk / 64)) flagged, blocks after the row's
//      position dropped) and the part's share of it taken.
//   2. K and V blocks arrive by TMA (64-column SW128 boxes) in a two-stage ring.
//   3. Scores: lane l holds head dimensions [DL l, DL l + DL) of all G query
//      rows in registers (DL = D / 32); each warp takes 64 / warps keys of the
//      block, reads each key row once (conflict-free through the swizzle) and
//      reduces the G partial dot products across lanes by halving transposes
//      (G - 1 + 5 - log2 G shuffles).
//   4. Online softmax per warp: each warp keeps its own running max and sum
//      of every query row and its own partial outputs over the keys it
//      handles (a split-K inside the CTA), so no block-wide barrier runs per
//      block; a stage is released by one arrival per warp.
//   5. P.V: lane l owns the same head dimensions of all G rows for the
//      warp's keys; the warps' partials are combined once at the end, each
//      rescaled by 2^(its max - the row's max).
#include <cfloat>
#include <climits>
#include <cmath>
#include <cstring>
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include "mfa.h"
#include "mfa_device.cuh"
#include "mfa_internal.h"

namespace mfa {
namespace {

constexpr int kBlk = 64;       // keys per selection block
constexpr int kCombineThreads = 256;
// 16 warps when the query rows and outputs fit 128 registers a thread
// (G * D <= 1024), else 8: more warps hide more of the shared-memory and
// shuffle latency of the one CTA that fits an SM.
template <int D, int G>
constexpr int kWarpsFor = G * D <= 1024 ? 16 : 8;

struct DecParams {
  int32_t B, Hq, Hkv, G, Nq, Nk, nblk, sel_k, n_split;
  float scale_log2;
  const int32_t* sel;  // [B, Hkv, Nq, sel_k]
  const __nv_bfloat16* q;
  int64_t qs0, qs1, qs2;
  __nv_bfloat16* out;
  int64_t os0, os1, os2;
  float* lse;          // [B, Hq, Nq]
  float* o_part;       // [B * Hkv * Nq][n_split][G][D]   (n_split > 1)
  float* ml_part;      // [B * Hkv * Nq][n_split][G][2]   (m, l)
  uint32_t* err;
};

template <int D>
struct DecCfg {
  static constexpr int kDL = D / 32;                 // head dimensions per lane
  static constexpr int kTile = kBlk * D * 2;         // one K (or V) block: D / 64 boxes of 64 rows x 128 B
  static constexpr int kStages = 3;                  // K/V ring: two blocks in flight while one is used
  static constexpr int kK = 0;                       // [kStages]
  static constexpr int kV = kK + kStages * kTile;    // [kStages]
  static constexpr int kS = kV + kStages * kTile;    // list scratch, then per-warp (m, l) at the end
  static constexpr int kList = kS + 2 * 16 * kBlk * 4;  // deduplicated list [kMaxSelK]
  static constexpr int kMisc = kList + kMaxSelK * 4; // softmax state, counters, barriers
  static constexpr int kBytes = kMisc + 1024;
  // The final combine of the warps' outputs reuses the K/V ring (16 warps with
  // G * D <= 1024 or 8 warps with G * D <= 2048); the warps' (m, l) go to the
  // space after the ring.
  static_assert(16 * 32 * (1024 / D * kDL + 1) * 4 <= kS, "output reduction space (16 warps)");
  static_assert(8 * 32 * (2048 / D * kDL + 1) * 4 <= kS, "output reduction space (8 warps)");
  static_assert(2 * 16 * 16 * 4 <= kList - kS, "per-warp (m, l)");
};

// Element offset of head dimensions [c0, c0 + n) of key row r in a K/V block
// written by TMA with 64-column SW128 boxes: box c0 / 64, 16-byte chunk
// (c0 % 64) / 8 placed at chunk ^ (r % 8). n <= 8 and within one chunk.
__device__ __forceinline__ uint32_t sw_off(int r, int c0) {
  const int box = c0 >> 6, ch = (c0 & 63) >> 3;
  return static_cast<uint32_t>(box * (kBlk * 128) + r * 128 + ((ch ^ (r & 7)) << 4) + (c0 & 7) * 2);
}

// A bf16 pair widened to a packed float pair: bf16 is the upper half of a float.
__device__ __forceinline__ uint64_t bf2_to_f2(uint32_t w) {
  return f2_pack(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}

// Head dimensions [DL lane, DL lane + DL) of key row r as DL / 2 packed pairs.
template <int DL>
__device__ __forceinline__ void load_row2(const uint8_t* tile, int r, int lane, uint64_t (&x)[DL / 2]) {
  const uint8_t* p = tile + sw_off(r, lane * DL);
  if constexpr (DL == 8) {
    const uint4 w = *reinterpret_cast<const uint4*>(p);
    x[0] = bf2_to_f2(w.x); x[1] = bf2_to_f2(w.y); x[2] = bf2_to_f2(w.z); x[3] = bf2_to_f2(w.w);
  } else {
    const uint2 w = *reinterpret_cast<const uint2*>(p);
    x[0] = bf2_to_f2(w.x); x[1] = bf2_to_f2(w.y);
  }
}

// Sum v[0 .. G) over the 32 lanes. Afterwards lane l holds the total of
// value index (l >> (5 - log2 G)) in v[0]: at distance 16, 8, ... each lane
// keeps the half of its values whose index bit matches its own lane bit and
// adds the partner's copy of that half; the remaining steps are a butterfly.
template <int G>
__device__ __forceinline__ float reduce_rows(float (&v)[G], int lane) {
  int n = G, dist = 16;
#pragma unroll
  for (int step = 0; step < 5; ++step, dist >>= 1) {
    if (n > 1) {
      const int half = n >> 1;
      const bool upper = (lane & dist) != 0;
#pragma unroll
      for (int x = 0; x < G / 2; ++x) {
        if (x < half) {
          const float send = upper ? v[x] : v[x + half];
          const float recv = __shfl_xor_sync(0xffffffffu, send, dist);
          v[x] = (upper ? v[x + half] : v[x]) + recv;
        }
      }
      n = half;
    } else {
      v[0] += __shfl_xor_sync(0xffffffffu, v[0], dist);
    }
  }
  return v[0];
}

template <int G>
__device__ __forceinline__ int row_of_lane(int lane) {
  constexpr int lg = G == 1 ? 0 : G == 2 ? 1 : G == 4 ? 2 : G == 8 ? 3 : 4;
  // value index bits were chosen at distances 16, 8, ...: the first step's
  // bit is the most significant bit of the index
  int idx = 0;
#pragma unroll
  for (int s = 0; s < lg; ++s) idx = (idx << 1) | ((lane >> (4 - s)) & 1);
  return idx;
}

// The first lane that holds row h's total after reduce_rows: h's bits from the
// most significant down sit at lane bits 4, 3, ... (the inverse of row_of_lane).
template <int G>
__device__ __forceinline__ int owner_lane(int h) {
  constexpr int lg = G == 1 ? 0 : G == 2 ? 1 : G == 4 ? 2 : G == 8 ? 3 : 4;
  int lane = 0;
#pragma unroll
  for (int s = 0; s < lg; ++s) lane |= ((h >> (lg - 1 - s)) & 1) << (4 - s);
  return lane;
}

template <int D, int G>
__global__ void __launch_bounds__(kWarpsFor<D, G> * 32, 1)
    mfa_decode_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                      const DecParams p) {
  using C = DecCfg<D>;
  constexpr int DL = C::kDL;
  constexpr int kWarps = kWarpsFor<D, G>;
  constexpr int kThreads = kWarps * 32;
  constexpr int kKeysPerWarp = kBlk / kWarps;
  constexpr int kCk = kKeysPerWarp < 4 ? kKeysPerWarp : 4;  // keys per softmax step
  extern __shared__ __align__(1024) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int part = blockIdx.x, i = blockIdx.y;
  const int bg = blockIdx.z, b = bg / p.Hkv, g = bg % p.Hkv;
  const size_t row_unit = (static_cast<size_t>(bg) * p.Nq + i);

  int* sList = reinterpret_cast<int*>(smem + C::kList);
  int* sCnt = reinterpret_cast<int*>(smem + C::kMisc + 192);   // [kWarps] list compaction, [16] total
  volatile int* sFlag = reinterpret_cast<volatile int*>(sCnt + 20);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kMisc + 512);  // [kStages] block landed
  uint64_t* empty = full + C::kStages;                                   // [kStages] every warp done with it

  if ((smem_u32(smem) & 1023u) != 0u) {  // SW128 boxes need a 1024-aligned base (uniform check)
    if (threadIdx.x == 0) atomicOr(p.err, MFA_DEVERR_TIMEOUT);
    return;
  }
  if (threadIdx.x == 0) {
    for (int st = 0; st < C::kStages; ++st) {
      mbar_init(&full[st], 1);
      mbar_init(&empty[st], kWarps);
    }
    *sFlag = 0;
    fence_mbarrier_init();
  }

  // ---- 1. the row's deduplicated list ----
  const int last = i + p.Nk - p.Nq;  // the row's position; keys after it are hidden
  const int32_t* lrow = p.sel + row_unit * p.sel_k;
  int* sRaw = reinterpret_cast<int*>(smem + C::kS);  // scratch until the first scores
  for (int e = threadIdx.x; e < p.sel_k; e += kThreads) sRaw[e] = lrow[e];
  __syncthreads();
  {
    const int e = threadIdx.x;  // sel_k <= kMaxSelK = 256 <= kThreads
    bool keep = false;
    if (e < p.sel_k) {
      const int v = sRaw[e];
      if (v < -1 || v >= p.nblk) atomicOr(p.err, MFA_DEVERR_SEL);
      keep = v >= 0 && v < p.nblk && static_cast<int64_t>(v) * kBlk <= last;
      for (int e2 = 0; keep && e2 < e; ++e2) keep = sRaw[e2] != v;
    }
    const unsigned bal = __ballot_sync(0xffffffffu, keep);
    if (lane == 0) sCnt[warp] = __popc(bal);
    __syncthreads();
    int base = 0;
    for (int w = 0; w < warp; ++w) base += sCnt[w];
    if (keep) sList[base + __popc(bal & ((1u << lane) - 1u))] = sRaw[e];
    if (threadIdx.x == 0) {
      int tot = 0;
      for (int w = 0; w < kWarps; ++w) tot += sCnt[w];
      sCnt[16] = tot;
    }
    __syncthreads();
  }
  const int n_valid = sCnt[16];
  const int per = (n_valid + p.n_split - 1) / p.n_split;
  const int j0 = min(part * per, n_valid), j1 = min(j0 + per, n_valid);
  const int nb = j1 - j0;

  // ---- query rows in registers (packed pairs), in log2 units ----
  uint64_t qr[G][DL / 2];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    const __nv_bfloat16* qp = p.q + b * p.qs0 + static_cast<int64_t>(g * G + h) * p.qs1 + i * p.qs2 + lane * DL;
#pragma unroll
    for (int e = 0; e < DL; e += 2) {
      const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(qp + e));
      qr[h][e / 2] = f2_pack(f.x * p.scale_log2, f.y * p.scale_log2);
    }
  }
  uint64_t acc[G][DL / 2];
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int e = 0; e < DL / 2; ++e) acc[h][e] = 0ull;  // +0.0f in both halves

  auto issue = [&](int n) {  // thread 0: K and V of the part's n-th block into stage n % kStages
    const int blk = sList[j0 + n], st = n % C::kStages;
    mbar_arrive_expect_tx(&full[st], 2 * C::kTile);
#pragma unroll
    for (int c = 0; c < D / 64; ++c) {
      tma_load_4d(smem + C::kK + st * C::kTile + c * (kBlk * 128), &tm_k, &full[st], c * 64, blk * kBlk, g, b);
      tma_load_4d(smem + C::kV + st * C::kTile + c * (kBlk * 128), &tm_v, &full[st], c * 64, blk * kBlk, g, b);
    }
  };
  int n_issued = 0;  // thread 0's count of blocks whose loads went out
  if (threadIdx.x == 0) {
    n_issued = min(nb, C::kStages);
    for (int n = 0; n < n_issued; ++n) issue(n);
  }
  int n_done = 0;  // blocks this warp has finished

  // Per-warp online softmax: every warp keeps its own running max and sum of
  // each query row (in every lane) and its own partial outputs, over the keys
  // it handles; the warps are combined once after the last block. No
  // block-wide barrier is needed per block: a stage is released by one
  // arrival per warp, and thread 0 refills it when all have arrived.
  float m_w[G], l_w[G];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    m_w[h] = -INFINITY;
    l_w[h] = 0.f;
  }
  for (int n = 0; n < nb; ++n) {
    const int st = n % C::kStages;
    if (!__all_sync(0xffffffffu, mbar_wait(&full[st], (n / C::kStages) & 1, sFlag))) {
      *sFlag = 1;
      break;
    }
    const uint8_t* tK = smem + C::kK + st * C::kTile;
    const uint8_t* tV = smem + C::kV + st * C::kTile;
    const int kbase = sList[j0 + n] * kBlk;

    // The warp's keys in chunks of kCk: scores, softmax update, P.V.
#pragma unroll
    for (int kc = 0; kc < kKeysPerWarp; kc += kCk) {
    // ---- 3. scores of this chunk, gathered into every lane ----
    float tot[kCk];
#pragma unroll
    for (int kk = 0; kk < kCk; ++kk) {
      const int r = warp * kKeysPerWarp + kc + kk;
      uint64_t kx[DL / 2];
      load_row2<DL>(tK, r, lane, kx);
      float part_dot[G];
#pragma unroll
      for (int h = 0; h < G; ++h) {
        uint64_t s2 = f2_fma(qr[h][0], kx[0], 0ull);
#pragma unroll
        for (int e = 1; e < DL / 2; ++e) s2 = f2_fma(qr[h][e], kx[e], s2);
        float lo, hi;
        f2_unpack(s2, lo, hi);
        part_dot[h] = lo + hi;
      }
      tot[kk] = reduce_rows<G>(part_dot, lane);
    }
    float pk[G][kCk];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      // ---- 4. online softmax of row h over these keys ----
      float mx = -INFINITY;
#pragma unroll
      for (int kk = 0; kk < kCk; ++kk) {
        const float v = __shfl_sync(0xffffffffu, tot[kk], owner_lane<G>(h));
        pk[h][kk] = (kbase + warp * kKeysPerWarp + kc + kk <= last) ? v : -INFINITY;
        mx = fmaxf(mx, pk[h][kk]);
      }
      const float m_new = fmaxf(m_w[h], mx);
      const float m_use = m_new == -INFINITY ? 0.f : m_new;
      const float alpha = ex2_approx(m_w[h] - m_use);  // 0 while nothing was visible
      float sum = 0.f;
#pragma unroll
      for (int kk = 0; kk < kCk; ++kk) {
        pk[h][kk] = ex2_approx(pk[h][kk] - m_use);
        sum += pk[h][kk];
      }
      l_w[h] = l_w[h] * alpha + sum;
      m_w[h] = m_new;
      if (alpha != 1.f) {  // the same in every lane: no divergence
        const uint64_t a2 = f2_pack(alpha, alpha);
#pragma unroll
        for (int e = 0; e < DL / 2; ++e) acc[h][e] = f2_fma(acc[h][e], a2, 0ull);
      }
    }

    // ---- 5. P.V of these keys ----
#pragma unroll
    for (int kk = 0; kk < kCk; ++kk) {
      const int r = warp * kKeysPerWarp + kc + kk;
      uint64_t vx[DL / 2];
      load_row2<DL>(tV, r, lane, vx);
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const uint64_t p2 = f2_pack(pk[h][kk], pk[h][kk]);
#pragma unroll
        for (int e = 0; e < DL / 2; ++e) acc[h][e] = f2_fma(p2, vx[e], acc[h][e]);
      }
    }
    }  // key chunks
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[st]);
    n_done = n + 1;
    // Thread 0 refills stage st with block n + kStages once every warp has released it.
    if (threadIdx.x == 0 && n + C::kStages < nb) {
      if (mbar_wait(&empty[st], (n / C::kStages) & 1, sFlag)) {
        issue(n + C::kStages);
        n_issued = n + C::kStages + 1;
      } else {
        *sFlag = 1;
      }
    }
  }
  __syncthreads();
  const bool aborted = *sFlag != 0;
  if (aborted && threadIdx.x == 0) {
    atomicOr(p.err, MFA_DEVERR_TIMEOUT);
    // let the copies already issued land before shared memory is released
    volatile int no_abort = 0;
    for (int n = n_done; n < n_issued; ++n) mbar_wait(&full[n % C::kStages], (n / C::kStages) & 1, &no_abort);
  }
  if (aborted) return;

  // ---- combine the warps (reusing the K/V ring and the score space) ----
  // Rows of G * DL + 1 floats, so the 32 lanes' stores fall in different banks.
  constexpr int kRow = G * DL + 1;
  float* red = reinterpret_cast<float*>(smem + C::kK);   // [kWarps][32 lanes][kRow]
  float* sMw = reinterpret_cast<float*>(smem + C::kS);    // [kWarps][G] running max
  float* sLw = sMw + kWarps * G;                          // [kWarps][G] running sum
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int e = 0; e < DL / 2; ++e) {
      float lo, hi;
      f2_unpack(acc[h][e], lo, hi);
      red[(warp * 32 + lane) * kRow + h * DL + 2 * e] = lo;
      red[(warp * 32 + lane) * kRow + h * DL + 2 * e + 1] = hi;
    }
  if (lane == 0) {
#pragma unroll
    for (int h = 0; h < G; ++h) {
      sMw[warp * G + h] = m_w[h];
      sLw[warp * G + h] = l_w[h];
    }
  }
  __syncthreads();
  // Element (h, dimension) = (h, DL * l + e) lives at lane l, slot h * DL + e of every warp.
  for (int it = threadIdx.x; it < G * D; it += kThreads) {
    const int h = it / D, d = it % D;
    const int l = d / DL, e = d % DL;
    float m = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) m = fmaxf(m, sMw[w * G + h]);
    const float m_use = m == -INFINITY ? 0.f : m;
    float o = 0.f, lsum = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const float wt = ex2_approx(sMw[w * G + h] - m_use);  // 0 for a warp that saw no key
      o = fmaf(wt, red[(w * 32 + l) * kRow + h * DL + e], o);
      lsum = fmaf(wt, sLw[w * G + h], lsum);
    }
    if (p.n_split == 1) {
      const bool has = lsum > 0.f;
      const float v = has ? o / lsum : 0.f;
      __nv_bfloat16* orow = p.out + b * p.os0 + static_cast<int64_t>(g * G + h) * p.os1 + i * p.os2;
      orow[d] = __float2bfloat16_rn(v);
      if (d == 0)
        p.lse[(static_cast<size_t>(b) * p.Hq + g * G + h) * p.Nq + i] =
            has ? (m + __log2f(lsum)) * 0.69314718055994530942f : -INFINITY;
    } else {
      const size_t pu = row_unit * p.n_split + part;
      p.o_part[(pu * G + h) * D + d] = o;
      if (d == 0) {
        // An empty part (or one that saw no visible key) carries m = -FLT_MAX, l = 0.
        p.ml_part[(pu * G + h) * 2] = (m == -INFINITY) ? -FLT_MAX : m;
        p.ml_part[(pu * G + h) * 2 + 1] = lsum;
      }
    }
  }
}

// Combine the n_split partials of every (batch, key/value head, row): with
// M = max m_s, out = sum o_s 2^(m_s - M) / sum l_s 2^(m_s - M). All parts
// empty gives M = -FLT_MAX, weights 1 on zeros, l = 0: out = 0, lse = -inf.
// One thread per output element, grid (rows, ceil(G * D / kCombineThreads)):
// every thread waits for two rounds of loads only (the parts' m, then their
// o and l), and the rows' CTAs spread over all SMs.
template <int D, int G>
__global__ void __launch_bounds__(kCombineThreads) mfa_decode_combine(const DecParams p) {
  const size_t ru = blockIdx.x;  // (bg, i)
  const int bg = static_cast<int>(ru / p.Nq), i = static_cast<int>(ru % p.Nq);
  const int b = bg / p.Hkv, g = bg % p.Hkv;
  const int it = blockIdx.y * kCombineThreads + threadIdx.x;
  if (it < G * D) {
    const int h = it / D, d = it % D;
    float M = -FLT_MAX;
    for (int s = 0; s < p.n_split; ++s) M = fmaxf(M, p.ml_part[((ru * p.n_split + s) * G + h) * 2]);
    float o = 0.f, l = 0.f;
    for (int s = 0; s < p.n_split; ++s) {
      const size_t pu = ru * p.n_split + s;
      const float w = ex2_approx(p.ml_part[(pu * G + h) * 2] - M);
      o = fmaf(w, p.o_part[(pu * G + h) * D + d], o);
      l = fmaf(w, p.ml_part[(pu * G + h) * 2 + 1], l);
    }
    const bool has = l > 0.f;
    __nv_bfloat16* orow = p.out + b * p.os0 + static_cast<int64_t>(g * G + h) * p.os1 + i * p.os2;
    orow[d] = __float2bfloat16_rn(has ? o / l : 0.f);
    if (d == 0)
      p.lse[(static_cast<size_t>(b) * p.Hq + g * G + h) * p.Nq + i] =
          has ? (M + __log2f(l)) * 0.69314718055994530942f : -INFINITY;
  }
}

// ------------------------------------------------------------------------
// host side
// ------------------------------------------------------------------------
bool map_kv(CUtensorMap* map, const mfa_tensor* t) {
  auto fn = tensor_map_encoder();
  if (!fn) return false;
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(t->D), static_cast<cuuint64_t>(t->N),
                        static_cast<cuuint64_t>(t->H), static_cast<cuuint64_t>(t->B)};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(t->stride[2]) * 2, static_cast<cuuint64_t>(t->stride[1]) * 2,
                           static_cast<cuuint64_t>(t->stride[0]) * 2};
  cuuint32_t box[4] = {64, static_cast<cuuint32_t>(kBlk), 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, t->data, dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

mfa_status check_dec_tensor(const mfa_tensor* t) {
  if (!t) return MFA_ERR_INVALID_ARG;
  if (t->B <= 0 || t->H <= 0 || t->N < 0 || t->D <= 0) return MFA_ERR_INVALID_ARG;
  if (!t->data && t->N > 0) return MFA_ERR_INVALID_ARG;
  if (t->dtype != MFA_BF16) return MFA_ERR_UNSUPPORTED;
  if (t->stride[3] != 1) return MFA_ERR_UNSUPPORTED;
  for (int a = 0; a < 3; ++a)
    if (t->stride[a] <= 0 || (t->stride[a] * 2) % 16 != 0) return MFA_ERR_UNSUPPORTED;
  if (reinterpret_cast<uintptr_t>(t->data) % 16 != 0) return MFA_ERR_UNSUPPORTED;
  return MFA_OK;
}

template <int D, int G>
mfa_status launch_dec(const CUtensorMap& mk, const CUtensorMap& mv, const DecParams& p, cudaStream_t s) {
  using C = DecCfg<D>;
  static std::atomic<uint64_t> attr_devs{0};
  if (!ensure_smem_attr(reinterpret_cast<const void*>(mfa_decode_kernel<D, G>), C::kBytes, attr_devs))
    return MFA_ERR_CUDA;
  const dim3 grid(p.n_split, p.Nq, p.B * p.Hkv);
  mfa_decode_kernel<D, G><<<grid, kWarpsFor<D, G> * 32, C::kBytes, s>>>(mk, mv, p);
  if (cudaGetLastError() != cudaSuccess) return MFA_ERR_CUDA;
  if (p.n_split > 1) {
    const dim3 cgrid(static_cast<unsigned>(p.B * p.Hkv * p.Nq), (G * D + kCombineThreads - 1) / kCombineThreads);
    mfa_decode_combine<D, G><<<cgrid, kCombineThreads, 0, s>>>(p);
    if (cudaGetLastError() != cudaSuccess) return MFA_ERR_CUDA;
  }
  return MFA_OK;
}

template <int D>
mfa_status launch_dec_g(const CUtensorMap& mk, const CUtensorMap& mv, const DecParams& p, cudaStream_t s) {
  switch (p.G) {
    case 1: return launch_dec<D, 1>(mk, mv, p, s);
    case 2: return launch_dec<D, 2>(mk, mv, p, s);
    case 4: return launch_dec<D, 4>(mk, mv, p, s);
    case 8: return launch_dec<D, 8>(mk, mv, p, s);
    case 16: return D * 16 <= 2048 ? launch_dec<(D > 128 ? 128 : D), 16>(mk, mv, p, s) : MFA_ERR_UNSUPPORTED;
    default: return MFA_ERR_UNSUPPORTED;
  }
}

// Parts per list: the fewest that give one wave of CTAs on at least 85 % of
// the SMs (CTAs per SM from the kernel's shared memory), at most half the
// list length. Every part pays the list deduplication, the query load and the
// output write, so fewer and longer parts are faster once the SMs are busy
// (decode_sel64k: 2 parts 2.35 TB/s, 4 parts 1.99, 16 parts 1.28).
int32_t auto_split(int64_t rows, int32_t sel_k, int D) {
  const int n_sm = device_sm_count();
  const int sms = n_sm > 0 ? n_sm : 148;
  const int bytes = D == 128 ? DecCfg<128>::kBytes : DecCfg<256>::kBytes;
  const int per_sm = (227 * 1024) / bytes > 0 ? (227 * 1024) / bytes : 1;
  const int64_t target = (static_cast<int64_t>(sms) * per_sm * 85 + 99) / 100;
  const int64_t max_ns = sel_k / 2 > 1 ? sel_k / 2 : 1;
  int64_t ns = (target + rows - 1) / rows;
  if (ns > max_ns) ns = max_ns;
  if (ns < 1) ns = 1;
  return static_cast<int32_t>(ns);
}

}  // namespace
}  // namespace mfa

extern "C" size_t mfa_decode_workspace_bytes(int32_t B, int32_t Hq, int32_t Hkv, int32_t Nq, int32_t D,
                                             int32_t sel_k, int32_t n_split) {
  using namespace mfa;
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Nq < 0 || D <= 0 || sel_k <= 0 || n_split < 0 || Hq % Hkv) return 0;
  const int64_t rows = static_cast<int64_t>(B) * Hkv * Nq;
  const int32_t ns = n_split == 0 ? auto_split(rows > 0 ? rows : 1, sel_k, D) : n_split;
  if (ns <= 1) return 256;
  const int64_t G = Hq / Hkv;
  const size_t o = align256(static_cast<size_t>(rows * ns * G * D) * 4);
  return o + align256(static_cast<size_t>(rows * ns * G * 2) * 4);
}

extern "C" mfa_status mfa_decode(const mfa_tensor* q, const mfa_tensor* k, const mfa_tensor* v, const int32_t* sel,
                                 int32_t sel_k, const mfa_tensor* out, float* lse, int32_t n_split, void* workspace,
                                 size_t workspace_bytes, uint32_t* dev_err, void* stream) {
  using namespace mfa;
  mfa_status st;
  if ((st = check_dec_tensor(q)) != MFA_OK || (st = check_dec_tensor(k)) != MFA_OK ||
      (st = check_dec_tensor(v)) != MFA_OK || (st = check_dec_tensor(out)) != MFA_OK)
    return st;
  if (!dev_err || (!lse && q->N > 0) || (!sel && q->N > 0)) return MFA_ERR_INVALID_ARG;
  if (sel_k <= 0 || n_split < 0) return MFA_ERR_INVALID_ARG;
  if (k->B != q->B || v->B != q->B || out->B != q->B || k->H != v->H || k->N != v->N) return MFA_ERR_SHAPE_MISMATCH;
  if (k->D != q->D || v->D != q->D || out->D != q->D || out->H != q->H || out->N != q->N)
    return MFA_ERR_SHAPE_MISMATCH;
  if (q->H % k->H != 0) return MFA_ERR_SHAPE_MISMATCH;
  if (q->D != 128 && q->D != 256) return MFA_ERR_UNSUPPORTED;
  const int64_t G = q->H / k->H;
  if (G != 1 && G != 2 && G != 4 && G != 8 && G != 16) return MFA_ERR_UNSUPPORTED;
  if (G * q->D > 2048) return MFA_ERR_UNSUPPORTED;  // query rows and outputs are held in registers
  if (sel_k > kMaxSelK || q->B * k->H > 65535 || q->N > 65535 || k->N > (int64_t(1) << 30))
    return MFA_ERR_UNSUPPORTED;
  const int64_t rows = q->B * k->H * q->N;
  if (rows > 0x7fffffff) return MFA_ERR_UNSUPPORTED;  // the combine grid has one CTA column per row
  const int32_t ns = n_split == 0 ? auto_split(rows > 0 ? rows : 1, sel_k, static_cast<int>(q->D)) : n_split;
  if (ns > 65535) return MFA_ERR_UNSUPPORTED;
  if (ns > 1) {
    const size_t o = align256(static_cast<size_t>(rows * ns * G * q->D) * 4);
    const size_t need = o + align256(static_cast<size_t>(rows * ns * G * 2) * 4);
    if (!workspace || workspace_bytes < need || reinterpret_cast<uintptr_t>(workspace) % 256 != 0)
      return MFA_ERR_INVALID_ARG;
  }
  if (rows == 0) return MFA_OK;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (k->N == 0) return MFA_ERR_UNSUPPORTED;  // no key blocks to describe by a tensor map
  CUtensorMap mk, mv;
  if (!map_kv(&mk, k) || !map_kv(&mv, v)) return MFA_ERR_CUDA;
  DecParams p;
  p.B = static_cast<int32_t>(q->B); p.Hq = static_cast<int32_t>(q->H); p.Hkv = static_cast<int32_t>(k->H);
  p.G = static_cast<int32_t>(G); p.Nq = static_cast<int32_t>(q->N); p.Nk = static_cast<int32_t>(k->N);
  p.nblk = static_cast<int32_t>(cdiv64(k->N, kBlk)); p.sel_k = sel_k; p.n_split = ns;
  p.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(q->D)));
  p.sel = sel;
  p.q = static_cast<const __nv_bfloat16*>(q->data); p.qs0 = q->stride[0]; p.qs1 = q->stride[1]; p.qs2 = q->stride[2];
  p.out = static_cast<__nv_bfloat16*>(out->data); p.os0 = out->stride[0]; p.os1 = out->stride[1]; p.os2 = out->stride[2];
  p.lse = lse;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  p.o_part = ns > 1 ? reinterpret_cast<float*>(ws) : nullptr;
  p.ml_part = ns > 1 ? reinterpret_cast<float*>(ws + align256(static_cast<size_t>(rows * ns * G * q->D) * 4))
                     : nullptr;
  p.err = dev_err;
  return q->D == 128 ? launch_dec_g<128>(mk, mv, p, s) : launch_dec_g<256>(mk, mv, p, s);
}
