// mfa_decode: selected-key attention for a few query rows (decode) on sm_100a.
//
// Each (batch b, key/value head g, query row i) has a list of 64-key blocks
// ("vulkan : selected-key flash attention for QSA block selection", overview
// and kernel description): -1 entries are skipped, a block listed twice counts
// once, and the list is shared by the G query heads of head g. Query row i
// sits at position i + Nk - Nq and sees only keys at or before it (the forward
// pass's block-selection rule when Nq == Nk). The work is a gather of whole
// 64-key K/V blocks and is bound by HBM; the two products run on the tensor
// cores, so that the CUDA cores only run the softmax of G rows.
//
// Split-K, as in the pull request, generalised to slot ranges: the lists of
// all rows are laid end to end (L slots per row, L >= sel_k, slots past sel_k
// empty) and every CTA takes the same number of consecutive slots, so a CTA
// may finish one row and start the next, and the grid fills the SMs whatever
// the number of rows. A row met by one CTA is written directly; a row split
// over several CTAs gets an unnormalised partial (m, l, o) from each, and a
// second kernel combines them. An empty part writes m = -FLT_MAX, not -inf,
// so the combination never evaluates exp(-inf - -inf).
#include <algorithm>
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
constexpr int kCombineFast = 8;  // partials per row merged with all loads in one round
constexpr int kMaxPer = 2048;  // list slots per CTA
constexpr int kMaxSeg = 64;    // rows (segments) per CTA

struct DecParams {
  int32_t B, Hq, Hkv, G, Nq, Nk, nblk, sel_k;
  int64_t rows;        // B * Hkv * Nq
  int64_t L;           // slots per row in the partition (>= sel_k)
  int32_t per;         // slots per CTA: CTA c takes slots [c * per, (c + 1) * per) of rows * L
  int32_t seg_max;     // partial slots per row in the workspace (0: no row is split)
  float scale_log2;
  const int32_t* sel;  // [B, Hkv, Nq, sel_k]
  __nv_bfloat16* out;
  int64_t os0, os1, os2;
  float* lse;          // [B, Hq, Nq]
  float* o_part;       // [rows][seg_max][G][D]
  float* ml_part;      // [rows][seg_max][G][2]   (m, l)
  uint32_t* err;
};

// CTAs that meet row r: the first and the last.
__host__ __device__ __forceinline__ int64_t first_cta(const DecParams& p, int64_t r) { return r * p.L / p.per; }
__host__ __device__ __forceinline__ int64_t last_cta(const DecParams& p, int64_t r) {
  return ((r + 1) * p.L - 1) / p.per;
}

__device__ __forceinline__ bool warp_all_dec(bool ok) { return __all_sync(0xffffffffu, ok); }

// ---------------------------------------------------------------------------
// The decode kernel on the tensor cores.
//
// S = Q K^T as one tcgen05 MMA of M = 128 rows with Q in TMEM (the TS form):
// lanes 0 .. G-1 hold the G query heads of the row, lanes G .. 31 zeros, and
// the results of the other lanes are never used. N = 64 keys (one block), K =
// D. With Q and P in TMEM, the tensor core reads only K and V from shared
// memory, once each: shared-memory bandwidth (TMA writes plus MMA operand
// reads) is what bounds a block's turn-around. Lane h of the
// softmax warp holds head h's 64 scores (TMEM lane = row), keeps its own
// online max and sum, and writes P (bf16) over its scores. O += P V as a TS
// MMA (P from TMEM) with N = D, into an accumulator of 128 x D fp32 columns.
// Two S buffers: S of block n + 1 is computed while the softmax works on block
// n. K and V of a block share a stage of a three-stage (D = 256) or six-stage
// (D = 128) TMA ring, with their own barriers: K is released when S of the
// block is done, V when its P.V is. The MMA warp issues whichever of the next
// S and the oldest pending P.V is ready first.
//
// A CTA's blocks form one stream across its rows (segments): the ring, the S
// buffers and the MMA order run on from one row into the next. Q arrives by
// TMA into one of two shared-memory buffers ahead of its row; the softmax
// warp copies it into TMEM when the previous row's S products are done (it
// has waited for the last of them) and releases the buffer. The first P.V
// of a row overwrites O; it follows the softmax warp's P of that row's first
// block, which the warp writes only after it has read the previous row's O.
//
// Warps: 0 softmax and epilogue (TMEM lanes 0-31), 1 MMA issuer and TMEM owner,
// 2 TMA producer, 3 idle. Every wait is bounded.
// ---------------------------------------------------------------------------
template <int D>
struct DecTc {
  static constexpr int kStages = D == 256 ? 3 : 6;
  static constexpr int kQChunk = 16 * 128;                  // 16 rows x 128 B per 64-column chunk
  static constexpr int kQBytes = (D / 64) * kQChunk;        // one Q buffer
  static constexpr int kQ = 0;                               // two Q buffers
  static constexpr int kTile = kBlk * D * 2;                 // one K (or V) block
  static constexpr int kStage0 = 16 * 1024;                  // stages start 1024-aligned after Q
  static constexpr int kK = 0, kV = kTile;                   // inside a stage
  static constexpr int kStageBytes = 2 * kTile;
  static constexpr int kRaw = kStage0 + kStages * kStageBytes;  // one row's raw list [kMaxSelK]
  static constexpr int kList = kRaw + kMaxSelK * 4 + 16;        // the CTA's kept blocks [kMaxPer]
  static constexpr int kSeg = kList + kMaxPer * 4;              // segment starts in the kept list [kMaxSeg + 1]
  static constexpr int kCoord = kSeg + ((kMaxSeg + 1) * 4 + 15) / 16 * 16;  // (b, g, i) per segment [kMaxSeg]
  static constexpr int kMisc = kCoord + kMaxSeg * 16;
  static constexpr int kBytes = kMisc + 512 + 1024;         // + slack for 1024-byte alignment
  static constexpr int kTmemCols = 512;        // S0 [0,64) S1 [64,128) O [128, 128 + D) Q [128 + D, 128 + 3D/2)
  static constexpr int kQCol = 128 + D;
  static_assert(kBytes <= 232448, "shared memory");
  static_assert(2 * kQBytes <= kStage0, "Q buffers");
  static_assert(kQCol + D / 2 <= kTmemCols, "TMEM columns");
};

template <int D, int G>
__global__ void __launch_bounds__(128, 1)
    mfa_decode_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const DecParams p) {
  using C = DecTc<D>;
  constexpr int S = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // This CTA's slots [v0, v1) of rows * L, rows r0 .. r0 + nseg - 1.
  const int64_t v0 = static_cast<int64_t>(blockIdx.x) * p.per;
  const int64_t v1 = v0 + p.per < p.rows * p.L ? v0 + p.per : p.rows * p.L;
  const int64_t r0 = v0 / p.L;
  const int nseg = static_cast<int>((v1 - 1) / p.L - r0 + 1);  // <= kMaxSeg (host)

  int* sRaw = reinterpret_cast<int*>(smem + C::kRaw);
  int* sList = reinterpret_cast<int*>(smem + C::kList);
  int* sSeg = reinterpret_cast<int*>(smem + C::kSeg);            // row k's blocks: sList[sSeg[k] .. sSeg[k + 1])
  int4* sCoord = reinterpret_cast<int4*>(smem + C::kCoord);     // row k's (b, g, i)
  int* sCnt = reinterpret_cast<int*>(smem + C::kMisc);          // [4] per-warp counts
  volatile int* s_abort = reinterpret_cast<volatile int*>(sCnt + 8);
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(sCnt + 9);
  int* s_early = sCnt + 10;                                     // Q, K, V of block 0 issued before the roles
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kMisc + 64);
  uint64_t* k_full = bars;              // [S]
  uint64_t* k_empty = k_full + S;       // [S]: S of the block is done with K
  uint64_t* v_full = k_empty + S;       // [S]
  uint64_t* v_empty = v_full + S;       // [S]: P.V of the block is done with V
  uint64_t* q_full = v_empty + S;       // [2]: Q of a row in shared memory
  uint64_t* q_empty = q_full + 2;       // [2]: copied into TMEM, the buffer is free
  uint64_t* q_ready = q_empty + 2;      // Q of the next row with blocks is in TMEM
  uint64_t* s_full = q_ready + 1;       // [2]
  uint64_t* p_full = s_full + 2;        // [2]
  uint64_t* pv_done = p_full + 2;       // one phase per P.V
  uint64_t* o_done = pv_done + 1;       // one phase per row with blocks
  uint64_t* drain = o_done + 1;

  // The first row's list is read before anything else, so that the latency
  // of that global load overlaps the barrier and TMEM set-up below.
  int pre0 = -1, pre1 = -1;
  {
    const int64_t e = v1 - r0 * p.L;
    const int eb0 = static_cast<int>(e < p.sel_k ? e : p.sel_k);
    const int32_t* lrow0 = p.sel + r0 * p.sel_k;
    if (static_cast<int>(threadIdx.x) < eb0) pre0 = __ldg(lrow0 + threadIdx.x);
    if (static_cast<int>(threadIdx.x) + 128 < eb0) pre1 = __ldg(lrow0 + threadIdx.x + 128);
  }
  // The combine kernel (a programmatic dependent launch) may be scheduled now:
  // it waits for this grid to complete before it reads anything.
  asm volatile("griddepcontrol.launch_dependents;");
  if (threadIdx.x == 0) {
    for (int st = 0; st < S; ++st) {
      mbar_init(&k_full[st], 1);
      mbar_init(&k_empty[st], 1);
      mbar_init(&v_full[st], 1);
      mbar_init(&v_empty[st], 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&q_full[t], 1);
      mbar_init(&q_empty[t], 1);
      mbar_init(&s_full[t], 1);
      mbar_init(&p_full[t], 32);
    }
    mbar_init(q_ready, 1);
    mbar_init(pv_done, 1);
    mbar_init(o_done, 1);
    mbar_init(drain, 1);
    *s_abort = 0;
    fence_mbarrier_init();
  }
  // The first block's loads go out before the deduplication when the first
  // slot of the CTA's range is a kept block of the first row: valid, at or
  // before the row's position, and not listed earlier in the row (its
  // earlier entries, fewer than 32, are in warp 0's registers). It is then
  // the first entry of the kept list, and the producer starts at block 1.
  if (warp == 0) {
    const int64_t a = v0 - r0 * p.L, e = v1 - r0 * p.L;
    const int ea0 = static_cast<int>(a < 0 ? 0 : (a < p.sel_k ? a : p.sel_k));
    const int eb0 = static_cast<int>(e < p.sel_k ? e : p.sel_k);
    int early = -1;
    if (ea0 < 32 && ea0 < eb0) {
      const int vf = __shfl_sync(0xffffffffu, pre0, ea0);
      const bool dup = __ballot_sync(0xffffffffu, lane < ea0 && pre0 == vf) != 0u;
      const int last0 = static_cast<int>(r0 % p.Nq) + p.Nk - p.Nq;
      if (!dup && vf >= 0 && vf < p.nblk && static_cast<int64_t>(vf) * kBlk <= last0) early = vf;
    }
    if (lane == 0) {
      *s_early = early >= 0 ? 1 : 0;
      if (early >= 0) {
        const int64_t bg = r0 / p.Nq;
        const int b = static_cast<int>(bg / p.Hkv), g = static_cast<int>(bg % p.Hkv), i = static_cast<int>(r0 % p.Nq);
        mbar_arrive_expect_tx(&q_full[0], G * 128 * (D / 64));
#pragma unroll
        for (int c = 0; c < D / 64; ++c)
          tma_load_4d(smem + C::kQ + c * C::kQChunk, &tm_q, &q_full[0], c * 64, i, g * G, b);
        mbar_arrive_expect_tx(&k_full[0], C::kTile);
#pragma unroll
        for (int c = 0; c < D / 64; ++c)
          tma_load_4d(smem + C::kStage0 + C::kK + c * (kBlk * 128), &tm_k, &k_full[0], c * 64, early * kBlk, g, b);
        mbar_arrive_expect_tx(&v_full[0], C::kTile);
#pragma unroll
        for (int c = 0; c < D / 64; ++c)
          tma_load_4d(smem + C::kStage0 + C::kV + c * (kBlk * 128), &tm_v, &v_full[0], c * 64, early * kBlk, g, b);
      }
    }
  }
  if (warp == 1) {
    tmem_alloc(s_tmem, C::kTmemCols);
    tmem_relinquish();
    tc_fence_before();
  }

  // ---- 1. every row's kept blocks in this CTA's slots (first occurrence in
  // the whole row kept, out-of-range entries flagged, blocks after the row's
  // position dropped) ----
  int total = 0;
  for (int k = 0; k < nseg; ++k) {
    const int64_t r = r0 + k;
    const int64_t a = v0 - r * p.L, e = v1 - r * p.L;  // the row's slots in this CTA: [a, e) clipped to [0, sel_k)
    const int ea = static_cast<int>(a < 0 ? 0 : (a < p.sel_k ? a : p.sel_k));
    const int eb = static_cast<int>(e < p.sel_k ? e : p.sel_k);
    const int last = static_cast<int>(r % p.Nq) + p.Nk - p.Nq;  // the row's position
    if (threadIdx.x == 0) {
      sSeg[k] = total;
      const int64_t bg = r / p.Nq;
      sCoord[k] = make_int4(static_cast<int>(bg / p.Hkv), static_cast<int>(bg % p.Hkv), static_cast<int>(r % p.Nq), 0);
    }
    if (eb <= ea) continue;
    const int32_t* lrow = p.sel + r * p.sel_k;
    if (k == 0) {
      if (static_cast<int>(threadIdx.x) < eb) sRaw[threadIdx.x] = pre0;
      if (static_cast<int>(threadIdx.x) + 128 < eb) sRaw[threadIdx.x + 128] = pre1;
    } else {
      for (int e = threadIdx.x; e < eb; e += 128) sRaw[e] = lrow[e];
    }
    // Entries up to the next multiple of 4 past eb are padding for the
    // vector compares below (never equal to a kept entry: -2).
    if (static_cast<int>(threadIdx.x) < 4) sRaw[eb + threadIdx.x] = -2;
    __syncthreads();
    for (int base = ea; base < eb; base += 128) {
      const int e = base + threadIdx.x;
      bool keep = false;
      if (e < eb) {
        const int v = sRaw[e];
        if (v < -1 || v >= p.nblk) atomicOr(p.err, MFA_DEVERR_SEL);
        keep = v >= 0 && v < p.nblk && static_cast<int64_t>(v) * kBlk <= last;
        // First occurrence: no equal entry before e. Four entries per
        // shared-memory load and no early exit, so the loads pipeline.
        if (keep) {
          const int4* raw4 = reinterpret_cast<const int4*>(sRaw);
          bool dup = false;
          for (int e2 = 0; e2 < e; e2 += 4) {
            const int4 w = raw4[e2 >> 2];
            dup |= (w.x == v) | ((w.y == v) & (e2 + 1 < e)) | ((w.z == v) & (e2 + 2 < e)) | ((w.w == v) & (e2 + 3 < e));
          }
          keep = !dup;
        }
      }
      const unsigned bal = __ballot_sync(0xffffffffu, keep);
      if (lane == 0) sCnt[warp] = __popc(bal);
      __syncthreads();
      int off = total;
      for (int w = 0; w < warp; ++w) off += sCnt[w];
      if (keep) sList[off + __popc(bal & ((1u << lane) - 1u))] = sRaw[e];
      total += sCnt[0] + sCnt[1] + sCnt[2] + sCnt[3];
      __syncthreads();
    }
  }
  if (threadIdx.x == 0) sSeg[nseg] = total;
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;
  // Moves (seg, q) to the row of block n: q counts the rows with blocks before it.
  auto seek = [&](int n, int& seg, int& q) {
    while (sSeg[seg + 1] <= n) {
      if (sSeg[seg + 1] > sSeg[seg]) ++q;
      ++seg;
    }
  };

  if (warp == 2) {
    // =================== TMA producer ===================
    // K and V of a block have their own barriers: K is released as soon as S
    // of the block is done, V after its P.V, and the K loads run one block
    // ahead of the V loads. A row's Q goes out just before its first K.
    if (lane == 0) {
      // The row's coordinates come from shared memory: 64-bit divisions here
      // would sit on the issue path of every load.
      auto load = [&](const CUtensorMap* map, uint64_t* full, int n, int off, int seg) {
        const int4 co = sCoord[seg];
        const int b = co.x, g = co.y;
        const int blk = sList[n];
        mbar_arrive_expect_tx(full, C::kTile);
        uint8_t* dst = smem + C::kStage0 + (n % S) * C::kStageBytes + off;
#pragma unroll
        for (int c = 0; c < D / 64; ++c) tma_load_4d(dst + c * (kBlk * 128), map, full, c * 64, blk * kBlk, g, b);
      };
      int nk = 0, nv = 0, nq = 0;  // K, V and Q loads issued
      if (*s_early) nk = nv = nq = 1;
      int kseg = 0, kq = 0, vseg = 0, vq = 0;
      bool stop = false;
      while (!stop && nv < total) {
        if (nk < total && nk <= nv + 1) {
          seek(nk, kseg, kq);
          if (nk == sSeg[kseg]) {
            // Q buffer nq & 1 is free once the S products of row nq - 2 are done.
            if (nq >= 2 && !mbar_wait(&q_empty[nq & 1], ((nq >> 1) - 1) & 1, s_abort)) { stop = true; break; }
            const int4 co = sCoord[kseg];
            const int b = co.x, g = co.y, i = co.z;
            mbar_arrive_expect_tx(&q_full[nq & 1], G * 128 * (D / 64));
#pragma unroll
            for (int c = 0; c < D / 64; ++c)
              tma_load_4d(smem + C::kQ + (nq & 1) * C::kQBytes + c * C::kQChunk, &tm_q, &q_full[nq & 1], c * 64, i,
                          g * G, b);
            ++nq;
          }
          if (nk >= S && !mbar_wait(&k_empty[nk % S], ((nk / S) - 1) & 1, s_abort)) { stop = true; break; }
          load(&tm_k, &k_full[nk % S], nk, C::kK, kseg);
          ++nk;
        } else {
          seek(nv, vseg, vq);
          if (nv >= S && !mbar_wait(&v_empty[nv % S], ((nv / S) - 1) & 1, s_abort)) { stop = true; break; }
          load(&tm_v, &v_full[nv % S], nv, C::kV, vseg);
          ++nv;
        }
      }
      if (*s_abort) {
        // Loads in flight land before the CTA exits.
        volatile int no_abort = 0;
        for (int j = (nk > S ? nk - S : 0); j < nk; ++j) mbar_wait(&k_full[j % S], (j / S) & 1, &no_abort);
        for (int j = (nv > S ? nv - S : 0); j < nv; ++j) mbar_wait(&v_full[j % S], (j / S) & 1, &no_abort);
        for (int j = (nq > 2 ? nq - 2 : 0); j < nq; ++j) mbar_wait(&q_full[j & 1], (j >> 1) & 1, &no_abort);
      }
    }
  } else if (warp == 1) {
    // =================== MMA issuer ===================
    constexpr uint32_t idesc_s = idesc_bf16_f32(128, kBlk, false);
    constexpr uint32_t idesc_o = idesc_bf16_f32(128, D, true);
    const uint32_t st_addr = smem_u32(smem + C::kStage0);
    bool ok = true;
    int sseg = 0, sq = 0, pseg = 0, pq = 0;  // rows of the next S and the next P.V
    auto issue_s_ready = [&](int n) {
      const int st = n % S;
      tc_fence_after();
      const uint32_t kb = st_addr + st * C::kStageBytes + C::kK;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t bd = sdesc_sw128_lo(kb + (kk >> 2) * (kBlk * 128) + (kk & 3) * 32, 16);
        umma_ts(tmem + (n & 1) * kBlk, tmem + C::kQCol + kk * 8, bd, idesc_s, kk > 0 ? 1u : 0u);
      }
      umma_commit(&s_full[n & 1]);
      umma_commit(&k_empty[st]);
    };
    auto issue_pv = [&](int n) {
      const int st = n % S;
      tc_fence_after();
      const uint32_t vd = sdesc_sw128_lo(st_addr + st * C::kStageBytes + C::kV, kBlk * 128);
      const uint32_t a_p = tmem + (n & 1) * kBlk;
      const bool first = n == sSeg[pseg];
#pragma unroll
      for (int kk = 0; kk < kBlk / 16; ++kk)
        umma_ts(tmem + 128, a_p + kk * 8, vd + kk * (16 * 128 / 16), idesc_o, (!first || kk > 0) ? 1u : 0u);
      umma_commit(pv_done);
      umma_commit(&v_empty[st]);
      if (n + 1 == sSeg[pseg + 1]) umma_commit(o_done);
    };
    // Whichever is ready first goes out: the P.V of the oldest block whose P
    // is written, or S of the next block once its K (and, for a row's first
    // block, its Q in TMEM) is there and its S buffer is free (S(n) overwrites the P
    // of block n - 2, so P.V(n - 2) must have gone out before it). A P.V never
    // waits for the next block's data, so a stage is released, and refilled,
    // as soon as its block is done.
    int ns = 0, np = 0;  // S and P.V issued
    uint64_t t_idle = 0;
    while (ok && np < total) {
      bool did = false;
      if (ns < total && ns <= np + 1) {
        seek(ns, sseg, sq);
        if ((ns != sSeg[sseg] || warp_all_dec(mbar_test_wait(q_ready, sq & 1))) &&
            warp_all_dec(mbar_test_wait(&k_full[ns % S], (ns / S) & 1))) {
          issue_s_ready(ns);
          ++ns;
          did = true;
        }
      }
      if (!did && np < ns) {
        seek(np, pseg, pq);
        if (warp_all_dec(mbar_test_wait(&p_full[np & 1], (np >> 1) & 1)) &&
            warp_all_dec(mbar_test_wait(&v_full[np % S], (np / S) & 1))) {
          issue_pv(np);
          ++np;
          did = true;
        }
      }
      if (did) {
        t_idle = 0;
      } else {
        // Bounded like every other wait: give up after kWaitTimeoutNs without progress.
        if (*s_abort) ok = false;
        const uint64_t now = global_timer_ns();
        if (t_idle == 0) t_idle = now;
        else if (now - t_idle > kWaitTimeoutNs) ok = false;
        ok = warp_all_dec(ok);
      }
    }
    if (!ok) *s_abort = 1;
    umma_commit(drain);
    volatile int no_abort = 0;
    mbar_wait(drain, 0, &no_abort);
  } else if (warp == 0) {
    // =================== softmax and epilogue (lane h = query head h) ===================
    const int h = lane;
    const bool real = h < G;
    const uint32_t lane_off = 0;  // warp 0 reads TMEM lanes 0-31
    bool ok = true;
    int n = 0, rows_done = 0;  // blocks done; rows with blocks whose O has been read
    for (int k = 0; k < nseg; ++k) {
      const int64_t r = r0 + k;
      const int64_t bg = r / p.Nq;
      const int i = static_cast<int>(r % p.Nq), b = static_cast<int>(bg / p.Hkv), g = static_cast<int>(bg % p.Hkv);
      const int last = i + p.Nk - p.Nq;
      const int nb = sSeg[k + 1] - sSeg[k];
      float m_run = -INFINITY, l_run = 0.f;
      if (nb > 0) {
        // Q of this row into TMEM lanes 0-31 (lane h: head h, zeros past G).
        // Every S product of the previous row is done: this warp has waited
        // for the last one.
        const int qb = rows_done & 1;
        if (!(ok = warp_all_dec(mbar_wait(&q_full[qb], (rows_done >> 1) & 1, s_abort)))) break;
        const uint8_t* qrow = smem + C::kQ + qb * C::kQBytes + lane * 128;
#pragma unroll 1
        for (int c = 0; c < D / 64; ++c) {
          uint32_t w[32];
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            uint4 x = make_uint4(0u, 0u, 0u, 0u);
            if (real) x = *reinterpret_cast<const uint4*>(qrow + c * C::kQChunk + ((u ^ (lane & 7)) << 4));
            w[4 * u] = x.x;
            w[4 * u + 1] = x.y;
            w[4 * u + 2] = x.z;
            w[4 * u + 3] = x.w;
          }
          tmem_st_32x32b_x32(tmem + lane_off + C::kQCol + c * 32, w);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(q_ready);
          mbar_arrive(&q_empty[qb]);
        }
      }
      for (int t = 0; t < nb; ++t, ++n) {
        const int kbase = sList[n] * kBlk;
        if (!(ok = warp_all_dec(mbar_wait(&s_full[n & 1], (n >> 1) & 1, s_abort)))) break;
        tc_fence_after();
        float sc[kBlk];
        {
          uint32_t sv[2][32];
          tmem_ld_32x32b_x32(tmem + lane_off + (n & 1) * kBlk, sv[0]);
          tmem_ld_32x32b_x32(tmem + lane_off + (n & 1) * kBlk + 32, sv[1]);
          tmem_ld_wait();
#pragma unroll
          for (int jj = 0; jj < kBlk; ++jj) sc[jj] = __uint_as_float(sv[jj >> 5][jj & 31]);
        }
        // Keys after the row's position are hidden (this also covers the keys
        // past Nk of a partial last block, which TMA fills with zeros).
        const int vis = last - kbase + 1;  // visible keys of this block: [0, vis)
        float mx = -INFINITY;
#pragma unroll
        for (int jj = 0; jj < kBlk; ++jj) {
          if (jj >= vis) sc[jj] = -INFINITY;
          mx = fmaxf(mx, sc[jj]);
        }
        const float mx_s = mx * p.scale_log2;
        const bool need = real && mx_s > m_run + 8.0f;
        const float m_new = need ? mx_s : m_run;
        const float m_use = m_new == -INFINITY ? 0.f : m_new;
        const float alpha = need ? ex2_approx(m_run - m_use) : 1.f;
        uint32_t pk[kBlk / 2];
        float sum = 0.f;
#pragma unroll
        for (int u = 0; u < kBlk / 2; ++u) {
          const float e0 = ex2_approx(fmaf(sc[2 * u], p.scale_log2, -m_use));
          const float e1 = ex2_approx(fmaf(sc[2 * u + 1], p.scale_log2, -m_use));
          sum += e0 + e1;
          pk[u] = pack_bf16x2(e0, e1);
        }
        l_run = l_run * alpha + sum;
        m_run = m_new;
        if (t > 0 && __any_sync(0xffffffffu, need)) {
          // Rare: O has every P.V of the row before this block's once
          // pv_done's phase n - 1 is complete (S of this block went out after
          // the P.V of block n - 2, so that phase is the only one pending).
          if (!(ok = warp_all_dec(mbar_wait(pv_done, (n - 1) & 1, s_abort)))) break;
          tc_fence_after();
#pragma unroll 1
          for (int c = 0; c < D / 32; ++c) {
            uint32_t o[32];
            tmem_ld_32x32b_x32(tmem + lane_off + 128 + c * 32, o);
            tmem_ld_wait();
#pragma unroll
            for (int u = 0; u < 32; ++u) o[u] = __float_as_uint(__uint_as_float(o[u]) * alpha);
            tmem_st_32x32b_x32(tmem + lane_off + 128 + c * 32, o);
          }
        }
        {
          uint32_t a16[16], b16[16];
#pragma unroll
          for (int u = 0; u < 16; ++u) {
            a16[u] = pk[u];
            b16[u] = pk[16 + u];
          }
          tmem_st_32x32b_x16(tmem + lane_off + (n & 1) * kBlk, a16);
          tmem_st_32x32b_x16(tmem + lane_off + (n & 1) * kBlk + 16, b16);
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&p_full[n & 1]);
      }
      if (!ok) break;
      if (nb > 0) {
        if (!(ok = warp_all_dec(mbar_wait(o_done, rows_done & 1, s_abort)))) break;
        ++rows_done;
        tc_fence_after();
      }
      // ---- epilogue of the row: head h's output, or this CTA's partial ----
      const bool whole = first_cta(p, r) == last_cta(p, r);
      const bool has = l_run > 0.f;
      const float inv = has ? 1.f / l_run : 0.f;
      const size_t pu = static_cast<size_t>(r) * p.seg_max + (blockIdx.x - first_cta(p, r));
      // Two 32-column TMEM loads per wait: the epilogue is on the CTA's tail.
      auto emit = [&](const uint32_t (&o)[32], int c) {
        if (whole) {
          __nv_bfloat16* orow = p.out + b * p.os0 + static_cast<int64_t>(g * G + h) * p.os1 + i * p.os2 + c * 32;
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            uint32_t w[4];
#pragma unroll
            for (int u = 0; u < 4; ++u)
              w[u] = pack_bf16x2(__uint_as_float(o[q4 * 8 + 2 * u]) * inv, __uint_as_float(o[q4 * 8 + 2 * u + 1]) * inv);
            reinterpret_cast<uint4*>(orow)[q4] = make_uint4(w[0], w[1], w[2], w[3]);
          }
        } else {
          float* op = p.o_part + (pu * G + h) * D + c * 32;
#pragma unroll
          for (int q4 = 0; q4 < 8; ++q4)
            reinterpret_cast<float4*>(op)[q4] =
                make_float4(__uint_as_float(o[4 * q4]), __uint_as_float(o[4 * q4 + 1]), __uint_as_float(o[4 * q4 + 2]),
                            __uint_as_float(o[4 * q4 + 3]));
        }
      };
#pragma unroll 1
      for (int c = 0; c < D / 32; c += 2) {
        uint32_t o0[32], o1[32];
        if (nb > 0) {
          tmem_ld_32x32b_x32(tmem + lane_off + 128 + c * 32, o0);
          tmem_ld_32x32b_x32(tmem + lane_off + 128 + (c + 1) * 32, o1);
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int u = 0; u < 32; ++u) o0[u] = o1[u] = 0u;
        }
        if (!real) continue;
        emit(o0, c);
        emit(o1, c + 1);
      }
      if (real) {
        if (whole) {
          p.lse[(static_cast<size_t>(b) * p.Hq + g * G + h) * p.Nq + i] =
              has ? (m_run + __log2f(l_run)) * 0.69314718055994530942f : -INFINITY;
        } else {
          // A part that saw no visible key carries m = -FLT_MAX, l = 0.
          p.ml_part[(pu * G + h) * 2] = m_run == -INFINITY ? -FLT_MAX : m_run;
          p.ml_part[(pu * G + h) * 2 + 1] = l_run;
        }
      }
      // The next row's first P (written after these TMEM reads) lets its
      // first P.V overwrite O.
    }
    if (!ok) {
      *s_abort = 1;
      if (lane == 0) atomicOr(p.err, MFA_DEVERR_TIMEOUT);
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// Combine the partials of every row met by more than one CTA: with
// M = max m_s, out = sum o_s 2^(m_s - M) / sum l_s 2^(m_s - M). All parts
// empty gives M = -FLT_MAX, weights 1 on zeros, l = 0: out = 0, lse = -inf.
// One thread per output element, grid (rows, ceil(G * D / kCombineThreads)):
// every thread waits for two rounds of loads only (the parts' m, then their
// o and l), and the rows' CTAs spread over all SMs. Launched as a
// programmatic dependent of the decode kernel: it is resident early and
// starts reading when that grid has completed and its writes are visible.
template <int D, int G>
__global__ void __launch_bounds__(kCombineThreads) mfa_decode_combine(const DecParams p) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int64_t ru = blockIdx.x;  // the row
  const int ns = static_cast<int>(last_cta(p, ru) - first_cta(p, ru) + 1);
  if (ns == 1) return;  // written by its only CTA
  const int64_t bg = ru / p.Nq;
  const int i = static_cast<int>(ru % p.Nq);
  const int b = static_cast<int>(bg / p.Hkv), g = static_cast<int>(bg % p.Hkv);
  const int it = blockIdx.y * kCombineThreads + threadIdx.x;
  if (it < G * D) {
    const int h = it / D, d = it % D;
    const size_t pu0 = static_cast<size_t>(ru) * p.seg_max;
    float M = -FLT_MAX, o = 0.f, l = 0.f;
    if (ns <= kCombineFast) {
      // Every load goes out before any is used: one round of L2 latency.
      float mv[kCombineFast], lv[kCombineFast], ov[kCombineFast];
#pragma unroll
      for (int s = 0; s < kCombineFast; ++s) {
        if (s < ns) {
          const size_t pu = pu0 + s;
          mv[s] = p.ml_part[(pu * G + h) * 2];
          lv[s] = p.ml_part[(pu * G + h) * 2 + 1];
          ov[s] = p.o_part[(pu * G + h) * D + d];
        }
      }
#pragma unroll
      for (int s = 0; s < kCombineFast; ++s)
        if (s < ns) M = fmaxf(M, mv[s]);
#pragma unroll
      for (int s = 0; s < kCombineFast; ++s) {
        if (s < ns) {
          const float w = ex2_approx(mv[s] - M);
          o = fmaf(w, ov[s], o);
          l = fmaf(w, lv[s], l);
        }
      }
    } else {
      for (int s = 0; s < ns; ++s) M = fmaxf(M, p.ml_part[((pu0 + s) * G + h) * 2]);
      for (int s = 0; s < ns; ++s) {
        const size_t pu = pu0 + s;
        const float w = ex2_approx(p.ml_part[(pu * G + h) * 2] - M);
        o = fmaf(w, p.o_part[(pu * G + h) * D + d], o);
        l = fmaf(w, p.ml_part[(pu * G + h) * 2 + 1], l);
      }
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
// A [B, H, N, D] bf16 tensor with boxes of 64 columns x box_n positions x
// box_h heads, 128-byte swizzle: K and V take whole 64-key blocks of one
// head, Q takes one row of the G heads of a key/value head.
bool map_bf16_4d(CUtensorMap* map, const mfa_tensor* t, uint32_t box_n, uint32_t box_h) {
  auto fn = tensor_map_encoder();
  if (!fn) return false;
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(t->D), static_cast<cuuint64_t>(t->N),
                        static_cast<cuuint64_t>(t->H), static_cast<cuuint64_t>(t->B)};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(t->stride[2]) * 2, static_cast<cuuint64_t>(t->stride[1]) * 2,
                           static_cast<cuuint64_t>(t->stride[0]) * 2};
  cuuint32_t box[4] = {64, box_n, box_h, 1};
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
mfa_status launch_dec(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const DecParams& p,
                      int64_t grid, cudaStream_t s) {
  using C = DecTc<D>;
  static std::atomic<uint64_t> attr_devs{0};
  if (!ensure_smem_attr(reinterpret_cast<const void*>(mfa_decode_kernel<D, G>), C::kBytes, attr_devs))
    return MFA_ERR_CUDA;
  mfa_decode_kernel<D, G><<<static_cast<unsigned>(grid), 128, C::kBytes, s>>>(mq, mk, mv, p);
  if (cudaGetLastError() != cudaSuccess) return MFA_ERR_CUDA;
  if (p.seg_max > 1) {
    // A programmatic dependent launch: the combine CTAs may start while the
    // decode grid runs and wait in griddepcontrol.wait for its completion.
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(p.rows), (G * D + kCombineThreads - 1) / kCombineThreads);
    cfg.blockDim = dim3(kCombineThreads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, mfa_decode_combine<D, G>, p) != cudaSuccess) return MFA_ERR_CUDA;
  }
  return MFA_OK;
}

template <int D>
mfa_status launch_dec_g(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const DecParams& p,
                        int64_t grid, cudaStream_t s) {
  switch (p.G) {
    case 1: return launch_dec<D, 1>(mq, mk, mv, p, grid, s);
    case 2: return launch_dec<D, 2>(mq, mk, mv, p, grid, s);
    case 4: return launch_dec<D, 4>(mq, mk, mv, p, grid, s);
    case 8: return launch_dec<D, 8>(mq, mk, mv, p, grid, s);
    case 16: return D * 16 <= 2048 ? launch_dec<(D > 128 ? 128 : D), 16>(mq, mk, mv, p, grid, s) : MFA_ERR_UNSUPPORTED;
    default: return MFA_ERR_UNSUPPORTED;
  }
}

// How the rows' list slots are cut among CTAs.
struct DecPlan {
  int64_t L = 0;        // slots per row (>= sel_k)
  int32_t per = 0;      // slots per CTA
  int64_t grid = 0;     // CTAs
  int32_t seg_max = 0;  // partials per row in the workspace (0: every row has one CTA)
};

// n_split >= 1: n_split parts of ceil(sel_k / n_split) slots per row, one CTA
// each (parts past the list's end are empty). n_split == 0: about one CTA
// per SM (shared memory allows no more), each over an equal range of the
// rows' slots laid end to end, at least 2 slots:
// - a range of a whole list or more is rounded up to whole lists (at most
//   kMaxPer slots and kMaxSeg lists, so very long jobs take more than one
//   wave), and no row is split;
// - a shorter range is widened to the next divisor of sel_k when that still
//   keeps three quarters of the SMs busy: every row is then cut at the same
//   places and no CTA holds parts of two rows (a CTA that moves on to a second
//   row pays for a second list read and a second epilogue; measured on
//   decode_sel64k, 16 slots per CTA: 36.0 us, 14 slots with rows spanning
//   CTAs: 38.3 us);
// - otherwise the ranges run across row ends.
bool plan_dec(int64_t rows, int32_t sel_k, int32_t n_split, DecPlan* pl) {
  if (rows <= 0 || sel_k <= 0 || sel_k > kMaxSelK || n_split < 0) return false;
  if (n_split >= 1) {
    pl->per = static_cast<int32_t>(cdiv64(sel_k, n_split));
    pl->L = static_cast<int64_t>(n_split) * pl->per;
    pl->grid = rows * n_split;
    pl->seg_max = n_split > 1 ? n_split : 0;
  } else {
    const int n_sm = device_sm_count();
    const int64_t sms = n_sm > 0 ? n_sm : 148;
    const int64_t total = rows * sel_k;
    int64_t per = cdiv64(total, sms);
    if (per < 2) per = 2;
    if (per >= sel_k) {
      int64_t lists = cdiv64(per, sel_k);
      const int64_t cap = std::min<int64_t>(kMaxPer / sel_k, kMaxSeg);
      if (lists > cap) lists = cap;
      per = lists * sel_k;
    } else {
      int64_t dv = per;
      while (sel_k % dv != 0) ++dv;
      if (rows * (sel_k / dv) * 4 >= sms * 3) per = dv;
    }
    pl->per = static_cast<int32_t>(per);
    pl->L = sel_k;
    pl->grid = cdiv64(total, per);
    if (per % sel_k == 0) pl->seg_max = 0;
    else if (sel_k % per == 0) pl->seg_max = static_cast<int32_t>(sel_k / per);
    else pl->seg_max = static_cast<int32_t>(cdiv64(sel_k - 1, per) + 1);
    if (pl->seg_max == 1) pl->seg_max = 0;
  }
  return pl->grid <= 0x7fffffff;
}

size_t dec_workspace(const DecPlan& pl, int64_t rows, int64_t G, int64_t D) {
  if (pl.seg_max <= 1) return 256;
  return align256(static_cast<size_t>(rows * pl.seg_max * G * D) * 4) +
         align256(static_cast<size_t>(rows * pl.seg_max * G * 2) * 4);
}

}  // namespace
}  // namespace mfa

extern "C" size_t mfa_decode_workspace_bytes(int32_t B, int32_t Hq, int32_t Hkv, int32_t Nq, int32_t D,
                                             int32_t sel_k, int32_t n_split) {
  using namespace mfa;
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Nq < 0 || D <= 0 || sel_k <= 0 || n_split < 0 || Hq % Hkv) return 0;
  const int64_t rows = static_cast<int64_t>(B) * Hkv * Nq;
  if (rows == 0) return 256;
  DecPlan pl;
  if (!plan_dec(rows, sel_k > kMaxSelK ? kMaxSelK : sel_k, n_split, &pl)) return 0;
  return dec_workspace(pl, rows, Hq / Hkv, D);
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
  if (G * q->D > 2048) return MFA_ERR_UNSUPPORTED;
  if (sel_k > kMaxSelK || q->B * k->H > 65535 || q->N > 65535 || k->N > (int64_t(1) << 30) || n_split > 65535)
    return MFA_ERR_UNSUPPORTED;
  const int64_t rows = q->B * k->H * q->N;
  if (rows > 0x7fffffff) return MFA_ERR_UNSUPPORTED;  // the combine grid has one CTA column per row
  DecPlan pl;
  if (rows > 0 && !plan_dec(rows, sel_k, n_split, &pl)) return MFA_ERR_UNSUPPORTED;
  if (rows > 0 && pl.seg_max > 1) {
    const size_t need = dec_workspace(pl, rows, G, q->D);
    if (!workspace || workspace_bytes < need || reinterpret_cast<uintptr_t>(workspace) % 256 != 0)
      return MFA_ERR_INVALID_ARG;
  }
  if (rows == 0) return MFA_OK;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (k->N == 0) return MFA_ERR_UNSUPPORTED;  // no key blocks to describe by a tensor map
  CUtensorMap mq, mk, mv;
  if (!map_bf16_4d(&mq, q, 1, static_cast<uint32_t>(G)) || !map_bf16_4d(&mk, k, kBlk, 1) ||
      !map_bf16_4d(&mv, v, kBlk, 1))
    return MFA_ERR_CUDA;
  DecParams p;
  p.B = static_cast<int32_t>(q->B); p.Hq = static_cast<int32_t>(q->H); p.Hkv = static_cast<int32_t>(k->H);
  p.G = static_cast<int32_t>(G); p.Nq = static_cast<int32_t>(q->N); p.Nk = static_cast<int32_t>(k->N);
  p.nblk = static_cast<int32_t>(cdiv64(k->N, kBlk)); p.sel_k = sel_k;
  p.rows = rows; p.L = pl.L; p.per = pl.per; p.seg_max = pl.seg_max;
  p.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(q->D)));
  p.sel = sel;
  p.out = static_cast<__nv_bfloat16*>(out->data); p.os0 = out->stride[0]; p.os1 = out->stride[1]; p.os2 = out->stride[2];
  p.lse = lse;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  p.o_part = pl.seg_max > 1 ? reinterpret_cast<float*>(ws) : nullptr;
  p.ml_part = pl.seg_max > 1 ? reinterpret_cast<float*>(ws + align256(static_cast<size_t>(rows * pl.seg_max * G * q->D) * 4))
                             : nullptr;
  p.err = dev_err;
  return q->D == 128 ? launch_dec_g<128>(mq, mk, mv, p, pl.grid, s) : launch_dec_g<256>(mq, mk, mv, p, pl.grid, s);
}
