// mfa_fwd: mask-aware flash-attention forward pass for sm_100a.
//
// out = softmax(Q K^T / sqrt(d) + mask) V and lse = log-sum-exp per row, where
// the mask is applied through the tile map: only the key tiles listed for a
// query tile are visited (Binary Block Masking, abstract: skip fully masked
// blocks), FULL tiles take no per-element mask work, and PARTIAL tiles apply
// the exact element mask of the compact description (FlashMask's column-wise
// intervals, the Ascend band, or 64-block selection lists).
//
// Persistent kernel, one CTA per SM. A work item is two 128-row query tiles
// that read the same key/value head:
//   kind 0  two head tiles of one key/value group at the same query block;
//           the mask is shared by all heads, so both tiles have the same list.
//   kind 1  two consecutive query tiles of one head tile (used when a group
//           holds an odd number of head tiles, or the mask has one head per
//           query head); the MMA warp walks the union of the two lists.
// A query tile is 128 queries of one head (block_q = 128) or 64 queries of two
// heads of one group (block_q = 64).
//
// Warp roles (384 threads, three warpgroups):
//   WG0 warp 0   TMA producer: Q of each tile once per item, then K and V of
//                every k-tile of the union list into shared-memory rings.
//   WG0 warp 1   TMEM owner and MMA issuer. Per k-tile and tile t: first the
//                pending O_t += P_t V of the previous k-tile (P_t read from
//                TMEM), then S_t = Q_t K^T. The two tiles alternate, so while
//                one softmax warpgroup works the tensor core runs the other
//                tile's MMAs.
//   WG1, WG2     softmax + epilogue of tile slot 0 and 1: one row per thread
//                (TMEM lane = row); load S, mask only PARTIAL tiles, online
//                max / exp2 / sum, rescale O in TMEM when the running max
//                grows by more than 2^8, write P (bf16) over S; at the end of
//                an item read O, release it to the next item, normalise and
//                store out and lse.
// TMEM columns: S0 [0, BK), S1 [BK, 2BK), O0 [2BK, 2BK+D), O1 [2BK+D, 2BK+2D).
// Every mbarrier wait is bounded; a wait that gives up raises an abort flag
// for the whole CTA and sets MFA_DEVERR_TIMEOUT in the map's error word.
#include <climits>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include "mfa.h"
#include "mfa_device.cuh"
#include "mfa_internal.h"

namespace mfa {
namespace {

constexpr int kRows = 128;  // MMA M: query rows per tile
constexpr int kThreads = 384;
constexpr float kRescaleThreshold = 8.0f;  // log2 units
// Register split (setmaxnreg): the launch gives 168 per thread (384 x 168 =
// 64512), shared as 128 x low + 256 x high = 64512. With BK = 128 the softmax
// holds a 128-score row and needs 200, leaving WG0 104; with BK = 64 it
// needs far fewer and WG0 (the MMA warp with two S buffers) gets 120.
template <int BK>
constexpr int kRegsLow = BK == 64 ? 120 : 104;
template <int BK>
constexpr int kRegsHigh = BK == 64 ? 192 : 200;
static_assert(128 * kRegsLow<64> + 256 * kRegsHigh<64> <= 384 * 168, "register split (BK = 64)");
static_assert(128 * kRegsLow<128> + 256 * kRegsHigh<128> <= 384 * 168, "register split (BK = 128)");

struct FwdParams {
  int32_t B, Hq, Hkv, G, Hm, Nq, Nk, nqt, nkt;
  int32_t item_kind, n_items, pairs, n_ht, nqp;
  float scale_log2;  // log2(e) / sqrt(d)
  MaskArgs mask;
  const uint8_t* cls;
  const int32_t* list;
  const int32_t* count;
  const int32_t* order;
  __nv_bfloat16* out;
  int64_t os0, os1, os2;
  float* lse;
  uint32_t* err;
  uint32_t* sched;  // [0] next work item, [1] CTAs finished (map scratch words)
  int32_t bias_kind;     // MFA_BIAS_* (kernels instantiated with kBias only)
  const float* slopes;   // [Hq] ALiBi slopes
  uint64_t wait_ns;      // limit of every bounded wait on the pipeline (kWaitTimeoutNs)
  int32_t withhold_k;    // test hook: 1 = CTA 0 never loads its first K tile (see mfa_test_arm_fwd_timeout)
};

constexpr int kRing = 4;  // decoded work items in flight from the producer to the other roles

template <int D, int BK>
struct Cfg {
  static constexpr int kStages = BK == 128 ? 2 : 4;
  static constexpr int kChunks = D / 64;  // 128-byte K chunks per row
  static constexpr int kQBytes = kRows * D * 2;
  static constexpr int kKVBytes = BK * D * 2;
  static constexpr int kQ = 0;  // two Q slots
  static constexpr int kK = kQ + 2 * kQBytes;
  static constexpr int kV = kK + kStages * kKVBytes;
  // Output staging for the TMA-store epilogue: one 32-row x 32-column bf16
  // tile (2 KB, 64-byte swizzle) per softmax warp.
  static constexpr int kStage = kV + kStages * kKVBytes;
  static constexpr int kStageBytes = 32 * 32 * 2;
  static constexpr int kBar = kStage + 8 * kStageBytes;
  // q_full[2] q_empty[2] k_full[S] k_empty[S] v_full[S] v_empty[S] s_full[2] p_full[2]
  // s_full[2][2] p_full[2][2] o_done[2] pv_done[2] bnd[2][2] drain sched_full[kRing] sched_empty[kRing]
  static constexpr int kNumBars = 4 + 4 * kStages + 12 + 4 + 1 + 2 * kRing;
  static constexpr int kBounds = kBar + ((kNumBars * 8 + 15) / 16) * 16;  // int4 [2 tiles][2 slots][BK]
  static constexpr int kRingOff = kBounds + 4 * BK * 16;                 // WorkItem [kRing]
  static constexpr int kMisc = kRingOff + kRing * 128;
  static constexpr int kBytes = kMisc + 16;
  static constexpr int kAlloc = kBytes + 1024;  // slack for 1024-byte alignment
  // S buffers per tile in TMEM: two when BK = 64 (4 x 64 S + 2 x 128 O columns
  // fit in 512), so S_t(u+1) is computed while the softmax works on S_t(u).
  static constexpr int kSBufs = BK == 64 ? 2 : 1;
  static constexpr int kTmemCols = (2 * kSBufs * BK + 2 * D) <= 256 ? 256 : 512;
  static constexpr int kOCol = 2 * kSBufs * BK;  // first O column
};

struct Tile {
  int n;         // listed k-tiles (0: no visible key in the tile)
  int h0, q0;    // first head and first query of the tile
  int b;
  bool valid;    // false when a kind-1 item runs past the last query tile
  size_t bh_mask;
  const int32_t* lst;
  const uint8_t* cls;
};

// One decoded work item as the producer publishes it to the MMA and softmax roles.
struct WorkItem {
  int32_t w;    // item index, -1 = no more work
  int32_t hkv;
  Tile t[2];
};
static_assert(sizeof(WorkItem) <= 128, "ring slot size");

template <int GP>
__device__ __forceinline__ void decode_item(const FwdParams& p, int w, Tile (&t)[2], int& hkv) {
  constexpr int BQ = kRows / GP;
  if (p.item_kind == 0) {
    const int e = p.order[w / p.pairs], pr = w % p.pairs;
    const int b = e / (p.Hm * p.nqt), hm = (e / p.nqt) % p.Hm, qt = e % p.nqt;
#pragma unroll
    for (int s = 0; s < 2; ++s) {
      t[s].valid = true;
      t[s].n = p.count[e];
      t[s].h0 = (2 * pr + s) * GP;
      t[s].q0 = qt * BQ;
      t[s].b = b;
      t[s].bh_mask = static_cast<size_t>(b) * p.Hm + hm;
      t[s].lst = p.list + static_cast<size_t>(e) * p.nkt;
      t[s].cls = p.cls + static_cast<size_t>(e) * p.nkt;
    }
  } else {
    const int qp = w % p.nqp, ht = (w / p.nqp) % p.n_ht, b = w / (p.nqp * p.n_ht);
    const int hm = p.Hm == 1 ? 0 : ht;
#pragma unroll
    for (int s = 0; s < 2; ++s) {
      const int qt = 2 * qp + s;
      const size_t e = (static_cast<size_t>(b) * p.Hm + hm) * p.nqt + qt;
      t[s].valid = qt < p.nqt;
      t[s].n = t[s].valid ? p.count[e] : 0;
      t[s].h0 = ht * GP;
      t[s].q0 = qt * BQ;
      t[s].b = b;
      t[s].bh_mask = static_cast<size_t>(b) * p.Hm + hm;
      t[s].lst = p.list + e * p.nkt;
      t[s].cls = p.cls + e * p.nkt;
    }
  }
  hkv = t[0].h0 / p.G;
}

// Walks the union of the two tiles' ascending k-tile lists.
struct Merge {
  const int32_t* l0;
  const int32_t* l1;
  int n0, n1, i0, i1;
  bool shared;
  __device__ __forceinline__ bool next(int& kt, bool& in0, bool& in1) {
    if (shared) {
      if (i0 >= n0) return false;
      kt = l0[i0++];
      in0 = in1 = true;
      return true;
    }
    const int a = i0 < n0 ? l0[i0] : INT_MAX;
    const int c = i1 < n1 ? l1[i1] : INT_MAX;
    if (a == INT_MAX && c == INT_MAX) return false;
    kt = min(a, c);
    in0 = a == kt;
    in1 = c == kt;
    i0 += in0;
    i1 += in1;
    return true;
  }
};

__device__ __forceinline__ Merge make_merge(const FwdParams& p, const Tile (&t)[2]) {
  Merge m;
  m.l0 = t[0].lst; m.l1 = t[1].lst;
  m.n0 = t[0].n; m.n1 = t[1].n;
  m.i0 = m.i1 = 0;
  m.shared = p.item_kind == 0;
  return m;
}

__device__ __forceinline__ bool warp_all(bool ok) { return __all_sync(0xffffffffu, ok); }

// Bits [a, b) of a 32-bit word, with a and b clamped to [0, 32].
__device__ __forceinline__ uint32_t rows_in_interval(int a, int b) {
  a = max(a, 0);
  b = min(b, 32);
  if (a >= b) return 0u;
  return static_cast<uint32_t>(((1ull << b) - 1ull) & ~((1ull << a) - 1ull));
}

// Transpose a 32x32 bit matrix held one row per lane (bit l of lane j's word
// is entry (j, l)): afterwards bit j of lane l's word is entry (j, l). Five
// butterfly stages; at distance d each lane keeps the half of its word whose
// bit index agrees with its own lane bit d and takes the other half from lane
// l ^ d, shifted by d.
__device__ __forceinline__ uint32_t transpose32_warp(uint32_t x, int lane) {
  const uint32_t masks[5] = {0x0000FFFFu, 0x00FF00FFu, 0x0F0F0F0Fu, 0x33333333u, 0x55555555u};
#pragma unroll
  for (int st = 0; st < 5; ++st) {
    const int d = 16 >> st;
    const uint32_t m = masks[st];
    const uint32_t y = __shfl_xor_sync(0xffffffffu, x, d);
    x = (lane & d) ? ((x & ~m) | ((y & ~m) >> d)) : ((x & m) | ((y & m) << d));
  }
  return x;
}

// kBias: 0 none, 1 linear ALiBi (right- or left-aligned), 2 square-root ALiBi.
template <int D, int BK, int GP, int kBias>
__global__ void __launch_bounds__(kThreads, 1)
    mfa_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                   const FwdParams p) {
  using C = Cfg<D, BK>;
  constexpr int S = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  uint8_t* sQ = smem + C::kQ;
  uint8_t* sK = smem + C::kK;
  uint8_t* sV = smem + C::kV;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBar);
  uint64_t* q_full = bars;
  uint64_t* q_empty = q_full + 2;
  uint64_t* k_full = q_empty + 2;
  uint64_t* k_empty = k_full + S;
  uint64_t* v_full = k_empty + S;
  uint64_t* v_empty = v_full + S;
  uint64_t* s_full = v_empty + S;
  uint64_t* p_full = s_full + 4;  // [tile][S buffer], like s_full
  uint64_t* o_done = p_full + 4;
  uint64_t* pv_done = o_done + 2;  // one phase per P.V of the tile
  uint64_t* bnd_full = pv_done + 2;  // [2 tiles][2 slots]
  uint64_t* drain = bnd_full + 4;
  uint64_t* sched_full = drain + 1;
  uint64_t* sched_empty = sched_full + kRing;
  int4* s_bounds = reinterpret_cast<int4*>(smem + C::kBounds);
  WorkItem* ring = reinterpret_cast<WorkItem*>(smem + C::kRingOff);
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + C::kMisc);
  volatile int* s_abort = reinterpret_cast<volatile int*>(smem + C::kMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int wg = warp >> 2;

  // ---- set-up ----------------------------------------------------------
  if (warp == 0 && lane == 0) {
    for (int t = 0; t < 2; ++t) {
      mbar_init(&q_full[t], 1);
      mbar_init(&q_empty[t], 1);
      mbar_init(&s_full[2 * t], 1);
      mbar_init(&s_full[2 * t + 1], 1);
      mbar_init(&p_full[2 * t], kRows);
      mbar_init(&p_full[2 * t + 1], kRows);
      mbar_init(&o_done[t], 1);
      mbar_init(&pv_done[t], 1);
      mbar_init(&bnd_full[2 * t], kRows);
      mbar_init(&bnd_full[2 * t + 1], kRows);
    }
    for (int s = 0; s < S; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 2);  // one arrival per tile slot for every k-tile
    }
    mbar_init(drain, 1);
    for (int i = 0; i < kRing; ++i) {
      mbar_init(&sched_full[i], 1);
      mbar_init(&sched_empty[i], 1 + 8);  // the MMA thread and one lane of each softmax warp
    }
    *s_abort = 0;
    fence_mbarrier_init();
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    tma_prefetch_desc(&tm_o);
  }
  if (warp == 1) {
    tmem_alloc(s_tmem, C::kTmemCols);
    tmem_relinquish();
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;

  if (wg == 0) {
   asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" :: "n"(kRegsLow<BK>));
   if (warp == 0) {
    // =================== TMA producer ===================
    if (lane == 0) {
      uint32_t kv_it = 0;
      int quse[2] = {0, 0};
      uint32_t k_inflight = 0, v_inflight = 0;  // loads issued (for the abort drain)
      bool stop = false;
      // Work items are handed out dynamically in LPT order: an idle CTA takes
      // the next one. The producer decodes it once and publishes it.
      for (int it = 0; !stop; ++it) {
        const int rs = it % kRing;
        if (it >= kRing && !mbar_wait(&sched_empty[rs], ((it / kRing) - 1) & 1, s_abort, p.wait_ns)) break;
        const uint32_t wu = atomicAdd(&p.sched[0], 1u);
        WorkItem info;
        info.w = wu < static_cast<uint32_t>(p.n_items) ? static_cast<int>(wu) : -1;
        info.hkv = 0;
        if (info.w >= 0) decode_item<GP>(p, info.w, info.t, info.hkv);
        ring[rs] = info;
        mbar_arrive(&sched_full[rs]);
        if (info.w < 0) break;
        const Tile (&t)[2] = info.t;
        const int hkv = info.hkv;
        for (int s = 0; s < 2 && !stop; ++s) {
          if (t[s].n == 0) continue;
          if (quse[s] > 0 && !mbar_wait(&q_empty[s], (quse[s] - 1) & 1, s_abort, p.wait_ns)) { stop = true; break; }
          mbar_arrive_expect_tx(&q_full[s], C::kQBytes);
          uint8_t* dst = sQ + s * C::kQBytes;
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            const int head = (GP == 2) ? t[s].h0 + hh : t[s].h0;
            const int row = (GP == 2) ? t[s].q0 : t[s].q0 + 64 * hh;
#pragma unroll
            for (int c = 0; c < C::kChunks; ++c)
              tma_load_4d(dst + c * (kRows * 128) + hh * (64 * 128), &tm_q, &q_full[s], c * 64, row, head, t[s].b);
          }
          ++quse[s];
        }
        Merge m = make_merge(p, t);
        int kt;
        bool in0, in1;
        while (!stop && m.next(kt, in0, in1)) {
          if (kt < 0 || kt >= p.nkt) {
            atomicOr(p.err, MFA_DEVERR_MAP);
            *s_abort = 1;
            stop = true;
            break;
          }
          const int st = kv_it % S;
          const uint32_t ph = (kv_it / S) & 1;
          if (kv_it >= S && !mbar_wait(&k_empty[st], ph ^ 1, s_abort, p.wait_ns)) { stop = true; break; }
          // Test hook: the first K tile of CTA 0 is neither loaded nor
          // announced, so the MMA warp's bounded wait for it runs out.
          const bool withhold = p.withhold_k && blockIdx.x == 0 && kv_it == 0;
          if (!withhold) {
            mbar_arrive_expect_tx(&k_full[st], C::kKVBytes);
#pragma unroll
            for (int c = 0; c < C::kChunks; ++c)
              tma_load_4d(sK + st * C::kKVBytes + c * (BK * 128), &tm_k, &k_full[st], c * 64, kt * BK, hkv, t[0].b);
          }
          k_inflight = kv_it + 1;
          if (kv_it >= S && !mbar_wait(&v_empty[st], ph ^ 1, s_abort, p.wait_ns)) { stop = true; break; }
          mbar_arrive_expect_tx(&v_full[st], C::kKVBytes);
#pragma unroll
          for (int c = 0; c < C::kChunks; ++c)
            tma_load_4d(sV + st * C::kKVBytes + c * (BK * 128), &tm_v, &v_full[st], c * 64, kt * BK, hkv, t[0].b);
          v_inflight = kv_it + 1;
          ++kv_it;
        }
      }
      if (*s_abort) {
        // Let the copies already issued land before shared memory is released.
        volatile int no_abort = 0;
        for (int s = 0; s < 2; ++s)
          if (quse[s] > 0) mbar_wait(&q_full[s], (quse[s] - 1) & 1, &no_abort);
        for (uint32_t j = (k_inflight > S ? k_inflight - S : 0); j < k_inflight; ++j)
          if (!(p.withhold_k && blockIdx.x == 0 && j == 0)) mbar_wait(&k_full[j % S], (j / S) & 1, &no_abort);
        for (uint32_t j = (v_inflight > S ? v_inflight - S : 0); j < v_inflight; ++j)
          mbar_wait(&v_full[j % S], (j / S) & 1, &no_abort);
      }
    }
  } else if (warp == 1) {
    // =================== MMA issuer ===================
    // The whole warp runs this loop converged (waits are made warp-uniform)
    // and the tcgen05 helpers issue from one elected lane.
    {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(kRows, BK, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(kRows, D, true);
      const uint32_t q_addr = smem_u32(sQ), k_addr = smem_u32(sK), v_addr = smem_u32(sV);
      uint32_t kv_it = 0;
      // nsq[t] counts the S_t issued so far; S number k of a tile uses S buffer
      // k % kSBufs and the phase (k / kSBufs) & 1 of that buffer's s_full and
      // p_full. psq[t] is the S number of the tile's pending P.V.
      uint32_t nsq[2] = {0, 0}, psq[2] = {0, 0};
      int quse[2] = {0, 0};
      bool ok = true;
      // The P.V of a tile's last k-tile is not issued at the end of its work
      // item but carried into the next item, where it goes out just before that
      // slot's first S like any pending P.V. The MMA warp thus reads the next
      // ring entry and sets up the next item while the softmax still works on
      // the last P, and the next S follows the carried P.V at once. Each
      // pending P.V records its V stage and whether it is the first (O is
      // overwritten) or last (o_done is committed) P.V of its item.
      // Per slot s, bits of `pv`: 1 << s pending, 4 << s first, 16 << s last;
      // pkv[s] = the k-tile counter of the pending P.V (stage and phase of V).
      uint32_t pv = 0;
      uint32_t pkv[2] = {0, 0};

      // O_t += P_t V for the tile's pending k-tile.
      auto issue_pv = [&](int s) -> bool {
        const uint32_t sb = psq[s] % C::kSBufs;
        if (!warp_all(mbar_wait(&p_full[2 * s + sb], (psq[s] / C::kSBufs) & 1, s_abort, p.wait_ns))) return false;
        const uint32_t vst = pkv[s] % S;
        if (!warp_all(mbar_wait(&v_full[vst], (pkv[s] / S) & 1, s_abort, p.wait_ns))) return false;
        tc_fence_after();
        const uint32_t a_p = tmem + (s * C::kSBufs + sb) * BK;
        const uint32_t d_o = tmem + C::kOCol + s * D;
        // Descriptor start addresses are in 16-byte units in the low bits, so
        // advancing by a byte offset adds offset >> 4 to the descriptor.
        // The MMAs are issued fully unrolled: a rolled issue loop costs about
        // twice the MMA's own 64 cycles per instruction.
        const uint32_t vd = sdesc_sw128_lo(v_addr + vst * C::kKVBytes, BK * 128);
        umma_ts(d_o, a_p, vd, idesc_pv, (pv & (4u << s)) ? 0u : 1u);
#pragma unroll
        for (int kk = 1; kk < BK / 16; ++kk) umma_ts(d_o, a_p + kk * 8, vd + kk * (16 * 128 / 16), idesc_pv, 1u);
        // With one S buffer the next S of this slot is issued after this P.V,
        // so its s_full commit also covers this MMA; o_done is needed only
        // after the item's last P.V.
        if (pv & (16u << s)) umma_commit(&o_done[s]);
        umma_commit(&pv_done[s]);
        umma_commit(&v_empty[vst]);
        pv &= ~(21u << s);
        return true;
      };

      for (int it = 0; ok; ++it) {
        const int rs = it % kRing;
        if (!(ok = warp_all(mbar_wait(&sched_full[rs], (it / kRing) & 1, s_abort, p.wait_ns)))) break;
        const WorkItem info = ring[rs];
        if (lane == 0) mbar_arrive(&sched_empty[rs]);
        if (info.w < 0) break;
        const Tile (&t)[2] = info.t;
        bool qready[2] = {false, false};
        uint32_t nS[2] = {0, 0};

        Merge m = make_merge(p, t);
        int kt;
        bool in[2];
        bool first_kt = true;
        while (ok && m.next(kt, in[0], in[1])) {
          const int st = kv_it % S;
          const uint32_t ph = (kv_it / S) & 1;
          // At an item's first k-tile the pending P.V are the previous item's
          // last ones: they need no K, and the item's first K tile may still be
          // loading, so slot 0's goes out before the K wait and slot 1's too if
          // K has not landed. Later k-tiles keep the order K, PV_0, S_0, PV_1,
          // S_1 (one S buffer per tile) or K, S_0, S_1, PV_0, PV_1 (two).
          if (first_kt) {
            first_kt = false;
            if ((pv & 1u) && !(ok = issue_pv(0))) break;
            if ((pv & 2u) && !warp_all(mbar_try_wait(&k_full[st], ph)) && !(ok = issue_pv(1))) break;
          }
          if (!(ok = warp_all(mbar_wait(&k_full[st], ph, s_abort, p.wait_ns)))) break;
          tc_fence_after();
          // S_s = Q_s K^T for k-tile st; returns the pending-P.V flags it adds.
          auto issue_s = [&](int s) -> uint32_t {
            const uint32_t sb = nsq[s] % C::kSBufs;
            const uint32_t qd = sdesc_sw128_lo(q_addr + s * C::kQBytes, 16);
            const uint32_t kd = sdesc_sw128_lo(k_addr + st * C::kKVBytes, 16);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              // K step of 16 bf16 = 32 bytes inside the 128-byte row; every 4
              // steps move to the next 64-column chunk of the tile.
              const uint32_t off = (kk & 3) * 32;
              const uint32_t a = qd + (((kk >> 2) * (kRows * 128) + off) >> 4);
              const uint32_t bd = kd + (((kk >> 2) * (BK * 128) + off) >> 4);
              umma_ss(tmem + (s * C::kSBufs + sb) * BK, a, bd, idesc_qk, kk > 0 ? 1u : 0u);
            }
            umma_commit(&s_full[2 * s + sb]);
            ++nsq[s];
            const bool last = ++nS[s] == t[s].n;
            if (last) umma_commit(&q_empty[s]);  // last read of Q_s in this item
            return (1u << s) | (nS[s] == 1 ? (4u << s) : 0u) | (last ? (16u << s) : 0u);
          };
          auto q_ready = [&](int s) -> bool {
            if (qready[s]) return true;
            if (!warp_all(mbar_wait(&q_full[s], quse[s] & 1, s_abort, p.wait_ns))) return false;
            tc_fence_after();
            qready[s] = true;
            return true;
          };
          if constexpr (C::kSBufs == 2) {
            // Two S buffers per tile: both S of this k-tile go out first (into
            // the buffers the pending P.V do not read), then the pending P.V.
            uint32_t added = 0;
#pragma unroll
            for (int s = 0; s < 2; ++s) {
              if (in[s]) {
                if (!(ok = q_ready(s))) break;
                added |= issue_s(s);
              } else {
                if (lane == 0) mbar_arrive(&v_empty[st]);  // this tile does not read V at this k-tile
              }
            }
            if (!ok) break;
#pragma unroll
            for (int s = 0; s < 2; ++s)
              if ((pv & (1u << s)) && !(ok = issue_pv(s))) break;
            if (!ok) break;
#pragma unroll
            for (int s = 0; s < 2; ++s) {
              if (in[s]) {
                pkv[s] = kv_it;
                psq[s] = nsq[s] - 1;
              }
            }
            pv |= added;
          } else {
#pragma unroll
            for (int s = 0; s < 2; ++s) {
              if ((pv & (1u << s)) && !(ok = issue_pv(s))) break;
              if (in[s]) {
                if (!(ok = q_ready(s))) break;
                pkv[s] = kv_it;
                psq[s] = nsq[s];
                pv |= issue_s(s);
              } else {
                if (lane == 0) mbar_arrive(&v_empty[st]);  // this tile does not read V at this k-tile
              }
            }
          }
          if (!ok) break;
          umma_commit(&k_empty[st]);
          ++kv_it;
        }
#pragma unroll
        for (int s = 0; s < 2; ++s)
          if (t[s].n > 0) ++quse[s];
      }
      // The P.V still pending when the work runs out.
#pragma unroll
      for (int s = 0; s < 2; ++s)
        if (ok && (pv & (1u << s))) ok = issue_pv(s);
      if (!ok) *s_abort = 1;
      // Wait for every MMA issued here before TMEM can be released.
      umma_commit(drain);
      volatile int no_abort = 0;
      mbar_wait(drain, 0, &no_abort);
    }
   }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" :: "n"(kRegsHigh<BK>));
    // =================== softmax / correction / epilogue ===================
    const int slot = wg - 1;
    const int sw = warp & 3;
    const int r = sw * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(sw * 32) << 16;
    const uint32_t tmem_o = tmem + C::kOCol + slot * D;
    const MaskArgs& mk = p.mask;
    const bool k_ragged = (p.Nk % BK) != 0;
    int4* my_bounds = s_bounds + slot * 2 * BK;
    uint64_t* my_bnd = bnd_full + 2 * slot;
    uint32_t s_cnt = 0, o_cnt = 0, n_bnd = 0;
    bool ok = true;

    for (int it = 0; ok; ++it) {
      const int rs = it % kRing;
      if (!(ok = warp_all(mbar_wait(&sched_full[rs], (it / kRing) & 1, s_abort, p.wait_ns)))) break;
      const WorkItem info = ring[rs];
      __syncwarp();
      if (lane == 0) mbar_arrive(&sched_empty[rs]);
      if (info.w < 0) break;
      const Tile T = slot == 0 ? info.t[0] : info.t[1];
      if (!T.valid) continue;
      const int qi = (GP == 2) ? T.q0 + (r & 63) : T.q0 + r;
      const int head = (GP == 2) ? T.h0 + (r >> 6) : T.h0;
      const int n = T.n;
      // ALiBi slope of this row's head in log2 units (additive bias variant only).
      const float slope2 = kBias != 0 ? __ldg(p.slopes + head) * 1.4426950408889634f : 0.f;
      float m_run = -INFINITY, l_run = 0.f;

      for (int i = 0; i < n; ++i) {
        const int kt = T.lst[i];
        if (kt < 0 || kt >= p.nkt) {
          if (lane == 0) atomicOr(p.err, MFA_DEVERR_MAP);
          *s_abort = 1;
          ok = false;
          break;
        }
        const uint32_t cb = T.cls[kt];
        const bool partial = ((cb & 3u) == 2u) || (k_ragged && kt == p.nkt - 1);
        const int4* bnd = nullptr;
        if (partial && mk.kind == MFA_MASK_COLWISE) {
          // Stage the tile's column bounds (double-buffered: a thread at partial
          // tile k+2 has passed tile k+1's barrier, so tile k's readers are done).
          const int bs = n_bnd & 1;
          int4* dst = my_bounds + bs * BK;
          if (r < BK) {
            const int j = kt * BK + r;
            int4 v = make_int4(0, 0x7fffffff, 0, 0);  // columns past Nk: masked for every row
            if (j < p.Nk) {
              const size_t idx = T.bh_mask * p.Nk + j;
              v.x = mk.lts ? mk.lts[idx] : 0;
              v.y = mk.lte ? mk.lte[idx] : 0;
              v.z = mk.uts ? mk.uts[idx] : 0;
              v.w = mk.ute ? mk.ute[idx] : 0;
            }
            dst[r] = v;
          }
          mbar_arrive(&my_bnd[bs]);
          if (!(ok = warp_all(mbar_wait(&my_bnd[bs], (n_bnd >> 1) & 1, s_abort, p.wait_ns)))) break;
          bnd = dst;
          ++n_bnd;
        }
        // Masked columns of this row in a PARTIAL tile, as BK / 32 words (bit
        // j of word c = column 32c + j), built before S is ready so that one
        // short loop applies every mask kind and only these words are live
        // beside the scores.
        //   column-wise: the warp's 32 lanes hold 32 consecutive queries from
        //     qbase; lane j turns column (32c + j)'s two intervals into a word
        //     of masked rows (bit l = query qbase + l), and a 32x32 bit
        //     transpose across the warp gives each lane its own row's columns
        //     (columns past Nk are staged as masked for every row);
        //   band: the visible columns form one interval per row;
        //   block selection: the causal interval, cleared in the 64-column
        //     halves that the tile's class byte does not select.
        uint32_t mrow[BK / 32];
#pragma unroll
        for (int c = 0; c < BK / 32; ++c) mrow[c] = 0u;
        if (partial) {
          const int jb = kt * BK;
          if (bnd != nullptr) {
            const int qbase = qi - lane;
#pragma unroll
            for (int c = 0; c < BK / 32; ++c) {
              const int4 v = bnd[c * 32 + lane];
              const uint32_t w =
                  rows_in_interval(v.x - qbase, v.y - qbase) | rows_in_interval(v.z - qbase, v.w - qbase);
              mrow[c] = transpose32_warp(w, lane);
            }
          } else if (mk.kind == MFA_MASK_BAND) {
            const int lo = qi - mk.pre - jb;                  // first visible column of the tile
            const int hi = min(qi + mk.nxt - jb + 1, p.Nk - jb);  // one past the last one
#pragma unroll
            for (int c = 0; c < BK / 32; ++c) mrow[c] = ~rows_in_interval(lo - 32 * c, hi - 32 * c);
          } else {
            const int qsl = (GP == 2) ? 0 : (r >> 6);
            const int hi = min(qi - jb + 1, p.Nk - jb);
#pragma unroll
            for (int c = 0; c < BK / 32; ++c) {
              const bool sel = (cb >> (4 + 2 * qsl + (c >> 1))) & 1u;
              mrow[c] = sel ? ~rows_in_interval(-32 * c, hi - 32 * c) : ~0u;
            }
          }
        }
        // S number s_cnt of this tile sits in buffer s_cnt % kSBufs.
        const uint32_t sb = s_cnt % C::kSBufs;
        const uint32_t tmem_s = tmem + (slot * C::kSBufs + sb) * BK;
        if (!(ok = warp_all(mbar_wait(&s_full[2 * slot + sb], (s_cnt / C::kSBufs) & 1, s_abort, p.wait_ns)))) break;
        ++s_cnt;
        tc_fence_after();

        float s[BK];
        {
          uint32_t sv[BK / 32][32];
#pragma unroll
          for (int c = 0; c < BK / 32; ++c) tmem_ld_32x32b_x32(tmem_s + lane_off + c * 32, sv[c]);
          tmem_ld_wait();
#pragma unroll
          for (int jj = 0; jj < BK; ++jj) s[jj] = __uint_as_float(sv[jj >> 5][jj & 31]);
        }
        if (partial) {
#pragma unroll
          for (int jj = 0; jj < BK; ++jj)
            if ((mrow[jj >> 5] >> (jj & 31)) & 1u) s[jj] = -INFINITY;
        }
        // Scores in log2 units: s * scale here, or, with an additive bias,
        // s * scale + bias(i, j) written into s (masked entries stay -inf)
        // and a unit scale from here on.
        float sc = p.scale_log2;
        if constexpr (kBias == 2) {
          // -slope sqrt(|j - i|); |j - i| < 2^24 is exact in fp32, sqrt.approx is one MUFU op
          const float dj0 = static_cast<float>(kt * BK - qi);  // j - i of column 0
#pragma unroll
          for (int jj = 0; jj < BK; ++jj) {
            float r;
            asm("sqrt.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(fabsf(dj0 + static_cast<float>(jj))));
            s[jj] = fmaf(s[jj], sc, -slope2 * r);
          }
          sc = 1.f;
        } else if constexpr (kBias == 1) {
          // linear: slope (j - i); left-aligned: slope j = slope (j - i) + slope i. (Packed
          // f32x2 running sums measured the same and spilled at 128-key tiles.)
          const float c0 = slope2 * static_cast<float>(p.bias_kind == MFA_BIAS_ALIBI_LEFT ? kt * BK : kt * BK - qi);
#pragma unroll
          for (int jj = 0; jj < BK; ++jj) s[jj] = fmaf(s[jj], sc, fmaf(slope2, static_cast<float>(jj), c0));
          sc = 1.f;
        }
        // Row max with 3-input max instructions over four independent chains.
        float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int jj = 0; jj < BK; jj += 8)
#pragma unroll
          for (int a = 0; a < 4; ++a) mx4[a] = fmax3(mx4[a], s[jj + 2 * a], s[jj + 2 * a + 1]);
        const float mx = fmax3(fmaxf(mx4[0], mx4[1]), mx4[2], mx4[3]);
        const float mx_s = mx * sc;
        const bool need = mx_s > m_run + kRescaleThreshold;
        const float m_new = need ? mx_s : m_run;
        const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
        // P = 2^(s * scale - m) as bf16 over S, 32 columns at a time so that
        // only 16 packed registers are live beside s[]. S_t(i) being complete
        // implies P_t(i-1).V is complete (MMAs finish in issue order), so S and
        // O of this slot are free here. Four partial sums keep the FADD chain
        // short.
        float sum4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int c = 0; c < BK / 32; ++c) {
          uint32_t pk[16];
#pragma unroll
          for (int u = 0; u < 16; ++u) {
            const float e0 = ex2_approx(fmaf(s[c * 32 + 2 * u], sc, -m_use));
            const float e1 = ex2_approx(fmaf(s[c * 32 + 2 * u + 1], sc, -m_use));
            sum4[u & 3] += e0 + e1;
            pk[u] = pack_bf16x2(e0, e1);
          }
          tmem_st_32x32b_x16(tmem_s + lane_off + c * 16, pk);
        }
        const float sum = (sum4[0] + sum4[1]) + (sum4[2] + sum4[3]);
        const float alpha = need ? ex2_approx(m_run - m_use) : 1.f;
        l_run = l_run * alpha + sum;
        m_run = m_new;
        if (i > 0 && __any_sync(0xffffffffu, need)) {
          // Rare (the running max grew by more than the threshold): kept
          // rolled to save instruction-cache space for the hot path. With two
          // S buffers, S number k is issued before the P.V of S number k - 1,
          // so that P.V (phase k - 1 of pv_done; at most one phase is pending)
          // must complete before O is rescaled.
          if (C::kSBufs == 2 && !(ok = warp_all(mbar_wait(&pv_done[slot], (s_cnt - 2) & 1, s_abort, p.wait_ns)))) break;
#pragma unroll 1
          for (int c = 0; c < D / 32; ++c) {
            uint32_t o[32];
            tmem_ld_32x32b_x32(tmem_o + lane_off + c * 32, o);
            tmem_ld_wait();
#pragma unroll
            for (int u = 0; u < 32; ++u) o[u] = __float_as_uint(__uint_as_float(o[u]) * alpha);
            tmem_st_32x32b_x32(tmem_o + lane_off + c * 32, o);
            tmem_st_wait();
          }
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&p_full[2 * slot + sb]);
      }
      if (!ok) break;

      // ---- epilogue of this tile ----
      // The next item's first P.V into this slot's O waits for this warpgroup's
      // next P, which is written after these reads, so O needs no other guard.
      if (n > 0) {
        if (!(ok = warp_all(mbar_wait(&o_done[slot], o_cnt & 1, s_abort, p.wait_ns)))) break;
        ++o_cnt;
        tc_fence_after();
      }
      const bool has = l_run > 0.f;
      const float inv = has ? 1.f / l_run : 0.f;
      const bool store = qi < p.Nq;
      // Each warp writes its 32 rows through its own staging tile, 32 columns
      // at a time: every lane puts its row's 64 bytes into shared memory
      // (64-byte swizzle: 16-byte unit j of row l at unit j ^ ((l >> 1) & 3),
      // conflict-free), and one lane hands the tile to a TMA store, which clips
      // rows past Nq. The stores leave the warp at once; a staging tile is
      // rewritten only after the TMA has read its previous contents.
      {
        const int row0 = (GP == 2) ? T.q0 + ((sw * 32) & 63) : T.q0 + sw * 32;
        const int hd = (GP == 2) ? T.h0 + (sw >> 1) : T.h0;
        const uint32_t stg = smem_u32(smem + C::kStage + (slot * 4 + sw) * C::kStageBytes);
        const uint32_t my_row = stg + lane * 64;
        const uint32_t swz = (lane >> 1) & 3;
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          if (n > 0) {
            tmem_ld_32x32b_x32(tmem_o + lane_off + c * 32, o);
            tmem_ld_wait();
          }
          uint32_t w[16];
#pragma unroll
          for (int u = 0; u < 16; ++u)
            w[u] = has ? pack_bf16x2(__uint_as_float(o[2 * u]) * inv, __uint_as_float(o[2 * u + 1]) * inv) : 0u;
          if (lane == 0) bulk_wait_read_all();
          __syncwarp();
#pragma unroll
          for (int j = 0; j < 4; ++j)
            st_shared_v4(my_row + ((j ^ swz) << 4), w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_4d(&tm_o, smem + C::kStage + (slot * 4 + sw) * C::kStageBytes, c * 32, row0, hd, T.b);
            bulk_commit_group();
          }
        }
      }
      if (store) {
        const float lse = has ? (m_run + __log2f(l_run)) * 0.69314718055994530942f : -INFINITY;
        p.lse[(static_cast<size_t>(T.b) * p.Hq + head) * p.Nq + qi] = lse;
      }
    }
    if (!ok && lane == 0) atomicOr(p.err, MFA_DEVERR_TIMEOUT);
    // The warp's TMA stores must be complete before its staging tile and the
    // CTA go away.
    if (lane == 0) bulk_wait_all();
    __syncwarp();
  }

  __syncthreads();
  if (threadIdx.x == 0) {
    // The producer (this thread) took its last item before this point; the CTA
    // that finishes last resets the scheduling words for the next launch.
    __threadfence();
    if (atomicAdd(&p.sched[1], 1u) == gridDim.x - 1) {
      atomicExch(&p.sched[0], 0u);
      atomicExch(&p.sched[1], 0u);
      __threadfence();
    }
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// ------------------------------------------------------------------------
// host side
// ------------------------------------------------------------------------
bool make_map(CUtensorMap* map, const mfa_tensor* t, int box_rows) {
  auto fn = tensor_map_encoder();
  if (!fn) return false;
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(t->D), static_cast<cuuint64_t>(t->N),
                        static_cast<cuuint64_t>(t->H), static_cast<cuuint64_t>(t->B)};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(t->stride[2]) * 2, static_cast<cuuint64_t>(t->stride[1]) * 2,
                           static_cast<cuuint64_t>(t->stride[0]) * 2};
  cuuint32_t box[4] = {64, static_cast<cuuint32_t>(box_rows), 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, t->data, dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// The output as TMA-store destination: 32-column x 32-row boxes with the
// 64-byte swizzle of the kernel's staging tiles.
bool make_store_map(CUtensorMap* map, const mfa_tensor* t) {
  auto fn = tensor_map_encoder();
  if (!fn) return false;
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(t->D), static_cast<cuuint64_t>(t->N),
                        static_cast<cuuint64_t>(t->H), static_cast<cuuint64_t>(t->B)};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(t->stride[2]) * 2, static_cast<cuuint64_t>(t->stride[1]) * 2,
                           static_cast<cuuint64_t>(t->stride[0]) * 2};
  cuuint32_t box[4] = {32, 32, 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, t->data, dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

mfa_status check_tensor(const mfa_tensor* t) {
  if (!t) return MFA_ERR_INVALID_ARG;
  if (t->B <= 0 || t->H <= 0 || t->N < 0 || t->D <= 0) return MFA_ERR_INVALID_ARG;
  if (!t->data && t->N > 0) return MFA_ERR_INVALID_ARG;  // an empty tensor may have no storage
  if (t->dtype != MFA_BF16 && t->dtype != MFA_F32) return MFA_ERR_INVALID_ARG;
  if (t->stride[3] != 1) return MFA_ERR_UNSUPPORTED;
  for (int a = 0; a < 3; ++a)
    if (t->stride[a] <= 0 || (t->stride[a] * 2) % 16 != 0) return MFA_ERR_UNSUPPORTED;
  if (reinterpret_cast<uintptr_t>(t->data) % 16 != 0) return MFA_ERR_UNSUPPORTED;
  return MFA_OK;
}

template <int D, int BK, int GP, int kBias>
mfa_status launch_b(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const CUtensorMap& mo,
                    const FwdParams& p, cudaStream_t s) {
  using C = Cfg<D, BK>;
  static std::atomic<uint64_t> attr_devs{0};
  if (!ensure_smem_attr(reinterpret_cast<const void*>(mfa_fwd_kernel<D, BK, GP, kBias>), C::kAlloc, attr_devs))
    return MFA_ERR_CUDA;
  const int sms = device_sm_count();
  if (sms <= 0) return MFA_ERR_CUDA;
  const int grid = p.n_items < sms ? p.n_items : sms;  // persistent: at most one CTA per SM
  mfa_fwd_kernel<D, BK, GP, kBias><<<grid, kThreads, C::kAlloc, s>>>(mq, mk, mv, mo, p);
  return cudaGetLastError() == cudaSuccess ? MFA_OK : MFA_ERR_CUDA;
}

template <int D, int BK, int GP>
mfa_status launch(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const CUtensorMap& mo,
                  const FwdParams& p, cudaStream_t s) {
  if (p.bias_kind == MFA_BIAS_NONE) return launch_b<D, BK, GP, 0>(mq, mk, mv, mo, p, s);
  if (p.bias_kind == MFA_BIAS_ALIBI_SQRT) return launch_b<D, BK, GP, 2>(mq, mk, mv, mo, p, s);
  return launch_b<D, BK, GP, 1>(mq, mk, mv, mo, p, s);
}

}  // namespace
}  // namespace mfa

namespace mfa {
namespace {
// Armed by mfa_test_arm_fwd_timeout: the wait limit in microseconds for the
// next bf16 forward launch, which then withholds one K tile (0 = not armed).
std::atomic<uint32_t> g_timeout_test_us{0};
mfa_status fwd_impl(const mfa_tensor* q, const mfa_tensor* k, const mfa_tensor* v, const mfa_mask_desc* mask,
                    const mfa_bias* bias, const mfa_tensor* out, float* lse, void* stream);
}  // namespace
}  // namespace mfa

extern "C" mfa_status mfa_fwd(const mfa_tensor* q, const mfa_tensor* k, const mfa_tensor* v,
                              const mfa_mask_desc* mask, const mfa_tensor* out, float* lse, void* stream) {
  return mfa::fwd_impl(q, k, v, mask, nullptr, out, lse, stream);
}

extern "C" mfa_status mfa_test_arm_fwd_timeout(uint32_t wait_us) {
  if (wait_us == 0 || wait_us > 1000000u) return MFA_ERR_INVALID_ARG;
  mfa::g_timeout_test_us.store(wait_us);
  return MFA_OK;
}

extern "C" mfa_status mfa_fwd_bias(const mfa_tensor* q, const mfa_tensor* k, const mfa_tensor* v,
                                   const mfa_mask_desc* mask, const mfa_bias* bias, const mfa_tensor* out, float* lse,
                                   void* stream) {
  if (!bias) return MFA_ERR_INVALID_ARG;
  return mfa::fwd_impl(q, k, v, mask, bias, out, lse, stream);
}

namespace mfa {

mfa_status check_fwd_args(const mfa_tensor* q, const mfa_tensor* k, const mfa_tensor* v, const mfa_mask_desc* mask,
                          const mfa_bias* bias, const mfa_tensor* out, const float* lse, int32_t block_q) {
  mfa_status st;
  const int32_t bias_kind = bias ? bias->kind : MFA_BIAS_NONE;
  if (bias_kind < MFA_BIAS_NONE || bias_kind > MFA_BIAS_ALIBI_LEFT) return MFA_ERR_INVALID_ARG;
  if (bias_kind != MFA_BIAS_NONE && !bias->slopes) return MFA_ERR_INVALID_ARG;
  if ((st = check_tensor(q)) != MFA_OK || (st = check_tensor(k)) != MFA_OK || (st = check_tensor(v)) != MFA_OK ||
      (st = check_tensor(out)) != MFA_OK)
    return st;
  if (!lse && q->N > 0) return MFA_ERR_INVALID_ARG;  // an empty lse may have no storage
  if ((st = check_mask(mask)) != MFA_OK) return st;
  if (q->dtype != k->dtype || q->dtype != v->dtype || out->dtype != q->dtype) return MFA_ERR_INVALID_ARG;
  if (k->B != q->B || v->B != q->B || out->B != q->B) return MFA_ERR_SHAPE_MISMATCH;
  if (k->H != v->H || k->N != v->N || k->D != q->D || v->D != q->D) return MFA_ERR_SHAPE_MISMATCH;
  if (out->H != q->H || out->N != q->N || out->D != q->D) return MFA_ERR_SHAPE_MISMATCH;
  if (q->H % k->H != 0) return MFA_ERR_SHAPE_MISMATCH;
  if (mask->B != q->B || mask->Nq != q->N || mask->Nk != k->N) return MFA_ERR_SHAPE_MISMATCH;
  if (mask->Hm != 1 && mask->Hm != q->H) return MFA_ERR_SHAPE_MISMATCH;
  if (q->D != 64 && q->D != 128) return MFA_ERR_UNSUPPORTED;
  if (q->N > (int64_t(1) << 30) || k->N > (int64_t(1) << 30) || q->H > 65535) return MFA_ERR_UNSUPPORTED;
  if (q->dtype == MFA_F32) return bias_kind != MFA_BIAS_NONE ? MFA_ERR_UNSUPPORTED : MFA_OK;  // no fp32 bias
  const int64_t G = q->H / k->H;
  if (block_q == 64 && (mask->Hm != 1 || G % 2 != 0)) return MFA_ERR_UNSUPPORTED;  // two heads per 64-row tile
  return MFA_OK;
}

namespace {
mfa_status fwd_impl(const mfa_tensor* q, const mfa_tensor* k, const mfa_tensor* v, const mfa_mask_desc* mask,
                    const mfa_bias* bias, const mfa_tensor* out, float* lse, void* stream) {
  mfa_status st;
  const int32_t bias_kind = bias ? bias->kind : MFA_BIAS_NONE;
  if ((st = check_mask(mask)) != MFA_OK) return st;
  if (!mask->map) return MFA_ERR_INVALID_ARG;
  const mfa_tile_map* map = mask->map;
  if ((st = check_map_matches(mask, map)) != MFA_OK) return st;
  if (map->kind != mask->kind) return MFA_ERR_SHAPE_MISMATCH;
  if ((st = check_fwd_args(q, k, v, mask, bias, out, lse, map->block_q)) != MFA_OK) return st;
  if (q->dtype == MFA_F32) return launch_fwd_f32(q, k, v, mask, map, out, lse, static_cast<cudaStream_t>(stream));
  const int G = static_cast<int>(q->H / k->H);
  const int GP = map->block_q == 64 ? 2 : 1;
  if (q->N == 0) return MFA_OK;

  FwdParams p;
  p.B = static_cast<int32_t>(q->B); p.Hq = static_cast<int32_t>(q->H); p.Hkv = static_cast<int32_t>(k->H);
  p.G = G; p.Hm = mask->Hm; p.Nq = static_cast<int32_t>(q->N); p.Nk = static_cast<int32_t>(k->N);
  p.nqt = map->nqt; p.nkt = map->nkt;
  // Work items pair two query tiles that read the same key/value head: two head
  // tiles of one group when the mask is shared and the group holds an even
  // number of head tiles (kind 0, same list), else two consecutive query tiles
  // of one head tile (kind 1, union of the two lists).
  const int tiles_per_group = G / GP;
  int64_t n_items64;
  if (mask->Hm == 1 && tiles_per_group % 2 == 0) {
    p.item_kind = 0;
    p.pairs = p.Hq / GP / 2;
    p.n_ht = 0; p.nqp = 0;
    n_items64 = static_cast<int64_t>(p.B) * p.nqt * p.pairs;
  } else {
    p.item_kind = 1;
    p.pairs = 0;
    p.n_ht = p.Hq / GP;
    p.nqp = (p.nqt + 1) / 2;
    n_items64 = static_cast<int64_t>(p.B) * p.n_ht * p.nqp;
  }
  p.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(q->D)));
  p.mask = mask_args(mask);
  p.cls = map->tile_class; p.list = map->tile_list; p.count = map->tile_count; p.order = map->order;
  p.out = static_cast<__nv_bfloat16*>(out->data);
  p.os0 = out->stride[0]; p.os1 = out->stride[1]; p.os2 = out->stride[2];
  p.lse = lse;
  p.err = map->err;
  p.sched = map->err + 1;
  p.bias_kind = bias_kind;
  p.slopes = bias_kind != MFA_BIAS_NONE ? bias->slopes : nullptr;
  p.wait_ns = kWaitTimeoutNs;
  p.withhold_k = 0;
  const uint32_t armed_us = g_timeout_test_us.exchange(0u);
  if (armed_us != 0) {
    p.wait_ns = static_cast<uint64_t>(armed_us) * 1000u;
    p.withhold_k = 1;
  }
  if (n_items64 <= 0) return MFA_OK;
  if (n_items64 > 0x7fffffff) return MFA_ERR_UNSUPPORTED;
  p.n_items = static_cast<int32_t>(n_items64);

  // With Nk == 0 every list is empty and the K/V maps are never read.
  CUtensorMap mq, mk, mv, mo;
  memset(&mk, 0, sizeof(mk));
  memset(&mv, 0, sizeof(mv));
  if (!make_map(&mq, q, 64)) return MFA_ERR_CUDA;
  if (!make_store_map(&mo, out)) return MFA_ERR_CUDA;
  if (k->N > 0 && (!make_map(&mk, k, map->block_k) || !make_map(&mv, v, map->block_k))) return MFA_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int D = static_cast<int>(q->D), BK = map->block_k;
  if (D == 128 && BK == 128) return GP == 2 ? launch<128, 128, 2>(mq, mk, mv, mo, p, s) : launch<128, 128, 1>(mq, mk, mv, mo, p, s);
  if (D == 128 && BK == 64) return GP == 2 ? launch<128, 64, 2>(mq, mk, mv, mo, p, s) : launch<128, 64, 1>(mq, mk, mv, mo, p, s);
  if (D == 64 && BK == 128) return GP == 2 ? launch<64, 128, 2>(mq, mk, mv, mo, p, s) : launch<64, 128, 1>(mq, mk, mv, mo, p, s);
  return GP == 2 ? launch<64, 64, 2>(mq, mk, mv, mo, p, s) : launch<64, 64, 1>(mq, mk, mv, mo, p, s);
}

}  // namespace
}  // namespace mfa
