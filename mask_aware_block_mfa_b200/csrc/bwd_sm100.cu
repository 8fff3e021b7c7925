// mfa_bwd: gradients of the mask-aware attention forward pass for sm_100a.
//
// For a loss whose gradient with respect to out is dout (lse is not used by
// the loss), with P = exp(S - lse) on visible pairs:
//   dV = P^T dout, dP = dout V^T, Delta = rowsum(dout * out),
//   dS = P * (dP - Delta), dQ = dS K / sqrt(d), dK = dS^T Q / sqrt(d);
// the key/value head of a group receives the sums over its query heads. The
// tile map of the forward pass decides which (query tile, key tile) pairs are
// computed: SKIP tiles are never visited, FULL tiles take no mask work and
// PARTIAL tiles apply the exact element mask (Binary Block Masking, abstract;
// FlashMask's column-wise intervals, the Ascend band, 64-block selection).
//
// Launches: (1) prep: Delta and lse in log2 units per query row, padded to the
// 64-row query tiles, and the fp32 dQ accumulator zeroed; (2) per key tile the
// ascending list of non-SKIP query tiles (the forward map transposed) and, in
// the last block, the key tiles ordered by list length; (3) the main kernel;
// (4) dQ accumulator -> dq (scaled, bf16).
//
// Main kernel: persistent, one CTA per SM, a work item is (batch, key/value
// head, 128-key tile). Its key/value tiles stay in shared memory while the
// item walks every query head g of the group and every listed 64-query tile
// (an "iteration"). TMEM (512 columns):
//   [128b, 128b+64)   S^T = K Q^T of iteration parity b (P^T in bf16 over its
//                     columns [16, 48), then dQ^T = K^T dS^T of the iteration)
//   [128b+64, 128b+128) dP^T = V dout^T (dS^T in bf16 over [80, 112))
//   [256, 384) dV,  [384, 512) dK   (accumulated over the item)
// Rows of S^T, dP^T, dV, dK are keys (TMEM lane = key); rows of dQ^T are head
// dimensions. Roles (512 threads):
//   warp 0        TMA producer: K, V once per item; Q, dout and the tile's lse
//                 and Delta per iteration into a three-stage ring.
//   warp 1        TMEM owner and MMA issuer: S^T, dP^T of iteration u + 1 go
//                 out before dV, dK, dQ^T of iteration u, so the tensor core
//                 works on one iteration while the key-row warps work on the
//                 other.
//   warps 4-11    two warpgroups, one key row per thread, query columns
//                 0-31 and 32-63: P^T = exp2(S^T c - lse2) (0 where masked),
//                 dS^T = P^T (dP^T - Delta), both to TMEM in bf16 and dS^T
//                 also to shared memory (the B operand of dQ^T); at the end of
//                 an item one warpgroup writes dV and the other dK.
//   warps 12-15   one head dimension per thread: dQ^T from TMEM to a staging
//                 tile, added into the fp32 accumulator by TMA reduces.
//   warps 2-3     idle.
// Every wait is bounded; a wait that gives up raises the CTA's abort flag and
// sets MFA_DEVERR_TIMEOUT in the map's error word.
#include <climits>
#include <cmath>
#include <cstring>
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include "mfa.h"
#include "mfa_device.cuh"
#include "mfa_internal.h"
#include "order.cuh"

namespace mfa {
namespace {

constexpr int kBQ = 64;    // queries per tile (the MMA N of S^T, dP^T, dQ^T)
constexpr int kBK = 128;   // keys per tile (the MMA M)
constexpr int kD = 128;    // head dimension
constexpr int kThreads = 512;
constexpr int kRing = 4;
constexpr int kStages = 3;  // Q / dout / lse2 / Delta ring
constexpr uint32_t kPCol = 16;   // packed P^T inside the S^T columns [0, 64) of a parity block
constexpr uint32_t kDSCol = 80;  // packed dS^T inside the dP^T columns [64, 128)

// ---- shared-memory layout (bytes from the 1024-aligned dynamic base) ----
constexpr int kKBytes = kBK * kD * 2;    // 32 KB: two 64-column chunks of 128 rows
constexpr int kQBytes = kBQ * kD * 2;    // 16 KB: two 64-column chunks of 64 rows
constexpr int kSK = 0;
constexpr int kSV = kSK + kKBytes;
constexpr int kSQ = kSV + kKBytes;                 // [kStages]
constexpr int kSDO = kSQ + kStages * kQBytes;     // [kStages]
constexpr int kDSBytes = kBK * kBQ * 2;           // dS^T: 128 key rows x 64 queries, SW128
constexpr int kSDS = kSDO + kStages * kQBytes;    // [2 buffers]
constexpr int kStgRows = 32;                      // dQ staging: two halves of 32 rows x 128 fp32
constexpr int kStgBytes = kStgRows * kD * 4;
constexpr int kSStg = kSDS + 2 * kDSBytes;        // [2 halves]
constexpr int kSLse = kSStg + 2 * kStgBytes;      // [kStages][64] lse2, then [kStages][64] Delta
constexpr int kSBar = kSLse + 2 * kStages * kBQ * 4;
constexpr int kNumBars = 2 + 2 * kStages + 2 * 6 + 1 + 4 + 1 + 2 * kRing;
constexpr int kSRing = kSBar + ((kNumBars * 8 + 127) / 128) * 128;
constexpr int kMeta = 8;  // per-iteration (query tile, head, class byte) published by the producer
constexpr int kSMeta = kSRing + kRing * 32;
constexpr int kSMisc = kSMeta + kMeta * 16;
constexpr int kSmemBytes = kSMisc + 32;
static_assert(kSmemBytes <= 227 * 1024, "shared memory");
static_assert(kSDS % 1024 == 0 && kSQ % 1024 == 0 && kSDO % 1024 == 0 && kDSBytes % 1024 == 0,
              "SW128 tiles need 1024-byte alignment");

struct BwdParams {
  int32_t B, Hq, Hkv, G, Nq, Nk;
  int32_t nqt, qsub;  // the map's query tiles and 64-row tiles per map tile (block_q / 64)
  int32_t nq64, nkt, nqp, n_items;  // 64-row query tiles, key tiles, nq64 * 64
  float scale_log2;  // log2(e) / sqrt(d)
  float scale;       // 1 / sqrt(d)
  MaskArgs mask;
  const uint8_t* cls;     // forward map classes [B][nqt][nkt] (mask heads = 1)
  const int32_t* tlist;   // [B][nkt][nq64] ascending non-SKIP 64-row query tiles
  const int32_t* tcount;  // [B][nkt]
  const int32_t* torder;  // [B * nkt] key tiles, longest list first
  int32_t order_lpt;      // 1: key tiles longest first; 0: ascending
  __nv_bfloat16* dk;
  int64_t dks0, dks1, dks2;
  __nv_bfloat16* dv;
  int64_t dvs0, dvs1, dvs2;
  uint32_t* err;
  uint32_t* sched;  // [0] next item, [1] finished CTAs
};

struct BwdItem {
  int32_t w;  // -1: no more work
  int32_t b, hkv, kt, n, e;
  int32_t pad[2];
};
static_assert(sizeof(BwdItem) == 32, "ring slot");

__device__ __forceinline__ bool warp_all(bool ok) { return __all_sync(0xffffffffu, ok); }

// Bits [a, b) of a 64-bit word, a and b clamped to [0, 64].
__device__ __forceinline__ uint64_t bits64(int a, int b) {
  a = max(a, 0);
  b = min(b, 64);
  if (a >= b) return 0ull;
  const uint64_t hi = b >= 64 ? ~0ull : ((1ull << b) - 1ull);
  return hi & ~((1ull << a) - 1ull);
}

// Instruction descriptor, kind::f16, bf16 A and B, f32 accumulator, with the
// major-ness of A (bit 15) and B (bit 16): 0 = K-major, 1 = MN-major.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool a_mn, bool b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16) |
         (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

__device__ __forceinline__ void bulk_load(void* smem_dst, const void* gsrc, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
               :: "r"(smem_u32(smem_dst)), "l"(gsrc), "r"(bytes), "r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void tma_reduce_add_4d(const CUtensorMap* map, const void* smem_src, int32_t c0,
                                                  int32_t c1, int32_t c2, int32_t c3) {
  asm volatile("cp.reduce.async.bulk.tensor.4d.global.shared::cta.add.tile.bulk_group [%0, {%1, %2, %3, %4}], [%5];"
               :: "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(smem_u32(smem_src))
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read1() { asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Items (batch, key tile, key/value head) go out with the heads of one key
// tile together, key tiles either longest list first or in ascending order
// (see order_lpt).
__device__ __forceinline__ void decode(const BwdParams& p, int w, BwdItem& it) {
  const int e = p.order_lpt ? p.torder[w / p.Hkv] : w / p.Hkv;
  it.w = w;
  it.hkv = w % p.Hkv;
  it.e = e;
  it.b = e / p.nkt;
  it.kt = e % p.nkt;
  it.n = p.tcount[e];
}

// ------------------------------------------------------------------------
// (1) prep: Delta_i = dout_i . out_i and lse2_i = lse_i log2(e) per query
// row, padded to nqp = nq64 * 64 rows per head (padding and rows without a
// visible key get lse2 = +inf, so their P is exactly 0); dQ accumulator rows
// zeroed. Half a warp per row: lane l of the half handles head dimensions
// 8l .. 8l + 7 with 16-byte loads.
// ------------------------------------------------------------------------
__global__ void __launch_bounds__(256) k_bwd_prep(const __nv_bfloat16* __restrict__ out, int64_t os0, int64_t os1,
                                                  int64_t os2, const __nv_bfloat16* __restrict__ dout, int64_t ds0,
                                                  int64_t ds1, int64_t ds2, const float* __restrict__ lse, int Hq,
                                                  int Nq, int nqp, int64_t rows, float* __restrict__ lse2,
                                                  float* __restrict__ delta, float* __restrict__ dq_acc,
                                                  uint32_t* __restrict__ words) {
  const int hl = threadIdx.x & 15;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 4) + (threadIdx.x >> 4);
  if (blockIdx.x == 0 && threadIdx.x < 4) words[threadIdx.x] = 0u;
  if (row >= rows) return;  // whole half-warps leave together (rows are per half-warp)
  const int64_t bh = row / nqp;
  const int i = static_cast<int>(row % nqp);
  const int b = static_cast<int>(bh / Hq), h = static_cast<int>(bh % Hq);
  float dl = 0.f, l2 = INFINITY;
  const unsigned half_mask = (threadIdx.x & 16) ? 0xffff0000u : 0x0000ffffu;
  if (i < Nq) {
    const uint4 o = *reinterpret_cast<const uint4*>(out + b * os0 + h * os1 + i * os2 + 8 * hl);
    const uint4 g = *reinterpret_cast<const uint4*>(dout + b * ds0 + h * ds1 + i * ds2 + 8 * hl);
    const uint32_t ow[4] = {o.x, o.y, o.z, o.w}, gw[4] = {g.x, g.y, g.z, g.w};
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&ow[c]));
      const float2 z = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&gw[c]));
      dl = fmaf(a.x, z.x, fmaf(a.y, z.y, dl));
    }
#pragma unroll
    for (int d = 8; d > 0; d >>= 1) dl += __shfl_xor_sync(half_mask, dl, d);
    const float l = lse[bh * Nq + i];
    l2 = l == -INFINITY ? INFINITY : l * 1.4426950408889634f;
    float4* acc = reinterpret_cast<float4*>(dq_acc + (bh * Nq + i) * kD);
    acc[2 * hl] = make_float4(0.f, 0.f, 0.f, 0.f);
    acc[2 * hl + 1] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  if (hl == 0) {
    lse2[row] = l2;
    delta[row] = dl;
  }
}

// ------------------------------------------------------------------------
// (2) transposed lists: one warp per (batch, key tile) compacts the 64-row
// query tiles whose class is not SKIP, in ascending order (a map built with
// 128-row query tiles gives both of its 64-row halves the tile's class); the
// last block to finish orders the key tiles by list length (longest first,
// stable).
// ------------------------------------------------------------------------
__global__ void __launch_bounds__(128) k_bwd_tlist(const uint8_t* __restrict__ cls, int nqt, int qsub, int nq64,
                                                   int nkt, int32_t* __restrict__ tlist, int32_t* __restrict__ tcount,
                                                   int32_t* __restrict__ torder, uint32_t* __restrict__ words) {
  extern __shared__ int s_hist[];
  __shared__ int s_last;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int b = blockIdx.y;
  const int kt = blockIdx.x * 4 + warp;
  if (kt < nkt) {
    const size_t e = static_cast<size_t>(b) * nkt + kt;
    int n = 0;
    for (int base = 0; base < nq64; base += 32) {
      const int qt = base + lane;
      const bool on = qt < nq64 && (cls[(static_cast<size_t>(b) * nqt + qt / qsub) * nkt + kt] & 3u) != 0u;
      const unsigned bal = __ballot_sync(0xffffffffu, on);
      if (on) tlist[e * nq64 + n + __popc(bal & ((1u << lane) - 1u))] = qt;
      n += __popc(bal);
    }
    if (lane == 0) tcount[e] = n;
  }
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) s_last = atomicAdd(&words[2], 1u) == gridDim.x * gridDim.y - 1;
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  order_by_count_desc(tcount, static_cast<int>(gridDim.y) * nkt, nq64, torder, s_hist);
  if (threadIdx.x == 0) words[2] = 0u;
}

// ------------------------------------------------------------------------
// (4) dq = bf16(dq_acc / sqrt(d)); eight elements per thread.
// ------------------------------------------------------------------------
__global__ void __launch_bounds__(256) k_bwd_dq_convert(const float* __restrict__ dq_acc, int Hq, int Nq,
                                                        int64_t n8, float scale, __nv_bfloat16* __restrict__ dq,
                                                        int64_t s0, int64_t s1, int64_t s2) {
  for (int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; t < n8;
       t += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t row = t / (kD / 8);
    const int c = static_cast<int>(t % (kD / 8));
    const int64_t bh = row / Nq;
    const int i = static_cast<int>(row % Nq);
    const int b = static_cast<int>(bh / Hq), h = static_cast<int>(bh % Hq);
    const float4 a = reinterpret_cast<const float4*>(dq_acc)[2 * t];
    const float4 z = reinterpret_cast<const float4*>(dq_acc)[2 * t + 1];
    uint4 o;
    o.x = pack_bf16x2(a.x * scale, a.y * scale);
    o.y = pack_bf16x2(a.z * scale, a.w * scale);
    o.z = pack_bf16x2(z.x * scale, z.y * scale);
    o.w = pack_bf16x2(z.z * scale, z.w * scale);
    *reinterpret_cast<uint4*>(dq + b * s0 + h * s1 + i * s2 + 8 * c) = o;
  }
}

// ------------------------------------------------------------------------
// (3) main kernel
// ------------------------------------------------------------------------
__global__ void __launch_bounds__(kThreads, 1)
    mfa_bwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                   const __grid_constant__ CUtensorMap tm_dq, const float* __restrict__ lse2,
                   const float* __restrict__ delta, const BwdParams p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  // The SW128 operand tiles need a 1024-byte aligned base; the declaration
  // asks for it and this checks it (uniformly, before any barrier exists).
  if ((smem_u32(smem) & 1023u) != 0u) {
    if (threadIdx.x == 0) atomicOr(p.err, MFA_DEVERR_TIMEOUT);
    return;
  }
  uint8_t* sK = smem + kSK;
  uint8_t* sV = smem + kSV;
  uint8_t* sQ = smem + kSQ;
  uint8_t* sDO = smem + kSDO;
  uint8_t* sDS = smem + kSDS;
  float* sStg = reinterpret_cast<float*>(smem + kSStg);       // [2][32][128]
  float* sLse = reinterpret_cast<float*>(smem + kSLse);       // [kStages][64]
  float* sDelta = sLse + kStages * kBQ;                       // [kStages][64]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kSBar);
  uint64_t* kv_full = bars;                  // 1
  uint64_t* kv_empty = kv_full + 1;          // 1
  uint64_t* q_full = kv_empty + 1;           // [kStages]
  uint64_t* q_empty = q_full + kStages;      // [kStages]
  uint64_t* s_full = q_empty + kStages;      // [2] S^T, dP^T of parity b ready
  uint64_t* p_full = s_full + 2;             // [2] P^T, dS^T of parity b written
  uint64_t* dq_full = p_full + 2 + 2;        // [2] dQ^T of parity b ready (and dS^T buffer b read)
  uint64_t* dq_free = dq_full + 2;           // [2] dQ^T of parity b read out
  uint64_t* kv_done = dq_free + 4;           // 1   (two spare slots above)
  uint64_t* stg_full = kv_done + 1;          // [2] staging half written
  uint64_t* stg_free = stg_full + 2;         // [2] staging half read by its reduce
  uint64_t* drain = stg_free + 2;            // 1
  uint64_t* sched_full = drain + 1;          // [kRing]
  uint64_t* sched_empty = sched_full + kRing;
  BwdItem* ring = reinterpret_cast<BwdItem*>(smem + kSRing);
  int4* meta = reinterpret_cast<int4*>(smem + kSMeta);  // [kMeta] {qt, head, class byte, 0}
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + kSMisc);
  volatile int* s_abort = reinterpret_cast<volatile int*>(smem + kSMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int wg = warp >> 2;

  if (warp == 0 && lane == 0) {
    mbar_init(kv_full, 1);
    mbar_init(kv_empty, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&q_full[s], 1);
      mbar_init(&q_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&s_full[s], 1);
      mbar_init(&p_full[s], 256);  // both key-row warpgroups
      mbar_init(&dq_full[s], 1);
      mbar_init(&dq_free[s], 128);
      mbar_init(&stg_full[s], 128);
      mbar_init(&stg_free[s], 1);
    }
    mbar_init(kv_done, 1);
    mbar_init(drain, 1);
    for (int i = 0; i < kRing; ++i) {
      mbar_init(&sched_full[i], 1);
      mbar_init(&sched_empty[i], 1 + 4 + 4 + 4);  // the MMA warp and one lane of every other consumer warp
    }
    *s_abort = 0;
    fence_mbarrier_init();
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    tma_prefetch_desc(&tm_do);
    tma_prefetch_desc(&tm_dq);
  }
  if (warp == 1) {
    tmem_alloc(s_tmem, 512);
    tmem_relinquish();
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;

  if (warp == 0) {
    // =================== TMA producer ===================
    if (lane == 0) {
      uint32_t u = 0, kv_loads = 0;
      bool stop = false;
      for (int it = 0; !stop; ++it) {
        const int rs = it % kRing;
        if (it >= kRing && !mbar_wait(&sched_empty[rs], ((it / kRing) - 1) & 1, s_abort)) break;
        const uint32_t wu = atomicAdd(&p.sched[0], 1u);
        BwdItem info;
        info.w = wu < static_cast<uint32_t>(p.n_items) ? static_cast<int>(wu) : -1;
        info.b = info.hkv = info.kt = info.n = info.e = 0;
        if (info.w >= 0) decode(p, info.w, info);
        ring[rs] = info;
        mbar_arrive(&sched_full[rs]);
        if (info.w < 0) break;
        if (info.n == 0) continue;
        if (kv_loads > 0 && !mbar_wait(kv_empty, (kv_loads - 1) & 1, s_abort)) break;
        mbar_arrive_expect_tx(kv_full, 2 * kKBytes);
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          tma_load_4d(sK + c * (kBK * 128), &tm_k, kv_full, c * 64, info.kt * kBK, info.hkv, info.b);
          tma_load_4d(sV + c * (kBK * 128), &tm_v, kv_full, c * 64, info.kt * kBK, info.hkv, info.b);
        }
        ++kv_loads;
        const int32_t* lst = p.tlist + static_cast<size_t>(info.e) * p.nq64;
        const uint8_t* crow = p.cls + static_cast<size_t>(info.b) * p.nqt * p.nkt + info.kt;
        for (int g = 0; g < p.G && !stop; ++g) {
          const int h = info.hkv * p.G + g;
          for (int i = 0; i < info.n; ++i, ++u) {
            const int qt = lst[i];
            const int cb = crow[static_cast<size_t>(qt / p.qsub) * p.nkt];
            const uint32_t st = u % kStages;
            if (u >= kStages && !mbar_wait(&q_empty[st], ((u - kStages) / kStages) & 1, s_abort)) {
              stop = true;
              break;
            }
            // Slot u % kMeta was last read for iteration u - kMeta: by the
            // key-row warps before p_full(u - kMeta) and by the dQ warps before
            // dq_free(u - kMeta). q_empty(u - kStages), waited for above, needs
            // the dQ^T MMA of u - 3, whose S^T waited for dq_free(u - 5), which
            // follows p_full(u - 5); kMeta = 8 > 5.
            meta[u % kMeta] = make_int4(qt, h, cb, 0);
            mbar_arrive_expect_tx(&q_full[st], 2 * kQBytes + 2 * kBQ * 4);
#pragma unroll
            for (int c = 0; c < 2; ++c) {
              tma_load_4d(sQ + st * kQBytes + c * (kBQ * 128), &tm_q, &q_full[st], c * 64, qt * kBQ, h, info.b);
              tma_load_4d(sDO + st * kQBytes + c * (kBQ * 128), &tm_do, &q_full[st], c * 64, qt * kBQ, h, info.b);
            }
            const size_t ro = (static_cast<size_t>(info.b) * p.Hq + h) * p.nqp + static_cast<size_t>(qt) * kBQ;
            bulk_load(sLse + st * kBQ, lse2 + ro, kBQ * 4, &q_full[st]);
            bulk_load(sDelta + st * kBQ, delta + ro, kBQ * 4, &q_full[st]);
          }
        }
      }
      if (*s_abort) {
        // Let the copies already issued land before shared memory is released.
        volatile int no_abort = 0;
        if (kv_loads > 0) mbar_wait(kv_full, (kv_loads - 1) & 1, &no_abort);
        for (uint32_t j = (u > kStages ? u - kStages : 0); j < u; ++j)
          mbar_wait(&q_full[j % kStages], (j / kStages) & 1, &no_abort);
      }
    }
  } else if (warp == 1) {
    // =================== MMA issuer ===================
    constexpr uint32_t idesc_s = idesc_bf16(kBK, kBQ, false, false);   // S^T, dP^T: A, B K-major
    constexpr uint32_t idesc_kv = idesc_bf16(kBK, kD, false, true);    // dV, dK: A in TMEM, B MN-major
    constexpr uint32_t idesc_dq = idesc_bf16(kD, kBQ, true, true);     // dQ^T: A = K^T, B = dS^T, both MN-major
    const uint32_t k_kmaj = sdesc_sw128_lo(smem_u32(sK), 16);
    const uint32_t v_kmaj = sdesc_sw128_lo(smem_u32(sV), 16);
    const uint32_t k_mn = sdesc_sw128_lo(smem_u32(sK), kBK * 128);       // 64-dim chunks 16 KB apart
    const uint32_t ds_mn0 = sdesc_sw128_lo(smem_u32(sDS), kBK * 128);   // one 64-query chunk per buffer
    uint32_t u = 0, kv_items = 0;
    bool ok = true;

    // S^T(u) = K Q(u)^T and dP^T(u) = V dout(u)^T into the TMEM columns of parity u & 1.
    auto issue_sdp = [&](uint32_t uu) -> bool {
      const uint32_t st = uu % kStages, b = uu & 1;
      if (!warp_all(mbar_wait(&q_full[st], (uu / kStages) & 1, s_abort))) return false;
      if (uu >= 2 && !warp_all(mbar_wait(&dq_free[b], ((uu - 2) >> 1) & 1, s_abort))) return false;
      tc_fence_after();
      const uint32_t q_kmaj = sdesc_sw128_lo(smem_u32(sQ + st * kQBytes), 16);
      const uint32_t do_kmaj = sdesc_sw128_lo(smem_u32(sDO + st * kQBytes), 16);
      const uint32_t d_s = tmem + b * 128;
#pragma unroll
      for (int kk = 0; kk < kD / 16; ++kk) {
        const uint32_t off = (kk & 3) * 32;
        umma_ss(d_s, k_kmaj + (((kk >> 2) * (kBK * 128) + off) >> 4), q_kmaj + (((kk >> 2) * (kBQ * 128) + off) >> 4),
                idesc_s, kk > 0 ? 1u : 0u);
      }
#pragma unroll
      for (int kk = 0; kk < kD / 16; ++kk) {
        const uint32_t off = (kk & 3) * 32;
        umma_ss(d_s + 64, v_kmaj + (((kk >> 2) * (kBK * 128) + off) >> 4),
                do_kmaj + (((kk >> 2) * (kBQ * 128) + off) >> 4), idesc_s, kk > 0 ? 1u : 0u);
      }
      umma_commit(&s_full[b]);
      return true;
    };

    for (int it = 0; ok; ++it) {
      const int rs = it % kRing;
      if (!(ok = warp_all(mbar_wait(&sched_full[rs], (it / kRing) & 1, s_abort)))) break;
      const BwdItem info = ring[rs];
      __syncwarp();
      if (lane == 0) mbar_arrive(&sched_empty[rs]);
      __syncwarp();
      if (info.w < 0) break;
      if (info.n == 0) continue;
      if (!(ok = warp_all(mbar_wait(kv_full, kv_items & 1, s_abort)))) break;
      tc_fence_after();
      const uint32_t n_it = static_cast<uint32_t>(p.G) * info.n;
      if (!(ok = issue_sdp(u))) break;
      for (uint32_t i = 0; i < n_it; ++i, ++u) {
        if (i + 1 < n_it && !(ok = issue_sdp(u + 1))) break;
        const uint32_t st = u % kStages, b = u & 1;
        if (!(ok = warp_all(mbar_wait(&p_full[b], (u >> 1) & 1, s_abort)))) break;
        tc_fence_after();
        const uint32_t buf = tmem + b * 128;
        const uint32_t q_mn = sdesc_sw128_lo(smem_u32(sQ + st * kQBytes), kBQ * 128);
        const uint32_t do_mn = sdesc_sw128_lo(smem_u32(sDO + st * kQBytes), kBQ * 128);
        // dV += P^T dout: K = the 64 queries, 16 per MMA (8 TMEM columns of
        // packed bf16 in A, 16 rows of 128 bytes in B).
#pragma unroll
        for (int kk = 0; kk < kBQ / 16; ++kk)
          umma_ts(tmem + 256, buf + kPCol + kk * 8, do_mn + kk * (16 * 128 / 16), idesc_kv, (i > 0 || kk > 0) ? 1u : 0u);
        // dK += dS^T Q
#pragma unroll
        for (int kk = 0; kk < kBQ / 16; ++kk)
          umma_ts(tmem + 384, buf + kDSCol + kk * 8, q_mn + kk * (16 * 128 / 16), idesc_kv, (i > 0 || kk > 0) ? 1u : 0u);
        // dQ^T = K^T dS^T over the 128 keys, into the S^T columns of this parity
        // (the dV MMAs above read P^T from them first; MMAs run in issue order).
        const uint32_t ds_mn = ds_mn0 + b * (kDSBytes >> 4);
#pragma unroll
        for (int kk = 0; kk < kBK / 16; ++kk)
          umma_ss(buf, k_mn + kk * (16 * 128 / 16), ds_mn + kk * (16 * 128 / 16), idesc_dq, kk > 0 ? 1u : 0u);
        umma_commit(&dq_full[b]);  // also frees dS^T buffer b
        umma_commit(&q_empty[st]);
        if (i + 1 == n_it) {
          umma_commit(kv_done);
          umma_commit(kv_empty);
        }
      }
      if (!ok) break;
      ++kv_items;
    }
    if (!ok) *s_abort = 1;
    umma_commit(drain);
    volatile int no_abort = 0;
    mbar_wait(drain, 0, &no_abort);
  } else if (wg == 1 || wg == 2) {
    // ============ key rows: P^T, dS^T for query columns 32 hq .. 32 hq + 31 ============
    // Two warpgroups share every key row (TMEM lane) and split the 64 query
    // columns; at the end of an item one writes dV and the other dK.
    const int hq = wg - 1;
    const int r = (warp & 3) * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const MaskArgs& mk = p.mask;
    uint32_t u = 0, items_done = 0;
    bool ok = true;
    for (int it = 0; ok; ++it) {
      const int rs = it % kRing;
      if (!(ok = warp_all(mbar_wait(&sched_full[rs], (it / kRing) & 1, s_abort)))) break;
      const BwdItem info = ring[rs];
      __syncwarp();
      if (lane == 0) mbar_arrive(&sched_empty[rs]);
      if (info.w < 0) break;
      const int j = info.kt * kBK + r;
      const bool key_ok = j < p.Nk;
      __nv_bfloat16* out_row = hq == 0
          ? p.dv + info.b * p.dvs0 + info.hkv * p.dvs1 + static_cast<int64_t>(j) * p.dvs2
          : p.dk + info.b * p.dks0 + info.hkv * p.dks1 + static_cast<int64_t>(j) * p.dks2;
      if (info.n == 0) {  // no query sees these keys
        if (key_ok)
#pragma unroll 1
          for (int c = 0; c < kD / 8; ++c) reinterpret_cast<uint4*>(out_row)[c] = make_uint4(0, 0, 0, 0);
        continue;
      }
      // The key's mask parameters (fixed for the item).
      int lts = 0, lte = 0, uts = 0, ute = 0;
      if (mk.kind == MFA_MASK_COLWISE && key_ok) {
        const size_t idx = static_cast<size_t>(info.b) * p.Nk + j;
        if (mk.lts) { lts = mk.lts[idx]; lte = mk.lte[idx]; }
        if (mk.uts) { uts = mk.uts[idx]; ute = mk.ute[idx]; }
      }
      const int half = r >> 6;  // which 64-key half of the tile (block selection bits)
      const uint32_t n_it = static_cast<uint32_t>(p.G) * info.n;
      for (uint32_t i = 0; i < n_it; ++i, ++u) {
        const uint32_t st = u % kStages, b = u & 1;
        if (!(ok = warp_all(mbar_wait(&q_full[st], (u / kStages) & 1, s_abort)))) break;  // meta, lse2, Delta
        const int4 mt = meta[u % kMeta];
        const int qt = mt.x;
        const uint32_t cb = static_cast<uint32_t>(mt.z);
        const int q0 = qt * kBQ + 32 * hq;  // first query of this warpgroup's columns
        uint32_t vis = ~0u;                 // bit c: query q0 + c visible
        if (!key_ok) {
          vis = 0u;
        } else if ((cb & 3u) == 2u) {
          if (mk.kind == MFA_MASK_COLWISE) {
            vis = ~static_cast<uint32_t>(bits64(lts - q0, lte - q0) | bits64(uts - q0, ute - q0));
          } else if (mk.kind == MFA_MASK_BAND) {
            vis = static_cast<uint32_t>(bits64(j - mk.nxt - q0, j + mk.pre + 1 - q0));
          } else {
            // selection bit of (64-query sub-block of the map tile, 64-key half)
            vis = ((cb >> (4 + 2 * (qt % p.qsub) + half)) & 1u) ? static_cast<uint32_t>(bits64(j - q0, 32)) : 0u;
          }
        }
        if (!(ok = warp_all(mbar_wait(&s_full[b], (u >> 1) & 1, s_abort)))) break;
        tc_fence_after();
        const uint32_t tb = tmem + lane_off + b * 128;
        uint32_t sv[32], dpv[32];
        tmem_ld_32x32b_x32(tb + 32 * hq, sv);
        tmem_ld_32x32b_x32(tb + 64 + 32 * hq, dpv);
        tmem_ld_wait();
        const float* l2 = sLse + st * kBQ + 32 * hq;
        const float* dl = sDelta + st * kBQ + 32 * hq;
        uint32_t pk[16], dsk[16];
        // P = 0 where masked. Fully visible 32-column blocks (FULL tiles, most
        // of the work) skip the per-element select.
        if (vis == ~0u) {
#pragma unroll
          for (int c2 = 0; c2 < 16; ++c2) {
            float pv[2], dsv[2];
#pragma unroll
            for (int e2 = 0; e2 < 2; ++e2) {
              const int c = 2 * c2 + e2;
              pv[e2] = ex2_approx(fmaf(__uint_as_float(sv[c]), p.scale_log2, -l2[c]));
              dsv[e2] = pv[e2] * (__uint_as_float(dpv[c]) - dl[c]);
            }
            pk[c2] = pack_bf16x2(pv[0], pv[1]);
            dsk[c2] = pack_bf16x2(dsv[0], dsv[1]);
          }
        } else {
#pragma unroll
          for (int c2 = 0; c2 < 16; ++c2) {
            float pv[2], dsv[2];
#pragma unroll
            for (int e2 = 0; e2 < 2; ++e2) {
              const int c = 2 * c2 + e2;
              const float x = fmaf(__uint_as_float(sv[c]), p.scale_log2, -l2[c]);
              const float pe = ((vis >> c) & 1u) ? ex2_approx(x) : 0.f;
              pv[e2] = pe;
              dsv[e2] = pe * (__uint_as_float(dpv[c]) - dl[c]);
            }
            pk[c2] = pack_bf16x2(pv[0], pv[1]);
            dsk[c2] = pack_bf16x2(dsv[0], dsv[1]);
          }
        }
        // Packed P^T sits at columns [16, 48) and dS^T at [80, 112) of the
        // parity's block: each warpgroup writes its 16 columns inside the 32 it
        // alone has just read, so neither overwrites scores the other still reads.
        tmem_st_32x32b_x16(tb + kPCol + 16 * hq, pk);
        tmem_st_32x32b_x16(tb + kDSCol + 16 * hq, dsk);
        // dS^T buffer b was last read by the dQ^T MMA of iteration u - 2, whose
        // completion is dq_full(u - 2).
        if (u >= 2 && !(ok = warp_all(mbar_wait(&dq_full[b], ((u - 2) >> 1) & 1, s_abort)))) break;
        // Row r, queries 32 hq .. 32 hq + 31 = 16-byte chunks 4 hq .. 4 hq + 3,
        // placed by the 128-byte swizzle (chunk c of row r at c ^ (r & 7)).
        uint8_t* ds_row = sDS + b * kDSBytes + r * 128;
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
          const int ch = 4 * hq + c4;
          *reinterpret_cast<uint4*>(ds_row + ((ch ^ (r & 7)) << 4)) =
              make_uint4(dsk[4 * c4], dsk[4 * c4 + 1], dsk[4 * c4 + 2], dsk[4 * c4 + 3]);
        }
        tmem_st_wait();
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&p_full[b]);
      }
      if (!ok) break;
      // ---- item epilogue: dV (hq = 0) or dK (hq = 1) row of this key ----
      if (!(ok = warp_all(mbar_wait(kv_done, items_done & 1, s_abort)))) break;
      ++items_done;
      tc_fence_after();
      const uint32_t col = hq == 0 ? 256u : 384u;
      const float sc = hq == 0 ? 1.f : p.scale;
#pragma unroll 1
      for (int c = 0; c < kD / 32; ++c) {
        uint32_t a[32];
        tmem_ld_32x32b_x32(tmem + lane_off + col + c * 32, a);
        tmem_ld_wait();
        if (key_ok) {
#pragma unroll
          for (int g4 = 0; g4 < 4; ++g4)
            reinterpret_cast<uint4*>(out_row)[c * 4 + g4] =
                make_uint4(pack_bf16x2(__uint_as_float(a[8 * g4]) * sc, __uint_as_float(a[8 * g4 + 1]) * sc),
                           pack_bf16x2(__uint_as_float(a[8 * g4 + 2]) * sc, __uint_as_float(a[8 * g4 + 3]) * sc),
                           pack_bf16x2(__uint_as_float(a[8 * g4 + 4]) * sc, __uint_as_float(a[8 * g4 + 5]) * sc),
                           pack_bf16x2(__uint_as_float(a[8 * g4 + 6]) * sc, __uint_as_float(a[8 * g4 + 7]) * sc));
        }
      }
      tc_fence_before();
    }
    if (!ok && lane == 0) atomicOr(p.err, MFA_DEVERR_TIMEOUT);
  } else if (wg == 3) {
    // =================== dQ: TMEM -> staging -> TMA reduce-add ===================
    // Staging is two halves of 32 query rows; the reduce of one half reads
    // shared memory while the other half is written. Reduce groups go out in
    // the order half 0, half 1, half 0, ...; after issuing group n, thread 0
    // waits until group n - 1 has been read and frees its half.
    const int t = (warp & 3) * 32 + lane;  // head dimension = TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    uint32_t u = 0, n_grp = 0;
    bool ok = true;
    for (int it = 0; ok; ++it) {
      const int rs = it % kRing;
      if (!(ok = warp_all(mbar_wait(&sched_full[rs], (it / kRing) & 1, s_abort)))) break;
      const BwdItem info = ring[rs];
      __syncwarp();
      if (lane == 0) mbar_arrive(&sched_empty[rs]);
      if (info.w < 0) break;
      // The iteration's query tile comes from the transposed list in global
      // memory (written by an earlier launch); it is loaded before the
      // dq_full wait, which hides the load latency.
      const int32_t* lst = p.tlist + static_cast<size_t>(info.e) * p.nq64;
      const uint32_t n_it = static_cast<uint32_t>(p.G) * info.n;
      for (uint32_t i = 0; i < n_it && ok; ++i, ++u) {
        const uint32_t b = u & 1;
        const int g = static_cast<int>(i / static_cast<uint32_t>(info.n));
        const int qt = lst[i - static_cast<uint32_t>(g) * info.n];
        const int h = info.hkv * p.G + g;
        if (!(ok = warp_all(mbar_wait(&dq_full[b], (u >> 1) & 1, s_abort)))) break;
        tc_fence_after();
        uint32_t a[64];
        tmem_ld_32x32b_x32(tmem + lane_off + b * 128, *reinterpret_cast<uint32_t(*)[32]>(a));
        tmem_ld_32x32b_x32(tmem + lane_off + b * 128 + 32, *reinterpret_cast<uint32_t(*)[32]>(a + 32));
        tmem_ld_wait();
        tc_fence_before();
        mbar_arrive(&dq_free[b]);
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          // Half hf's previous group is n_grp - 2; it was freed after group n_grp - 1 went out.
          if (n_grp >= 2 && !(ok = warp_all(mbar_wait(&stg_free[hf], ((n_grp - 2) >> 1) & 1, s_abort)))) break;
          float* dst = sStg + hf * (kStgRows * kD);
#pragma unroll
          for (int c = 0; c < kStgRows; ++c) dst[c * kD + t] = __uint_as_float(a[kStgRows * hf + c]);
          fence_proxy_async_smem();
          mbar_arrive(&stg_full[hf]);
          if (t == 0) {
            // All 128 threads arrive right above, so this wait ends unless a
            // warp has left on an abort; then it gives up after the bound.
            if (mbar_wait(&stg_full[hf], (n_grp >> 1) & 1, s_abort)) {
              tma_reduce_add_4d(&tm_dq, dst, 0, qt * kBQ + kStgRows * hf, h, info.b);
              bulk_commit();
              if (n_grp >= 1) {
                bulk_wait_read1();
                mbar_arrive(&stg_free[hf ^ 1]);
              }
            }
          }
          __syncwarp();  // reconverge before the next warp-collective instruction
          ++n_grp;
        }
      }
    }
    if (t == 0) bulk_wait0();
    if (!ok && lane == 0) atomicOr(p.err, MFA_DEVERR_TIMEOUT);
  }

  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    if (atomicAdd(&p.sched[1], 1u) == gridDim.x - 1) {
      atomicExch(&p.sched[0], 0u);
      atomicExch(&p.sched[1], 0u);
      __threadfence();
    }
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------------
// host side
// ------------------------------------------------------------------------
struct BwdLayout {
  size_t dq_acc, lse2, delta, tlist, tcount, torder, words, total;
};

bool bwd_layout(int64_t B, int64_t Hq, int64_t Nq, int64_t D, int64_t nqt, int64_t nkt, BwdLayout* L) {
  if (B <= 0 || Hq <= 0 || Nq < 0 || D <= 0 || nqt < 0 || nkt < 0) return false;
  const size_t nqp = static_cast<size_t>(nqt) * kBQ;
  size_t off = 0;
  L->dq_acc = off; off = align256(off + static_cast<size_t>(B * Hq * Nq * D) * 4);
  L->lse2 = off;   off = align256(off + static_cast<size_t>(B * Hq) * nqp * 4);
  L->delta = off;  off = align256(off + static_cast<size_t>(B * Hq) * nqp * 4);
  L->tlist = off;  off = align256(off + static_cast<size_t>(B * nkt * nqt) * 4);
  L->tcount = off; off = align256(off + static_cast<size_t>(B * nkt) * 4);
  L->torder = off; off = align256(off + static_cast<size_t>(B * nkt) * 4);
  L->words = off;  off = align256(off + 4 * 4);
  L->total = off;
  return true;
}

// bf16 [B, H, N, D] tensor, 64-column SW128 boxes of `rows` rows.
bool map_bf16(CUtensorMap* map, const mfa_tensor* t, int rows) {
  auto fn = tensor_map_encoder();
  if (!fn) return false;
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(t->D), static_cast<cuuint64_t>(t->N),
                        static_cast<cuuint64_t>(t->H), static_cast<cuuint64_t>(t->B)};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(t->stride[2]) * 2, static_cast<cuuint64_t>(t->stride[1]) * 2,
                           static_cast<cuuint64_t>(t->stride[0]) * 2};
  cuuint32_t box[4] = {64, static_cast<cuuint32_t>(rows), 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, t->data, dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The fp32 dQ accumulator [B, Hq, Nq, D] (contiguous), 32 rows x 128 columns per box, no swizzle.
bool map_dq(CUtensorMap* map, void* base, int64_t B, int64_t Hq, int64_t Nq) {
  auto fn = tensor_map_encoder();
  if (!fn) return false;
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(kD), static_cast<cuuint64_t>(Nq), static_cast<cuuint64_t>(Hq),
                        static_cast<cuuint64_t>(B)};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(kD) * 4, static_cast<cuuint64_t>(Nq * kD) * 4,
                           static_cast<cuuint64_t>(Hq * Nq * kD) * 4};
  cuuint32_t box[4] = {static_cast<cuuint32_t>(kD), static_cast<cuuint32_t>(kStgRows), 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

mfa_status check_bf16(const mfa_tensor* t) {
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

bool same_shape(const mfa_tensor* a, const mfa_tensor* b) {
  return a->B == b->B && a->H == b->H && a->N == b->N && a->D == b->D;
}

}  // namespace
}  // namespace mfa

extern "C" size_t mfa_bwd_workspace_bytes(int32_t B, int32_t Hq, int32_t Nq, int32_t Nk, int32_t D) {
  using namespace mfa;
  BwdLayout L;
  if (!bwd_layout(B, Hq, Nq, D, cdiv64(Nq, kBQ), cdiv64(Nk, kBK), &L)) return 0;
  return L.total;
}

extern "C" mfa_status mfa_bwd(const mfa_tensor* q, const mfa_tensor* k, const mfa_tensor* v,
                              const mfa_tensor* out, const mfa_tensor* dout, const float* lse,
                              const mfa_mask_desc* mask, const mfa_tensor* dq, const mfa_tensor* dk,
                              const mfa_tensor* dv, void* workspace, size_t workspace_bytes, void* stream) {
  using namespace mfa;
  mfa_status st;
  const mfa_tensor* all[8] = {q, k, v, out, dout, dq, dk, dv};
  for (const mfa_tensor* t : all)
    if ((st = check_bf16(t)) != MFA_OK) return st;
  if ((!lse && q->N > 0) || !workspace) return MFA_ERR_INVALID_ARG;  // an empty lse may have no storage
  if ((st = check_mask(mask)) != MFA_OK) return st;
  if (!mask->map) return MFA_ERR_INVALID_ARG;
  const mfa_tile_map* map = mask->map;
  if ((st = check_map_matches(mask, map)) != MFA_OK) return st;
  if (map->kind != mask->kind) return MFA_ERR_SHAPE_MISMATCH;
  if (!same_shape(out, q) || !same_shape(dout, q) || !same_shape(dq, q)) return MFA_ERR_SHAPE_MISMATCH;
  if (!same_shape(v, k) || !same_shape(dk, k) || !same_shape(dv, k)) return MFA_ERR_SHAPE_MISMATCH;
  if (k->B != q->B || k->D != q->D || q->H % k->H != 0) return MFA_ERR_SHAPE_MISMATCH;
  if (mask->B != q->B || mask->Nq != q->N || mask->Nk != k->N) return MFA_ERR_SHAPE_MISMATCH;
  if (q->D != kD || mask->Hm != 1 || map->block_k != kBK) return MFA_ERR_UNSUPPORTED;
  if (map->block_q != 64 && map->block_q != 128) return MFA_ERR_UNSUPPORTED;
  if (q->N > (int64_t(1) << 30) || k->N > (int64_t(1) << 30) || q->H > 65535) return MFA_ERR_UNSUPPORTED;
  if (reinterpret_cast<uintptr_t>(workspace) % 256 != 0) return MFA_ERR_INVALID_ARG;
  const int nq64 = static_cast<int>(cdiv64(q->N, kBQ));
  BwdLayout L;
  if (!bwd_layout(q->B, q->H, q->N, q->D, nq64, map->nkt, &L)) return MFA_ERR_INVALID_ARG;
  if (workspace_bytes < L.total) return MFA_ERR_INVALID_ARG;
  if (static_cast<size_t>(nq64 + 1) * sizeof(int) > 200 * 1024) return MFA_ERR_UNSUPPORTED;

  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* dq_acc = reinterpret_cast<float*>(ws + L.dq_acc);
  float* lse2 = reinterpret_cast<float*>(ws + L.lse2);
  float* delta = reinterpret_cast<float*>(ws + L.delta);
  int32_t* tlist = reinterpret_cast<int32_t*>(ws + L.tlist);
  int32_t* tcount = reinterpret_cast<int32_t*>(ws + L.tcount);
  int32_t* torder = reinterpret_cast<int32_t*>(ws + L.torder);
  uint32_t* words = reinterpret_cast<uint32_t*>(ws + L.words);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int nqp = nq64 * kBQ;

  // (1) prep
  const int64_t rows = q->B * q->H * static_cast<int64_t>(nqp);
  {
    const int64_t blocks = (rows + 15) / 16;
    if (blocks > 0x7fffffff) return MFA_ERR_UNSUPPORTED;
    k_bwd_prep<<<static_cast<unsigned>(blocks > 0 ? blocks : 1), 256, 0, s>>>(
        static_cast<const __nv_bfloat16*>(out->data), out->stride[0], out->stride[1], out->stride[2],
        static_cast<const __nv_bfloat16*>(dout->data), dout->stride[0], dout->stride[1], dout->stride[2], lse,
        static_cast<int>(q->H), static_cast<int>(q->N), nqp, rows, lse2, delta, dq_acc, words);
    if (cudaGetLastError() != cudaSuccess) return MFA_ERR_CUDA;
  }
  // (2) transposed lists and key-tile order
  if (map->nkt > 0) {
    const size_t hist = static_cast<size_t>(nq64 + 1) * sizeof(int);
    if (hist > 48 * 1024 &&
        cudaFuncSetAttribute(k_bwd_tlist, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(hist)) !=
            cudaSuccess)
      return MFA_ERR_CUDA;
    k_bwd_tlist<<<dim3((map->nkt + 3) / 4, static_cast<unsigned>(q->B)), 128, hist, s>>>(
        map->tile_class, map->nqt, map->block_q / kBQ, nq64, map->nkt, tlist, tcount, torder, words);
    if (cudaGetLastError() != cudaSuccess) return MFA_ERR_CUDA;
  }
  // (3) main kernel
  const int64_t n_items64 = q->B * k->H * static_cast<int64_t>(map->nkt);
  if (n_items64 > 0x7fffffff) return MFA_ERR_UNSUPPORTED;
  if (n_items64 > 0) {
    CUtensorMap mq, mk, mv, mdo, mdq;
    if (!map_bf16(&mk, k, kBK) || !map_bf16(&mv, v, kBK)) return MFA_ERR_CUDA;
    if (q->N > 0) {
      if (!map_bf16(&mq, q, kBQ) || !map_bf16(&mdo, dout, kBQ) || !map_dq(&mdq, dq_acc, q->B, q->H, q->N))
        return MFA_ERR_CUDA;
    } else {  // never read: every list is empty and the kernel only writes dk = dv = 0
      memset(&mq, 0, sizeof(mq));
      memset(&mdo, 0, sizeof(mdo));
      memset(&mdq, 0, sizeof(mdq));
    }
    BwdParams p;
    p.B = static_cast<int32_t>(q->B); p.Hq = static_cast<int32_t>(q->H); p.Hkv = static_cast<int32_t>(k->H);
    p.G = p.Hq / p.Hkv; p.Nq = static_cast<int32_t>(q->N); p.Nk = static_cast<int32_t>(k->N);
    p.nqt = map->nqt; p.qsub = map->block_q / kBQ; p.nq64 = nq64; p.nkt = map->nkt; p.nqp = nqp;
    p.n_items = static_cast<int32_t>(n_items64);
    p.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(q->D)));
    p.scale = static_cast<float>(1.0 / std::sqrt(static_cast<double>(q->D)));
    p.mask = mask_args(mask);
    p.cls = map->tile_class; p.tlist = tlist; p.tcount = tcount; p.torder = torder;
    // Work order. With many items per CTA and a contiguous mask (documents,
    // bands), ascending key tiles keep the CTAs working at any moment on
    // neighbouring key tiles, which share their query tiles: Q / dout tiles
    // and dQ accumulator rows stay in L2 (doc32k: 11 % faster than longest
    // first, which re-read them from DRAM). With few items per CTA the end of
    // the launch dominates and longest first balances it (doc8k: 10 % faster);
    // block-selection lists are scattered, so there only the balance counts.
    const int sms_ = device_sm_count();
    p.order_lpt = (mask->kind == MFA_MASK_BLOCKSEL || n_items64 < 8 * static_cast<int64_t>(sms_ > 0 ? sms_ : 148)) ? 1 : 0;
    p.dk = static_cast<__nv_bfloat16*>(dk->data); p.dks0 = dk->stride[0]; p.dks1 = dk->stride[1]; p.dks2 = dk->stride[2];
    p.dv = static_cast<__nv_bfloat16*>(dv->data); p.dvs0 = dv->stride[0]; p.dvs1 = dv->stride[1]; p.dvs2 = dv->stride[2];
    p.err = map->err;
    p.sched = words;
    static std::atomic<uint64_t> attr_devs{0};
    if (!ensure_smem_attr(reinterpret_cast<const void*>(mfa_bwd_kernel), kSmemBytes, attr_devs)) return MFA_ERR_CUDA;
    const int sms = device_sm_count();
    if (sms <= 0) return MFA_ERR_CUDA;
    const int grid = p.n_items < sms ? p.n_items : sms;
    mfa_bwd_kernel<<<grid, kThreads, kSmemBytes, s>>>(mq, mk, mv, mdo, mdq, lse2, delta, p);
    if (cudaGetLastError() != cudaSuccess) return MFA_ERR_CUDA;
  }
  // (4) dq
  const int64_t n8 = q->B * q->H * q->N * (kD / 8);
  if (n8 > 0) {
    const int64_t blocks = (n8 + 255) / 256;
    k_bwd_dq_convert<<<static_cast<unsigned>(blocks < 4 * 148 ? blocks : 4 * 148), 256, 0, s>>>(
        dq_acc, static_cast<int>(q->H), static_cast<int>(q->N), n8, static_cast<float>(1.0 / std::sqrt(double(kD))),
        static_cast<__nv_bfloat16*>(dq->data), dq->stride[0], dq->stride[1], dq->stride[2]);
    if (cudaGetLastError() != cudaSuccess) return MFA_ERR_CUDA;
  }
  return MFA_OK;
}
