// mfa_fwd: mask-aware flash-attention forward pass for sm_100a.
//
// out = softmax(Q K^T / sqrt(d) + mask) V and lse = log-sum-exp per row, where
// the mask is applied through the tile map: only the key tiles listed for a
// query tile are visited (Binary Block Masking, abstract: skip fully masked
// blocks), FULL tiles take no per-element mask work, and PARTIAL tiles apply
// the exact element mask of the compact description (FlashMask's column-wise
// intervals, the Ascend band, or 64-block selection lists).
//
// One CTA computes one 128-row query tile (128 queries of one head, or 64
// queries of two heads of one key/value group when the map is built at
// block_q = 64). Warp roles:
//   warp 0     TMA producer: Q tile once, then K and V tiles of the listed
//              k-tiles into two-stage shared-memory rings.
//   warp 1     TMEM owner and MMA issuer: S = Q K^T into one of two TMEM S
//              buffers, then O += P V with P read from TMEM.
//   warps 4-7  softmax: one query row per thread (TMEM lane = row). Load S,
//              mask (PARTIAL tiles only), online max / exp2 / sum, rescale O
//              in TMEM when the running max grows, write P as bf16 over S,
//              and finally normalise O and store out and lse.
// Every mbarrier wait is bounded; a wait that gives up raises an abort flag
// for the whole CTA and sets MFA_DEVERR_TIMEOUT in the map's error word.
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

constexpr int kRows = 128;       // MMA M: query rows per tile
constexpr int kStagesK = 2;
constexpr int kStagesV = 2;
constexpr int kThreads = 256;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: rescale only when the max grows by > 2^8

struct FwdParams {
  int32_t B, Hq, Hkv, G, Hm, Nq, Nk, nqt, nkt, hpe;
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
};

template <int D, int BK>
struct Smem {
  static constexpr int kChunks = D / 64;                 // 128-byte K chunks per row
  static constexpr int kQBytes = kRows * D * 2;
  static constexpr int kKVBytes = BK * D * 2;
  static constexpr int kQ = 0;
  static constexpr int kK = kQ + kQBytes;
  static constexpr int kV = kK + kStagesK * kKVBytes;
  static constexpr int kBar = kV + kStagesV * kKVBytes;
  // barriers: q_full, k_full[2], k_empty[2], v_full[2], v_empty[2], s_full[2], p_full[2], o_done,
  // drain, bnd_full[2]
  static constexpr int kNumBars = 1 + 2 * kStagesK + 2 * kStagesV + 2 + 2 + 1 + 1 + 2;
  static constexpr int kBounds = kBar + ((kNumBars * 8 + 15) / 16) * 16;  // int4 [2][BK]
  static constexpr int kMisc = kBounds + 2 * BK * 16;
  static constexpr int kBytes = kMisc + 16;
  static constexpr int kAlloc = kBytes + 1024;           // slack for 1024-byte alignment
  static constexpr int kTmemCols = (2 * BK + D) <= 256 ? 256 : 512;
};

__device__ __forceinline__ bool warp_all(bool ok) { return __all_sync(0xffffffffu, ok); }

template <int D, int BK, int GP>
__global__ void __launch_bounds__(kThreads, 1)
    mfa_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
  using L = Smem<D, BK>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  uint8_t* sQ = smem + L::kQ;
  uint8_t* sK = smem + L::kK;
  uint8_t* sV = smem + L::kV;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* k_empty = k_full + kStagesK;
  uint64_t* v_full = k_empty + kStagesK;
  uint64_t* v_empty = v_full + kStagesV;
  uint64_t* s_full = v_empty + kStagesV;
  uint64_t* p_full = s_full + 2;
  uint64_t* o_done = p_full + 2;
  uint64_t* drain = o_done + 1;
  uint64_t* bnd_full = drain + 1;
  int4* s_bounds = reinterpret_cast<int4*>(smem + L::kBounds);
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* s_abort = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // ---- work item -------------------------------------------------------
  const int w = blockIdx.x;
  const int ent = p.order[w / p.hpe];
  const int ht = w % p.hpe;
  const int b = ent / (p.Hm * p.nqt);
  const int hm = (ent / p.nqt) % p.Hm;
  const int qt = ent % p.nqt;
  const int h0 = (p.Hm == 1) ? ht * GP : hm;
  const int hkv = h0 / p.G;
  const int BQ = kRows / GP;
  const int q0 = qt * BQ;
  const int n = p.count[ent];
  const int32_t* lst = p.list + static_cast<size_t>(ent) * p.nkt;
  const uint8_t* ccls = p.cls + static_cast<size_t>(ent) * p.nkt;

  // ---- set-up ----------------------------------------------------------
  if (warp == 0 && lane == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < kStagesK; ++s) { mbar_init(&k_full[s], 1); mbar_init(&k_empty[s], 1); }
    for (int s = 0; s < kStagesV; ++s) { mbar_init(&v_full[s], 1); mbar_init(&v_empty[s], 1); }
    for (int s = 0; s < 2; ++s) { mbar_init(&s_full[s], 1); mbar_init(&p_full[s], kRows); }
    mbar_init(o_done, 1);
    mbar_init(drain, 1);
    mbar_init(&bnd_full[0], kRows);
    mbar_init(&bnd_full[1], kRows);
    *s_abort = 0;
    fence_mbarrier_init();
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  if (warp == 1) {
    tmem_alloc(s_tmem, L::kTmemCols);
    tmem_relinquish();
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;
  const uint32_t tmem_o = tmem + 2 * BK;

  if (warp == 0) {
    // =================== TMA producer ===================
    if (lane == 0 && n > 0) {
      mbar_arrive_expect_tx(q_full, L::kQBytes);
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int head = (GP == 2) ? h0 + hh : h0;
        const int row = (GP == 2) ? q0 : q0 + 64 * hh;
#pragma unroll
        for (int c = 0; c < L::kChunks; ++c)
          tma_load_4d(sQ + c * (kRows * 128) + hh * (64 * 128), &tm_q, q_full, c * 64, row, head, b);
      }
      int k_issued = 0, v_issued = 0;
      for (int i = 0; i < n; ++i) {
        const int kt = lst[i];
        if (kt < 0 || kt >= p.nkt) {
          atomicOr(p.err, MFA_DEVERR_MAP);
          *s_abort = 1;
          break;
        }
        const int ks = i % kStagesK;
        if (i >= kStagesK && !mbar_wait(&k_empty[ks], ((i / kStagesK) - 1) & 1, s_abort)) break;
        mbar_arrive_expect_tx(&k_full[ks], L::kKVBytes);
#pragma unroll
        for (int c = 0; c < L::kChunks; ++c)
          tma_load_4d(sK + ks * L::kKVBytes + c * (BK * 128), &tm_k, &k_full[ks], c * 64, kt * BK, hkv, b);
        k_issued = i + 1;
        const int vs = i % kStagesV;
        if (i >= kStagesV && !mbar_wait(&v_empty[vs], ((i / kStagesV) - 1) & 1, s_abort)) break;
        mbar_arrive_expect_tx(&v_full[vs], L::kKVBytes);
#pragma unroll
        for (int c = 0; c < L::kChunks; ++c)
          tma_load_4d(sV + vs * L::kKVBytes + c * (BK * 128), &tm_v, &v_full[vs], c * 64, kt * BK, hkv, b);
        v_issued = i + 1;
      }
      if (*s_abort) {
        // Let the copies already issued land before the CTA's shared memory goes away.
        volatile int no_abort = 0;
        mbar_wait(q_full, 0, &no_abort);
        for (int j = (k_issued > kStagesK ? k_issued - kStagesK : 0); j < k_issued; ++j)
          mbar_wait(&k_full[j % kStagesK], (j / kStagesK) & 1, &no_abort);
        for (int j = (v_issued > kStagesV ? v_issued - kStagesV : 0); j < v_issued; ++j)
          mbar_wait(&v_full[j % kStagesV], (j / kStagesV) & 1, &no_abort);
      }
    }
  } else if (warp == 1) {
    // =================== MMA issuer ===================
    if (lane == 0 && n > 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(kRows, BK, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(kRows, D, true);
      const uint32_t q_addr = smem_u32(sQ), k_addr = smem_u32(sK), v_addr = smem_u32(sV);
      bool ok = mbar_wait(q_full, 0, s_abort);
      tc_fence_after();
      for (int i = 0; ok && i <= n; ++i) {
        if (i < n) {
          const int ks = i % kStagesK;
          if (!(ok = mbar_wait(&k_full[ks], (i / kStagesK) & 1, s_abort))) break;
          tc_fence_after();
          const uint32_t d_s = tmem + (i & 1) * BK;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk & 3) * 32;  // 16 bf16 along K inside the 128-byte row
            const uint64_t a = sdesc_sw128(q_addr + (kk >> 2) * (kRows * 128) + off, 16, 1024);
            const uint64_t bd = sdesc_sw128(k_addr + ks * L::kKVBytes + (kk >> 2) * (BK * 128) + off, 16, 1024);
            umma_ss(d_s, a, bd, idesc_qk, kk > 0 ? 1u : 0u);
          }
          umma_commit(&s_full[i & 1]);
          umma_commit(&k_empty[ks]);
        }
        if (i >= 1) {
          const int j = i - 1;
          if (!(ok = mbar_wait(&p_full[j & 1], (j >> 1) & 1, s_abort))) break;
          const int vs = j % kStagesV;
          if (!(ok = mbar_wait(&v_full[vs], (j / kStagesV) & 1, s_abort))) break;
          tc_fence_after();
          const uint32_t a_p = tmem + (j & 1) * BK;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t bd = sdesc_sw128(v_addr + vs * L::kKVBytes + kk * (16 * 128), BK * 128, 1024);
            umma_ts(tmem_o, a_p + kk * 8, bd, idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(o_done);
          umma_commit(&v_empty[vs]);
        }
      }
      // Wait for every MMA issued here before TMEM can be released.
      umma_commit(drain);
      volatile int no_abort = 0;
      mbar_wait(drain, 0, &no_abort);
    }
  } else if (warp >= 4) {
    // =================== softmax / correction / epilogue ===================
    const int sw = warp - 4;
    const int r = sw * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(sw * 32) << 16;
    const int qi = (GP == 2) ? q0 + (r & 63) : q0 + r;
    const int head = (GP == 2) ? h0 + (r >> 6) : h0;
    const MaskArgs& mk = p.mask;
    const size_t bh_mask = static_cast<size_t>(b) * p.Hm + hm;
    const bool k_ragged = (p.Nk % BK) != 0;

    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    int n_bnd = 0;  // colwise partial tiles staged so far
    for (int i = 0; i < n; ++i) {
      const int kt = lst[i];
      if (kt < 0 || kt >= p.nkt) {
        if (lane == 0) atomicOr(p.err, MFA_DEVERR_MAP);
        *s_abort = 1;
        ok = false;
        break;
      }
      const uint32_t cb = ccls[kt];
      const bool partial = ((cb & 3u) == 2u) || (k_ragged && kt == p.nkt - 1);
      const int4* bnd = nullptr;
      if (partial && mk.kind == MFA_MASK_COLWISE) {
        // Stage the tile's column bounds in shared memory (double-buffered; a
        // thread reaching partial tile t+2 has passed tile t+1's barrier, so
        // every reader of tile t is done with the slot it overwrites).
        const int slot = n_bnd & 1;
        int4* dst = s_bounds + slot * BK;
        if (r < BK) {
          const int j = kt * BK + r;
          int4 v = make_int4(0, 0x7fffffff, 0, 0);  // columns past Nk: masked for every row
          if (j < p.Nk) {
            const size_t idx = bh_mask * p.Nk + j;
            v.x = mk.lts ? mk.lts[idx] : 0;
            v.y = mk.lte ? mk.lte[idx] : 0;
            v.z = mk.uts ? mk.uts[idx] : 0;
            v.w = mk.ute ? mk.ute[idx] : 0;
          }
          dst[r] = v;
        }
        mbar_arrive(&bnd_full[slot]);
        if (!(ok = warp_all(mbar_wait(&bnd_full[slot], (n_bnd >> 1) & 1, s_abort)))) break;
        bnd = dst;
        ++n_bnd;
      }
      if (!(ok = warp_all(mbar_wait(&s_full[i & 1], (i >> 1) & 1, s_abort)))) break;
      tc_fence_after();

      float s[BK];
      {
        uint32_t* su = reinterpret_cast<uint32_t*>(s);
#pragma unroll
        for (int c = 0; c < BK / 32; ++c)
          tmem_ld_32x32b_x32(tmem + lane_off + (i & 1) * BK + c * 32,
                             *reinterpret_cast<uint32_t(*)[32]>(su + c * 32));
        tmem_ld_wait();
      }
      if (partial) {
        const int jb = kt * BK;
        if (mk.kind == MFA_MASK_COLWISE) {
#pragma unroll
          for (int jj = 0; jj < BK; ++jj) {
            const int4 v = bnd[jj];
            const bool masked = (v.x <= qi && qi < v.y) || (v.z <= qi && qi < v.w);
            if (masked) s[jj] = -INFINITY;
          }
        } else if (mk.kind == MFA_MASK_BAND) {
#pragma unroll
          for (int jj = 0; jj < BK; ++jj) {
            const int dj = jb + jj - qi;
            const bool vis = (jb + jj < p.Nk) && dj >= -mk.pre && dj <= mk.nxt;
            if (!vis) s[jj] = -INFINITY;
          }
        } else {
          const int qsl = (GP == 2) ? 0 : (r >> 6);
#pragma unroll
          for (int jj = 0; jj < BK; ++jj) {
            const int ksl = jj >> 6;
            const bool vis = (jb + jj < p.Nk) && (jb + jj <= qi) && ((cb >> (4 + 2 * qsl + ksl)) & 1u);
            if (!vis) s[jj] = -INFINITY;
          }
        }
      }
      float mx = -INFINITY;
#pragma unroll
      for (int jj = 0; jj < BK; ++jj) mx = fmaxf(mx, s[jj]);
      const float mx_s = mx * p.scale_log2;
      const bool need = mx_s > m_run + kRescaleThreshold;
      const float m_new = need ? mx_s : m_run;
      const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
      float sum = 0.f;
#pragma unroll
      for (int jj = 0; jj < BK; ++jj) {
        const float e = ex2_approx(fmaf(s[jj], p.scale_log2, -m_use));
        s[jj] = e;
        sum += e;
      }
      if (i > 0) {
        if (!(ok = warp_all(mbar_wait(o_done, (i - 1) & 1, s_abort)))) break;
        tc_fence_after();
      }
      const float alpha = need ? ex2_approx(m_run - m_use) : 1.f;
      l_run = l_run * alpha + sum;
      m_run = m_new;
      if (i > 0 && __any_sync(0xffffffffu, need)) {
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          tmem_ld_32x32b_x32(tmem_o + lane_off + c * 32, o);
          tmem_ld_wait();
#pragma unroll
          for (int t = 0; t < 32; ++t) o[t] = __float_as_uint(__uint_as_float(o[t]) * alpha);
          tmem_st_32x32b_x32(tmem_o + lane_off + c * 32, o);
        }
      }
#pragma unroll
      for (int c = 0; c < BK / 64; ++c) {
        uint32_t pk[32];
#pragma unroll
        for (int t = 0; t < 32; ++t) pk[t] = pack_bf16x2(s[c * 64 + 2 * t], s[c * 64 + 2 * t + 1]);
        tmem_st_32x32b_x32(tmem + lane_off + (i & 1) * BK + c * 32, pk);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&p_full[i & 1]);
    }

    // ---- epilogue ----
    if (ok && n > 0) {
      ok = warp_all(mbar_wait(o_done, (n - 1) & 1, s_abort));
      tc_fence_after();
    }
    const bool has = ok && l_run > 0.f;
    const float inv = has ? 1.f / l_run : 0.f;
    const bool store = qi < p.Nq;
    __nv_bfloat16* orow = p.out + static_cast<int64_t>(b) * p.os0 + static_cast<int64_t>(head) * p.os1 +
                          static_cast<int64_t>(qi) * p.os2;
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
      uint32_t o[32] = {};
      if (ok && n > 0) {
        tmem_ld_32x32b_x32(tmem_o + lane_off + c * 32, o);
        tmem_ld_wait();
      }
      uint32_t pk[16];
#pragma unroll
      for (int t = 0; t < 16; ++t)
        pk[t] = has ? pack_bf16x2(__uint_as_float(o[2 * t]) * inv, __uint_as_float(o[2 * t + 1]) * inv) : 0u;
      if (store) {
        uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
        for (int t = 0; t < 4; ++t) dst[t] = make_uint4(pk[4 * t], pk[4 * t + 1], pk[4 * t + 2], pk[4 * t + 3]);
      }
    }
    if (store) {
      const float lse = has ? (m_run + __log2f(l_run)) * 0.69314718055994530942f : -INFINITY;
      p.lse[(static_cast<size_t>(b) * p.Hq + head) * p.Nq + qi] = lse;
    }
    if (!ok && lane == 0) atomicOr(p.err, MFA_DEVERR_TIMEOUT);
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

// ------------------------------------------------------------------------
// host side
// ------------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

bool make_map(CUtensorMap* map, const mfa_tensor* t, int box_rows) {
  auto fn = encode_fn();
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

template <int D, int BK, int GP>
mfa_status launch(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const FwdParams& p,
                  int n_items, cudaStream_t s) {
  using L = Smem<D, BK>;
  static bool attr_set = false;
  if (!attr_set) {
    if (cudaFuncSetAttribute(mfa_fwd_kernel<D, BK, GP>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc) !=
        cudaSuccess)
      return MFA_ERR_CUDA;
    attr_set = true;
  }
  mfa_fwd_kernel<D, BK, GP><<<n_items, kThreads, L::kAlloc, s>>>(mq, mk, mv, p);
  return cudaGetLastError() == cudaSuccess ? MFA_OK : MFA_ERR_CUDA;
}

}  // namespace
}  // namespace mfa

extern "C" mfa_status mfa_fwd(const mfa_tensor* q, const mfa_tensor* k, const mfa_tensor* v,
                              const mfa_mask_desc* mask, const mfa_tensor* out, float* lse, void* stream) {
  using namespace mfa;
  mfa_status st;
  if ((st = check_tensor(q)) != MFA_OK || (st = check_tensor(k)) != MFA_OK || (st = check_tensor(v)) != MFA_OK ||
      (st = check_tensor(out)) != MFA_OK)
    return st;
  if (!lse) return MFA_ERR_INVALID_ARG;
  if ((st = check_mask(mask)) != MFA_OK) return st;
  if (!mask->map) return MFA_ERR_INVALID_ARG;
  const mfa_tile_map* map = mask->map;
  if ((st = check_map_matches(mask, map)) != MFA_OK) return st;
  if (map->kind != mask->kind) return MFA_ERR_SHAPE_MISMATCH;
  if (q->dtype != k->dtype || q->dtype != v->dtype || out->dtype != q->dtype) return MFA_ERR_INVALID_ARG;
  if (q->dtype != MFA_BF16) return MFA_ERR_UNSUPPORTED;
  if (k->B != q->B || v->B != q->B || out->B != q->B) return MFA_ERR_SHAPE_MISMATCH;
  if (k->H != v->H || k->N != v->N || k->D != q->D || v->D != q->D) return MFA_ERR_SHAPE_MISMATCH;
  if (out->H != q->H || out->N != q->N || out->D != q->D) return MFA_ERR_SHAPE_MISMATCH;
  if (q->H % k->H != 0) return MFA_ERR_SHAPE_MISMATCH;
  if (mask->B != q->B || mask->Nq != q->N || mask->Nk != k->N) return MFA_ERR_SHAPE_MISMATCH;
  if (mask->Hm != 1 && mask->Hm != q->H) return MFA_ERR_SHAPE_MISMATCH;
  if (q->D != 64 && q->D != 128) return MFA_ERR_UNSUPPORTED;
  if (q->N > (int64_t(1) << 30) || k->N > (int64_t(1) << 30) || q->H > 65535) return MFA_ERR_UNSUPPORTED;
  const int G = static_cast<int>(q->H / k->H);
  const int GP = map->block_q == 64 ? 2 : 1;
  if (GP == 2 && (mask->Hm != 1 || G % 2 != 0)) return MFA_ERR_UNSUPPORTED;
  if (q->N == 0) return MFA_OK;

  FwdParams p;
  p.B = static_cast<int32_t>(q->B); p.Hq = static_cast<int32_t>(q->H); p.Hkv = static_cast<int32_t>(k->H);
  p.G = G; p.Hm = mask->Hm; p.Nq = static_cast<int32_t>(q->N); p.Nk = static_cast<int32_t>(k->N);
  p.nqt = map->nqt; p.nkt = map->nkt;
  p.hpe = mask->Hm == 1 ? p.Hq / GP : 1;
  p.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(q->D)));
  p.mask = mask_args(mask);
  p.cls = map->tile_class; p.list = map->tile_list; p.count = map->tile_count; p.order = map->order;
  p.out = static_cast<__nv_bfloat16*>(out->data);
  p.os0 = out->stride[0]; p.os1 = out->stride[1]; p.os2 = out->stride[2];
  p.lse = lse;
  p.err = map->err;
  const int64_t n_items64 = static_cast<int64_t>(p.B) * p.Hm * p.nqt * p.hpe;
  if (n_items64 <= 0) return MFA_OK;
  if (n_items64 > 0x7fffffff) return MFA_ERR_UNSUPPORTED;
  const int n_items = static_cast<int>(n_items64);

  // With Nk == 0 every list is empty and the K/V maps are never read.
  CUtensorMap mq, mk, mv;
  memset(&mk, 0, sizeof(mk));
  memset(&mv, 0, sizeof(mv));
  if (!make_map(&mq, q, 64)) return MFA_ERR_CUDA;
  if (k->N > 0 && (!make_map(&mk, k, map->block_k) || !make_map(&mv, v, map->block_k))) return MFA_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int D = static_cast<int>(q->D), BK = map->block_k;
  if (D == 128 && BK == 128) return GP == 2 ? launch<128, 128, 2>(mq, mk, mv, p, n_items, s) : launch<128, 128, 1>(mq, mk, mv, p, n_items, s);
  if (D == 128 && BK == 64) return GP == 2 ? launch<128, 64, 2>(mq, mk, mv, p, n_items, s) : launch<128, 64, 1>(mq, mk, mv, p, n_items, s);
  if (D == 64 && BK == 128) return GP == 2 ? launch<64, 128, 2>(mq, mk, mv, p, n_items, s) : launch<64, 128, 1>(mq, mk, mv, p, n_items, s);
  return GP == 2 ? launch<64, 64, 2>(mq, mk, mv, p, n_items, s) : launch<64, 64, 1>(mq, mk, mv, p, n_items, s);
}
