// mfa_fwd for fp32 inputs: the same masked attention through the same tile
// map, computed in fp32 on the CUDA cores.
//
// The tensor cores read fp32 operands as tf32 (10-bit mantissa); on fp32 inputs
// that moves the log-sum-exp by about 2e-3, outside the 1e-3 the outputs are
// held to, so fp32 problems are computed with fp32 fused multiply-adds instead.
// They are the small correctness workloads (d = 64, a few hundred rows).
//
// One thread owns one query row; a block holds 64 consecutive rows of one head,
// which always fall in one query tile of the map (block_q is 64 or 128). The
// block walks the tile's listed key tiles 32 keys at a time: K and V rows are
// staged in shared memory, scores are masked only on PARTIAL tiles (and past
// Nk), and the row keeps a running max, sum and output (online softmax).
#include <cmath>
#include <cuda_runtime.h>

#include "mfa.h"
#include "mfa_internal.h"

namespace mfa {
namespace {

constexpr int kRowsPerBlock = 64;
constexpr int kChunk = 32;

struct F32Params {
  int32_t B, Hq, G, Hm, Nq, Nk, nqt, nkt, BQ, BK;
  float scale;  // 1 / sqrt(d)
  MaskArgs mask;
  const uint8_t* cls;
  const int32_t* list;
  const int32_t* count;
  const float *q, *k, *v;
  int64_t qs0, qs1, qs2, ks0, ks1, ks2, vs0, vs1, vs2, os0, os1, os2;
  float* out;
  float* lse;
  uint32_t* err;
};

template <int D>
__global__ void __launch_bounds__(kRowsPerBlock) mfa_fwd_f32_kernel(const F32Params p) {
  extern __shared__ float smem[];
  float* sq = smem;                                 // [64][D + 1], padded against bank conflicts
  float* sk = sq + kRowsPerBlock * (D + 1);         // [32][D]
  float* sv = sk + kChunk * D;                      // [32][D]
  int4* sb = reinterpret_cast<int4*>(sv + kChunk * D);  // [32] column bounds

  const int t = threadIdx.x;
  const int head = blockIdx.y, b = blockIdx.z;
  const int row0 = blockIdx.x * kRowsPerBlock;
  const int qi = row0 + t;
  const int hkv = head / p.G;
  const int hm = p.Hm == 1 ? 0 : head;
  const int qt = row0 / p.BQ;
  const size_t e = (static_cast<size_t>(b) * p.Hm + hm) * p.nqt + qt;
  const int n = p.count[e];
  const int32_t* lst = p.list + e * p.nkt;
  const uint8_t* cls = p.cls + e * p.nkt;
  const size_t bh_mask = static_cast<size_t>(b) * p.Hm + hm;

  for (int i = t; i < kRowsPerBlock * D; i += kRowsPerBlock) {
    const int r = i / D, c = i % D;
    const int qr = row0 + r;
    sq[r * (D + 1) + c] = qr < p.Nq ? p.q[b * p.qs0 + head * p.qs1 + static_cast<int64_t>(qr) * p.qs2 + c] : 0.f;
  }

  float o[D];
#pragma unroll
  for (int c = 0; c < D; ++c) o[c] = 0.f;
  float m = -INFINITY, l = 0.f;

  for (int it = 0; it < n; ++it) {
    const int kt = lst[it];
    if (kt < 0 || kt >= p.nkt) {
      if (t == 0) atomicOr(p.err, MFA_DEVERR_MAP);
      break;
    }
    const uint32_t cb = cls[kt];
    const bool partial = (cb & 3u) == 2u;
    for (int c0 = 0; c0 < p.BK; c0 += kChunk) {
      const int j0 = kt * p.BK + c0;
      __syncthreads();  // previous chunk fully consumed
      for (int i = t; i < kChunk * D; i += kRowsPerBlock) {
        const int r = i / D, c = i % D;
        const int j = j0 + r;
        const bool ok = j < p.Nk && c0 + r < p.BK;
        sk[i] = ok ? p.k[b * p.ks0 + hkv * p.ks1 + static_cast<int64_t>(j) * p.ks2 + c] : 0.f;
        sv[i] = ok ? p.v[b * p.vs0 + hkv * p.vs1 + static_cast<int64_t>(j) * p.vs2 + c] : 0.f;
      }
      if (partial && p.mask.kind == MFA_MASK_COLWISE && t < kChunk) {
        const int j = j0 + t;
        int4 bv = make_int4(0, 0, 0, 0);
        if (j < p.Nk) {
          const size_t idx = bh_mask * p.Nk + j;
          bv.x = p.mask.lts ? p.mask.lts[idx] : 0;
          bv.y = p.mask.lte ? p.mask.lte[idx] : 0;
          bv.z = p.mask.uts ? p.mask.uts[idx] : 0;
          bv.w = p.mask.ute ? p.mask.ute[idx] : 0;
        }
        sb[t] = bv;
      }
      __syncthreads();

      float s[kChunk];
      float cmax = -INFINITY;
#pragma unroll 4
      for (int jj = 0; jj < kChunk; ++jj) {
        const int j = j0 + jj;
        bool vis = j < p.Nk && c0 + jj < p.BK;
        if (vis && partial) {
          if (p.mask.kind == MFA_MASK_COLWISE) {
            const int4 bv = sb[jj];
            vis = !((bv.x <= qi && qi < bv.y) || (bv.z <= qi && qi < bv.w));
          } else if (p.mask.kind == MFA_MASK_BAND) {
            const int dj = j - qi;
            vis = dj >= -p.mask.pre && dj <= p.mask.nxt;
          } else {
            const int qsl = (qi / 64) - (qt * p.BQ) / 64;
            const int ksl = (j / 64) - (kt * p.BK) / 64;
            vis = j <= qi && ((cb >> (4 + 2 * qsl + ksl)) & 1u);
          }
        }
        float acc = 0.f;
        if (vis) {
          const float* kr = sk + jj * D;
          const float* qr = sq + t * (D + 1);
#pragma unroll 16
          for (int c = 0; c < D; ++c) acc = fmaf(qr[c], kr[c], acc);
        }
        s[jj] = vis ? acc * p.scale : -INFINITY;
        cmax = fmaxf(cmax, s[jj]);
      }
      if (cmax == -INFINITY) continue;  // nothing visible to this row in the chunk
      const float m_new = fmaxf(m, cmax);
      const float alpha = expf(m - m_new);  // 0 when m is -inf
      l *= alpha;
#pragma unroll
      for (int c = 0; c < D; ++c) o[c] *= alpha;
      m = m_new;
#pragma unroll 2
      for (int jj = 0; jj < kChunk; ++jj) {
        const float pj = expf(s[jj] - m);  // 0 for masked scores
        l += pj;
        const float* vr = sv + jj * D;
#pragma unroll
        for (int c = 0; c < D; ++c) o[c] = fmaf(pj, vr[c], o[c]);
      }
    }
  }

  if (qi < p.Nq) {
    const bool has = l > 0.f;
    const float inv = has ? 1.f / l : 0.f;
    float* orow = p.out + b * p.os0 + head * p.os1 + static_cast<int64_t>(qi) * p.os2;
#pragma unroll
    for (int c = 0; c < D; ++c) orow[c] = has ? o[c] * inv : 0.f;
    p.lse[(static_cast<size_t>(b) * p.Hq + head) * p.Nq + qi] = has ? m + logf(l) : -INFINITY;
  }
}

template <int D>
mfa_status launch_d(const F32Params& p, cudaStream_t s) {
  const size_t smem = (kRowsPerBlock * (D + 1) + 2 * kChunk * D) * sizeof(float) + kChunk * sizeof(int4);
  static std::atomic<uint64_t> attr_devs{0};
  if (!ensure_smem_attr(reinterpret_cast<const void*>(mfa_fwd_f32_kernel<D>), static_cast<int>(smem), attr_devs))
    return MFA_ERR_CUDA;
  const dim3 grid((p.Nq + kRowsPerBlock - 1) / kRowsPerBlock, p.Hq, p.B);
  mfa_fwd_f32_kernel<D><<<grid, kRowsPerBlock, smem, s>>>(p);
  return cudaGetLastError() == cudaSuccess ? MFA_OK : MFA_ERR_CUDA;
}

}  // namespace

mfa_status launch_fwd_f32(const mfa_tensor* q, const mfa_tensor* k, const mfa_tensor* v, const mfa_mask_desc* mask,
                          const mfa_tile_map* map, const mfa_tensor* out, float* lse, cudaStream_t s) {
  if (q->B > 65535 || q->H > 65535) return MFA_ERR_UNSUPPORTED;
  F32Params p;
  p.B = static_cast<int32_t>(q->B);
  p.Hq = static_cast<int32_t>(q->H);
  p.G = static_cast<int32_t>(q->H / k->H);
  p.Hm = mask->Hm;
  p.Nq = static_cast<int32_t>(q->N);
  p.Nk = static_cast<int32_t>(k->N);
  p.nqt = map->nqt;
  p.nkt = map->nkt;
  p.BQ = map->block_q;
  p.BK = map->block_k;
  p.scale = static_cast<float>(1.0 / std::sqrt(static_cast<double>(q->D)));
  p.mask = mask_args(mask);
  p.cls = map->tile_class;
  p.list = map->tile_list;
  p.count = map->tile_count;
  p.q = static_cast<const float*>(q->data);
  p.k = static_cast<const float*>(k->data);
  p.v = static_cast<const float*>(v->data);
  p.qs0 = q->stride[0]; p.qs1 = q->stride[1]; p.qs2 = q->stride[2];
  p.ks0 = k->stride[0]; p.ks1 = k->stride[1]; p.ks2 = k->stride[2];
  p.vs0 = v->stride[0]; p.vs1 = v->stride[1]; p.vs2 = v->stride[2];
  p.os0 = out->stride[0]; p.os1 = out->stride[1]; p.os2 = out->stride[2];
  p.out = static_cast<float*>(out->data);
  p.lse = lse;
  p.err = map->err;
  if (p.Nq == 0) return MFA_OK;
  return q->D == 64 ? launch_d<64>(p, s) : launch_d<128>(p, s);
}

}  // namespace mfa
