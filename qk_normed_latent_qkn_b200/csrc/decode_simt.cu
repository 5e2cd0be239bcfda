// CUDA-core split-KV decode: the same computation as the tcgen05 kernel, on
// fp32 FMA units.  It serves fp32 workloads (where bf16 tensor-core operands
// would not meet fp32 accuracy) and any shape the tcgen05 kernel does not
// take.  Decode logit ("QK-Normed MLA: QK normalization without full key
// caching", technical summary, Metodología, decode-logit equation):
//   l[t] = a_q * a_k[t, g(h)] * (q~ . c_t) + q^R^ . k^R^_t
// followed by an online softmax over the item's pages and the weighted sum of
// the latents.  One CTA per schedule slot; one warp per query row; each lane
// holds latent elements lane, lane+32, ... of q~ and of the running output.
#include "common.cuh"
#include "kernels.h"

namespace qkn {

template <typename T, int NK>
__global__ void __launch_bounds__(kSimtRows * 32) decode_simt_kernel(DecodeArgs a) {
  extern __shared__ float4 smem4[];
  T* cs = reinterpret_cast<T*>(smem4);                          // [64][r]
  T* krs = cs + kBlockSize * a.r;                               // [64][d_rope]
  float* aks = reinterpret_cast<float*>(krs + kBlockSize * a.d_rope);   // [64][groups]
  __shared__ Cursor cur_s;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_trigger();
  pdl_wait();
  SchedParams sp{a.seq_lens, a.batch, a.s_q, a.max_blocks, a.ht_count, a.ncta, a.item_cost,
                 a.heads, a.rows, a.vis_end};
  if (warp == 0) {
    Cursor c = sched_begin(sp, blockIdx.x);
    if (lane == 0) cur_s = c;
  }
  __syncthreads();
  Cursor cur = cur_s;
  const int ng = a.heads / a.groups;
  const int qrows = a.s_q * a.heads;
  Item it;
  while (sched_next(cur, sp, blockIdx.x, it)) {
    const int rho = it.ht * a.rows + warp;
    const bool valid = rho < qrows;
    const int j = valid ? rho / a.heads : 0;
    const int h = valid ? rho - j * a.heads : 0;
    const int grp = h / ng;
    const int32_t qpos = (a.vis_end ? a.vis_end[it.b] : it.L) - a.s_q + j;
    const int64_t qrow = (int64_t)it.b * qrows + (valid ? rho : 0);

    float qv[NK], ov[NK];
    const T* qt = static_cast<const T*>(a.q_tilde) + qrow * a.r;
#pragma unroll
    for (int i = 0; i < NK; ++i) {
      const int k = lane + 32 * i;
      qv[i] = (k < a.r) ? to_f32(qt[k]) : 0.f;
      ov[i] = 0.f;
    }
    float qr[4];
    const T* qrp = static_cast<const T*>(a.q_rope_hat) + qrow * a.d_rope;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int k = lane + 32 * i;
      qr[i] = (k < a.d_rope) ? to_f32(qrp[k]) : 0.f;
    }
    const float aq = a.a_q[qrow];
    float m = -INFINITY, lsum = 0.f;

    for (int p = it.p0; p < it.p1; ++p) {
      int32_t blk = a.block_table[(int64_t)it.b * a.max_blocks + p];
      if (blk < 0 || blk >= a.num_blocks) {
        record_status(a.status, QKN_ERR_BOUNDS);
        blk = 0;
      }
      __syncthreads();
      {   // stage the page: latent, RoPE key, a_k
        const uint4* src = reinterpret_cast<const uint4*>(static_cast<const T*>(a.latent) +
                                                          (int64_t)blk * kBlockSize * a.r);
        uint4* dst = reinterpret_cast<uint4*>(cs);
        const int n16 = kBlockSize * a.r * (int)sizeof(T) / 16;
        for (int e = threadIdx.x; e < n16; e += blockDim.x) dst[e] = src[e];
        const uint4* srk = reinterpret_cast<const uint4*>(static_cast<const T*>(a.k_rope) +
                                                          (int64_t)blk * kBlockSize * a.d_rope);
        uint4* dsk = reinterpret_cast<uint4*>(krs);
        const int k16 = kBlockSize * a.d_rope * (int)sizeof(T) / 16;
        for (int e = threadIdx.x; e < k16; e += blockDim.x) dsk[e] = srk[e];
        const float* sak = a.a_k + (int64_t)blk * kBlockSize * a.groups;
        for (int e = threadIdx.x; e < kBlockSize * a.groups; e += blockDim.x) aks[e] = sak[e];
      }
      __syncthreads();
      if (!valid) continue;
      const int t0 = p * kBlockSize;
      // tokens t0 + tt with tt < nvis are visible to this query row
      const int nvis = min(kBlockSize, qpos + 1 - t0);
      if (nvis <= 0) continue;
      float l0 = -INFINITY, l1 = -INFINITY;
      for (int tt = 0; tt < nvis; ++tt) {
        const T* crow = cs + tt * a.r;
        float dot = 0.f;
#pragma unroll
        for (int i = 0; i < NK; ++i) {
          const int k = lane + 32 * i;
          if (k < a.r) dot = fmaf(qv[i], to_f32(crow[k]), dot);
        }
        float rdot = 0.f;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int k = lane + 32 * i;
          if (k < a.d_rope) rdot = fmaf(qr[i], to_f32(krs[tt * a.d_rope + k]), rdot);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          dot += __shfl_xor_sync(0xffffffffu, dot, o);
          rdot += __shfl_xor_sync(0xffffffffu, rdot, o);
        }
        const float ak = a.ak_one ? 1.f : aks[tt * a.groups + grp];
        const float l = aq * ak * dot + rdot;
        if ((tt & 31) == lane) {
          if (tt < 32) l0 = l; else l1 = l;
        }
      }
      float mt = fmaxf(l0, l1);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, o));
      const float mn = fmaxf(m, mt);
      const float corr = (m == -INFINITY) ? 0.f : __expf(m - mn);
      const float p0 = (l0 == -INFINITY) ? 0.f : __expf(l0 - mn);
      const float p1 = (l1 == -INFINITY) ? 0.f : __expf(l1 - mn);
      float ps = p0 + p1;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o);
      lsum = lsum * corr + ps;
#pragma unroll
      for (int i = 0; i < NK; ++i) ov[i] *= corr;
      for (int tt = 0; tt < nvis; ++tt) {
        const float pt = __shfl_sync(0xffffffffu, tt < 32 ? p0 : p1, tt & 31);
        const T* crow = cs + tt * a.r;
#pragma unroll
        for (int i = 0; i < NK; ++i) {
          const int k = lane + 32 * i;
          if (k < a.r) ov[i] = fmaf(pt, to_f32(crow[k]), ov[i]);
        }
      }
      m = mn;
    }
    if (valid) {
      const int64_t prow = (int64_t)it.slot * a.rows + warp;
      float* po = a.part_o + prow * a.r;
      const float inv = lsum > 0.f ? 1.f / lsum : 0.f;
#pragma unroll
      for (int i = 0; i < NK; ++i) {
        const int k = lane + 32 * i;
        if (k < a.r) po[k] = ov[i] * inv;
      }
      if (lane == 0) a.part_lse[prow] = lsum > 0.f ? m + logf(lsum) : -INFINITY;
    }
  }
}

template <typename T, int NK>
static cudaError_t launch_simt_nk(const DecodeArgs& a, cudaStream_t st) {
  const size_t smem = (size_t)kBlockSize * (a.r + a.d_rope) * sizeof(T) +
                      (size_t)kBlockSize * a.groups * sizeof(float);
  static PerDeviceOnce attrs;
  cudaError_t e = once_per_device(attrs, [] { return set_smem_attrs(decode_simt_kernel<T, NK>, 200 * 1024); });
  if (e != cudaSuccess) return e;
  return launch_chained(decode_simt_kernel<T, NK>, dim3(a.ncta), dim3(kSimtRows * 32), smem, st, a);
}

template <typename T>
static cudaError_t launch_simt_t(const DecodeArgs& a, cudaStream_t st) {
  const int nk = (a.r + 31) / 32;
  if (nk <= 2) return launch_simt_nk<T, 2>(a, st);
  if (nk <= 4) return launch_simt_nk<T, 4>(a, st);
  if (nk <= 8) return launch_simt_nk<T, 8>(a, st);
  if (nk <= 16) return launch_simt_nk<T, 16>(a, st);
  return launch_simt_nk<T, 32>(a, st);
}

cudaError_t launch_decode_simt(const DecodeArgs& a, bool bf16, cudaStream_t st) {
  return bf16 ? launch_simt_t<__nv_bfloat16>(a, st) : launch_simt_t<float>(a, st);
}

}  // namespace qkn
