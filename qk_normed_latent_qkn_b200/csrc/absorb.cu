// qkn_absorb_query kernels: fold the static norm weights into the query
// ("QK-Normed MLA: QK normalization without full key caching", technical
// summary, Metodología item 1 and the decode-logit equation).
//
//   q~[i,h]  = W^K_{g,h} (gamma_q[h] * gamma_k[h] * q[i,h])        (absorb_qtilde)
//   a_q[i,h] = sigma / S(q[i,h])                                   (absorb_row)
//   q^R^[i,h] = sigma * RoPE_pos(gamma_qR[h] * q^R / S(q^R))        (absorb_row)
// One launch: the CTAs of the first latent block also do the per-row work.
#include "common.cuh"
#include "kernels.h"

namespace qkn {

// a_q[i,h] and the rotated RoPE query of one (query row i, head h), by one warp.
template <typename T>
__device__ __forceinline__ void absorb_row(const AbsorbArgs& a, int i, int h, float* row, int lane) {
  const int64_t wid = (int64_t)i * a.heads + h;
  const T* q = static_cast<const T*>(a.q) + wid * a.d_h;
  float ss = 0.f;
  for (int d = lane; d < a.d_h; d += 32) {
    const float v = to_f32(q[d]);
    ss += v * v;
  }
  const T* qr = static_cast<const T*>(a.q_rope) + wid * a.d_rope;
  float sr = 0.f;
  for (int d = lane; d < a.d_rope; d += 32) {
    const float v = to_f32(qr[d]);
    row[d] = v;
    sr += v * v;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    ss += __shfl_xor_sync(0xffffffffu, ss, o);
    sr += __shfl_xor_sync(0xffffffffu, sr, o);
  }
  if (lane == 0) a.a_q[wid] = a.softmax_scale / sqrtf(ss / (float)a.d_h + a.eps);
  const float inv = a.softmax_scale / sqrtf(sr / (float)a.d_rope + a.eps);
  __syncwarp();
  const int half = a.d_rope / 2;
  const int32_t pos = a.pos[i];
  T* out = static_cast<T*>(a.q_rope_hat) + wid * a.d_rope;
  for (int d = lane; d < half; d += 32) {
    const float x1 = row[d] * inv * a.gamma_qr[h * a.d_rope + d];
    const float x2 = row[d + half] * inv * a.gamma_qr[h * a.d_rope + d + half];
    float sn, cs;
    rope_sincos(pos, a.freq.f[d], sn, cs);
    out[d] = from_f32<T>(x1 * cs - x2 * sn);
    out[d + half] = from_f32<T>(x2 * cs + x1 * sn);
  }
  __syncwarp();
}

constexpr int kAbsK = 64;        // latent rows of W^K_{g,h} per CTA
constexpr int kAbsQ = 64;        // query rows per pass (16 quads of 4)

// grid (H, ceil(r / kAbsK)); block 256.  The CTA stages its 64 x d_h slice of
// W^K_{g,h} once (rows padded by one float), then computes q~[i, h, k] for its
// 64 values of k and every query row i, 4 x 4 outputs per thread.
template <typename T>
__global__ void __launch_bounds__(256) absorb_qtilde_kernel(const __grid_constant__ AbsorbArgs a) {
  extern __shared__ float4 smem4[];
  const int pitch = a.d_h + 1;
  float* wc = reinterpret_cast<float*>(smem4);             // [kAbsK][d_h + 1]
  float* sv = wc + kAbsK * pitch;                          // [kAbsQ][d_h]
  const int h = blockIdx.x;
  const int kbase = blockIdx.y * kAbsK;
  const int ng = a.heads / a.groups;
  const int g = h / ng, m = h - g * ng;
  const int width = ng * a.d_h;
  const float* w = a.w_k + (int64_t)g * a.r * width + (int64_t)m * a.d_h;
  pdl_trigger();
  pdl_wait();
  // stage the slice with batches of independent loads (d_h is a multiple of 4 here)
  const int nvec = kAbsK * (a.d_h / 4);
  for (int e0 = threadIdx.x; e0 < nvec; e0 += 8 * blockDim.x) {
    float4 v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int e = e0 + u * blockDim.x;
      const int rr = e / (a.d_h / 4), d4 = e - rr * (a.d_h / 4);
      v[u] = (e < nvec && kbase + rr < a.r)
                 ? *reinterpret_cast<const float4*>(w + (int64_t)(kbase + rr) * width + d4 * 4)
                 : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int e = e0 + u * blockDim.x;
      if (e < nvec) {
        const int rr = e / (a.d_h / 4), d4 = e - rr * (a.d_h / 4);
        float* dst = wc + rr * pitch + d4 * 4;
        dst[0] = v[u].x;
        dst[1] = v[u].y;
        dst[2] = v[u].z;
        dst[3] = v[u].w;
      }
    }
  }
  const T* q = static_cast<const T*>(a.q);
  T* out = static_cast<T*>(a.q_tilde);
  // 256 threads = 16 latent quads x 16 query quads: each thread computes a 4 x 4 block of
  // q~ (latent rows kq*4.., query rows qq*4..), reusing every shared-memory value four times
  const int kq = threadIdx.x & 15, qq = threadIdx.x >> 4;
  for (int i0 = 0; i0 < a.n_q; i0 += kAbsQ) {
    const int nq = min(kAbsQ, a.n_q - i0);
    __syncthreads();
    // stage gamma_q * gamma_k * q for the pass, loads batched four deep
    for (int e0 = threadIdx.x; e0 < kAbsQ * a.d_h; e0 += 4 * blockDim.x) {
      float qv[4], gq[4], gk[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int e = e0 + u * blockDim.x;
        const int qi = e / a.d_h, d = e - qi * a.d_h;
        const bool ok = e < kAbsQ * a.d_h && qi < nq;
        qv[u] = ok ? to_f32(q[((int64_t)(i0 + qi) * a.heads + h) * a.d_h + d]) : 0.f;
        gq[u] = ok ? a.gamma_q[h * a.d_h + d] : 0.f;
        gk[u] = ok ? a.gamma_k[h * a.d_h + d] : 0.f;
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int e = e0 + u * blockDim.x;
        if (e < kAbsQ * a.d_h) sv[e] = qv[u] * gq[u] * gk[u];
      }
    }
    __syncthreads();
    if (qq * 4 < nq) {
      float acc[4][4];
#pragma unroll
      for (int x = 0; x < 4; ++x)
#pragma unroll
        for (int y = 0; y < 4; ++y) acc[x][y] = 0.f;
      const float* w0 = wc + (kq * 4) * pitch;
      const float* s0 = sv + (qq * 4) * a.d_h;
      for (int d = 0; d < a.d_h; ++d) {
        float wv[4], qv[4];
#pragma unroll
        for (int x = 0; x < 4; ++x) wv[x] = w0[x * pitch + d];
#pragma unroll
        for (int y = 0; y < 4; ++y) qv[y] = s0[y * a.d_h + d];
#pragma unroll
        for (int x = 0; x < 4; ++x)
#pragma unroll
          for (int y = 0; y < 4; ++y) acc[x][y] = fmaf(wv[x], qv[y], acc[x][y]);
      }
#pragma unroll
      for (int y = 0; y < 4; ++y) {
        const int qi = qq * 4 + y;
        if (qi >= nq) break;
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          const int k = kbase + kq * 4 + x;
          if (k < a.r) out[((int64_t)(i0 + qi) * a.heads + h) * a.r + k] = from_f32<T>(acc[x][y]);
        }
      }
    }
  }
  // the first latent block's CTA of each head also produces a_q and the RoPE query of that head
  if (blockIdx.y == 0) {
    __shared__ float rowbuf[8][128];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int i = warp; i < a.n_q; i += 8) absorb_row<T>(a, i, h, rowbuf[warp], lane);
  }
}

template <typename T>
static cudaError_t launch_absorb_t(const AbsorbArgs& a, cudaStream_t st) {
  const size_t smem = ((size_t)kAbsK * (a.d_h + 1) + (size_t)kAbsQ * a.d_h) * sizeof(float);
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(absorb_qtilde_kernel<T>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  dim3 grid(a.heads, (a.r + kAbsK - 1) / kAbsK);
  return launch_chained(absorb_qtilde_kernel<T>, grid, dim3(256), smem, st, a);
}

cudaError_t launch_absorb(const AbsorbArgs& a, bool bf16, cudaStream_t st) {
  return bf16 ? launch_absorb_t<__nv_bfloat16>(a, st) : launch_absorb_t<float>(a, st);
}

}  // namespace qkn
