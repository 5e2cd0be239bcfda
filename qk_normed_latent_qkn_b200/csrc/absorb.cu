// qkn_absorb_query kernels: fold the static norm weights into the query
// ("QK-Normed MLA: QK normalization without full key caching", technical
// summary, Metodología item 1 and the decode-logit equation).
//
//   q~[i,h]  = W^K_{g,h} (gamma_q[h] * gamma_k[h] * q[i,h])        (absorb_qtilde)
//   a_q[i,h] = sigma / S(q[i,h])                                   (absorb_row)
//   q^R^[i,h] = sigma * RoPE_pos(gamma_qR[h] * q^R / S(q^R))        (absorb_row)
// One launch: one extra CTA per head does the per-row work beside the q~ CTAs.
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

constexpr int kAbsK = 32;        // latent rows of W^K_{g,h} per CTA (one per lane)
constexpr int kAbsQ = 32;        // query rows per pass (four per warp)

// grid (H, ceil(r / kAbsK) + 1); block 256.  CTA (h, y < last) stages its
// 32 x d_h slice of W^K_{g,h} once, with gamma_q * gamma_k folded into its
// columns, and computes q~[i, h, k] for its 32 values of k and every query
// row i: lane = latent row k, warp w = query rows w, w + 8, ... of the pass,
// so a warp's W reads hit 32 banks and its query reads are broadcasts.  The
// CTA with y == last produces a_q and the RoPE query of head h.
template <typename T>
__global__ void __launch_bounds__(256) absorb_qtilde_kernel(const __grid_constant__ AbsorbArgs a) {
  extern __shared__ float4 smem4[];
  // row pitch d_h + 4: 16-byte aligned rows, and the eight lanes of a quarter-warp read distinct banks
  const int pitch = a.d_h + 4;
  float* wc = reinterpret_cast<float*>(smem4);             // [kAbsK][d_h + 4]
  float* sv = wc + kAbsK * pitch;                          // [kAbsQ][d_h]
  const int h = blockIdx.x;
  const int nkb = (a.r + kAbsK - 1) / kAbsK;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_trigger();
  pdl_wait();
  if ((int)blockIdx.y == nkb) {
    __shared__ float rowbuf[8][128];
    for (int i = warp; i < a.n_q; i += 8) absorb_row<T>(a, i, h, rowbuf[warp], lane);
    return;
  }
  const int kbase = blockIdx.y * kAbsK;
  const int ng = a.heads / a.groups;
  const int g = h / ng, m = h - g * ng;
  const int width = ng * a.d_h;
  const float* w = a.w_k + (int64_t)g * a.r * width + (int64_t)m * a.d_h;
  const int dq = a.d_h / 4;
  // stage the slice, gamma_q * gamma_k folded in; one batch of independent 16-byte loads
  for (int e0 = threadIdx.x; e0 < kAbsK * dq; e0 += 4 * blockDim.x) {
    float4 v[4], gq[4], gk[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int e = e0 + u * blockDim.x;
      const int rr = e / dq, d4 = e - rr * dq;
      const bool ok = e < kAbsK * dq && kbase + rr < a.r;
      v[u] = ok ? *reinterpret_cast<const float4*>(w + (int64_t)(kbase + rr) * width + d4 * 4)
                : make_float4(0.f, 0.f, 0.f, 0.f);
      gq[u] = ok ? *reinterpret_cast<const float4*>(a.gamma_q + h * a.d_h + d4 * 4) : make_float4(0.f, 0.f, 0.f, 0.f);
      gk[u] = ok ? *reinterpret_cast<const float4*>(a.gamma_k + h * a.d_h + d4 * 4) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int e = e0 + u * blockDim.x;
      if (e < kAbsK * dq) {
        const int rr = e / dq, d4 = e - rr * dq;
        *reinterpret_cast<float4*>(wc + rr * pitch + d4 * 4) =
            make_float4(v[u].x * gq[u].x * gk[u].x, v[u].y * gq[u].y * gk[u].y, v[u].z * gq[u].z * gk[u].z,
                        v[u].w * gq[u].w * gk[u].w);
      }
    }
  }
  const T* q = static_cast<const T*>(a.q);
  T* out = static_cast<T*>(a.q_tilde);
  const float* wrow = wc + lane * pitch;
  const bool k_ok = kbase + lane < a.r;
  for (int i0 = 0; i0 < a.n_q; i0 += kAbsQ) {
    const int nq = min(kAbsQ, a.n_q - i0);
    __syncthreads();
    // stage the pass's query rows of head h as fp32
    for (int e0 = threadIdx.x; e0 < kAbsQ * dq; e0 += 2 * blockDim.x) {
      float4 v[2];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int e = e0 + u * blockDim.x;
        const int qi = e / dq, d4 = e - qi * dq;
        v[u] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (e < kAbsQ * dq && qi < nq) {
          const T* src = q + ((int64_t)(i0 + qi) * a.heads + h) * a.d_h + d4 * 4;
          v[u] = make_float4(to_f32(src[0]), to_f32(src[1]), to_f32(src[2]), to_f32(src[3]));
        }
      }
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int e = e0 + u * blockDim.x;
        if (e < kAbsQ * dq) reinterpret_cast<float4*>(sv)[e] = v[u];
      }
    }
    __syncthreads();
    float acc[kAbsQ / 8];
#pragma unroll
    for (int j = 0; j < kAbsQ / 8; ++j) acc[j] = 0.f;
    // query rows warp, warp + 8, ... of the pass that exist (warp-uniform)
    const int nj = (nq - warp + 7) / 8;
    for (int d = 0; d < a.d_h; d += 4) {
      const float4 wq = *reinterpret_cast<const float4*>(wrow + d);
#pragma unroll
      for (int j = 0; j < kAbsQ / 8; ++j) {
        if (j < nj) {
          const float4 sq = *reinterpret_cast<const float4*>(sv + (warp + 8 * j) * a.d_h + d);
          acc[j] = fmaf(wq.x, sq.x, fmaf(wq.y, sq.y, fmaf(wq.z, sq.z, fmaf(wq.w, sq.w, acc[j]))));
        }
      }
    }
#pragma unroll
    for (int j = 0; j < kAbsQ / 8; ++j) {
      const int qi = warp + 8 * j;
      if (qi < nq && k_ok) out[((int64_t)(i0 + qi) * a.heads + h) * a.r + kbase + lane] = from_f32<T>(acc[j]);
    }
  }
}

template <typename T>
static cudaError_t launch_absorb_t(const AbsorbArgs& a, cudaStream_t st) {
  const size_t smem = ((size_t)kAbsK * (a.d_h + 4) + (size_t)kAbsQ * a.d_h) * sizeof(float);
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(absorb_qtilde_kernel<T>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  dim3 grid(a.heads, (a.r + kAbsK - 1) / kAbsK + 1);
  return launch_chained(absorb_qtilde_kernel<T>, grid, dim3(256), smem, st, a);
}

cudaError_t launch_absorb(const AbsorbArgs& a, bool bf16, cudaStream_t st) {
  return bf16 ? launch_absorb_t<__nv_bfloat16>(a, st) : launch_absorb_t<float>(a, st);
}

}  // namespace qkn
