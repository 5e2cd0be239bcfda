// qkn_absorb_query kernels: fold the static norm weights into the query
// ("QK-Normed MLA: QK normalization without full key caching", technical
// summary, Metodología item 1 and the decode-logit equation).
//
//   q~[i,h]  = W^K_{g,h} (gamma_q[h] * gamma_k[h] * q[i,h])        (absorb_qtilde)
//   a_q[i,h] = sigma / S(q[i,h])                                   (absorb_rows)
//   q^R^[i,h] = sigma * RoPE_pos(gamma_qR[h] * q^R / S(q^R))        (absorb_rows)
#include "common.cuh"
#include "kernels.h"

namespace qkn {

constexpr int kAbsQ = 16;        // query rows per CTA
constexpr int kAbsK = 32;        // latent rows of W per staged chunk

// grid (H, ceil(n_q / kAbsQ)); block 256.  Stages W^K_{g,h} (r x d_h) through
// shared memory in chunks of kAbsK latent rows.
template <typename T>
__global__ void __launch_bounds__(256) absorb_qtilde_kernel(AbsorbArgs a) {
  extern __shared__ float4 smem4[];
  float* sv = reinterpret_cast<float*>(smem4);            // [kAbsQ][d_h]
  float* wc = sv + kAbsQ * a.d_h;                          // [kAbsK][d_h + 1]
  const int h = blockIdx.x;
  const int i0 = blockIdx.y * kAbsQ;
  const int nq = min(kAbsQ, a.n_q - i0);
  const int ng = a.heads / a.groups;
  const int g = h / ng, m = h - g * ng;
  const int width = ng * a.d_h;
  const int pitch = a.d_h + 1;
  const T* q = static_cast<const T*>(a.q);
  for (int e = threadIdx.x; e < kAbsQ * a.d_h; e += blockDim.x) {
    const int qi = e / a.d_h, d = e - qi * a.d_h;
    float v = 0.f;
    if (qi < nq)
      v = to_f32(q[((int64_t)(i0 + qi) * a.heads + h) * a.d_h + d]) * a.gamma_q[h * a.d_h + d] *
          a.gamma_k[h * a.d_h + d];
    sv[e] = v;
  }
  const float* w = a.w_k + (int64_t)g * a.r * width + (int64_t)m * a.d_h;
  T* out = static_cast<T*>(a.q_tilde);
  const int kk = threadIdx.x & 31;
  const int qsub = threadIdx.x >> 5;                       // 8 warps -> 8 query rows per pass
  for (int k0 = 0; k0 < a.r; k0 += kAbsK) {
    __syncthreads();
    for (int e = threadIdx.x; e < kAbsK * a.d_h; e += blockDim.x) {
      const int rr = e / a.d_h, d = e - rr * a.d_h;
      wc[rr * pitch + d] = (k0 + rr < a.r) ? w[(int64_t)(k0 + rr) * width + d] : 0.f;
    }
    __syncthreads();
    for (int qi = qsub; qi < nq; qi += 8) {
      float acc = 0.f;
      const float* wr = wc + kk * pitch;
      const float* sr = sv + qi * a.d_h;
      for (int d = 0; d < a.d_h; ++d) acc = fmaf(wr[d], sr[d], acc);
      if (k0 + kk < a.r) out[((int64_t)(i0 + qi) * a.heads + h) * a.r + k0 + kk] = from_f32<T>(acc);
    }
  }
}

// One warp per (query row, head): a_q and the rotated RoPE query.
template <typename T>
__global__ void __launch_bounds__(256) absorb_rows_kernel(AbsorbArgs a) {
  const int wid = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (wid >= a.n_q * a.heads) return;
  const int i = wid / a.heads, h = wid - i * a.heads;
  const T* q = static_cast<const T*>(a.q) + (int64_t)wid * a.d_h;
  float ss = 0.f;
  for (int d = lane; d < a.d_h; d += 32) {
    const float v = to_f32(q[d]);
    ss += v * v;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if (lane == 0) a.a_q[wid] = a.softmax_scale / sqrtf(ss / (float)a.d_h + a.eps);

  const T* qr = static_cast<const T*>(a.q_rope) + (int64_t)wid * a.d_rope;
  __shared__ float buf[8][128];
  float* row = buf[threadIdx.x >> 5];
  float sr = 0.f;
  for (int d = lane; d < a.d_rope; d += 32) {
    const float v = to_f32(qr[d]);
    row[d] = v;
    sr += v * v;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sr += __shfl_xor_sync(0xffffffffu, sr, o);
  const float inv = a.softmax_scale / sqrtf(sr / (float)a.d_rope + a.eps);
  __syncwarp();
  const int half = a.d_rope / 2;
  const int32_t pos = a.pos[i];
  T* out = static_cast<T*>(a.q_rope_hat) + (int64_t)wid * a.d_rope;
  for (int d = lane; d < half; d += 32) {
    float x1 = row[d] * inv * a.gamma_qr[h * a.d_rope + d];
    float x2 = row[d + half] * inv * a.gamma_qr[h * a.d_rope + d + half];
    const double freq = pow((double)a.rope_theta, -2.0 * (double)d / (double)a.d_rope);
    double s, c;
    sincos((double)pos * freq, &s, &c);
    const float cs = (float)c, sn = (float)s;
    out[d] = from_f32<T>(x1 * cs - x2 * sn);
    out[d + half] = from_f32<T>(x2 * cs + x1 * sn);
  }
}

template <typename T>
static cudaError_t launch_absorb_t(const AbsorbArgs& a, cudaStream_t st) {
  const size_t smem = ((size_t)kAbsQ * a.d_h + (size_t)kAbsK * (a.d_h + 1)) * sizeof(float);
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(absorb_qtilde_kernel<T>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, 96 * 1024);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  dim3 grid(a.heads, (a.n_q + kAbsQ - 1) / kAbsQ);
  absorb_qtilde_kernel<T><<<grid, 256, smem, st>>>(a);
  const int warps = a.n_q * a.heads;
  absorb_rows_kernel<T><<<(warps + 7) / 8, 256, 0, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_absorb(const AbsorbArgs& a, bool bf16, cudaStream_t st) {
  return bf16 ? launch_absorb_t<__nv_bfloat16>(a, st) : launch_absorb_t<float>(a, st);
}

}  // namespace qkn
