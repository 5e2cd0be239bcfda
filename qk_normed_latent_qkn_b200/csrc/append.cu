// qkn_append kernels: write new tokens into the latent cache, the normalised
// and rotated RoPE key, and the per-token, per-group inverse RMS a_k of the
// up-projected key ("QK-Normed MLA: QK normalization without full key
// caching", technical summary, Metodología items 2 and 4).
//
// Three launches on the caller's stream:
//   1. append_copy:     one warp per token — latent copy, RoPE key
//                       (RMS-normalise, weight, rotate), a_k slots zeroed;
//   2. append_keyrms:   z = c W^K_g tiled over (column block, token tile,
//                       group); each CTA adds sum(z^2) of its columns into
//                       the token's a_k slot;
//   3. append_finalize: a_k = 1 / sqrt(sum / (n_g d_h) + eps).
// The key z is only ever held in registers; it is never written anywhere.
#include "common.cuh"
#include "kernels.h"

namespace qkn {

// Rotate pairs (i, i + d/2) of x (length d, lanes hold x[lane], x[lane+32], ...)
// by angle pos * theta^(-2i/d).  Angles are formed in fp64 so that positions in
// the hundreds of thousands keep full fp32 accuracy after the rotation.
__device__ __forceinline__ void rope_pair(float& x1, float& x2, int i, int d, int32_t pos, float theta) {
  const double freq = pow((double)theta, -2.0 * (double)i / (double)d);
  double s, c;
  sincos((double)pos * freq, &s, &c);
  const float cs = (float)c, sn = (float)s;
  const float a = x1 * cs - x2 * sn;
  const float b = x2 * cs + x1 * sn;
  x1 = a;
  x2 = b;
}

template <typename T>
__global__ void __launch_bounds__(256) append_copy_kernel(AppendArgs a) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= a.n_tok) return;
  const int64_t slot = a.slot[warp];
  const int32_t pos = a.pos[warp];
  const T* src = static_cast<const T*>(a.c_new) + (int64_t)warp * a.r;
  T* dst = static_cast<T*>(a.latent) + slot * a.r;
  for (int k = lane; k < a.r; k += 32) dst[k] = src[k];

  // RoPE key: d_R <= 128, so each lane holds at most 4 elements.
  const T* kr = static_cast<const T*>(a.k_rope_raw) + (int64_t)warp * a.d_rope;
  float x[4];
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int k = lane + 32 * i;
    x[i] = k < a.d_rope ? to_f32(kr[k]) : 0.f;
    ss += x[i] * x[i];
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const float inv = 1.0f / sqrtf(ss / (float)a.d_rope + a.eps);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int k = lane + 32 * i;
    if (k < a.d_rope) x[i] = x[i] * inv * a.gamma_kr[k];
  }
  // Pair element k (< d/2) with k + d/2, which sits in lane (k + d/2) % 32 of
  // slot (k + d/2) / 32.  Gather the partner through a small shared buffer.
  __shared__ float buf[8][128];
  float* row = buf[threadIdx.x >> 5];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int k = lane + 32 * i;
    if (k < a.d_rope) row[k] = x[i];
  }
  __syncwarp();
  T* kout = static_cast<T*>(a.k_rope) + slot * a.d_rope;
  const int half = a.d_rope / 2;
  for (int i = lane; i < half; i += 32) {
    float x1 = row[i], x2 = row[i + half];
    rope_pair(x1, x2, i, a.d_rope, pos, a.rope_theta);
    kout[i] = from_f32<T>(x1);
    kout[i + half] = from_f32<T>(x2);
  }
  for (int g = lane; g < a.groups; g += 32) a.a_k[slot * a.groups + g] = 0.f;
}

constexpr int kRmsTok = 32;      // tokens per CTA
constexpr int kRmsCols = 256;    // key columns per CTA (one per thread)

template <typename T>
__global__ void __launch_bounds__(kRmsCols) append_keyrms_kernel(AppendArgs a) {
  extern __shared__ float4 smem4[];
  float* cs = reinterpret_cast<float*>(smem4);          // [kRmsTok][r]
  __shared__ float red[kRmsCols / 32][kRmsTok];
  const int g = blockIdx.z;
  const int t0 = blockIdx.y * kRmsTok;
  const int ntok = min(kRmsTok, a.n_tok - t0);
  const int width = a.width;                            // n_g * d_h
  const int n = blockIdx.x * kRmsCols + threadIdx.x;

  const T* c = static_cast<const T*>(a.c_new);
  for (int e = threadIdx.x; e < kRmsTok * a.r; e += blockDim.x) {
    const int t = e / a.r, k = e - t * a.r;
    cs[e] = t < ntok ? to_f32(c[(int64_t)(t0 + t) * a.r + k]) : 0.f;
  }
  __syncthreads();

  float acc[kRmsTok];
#pragma unroll
  for (int t = 0; t < kRmsTok; ++t) acc[t] = 0.f;
  if (n < width) {
    const float* w = a.w_k + (int64_t)g * a.r * width + n;
    for (int k = 0; k < a.r; k += 4) {
      const float w0 = w[(int64_t)(k + 0) * width], w1 = w[(int64_t)(k + 1) * width];
      const float w2 = w[(int64_t)(k + 2) * width], w3 = w[(int64_t)(k + 3) * width];
#pragma unroll
      for (int t = 0; t < kRmsTok; ++t) {
        const float4 cv = *reinterpret_cast<const float4*>(cs + t * a.r + k);
        acc[t] = fmaf(cv.x, w0, acc[t]);
        acc[t] = fmaf(cv.y, w1, acc[t]);
        acc[t] = fmaf(cv.z, w2, acc[t]);
        acc[t] = fmaf(cv.w, w3, acc[t]);
      }
    }
  }
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
#pragma unroll
  for (int t = 0; t < kRmsTok; ++t) {
    float v = acc[t] * acc[t];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0) red[wid][t] = v;
  }
  __syncthreads();
  if (threadIdx.x < ntok) {
    float s = 0.f;
#pragma unroll
    for (int w8 = 0; w8 < kRmsCols / 32; ++w8) s += red[w8][threadIdx.x];
    atomicAdd(a.a_k + (int64_t)a.slot[t0 + threadIdx.x] * a.groups + g, s);
  }
}

__global__ void append_finalize_kernel(AppendArgs a) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= a.n_tok * a.groups) return;
  const int t = i / a.groups, g = i - t * a.groups;
  float* p = a.a_k + (int64_t)a.slot[t] * a.groups + g;
  *p = 1.0f / sqrtf(*p / (float)a.width + a.eps);
}

template <typename T>
static cudaError_t launch_append_t(const AppendArgs& a, cudaStream_t st) {
  append_copy_kernel<T><<<(a.n_tok + 7) / 8, 256, 0, st>>>(a);
  const size_t smem = (size_t)kRmsTok * a.r * sizeof(float);
  static bool attr_set = false;   // one attribute per instantiation
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(append_keyrms_kernel<T>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, 160 * 1024);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  dim3 grid((a.width + kRmsCols - 1) / kRmsCols, (a.n_tok + kRmsTok - 1) / kRmsTok, a.groups);
  append_keyrms_kernel<T><<<grid, kRmsCols, smem, st>>>(a);
  append_finalize_kernel<<<(a.n_tok * a.groups + 255) / 256, 256, 0, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_append(const AppendArgs& a, bool bf16, cudaStream_t st) {
  return bf16 ? launch_append_t<__nv_bfloat16>(a, st) : launch_append_t<float>(a, st);
}

}  // namespace qkn
