// qkn_append kernels: write new tokens into the latent cache, the normalised
// and rotated RoPE key, and the per-token, per-group inverse RMS a_k of the
// up-projected key ("QK-Normed MLA: QK normalization without full key
// caching", technical summary, Metodología items 2 and 4).
//
// With the cache's ak_scratch: one launch of append_keyrms<FUSED>, whose
// extra CTA column copies the latents and RoPE keys while the column CTAs
// compute the key statistic and the last of them finalises a_k.  Without it,
// three launches on the caller's stream:
//   1. append_copy:     one warp per token — latent copy, RoPE key
//                       (RMS-normalise, weight, rotate), a_k slots zeroed;
//   2. append_keyrms:   z = c W^K_g tiled over (16-column block, token
//                       tile, group); each CTA adds sum(z^2) of its columns
//                       into the token's a_k slot;
//   3. append_finalize: a_k = 1 / sqrt(sum / (n_g d_h) + eps).
// The key z is only ever held in registers; it is never written anywhere.
#include "common.cuh"
#include "kernels.h"

namespace qkn {

// Token i of the call, by one warp: the latent row copied, the RoPE key
// RMS-normalised, weighted and rotated.  `row` is the warp's 128-float
// shared-memory buffer (d_R <= 128).
template <typename T>
__device__ __forceinline__ void append_token(const AppendArgs& a, int i, int lane, float* row) {
  const int64_t slot = a.slot[i];
  const int32_t pos = a.pos[i];
  // latent row: 16-byte vectors (rows are a multiple of 16 bytes)
  const uint4* src = reinterpret_cast<const uint4*>(static_cast<const T*>(a.c_new) + (int64_t)i * a.r);
  uint4* dst = reinterpret_cast<uint4*>(static_cast<T*>(a.latent) + slot * a.r);
  const int nvec = a.r * (int)sizeof(T) / 16;
  uint4 cv[4];
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int k = lane + 32 * u;
    if (k < nvec) cv[u] = src[k];
  }
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int k = lane + 32 * u;
    if (k < nvec) dst[k] = cv[u];
  }
  for (int k = lane + 128; k < nvec; k += 32) dst[k] = src[k];

  // RoPE key: d_R <= 128, so each lane holds at most 4 elements.
  const T* kr = static_cast<const T*>(a.k_rope_raw) + (int64_t)i * a.d_rope;
  float x[4];
  float ss = 0.f;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int k = lane + 32 * q;
    x[q] = k < a.d_rope ? to_f32(kr[k]) : 0.f;
    ss += x[q] * x[q];
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const float inv = 1.0f / sqrtf(ss / (float)a.d_rope + a.eps);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int k = lane + 32 * q;
    if (k < a.d_rope) x[q] = x[q] * inv * a.gamma_kr[k];
  }
  // Pair element k (< d/2) with k + d/2, which sits in lane (k + d/2) % 32 of
  // slot (k + d/2) / 32.  Gather the partner through the warp's shared buffer.
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int k = lane + 32 * q;
    if (k < a.d_rope) row[k] = x[q];
  }
  __syncwarp();
  T* kout = static_cast<T*>(a.k_rope) + slot * a.d_rope;
  const int half = a.d_rope / 2;
  for (int k = lane; k < half; k += 32) {
    const float x1 = row[k], x2 = row[k + half];
    float sn, cs;
    rope_sincos(pos, a.freq.f[k], sn, cs);
    kout[k] = from_f32<T>(x1 * cs - x2 * sn);
    kout[k + half] = from_f32<T>(x2 * cs + x1 * sn);
  }
  __syncwarp();
}

// Three-launch path, step 1: one warp per token; the a_k slots are zeroed for
// the key-statistic atomics of step 2.
template <typename T>
__global__ void __launch_bounds__(256) append_copy_kernel(const __grid_constant__ AppendArgs a) {
  pdl_trigger();
  pdl_wait();
  __shared__ float buf[8][128];
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= a.n_tok) return;
  append_token<T>(a, warp, lane, buf[threadIdx.x >> 5]);
  const int64_t slot = a.slot[warp];
  for (int g = lane; g < a.groups; g += 32) a.a_k[slot * a.groups + g] = 0.f;
}

// Key statistic sum(z^2), z = c W^K_g.  CTA = (16 key columns, TT tokens,
// group); its 512 threads are 16 columns x 32 slices of the latent
// dimension, so a decode step's handful of tokens still spreads over about a
// hundred CTAs per group.  Every thread loads its slice of one W column in
// one batch of independent loads and applies it to the TT tokens held in
// shared memory; slices are summed in shared memory, squared, reduced over
// the CTA's 16 columns and added into the token's a_k slot (zeroed by
// append_copy_kernel).
constexpr int kRmsCols = 16;
constexpr int kRmsSlices = 32;

// FUSED (the cache has ak_scratch): the whole append in this one launch.  One
// more CTA column (blockIdx.x == number of column blocks) copies the tile's
// latents and RoPE keys; the column CTAs add their sums into the slot's
// accumulator in ak_scratch and count themselves in, and the CTA whose count
// completes a token writes a_k = 1 / sqrt(sum / width + eps) and returns the
// accumulator and the count to zero.
template <typename T, int TT, bool FUSED>
__global__ void __launch_bounds__(kRmsCols * kRmsSlices) append_keyrms_kernel(AppendArgs a) {
  extern __shared__ float4 smem4[];
  float* cs = reinterpret_cast<float*>(smem4);                    // [TT][r]
  float* zp = cs + TT * a.r;                                      // [kRmsSlices][TT][kRmsCols]
  const int g = blockIdx.z;
  const int t0 = blockIdx.y * TT;
  const int ntok = min(TT, a.n_tok - t0);
  const int width = a.width;
  const int col = threadIdx.x % kRmsCols, slice = threadIdx.x / kRmsCols;
  const int n = blockIdx.x * kRmsCols + col;
  const int nblk = (width + kRmsCols - 1) / kRmsCols;
  pdl_trigger();
  pdl_wait();
  if constexpr (FUSED) {
    if ((int)blockIdx.x == nblk) {
      __shared__ float rows[kRmsCols * kRmsSlices / 32][128];
      const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
      if (blockIdx.z == 0)
        for (int i = warp; i < ntok; i += kRmsCols * kRmsSlices / 32) append_token<T>(a, t0 + i, lane, rows[warp]);
      return;
    }
  }

  // latent rows [k0, k1) of this slice; W loads are issued before the token tile is staged
  const int k0 = (int)((int64_t)slice * a.r / kRmsSlices);
  const int k1 = (int)((int64_t)(slice + 1) * a.r / kRmsSlices);
  const float* w = a.w_k + (int64_t)g * a.r * width + min(n, width - 1);
  constexpr int kBatch = 16;
  float wv[kBatch];
#pragma unroll
  for (int u = 0; u < kBatch; ++u) wv[u] = (k0 + u < k1) ? w[(int64_t)(k0 + u) * width] : 0.f;

  {   // stage the token tile as fp32, 16 bytes of input per load
    constexpr int kPer = 16 / (int)sizeof(T);          // elements per 16-byte load
    const uint4* c4 = reinterpret_cast<const uint4*>(static_cast<const T*>(a.c_new) + (int64_t)t0 * a.r);
    const int nvec = TT * a.r / kPer;
    for (int e0 = threadIdx.x; e0 < nvec; e0 += 4 * blockDim.x) {
      uint4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int e = e0 + u * blockDim.x;
        v[u] = (e < nvec && (e * kPer) / a.r < ntok) ? c4[e] : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int e = e0 + u * blockDim.x;
        if (e < nvec) {
          const T* x = reinterpret_cast<const T*>(&v[u]);
#pragma unroll
          for (int q = 0; q < kPer; ++q) cs[e * kPer + q] = to_f32(x[q]);
        }
      }
    }
  }
  __syncthreads();

  float acc[TT];
#pragma unroll
  for (int t = 0; t < TT; ++t) acc[t] = 0.f;
  for (int kb = k0;; ) {
    const int nk = min(kBatch, k1 - kb);
    if (nk == kBatch && (kb & 3) == 0 && (a.r & 3) == 0) {
      // 16-byte token reads: four FMAs per shared-memory load
#pragma unroll
      for (int t = 0; t < TT; ++t) {
        const float4* crow = reinterpret_cast<const float4*>(cs + t * a.r + kb);
#pragma unroll
        for (int u4 = 0; u4 < kBatch / 4; ++u4) {
          const float4 cv = crow[u4];
          acc[t] = fmaf(cv.x, wv[4 * u4 + 0], acc[t]);
          acc[t] = fmaf(cv.y, wv[4 * u4 + 1], acc[t]);
          acc[t] = fmaf(cv.z, wv[4 * u4 + 2], acc[t]);
          acc[t] = fmaf(cv.w, wv[4 * u4 + 3], acc[t]);
        }
      }
    } else {
#pragma unroll
      for (int t = 0; t < TT; ++t) {
        const float* crow = cs + t * a.r + kb;
#pragma unroll
        for (int u = 0; u < kBatch; ++u)
          if (u < nk) acc[t] = fmaf(crow[u], wv[u], acc[t]);
      }
    }
    kb += kBatch;
    if (kb >= k1) break;
#pragma unroll
    for (int u = 0; u < kBatch; ++u) wv[u] = (kb + u < k1) ? w[(int64_t)(kb + u) * width] : 0.f;
  }
#pragma unroll
  for (int t = 0; t < TT; ++t) zp[(slice * TT + t) * kRmsCols + col] = acc[t];
  __syncthreads();
  // thread (slice, col) finishes tokens slice, slice + 16, ...: z summed over slices, squared,
  // then summed over the 16 columns of its half-warp
  for (int t = slice; t < TT; t += kRmsSlices) {
    float z = 0.f;
#pragma unroll
    for (int sl = 0; sl < kRmsSlices; ++sl) z += zp[(sl * TT + t) * kRmsCols + col];
    float v = (n < width) ? z * z : 0.f;
#pragma unroll
    for (int o = kRmsCols / 2; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (col == 0 && t < ntok) {
      const int64_t i = (int64_t)a.slot[t0 + t] * a.groups + g;
      if constexpr (FUSED) {
        float* acc = reinterpret_cast<float*>(a.ak_scratch + 2 * i);
        unsigned int* cnt = a.ak_scratch + 2 * i + 1;
        atomicAdd(acc, v);
        __threadfence();
        if (atomicAdd(cnt, 1u) == (unsigned int)(nblk - 1)) {
          __threadfence();
          const float total = atomicExch(acc, 0.f);
          a.a_k[i] = 1.0f / sqrtf(total / (float)width + a.eps);
          atomicExch(cnt, 0u);
        }
      } else {
        atomicAdd(a.a_k + i, v);
      }
    }
  }
}

__global__ void append_finalize_kernel(AppendArgs a) {
  pdl_trigger();
  pdl_wait();
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= a.n_tok * a.groups) return;
  const int t = i / a.groups, g = i - t * a.groups;
  float* p = a.a_k + (int64_t)a.slot[t] * a.groups + g;
  *p = 1.0f / sqrtf(*p / (float)a.width + a.eps);
}

template <typename T, int TT, bool FUSED>
static cudaError_t launch_keyrms(const AppendArgs& a, cudaStream_t st) {
  const size_t smem = ((size_t)TT * a.r + (size_t)kRmsSlices * TT * kRmsCols) * sizeof(float);
  static bool attr_set = false;   // one attribute per instantiation
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(append_keyrms_kernel<T, TT, FUSED>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  const int nblk = (a.width + kRmsCols - 1) / kRmsCols;
  dim3 grid(nblk + (FUSED ? 1 : 0), (a.n_tok + TT - 1) / TT, a.groups);
  return launch_chained(append_keyrms_kernel<T, TT, FUSED>, grid, dim3(kRmsCols * kRmsSlices), smem, st, a);
}

template <typename T>
static cudaError_t launch_append_t(const AppendArgs& a, cudaStream_t st) {
  // few tokens (a decode step): small token tiles spread over many CTAs;
  // many tokens (filling a cache): larger tiles re-read W less often
  if (a.ak_scratch)
    return a.n_tok <= 256 ? launch_keyrms<T, 16, true>(a, st) : launch_keyrms<T, 32, true>(a, st);
  cudaError_t e0 = launch_chained(append_copy_kernel<T>, dim3((a.n_tok + 7) / 8), dim3(256), 0, st, a);
  if (e0 != cudaSuccess) return e0;
  cudaError_t e = a.n_tok <= 256 ? launch_keyrms<T, 16, false>(a, st) : launch_keyrms<T, 32, false>(a, st);
  if (e != cudaSuccess) return e;
  return launch_chained(append_finalize_kernel, dim3((a.n_tok * a.groups + 255) / 256), dim3(256), 0, st, a);
}

cudaError_t launch_append(const AppendArgs& a, bool bf16, cudaStream_t st) {
  return bf16 ? launch_append_t<__nv_bfloat16>(a, st) : launch_append_t<float>(a, st);
}

}  // namespace qkn
