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
//   2. append_keyrms:   z = c W^K_g (or c G_g with the Gram matrix) tiled
//                       over (16-column block, token tile, group); each CTA
//                       adds its columns' terms of sum(z^2) into the token's
//                       a_k slot;
//   3. append_finalize: a_k = 1 / sqrt(sum / (n_g d_h) + eps).
// The key z is only ever held in registers; it is never written anywhere.
#include "prep_blocks.cuh"

namespace qkn {

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

template <typename T, int TT, bool FUSED>
__global__ void __launch_bounds__(kRmsCols * kRmsSlices, 2) append_keyrms_kernel(AppendArgs a) {
  extern __shared__ float4 smem4[];
  // dependents may launch only once everything before this kernel is complete (see prep.cu)
  pdl_wait();
  pdl_trigger();
  __shared__ float rows[kRmsCols * kRmsSlices / 32][128];
  keyrms_block<T, TT, FUSED>(a, blockIdx.x, blockIdx.y, blockIdx.z, reinterpret_cast<float*>(smem4), rows);
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
  static PerDeviceOnce attrs;   // one per instantiation
  cudaError_t e =
      once_per_device(attrs, [] { return set_smem_attrs(append_keyrms_kernel<T, TT, FUSED>, 200 * 1024); });
  if (e != cudaSuccess) return e;
  const int nblk = (a.ncols + kRmsCols - 1) / kRmsCols;
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
