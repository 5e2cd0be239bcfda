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
//
// Many tokens at once (more than 256: a prefill chunk, a cache fill) take the
// key statistic as a register-blocked fp32 GEMM instead (keystat_gemm_kernel):
// CTA tiles of 64 tokens x 64 matrix columns over K = r in steps of 32, each
// thread 4 tokens x 4 columns, the next K step's tiles loaded into registers
// while the current one is multiplied; the column-block sums meet in the
// same accumulators (and, with ak_scratch, the same arrival count) as above.
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
  if (slot < 0 || slot >= a.n_slots) return;       // outside the pool: the token is skipped
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
  const int64_t slot = a.slot[t];
  if (slot < 0 || slot >= a.n_slots) return;
  float* p = a.a_k + slot * a.groups + g;
  *p = 1.0f / sqrtf(*p / (float)a.width + a.eps);
}

// ---------------------------------------------------------------- key statistic as a GEMM
constexpr int kGM = 64, kGN = 64, kGK = 32;   // tokens, matrix columns, K step per CTA tile
constexpr int kGThreads = 256;                // 16 x 16 threads, 4 x 4 outputs each

// CTA (column block bx, token tile by, group bz); FUSED: block bx == number of column blocks copies
// the tile's latents and RoPE keys.
template <typename T, bool FUSED>
__global__ void __launch_bounds__(kGThreads) keystat_gemm_kernel(const __grid_constant__ AppendArgs a) {
  __shared__ __align__(16) float As[2][kGK][kGM];   // c^T tile: [k][token]
  __shared__ __align__(16) float Bs[2][kGK][kGN];   // matrix tile: [k][column]
  __shared__ float rows[kGThreads / 32][128];
  pdl_wait();
  pdl_trigger();
  const int g = blockIdx.z, t0 = blockIdx.y * kGM, n0 = blockIdx.x * kGN;
  const int ncols = a.ncols;
  const int nblk = (ncols + kGN - 1) / kGN;
  const int ntok = min(kGM, a.n_tok - t0);
  if (FUSED && (int)blockIdx.x == nblk) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (g == 0)
      for (int i = warp; i < ntok; i += kGThreads / 32) append_token<T>(a, t0 + i, lane, rows[warp]);
    return;
  }
  const bool gram = a.key_gram != nullptr;
  const float* M = (gram ? a.key_gram : a.w_k) + (int64_t)g * a.r * ncols;
  const T* C = static_cast<const T*>(a.c_new);
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  // loads of one K step, 16 or 32 contiguous bytes per thread: the c tile (64 tokens x 32 k: thread
  // -> token threadIdx / 4, k values 8 (threadIdx % 4) ..) and the matrix tile (32 k x 64 columns:
  // thread -> k row threadIdx / 8, columns 8 (threadIdx % 8) ..)
  const int la_t = threadIdx.x >> 2, la_k = (threadIdx.x & 3) * 8;
  const int lb_k = threadIdx.x >> 3, lb_n = (threadIdx.x & 7) * 8;
  const bool vec_b = (ncols & 3) == 0;
  float ra[8], rb[8];
  auto load = [&](int k0) {
    const int ka = k0 + la_k;
    const T* crow = C + (int64_t)(t0 + la_t) * a.r + ka;
    if (la_t < ntok && ka + 8 <= a.r) {
      if constexpr (sizeof(T) == 2) {
        const uint4 v = *reinterpret_cast<const uint4*>(crow);         // rows are 16-byte multiples
        const T* x = reinterpret_cast<const T*>(&v);
#pragma unroll
        for (int u = 0; u < 8; ++u) ra[u] = to_f32(x[u]);
      } else {
        const float4 v0 = *reinterpret_cast<const float4*>(crow), v1 = *reinterpret_cast<const float4*>(crow + 4);
        ra[0] = v0.x; ra[1] = v0.y; ra[2] = v0.z; ra[3] = v0.w; ra[4] = v1.x; ra[5] = v1.y; ra[6] = v1.z; ra[7] = v1.w;
      }
    } else {
#pragma unroll
      for (int u = 0; u < 8; ++u) ra[u] = (la_t < ntok && ka + u < a.r) ? to_f32(crow[u]) : 0.f;
    }
    const int kb = k0 + lb_k, nb = n0 + lb_n;
    const float* mrow = M + (int64_t)kb * ncols + nb;
    if (kb < a.r && nb + 8 <= ncols && vec_b) {
      const float4 v0 = *reinterpret_cast<const float4*>(mrow), v1 = *reinterpret_cast<const float4*>(mrow + 4);
      rb[0] = v0.x; rb[1] = v0.y; rb[2] = v0.z; rb[3] = v0.w; rb[4] = v1.x; rb[5] = v1.y; rb[6] = v1.z; rb[7] = v1.w;
    } else {
#pragma unroll
      for (int u = 0; u < 8; ++u) rb[u] = (kb < a.r && nb + u < ncols) ? mrow[u] : 0.f;
    }
  };
  auto store = [&](int buf) {
#pragma unroll
    for (int u = 0; u < 8; ++u) As[buf][la_k + u][la_t] = ra[u];
    *reinterpret_cast<float4*>(&Bs[buf][lb_k][lb_n]) = make_float4(rb[0], rb[1], rb[2], rb[3]);
    *reinterpret_cast<float4*>(&Bs[buf][lb_k][lb_n + 4]) = make_float4(rb[4], rb[5], rb[6], rb[7]);
  };
  float acc[4][4] = {};
  load(0);
  store(0);
  __syncthreads();
  const int nk = (a.r + kGK - 1) / kGK;
  for (int ks = 0; ks < nk; ++ks) {
    const int buf = ks & 1;
    if (ks + 1 < nk) load((ks + 1) * kGK);          // in flight while this step multiplies
#pragma unroll
    for (int k = 0; k < kGK; ++k) {
      const float4 av = *reinterpret_cast<const float4*>(&As[buf][k][ty * 4]);
      const float4 bv = *reinterpret_cast<const float4*>(&Bs[buf][k][tx * 4]);
      const float am[4] = {av.x, av.y, av.z, av.w}, bm[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(am[i], bm[j], acc[i][j]);
    }
    if (ks + 1 < nk) store(buf ^ 1);                 // the other buffer was last read a step ago
    __syncthreads();
  }
  // each token's term over this block's columns: z^2 (direct form) or z c_n (Gram form), summed over
  // the 16 threads that hold the token's columns (tx, lanes of one half-warp)
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int t = ty * 4 + i;
    float v = 0.f;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx * 4 + j;
      if (t < ntok && n < ncols) v += acc[i][j] * (gram ? to_f32(C[(int64_t)(t0 + t) * a.r + n]) : acc[i][j]);
    }
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    const int64_t s_t = t < ntok ? (int64_t)a.slot[t0 + t] : -1;
    if (tx == 0 && t < ntok && s_t >= 0 && s_t < a.n_slots) {
      const int64_t idx = s_t * a.groups + g;
      if constexpr (FUSED) {
        float* accp = reinterpret_cast<float*>(a.ak_scratch + 2 * idx);
        unsigned int* cnt = a.ak_scratch + 2 * idx + 1;
        atomicAdd(accp, v);
        __threadfence();
        if (atomicAdd(cnt, 1u) == (unsigned int)(nblk - 1)) {
          __threadfence();
          const float total = atomicExch(accp, 0.f);
          a.a_k[idx] = 1.0f / sqrtf(total / (float)a.width + a.eps);
          atomicExch(cnt, 0u);
        }
      } else {
        atomicAdd(a.a_k + idx, v);
      }
    }
  }
}

template <typename T, bool FUSED>
static cudaError_t launch_keystat_gemm(const AppendArgs& a, cudaStream_t st) {
  const int nblk = (a.ncols + kGN - 1) / kGN;
  const dim3 grid(nblk + (FUSED ? 1 : 0), (a.n_tok + kGM - 1) / kGM, a.groups);
  return launch_chained(keystat_gemm_kernel<T, FUSED>, grid, dim3(kGThreads), 0, st, a);
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
    return a.n_tok <= 256 ? launch_keyrms<T, 16, true>(a, st) : launch_keystat_gemm<T, true>(a, st);
  cudaError_t e0 = launch_chained(append_copy_kernel<T>, dim3((a.n_tok + 7) / 8), dim3(256), 0, st, a);
  if (e0 != cudaSuccess) return e0;
  cudaError_t e = a.n_tok <= 256 ? launch_keyrms<T, 16, false>(a, st) : launch_keystat_gemm<T, false>(a, st);
  if (e != cudaSuccess) return e;
  return launch_chained(append_finalize_kernel, dim3((a.n_tok * a.groups + 255) / 256), dim3(256), 0, st, a);
}

cudaError_t launch_append(const AppendArgs& a, bool bf16, cudaStream_t st) {
  return bf16 ? launch_append_t<__nv_bfloat16>(a, st) : launch_append_t<float>(a, st);
}

}  // namespace qkn
