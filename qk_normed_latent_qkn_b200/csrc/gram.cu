// qkn_key_gram: G_g = W^K_g (W^K_g)^T for every KV group, the r x r matrix
// with which the append computes the key statistic without forming the key:
// sum_n (c W^K_g)_n^2 = c G_g c^T ("QK-Normed MLA: QK normalization without
// full key caching", technical summary, Metodología items 2-4: the statistic
// is the RMS of the up-projected key c W^K_g over its n_g d_h columns).
// Computed once per weight set, accumulated in fp64 and stored in fp32.
#include "common.cuh"
#include "kernels.h"

namespace qkn {

namespace {

constexpr int kGT = 32;     // output tile (rows and columns)
constexpr int kGK = 32;     // columns of W per pass

// CTA (column tile, row tile, group), 256 threads: thread (ty, tx) accumulates
// G[i0 + ty + 16a][j0 + tx + 16b] for a, b in {0, 1}.
__global__ void __launch_bounds__(256) key_gram_kernel(const float* __restrict__ w_k, float* __restrict__ gram,
                                                       int r, int width) {
  __shared__ double wi[kGT][kGK + 1];
  __shared__ double wj[kGT][kGK + 1];
  const int g = blockIdx.z;
  const int i0 = blockIdx.y * kGT, j0 = blockIdx.x * kGT;
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  const float* w = w_k + (int64_t)g * r * width;
  double acc[2][2] = {{0.0, 0.0}, {0.0, 0.0}};
  for (int k0 = 0; k0 < width; k0 += kGK) {
    for (int e = threadIdx.x; e < kGT * kGK; e += blockDim.x) {
      const int row = e / kGK, k = e % kGK;
      const bool kin = k0 + k < width;
      wi[row][k] = (i0 + row < r && kin) ? (double)w[(int64_t)(i0 + row) * width + k0 + k] : 0.0;
      wj[row][k] = (j0 + row < r && kin) ? (double)w[(int64_t)(j0 + row) * width + k0 + k] : 0.0;
    }
    __syncthreads();
#pragma unroll 8
    for (int k = 0; k < kGK; ++k) {
      const double a0 = wi[ty][k], a1 = wi[ty + 16][k];
      const double b0 = wj[tx][k], b1 = wj[tx + 16][k];
      acc[0][0] = fma(a0, b0, acc[0][0]);
      acc[0][1] = fma(a0, b1, acc[0][1]);
      acc[1][0] = fma(a1, b0, acc[1][0]);
      acc[1][1] = fma(a1, b1, acc[1][1]);
    }
    __syncthreads();
  }
  float* out = gram + (int64_t)g * r * r;
#pragma unroll
  for (int a = 0; a < 2; ++a) {
#pragma unroll
    for (int b = 0; b < 2; ++b) {
      const int i = i0 + ty + 16 * a, j = j0 + tx + 16 * b;
      if (i < r && j < r) out[(int64_t)i * r + j] = (float)acc[a][b];
    }
  }
}

}  // namespace

cudaError_t launch_key_gram(const float* w_k, float* gram, int groups, int r, int width, cudaStream_t st) {
  const dim3 grid((r + kGT - 1) / kGT, (r + kGT - 1) / kGT, groups);
  key_gram_kernel<<<grid, 256, 0, st>>>(w_k, gram, r, width);
  return cudaGetLastError();
}

}  // namespace qkn
