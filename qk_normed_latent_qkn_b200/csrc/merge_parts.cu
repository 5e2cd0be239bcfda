// Merge of normalised partial attention outputs of the same query rows: the
// exchange end of a context-parallel decode, where each rank decodes a slice
// of every sequence's pages and the ranks' (o_p, lse_p) meet after an
// all-gather.  For every row
//   lse = log sum_p exp(lse_p),   o = sum_p exp(lse_p - lse) o_p,
// which is the softmax over the union of the slices' tokens (the same
// identity as the split-KV merge).  A part with lse_p = -inf (no visible
// token) contributes nothing; a row with no visible token in any part comes
// out as zeros with lse = -inf.  One CTA per four rows; every thread owns 16
// bytes of a row and merges them over the parts in one pass with a running
// maximum, loading four parts at a time.
#include "common.cuh"
#include "kernels.h"

namespace qkn {

namespace {

constexpr int kMergeRows = 4;
constexpr int kMergeThreads = 128;

template <typename T>
__device__ __forceinline__ float4 load4(const T* p);
template <>
__device__ __forceinline__ float4 load4<float>(const float* p) {
  return *reinterpret_cast<const float4*>(p);
}
template <>
__device__ __forceinline__ float4 load4<__nv_bfloat16>(const __nv_bfloat16* p) {
  const uint2 u = *reinterpret_cast<const uint2*>(p);
  const __nv_bfloat162 lo = *reinterpret_cast<const __nv_bfloat162*>(&u.x);
  const __nv_bfloat162 hi = *reinterpret_cast<const __nv_bfloat162*>(&u.y);
  const float2 a = __bfloat1622float2(lo), b = __bfloat1622float2(hi);
  return make_float4(a.x, a.y, b.x, b.y);
}
template <typename T>
__device__ __forceinline__ void store4(T* p, float4 v);
template <>
__device__ __forceinline__ void store4<float>(float* p, float4 v) {
  *reinterpret_cast<float4*>(p) = v;
}
template <>
__device__ __forceinline__ void store4<__nv_bfloat16>(__nv_bfloat16* p, float4 v) {
  __nv_bfloat162 lo = __floats2bfloat162_rn(v.x, v.y), hi = __floats2bfloat162_rn(v.z, v.w);
  uint2 u;
  u.x = *reinterpret_cast<uint32_t*>(&lo);
  u.y = *reinterpret_cast<uint32_t*>(&hi);
  *reinterpret_cast<uint2*>(p) = u;
}

template <typename T>
__global__ void __launch_bounds__(kMergeThreads) merge_parts_kernel(const T* parts, const float* lse_parts, int n_parts,
                                                                    int64_t rows, int r, T* out, float* lse) {
  pdl_trigger();
  pdl_wait();
  const int nvec = r / 4;                                  // 4-element pieces of a row
  for (int e = threadIdx.x; e < kMergeRows * nvec; e += kMergeThreads) {
    const int rr = e / nvec, v = e - rr * nvec;
    const int64_t row = (int64_t)blockIdx.x * kMergeRows + rr;
    if (row >= rows) break;
    float m = -INFINITY, den = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int p0 = 0; p0 < n_parts; p0 += 4) {
      float ls[4];
      float4 x[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const bool in = p0 + u < n_parts;
        ls[u] = in ? lse_parts[(int64_t)(p0 + u) * rows + row] : -INFINITY;
        x[u] = in ? load4<T>(parts + ((int64_t)(p0 + u) * rows + row) * r + v * 4) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
      float mc = m;
#pragma unroll
      for (int u = 0; u < 4; ++u) mc = fmaxf(mc, ls[u]);
      if (mc == -INFINITY) continue;                       // nothing visible so far
      const float sc = __expf(m - mc);                     // m == -inf gives 0
      acc.x *= sc; acc.y *= sc; acc.z *= sc; acc.w *= sc;
      den *= sc;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float w = __expf(ls[u] - mc);                // ls == -inf gives 0
        den += w;
        acc.x = fmaf(w, x[u].x, acc.x);
        acc.y = fmaf(w, x[u].y, acc.y);
        acc.z = fmaf(w, x[u].z, acc.z);
        acc.w = fmaf(w, x[u].w, acc.w);
      }
      m = mc;
    }
    const float inv = den > 0.f ? 1.f / den : 0.f;
    store4<T>(out + row * r + v * 4, make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv));
    if (v == 0) lse[row] = den > 0.f ? m + logf(den) : -INFINITY;
  }
}

}  // namespace

cudaError_t launch_merge_parts(const void* parts, const float* lse_parts, int n_parts, int64_t rows, int r,
                               void* out, float* lse, bool bf16, cudaStream_t st) {
  const dim3 grid((unsigned)((rows + kMergeRows - 1) / kMergeRows));
  if (bf16)
    return launch_chained(merge_parts_kernel<__nv_bfloat16>, grid, dim3(kMergeThreads), 0, st,
                          static_cast<const __nv_bfloat16*>(parts), lse_parts, n_parts, rows, r,
                          static_cast<__nv_bfloat16*>(out), lse);
  return launch_chained(merge_parts_kernel<float>, grid, dim3(kMergeThreads), 0, st, static_cast<const float*>(parts),
                        lse_parts, n_parts, rows, r, static_cast<float*>(out), lse);
}

}  // namespace qkn
