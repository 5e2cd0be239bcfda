// Split-KV combine: merge the per-split partial results of one decode step.
// Each split s of a query row carries a normalised partial output o_s and its
// log-sum-exp lse_s; the row's result is
//   lse = log sum_s exp(lse_s),   o = sum_s exp(lse_s - lse) * o_s,
// which is exactly the softmax over the union of the splits' tokens.
// One CTA per query row: warp 0 turns the row's split lse values into weights
// (shared memory), then every thread owns 16 bytes of the row and streams the
// splits' partials for them with independent loads.
#include "common.cuh"
#include "kernels.h"

namespace qkn {

constexpr int kCombThreads = 128;

template <typename T>
__device__ __forceinline__ void store4(T* dst, float4 v);
template <>
__device__ __forceinline__ void store4<float>(float* dst, float4 v) {
  *reinterpret_cast<float4*>(dst) = v;
}
template <>
__device__ __forceinline__ void store4<__nv_bfloat16>(__nv_bfloat16* dst, float4 v) {
  __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y), b = __floats2bfloat162_rn(v.z, v.w);
  uint2 u;
  u.x = *reinterpret_cast<uint32_t*>(&a);
  u.y = *reinterpret_cast<uint32_t*>(&b);
  *reinterpret_cast<uint2*>(dst) = u;
}

template <typename T>
__global__ void __launch_bounds__(kCombThreads) combine_kernel(CombineArgs a) {
  extern __shared__ float wsm[];                          // [max_items] split weights
  __shared__ int64_t first_s;
  __shared__ int nitems_s;
  __shared__ float lse_s;
  pdl_trigger();
  pdl_wait();
  const int grow = blockIdx.x;                            // (segment, row)
  const int seg = grow / a.rows, row = grow - seg * a.rows;
  const int b = seg / a.ht_count, ht = seg - b * a.ht_count;
  const int qrows = a.s_q * a.heads;
  const int rho = ht * a.rows + row;
  if (b >= a.batch || rho >= qrows) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (a.seg_desc) {
    // a sequence with a rejected length has no splits: the tcgen05 kernel wrote its rows itself
    const int2 d = a.seg_desc[seg];
    if (d.y <= 0) return;
  }
  if (warp == 0) {
    int64_t first;
    int nitems;
    if (a.seg_desc) {
      const int2 d = a.seg_desc[seg];
      first = (int64_t)d.x * a.rows + row;
      nitems = d.y;
    } else {
      SchedParams sp{a.seq_lens, a.batch, a.s_q, a.max_blocks, a.ht_count, a.ncta};
      const int64_t total = sched_total_units(sp);
      const int64_t before = sched_pages_before(sp, b);
      const int32_t n = pages_of(a.seq_lens[b], sp);
      if (n == 0 && ht == 0 && row == 0 && lane == 0) record_status(a.status, QKN_ERR_BOUNDS);
      const int64_t q = total > 0 ? (total + a.ncta - 1) / a.ncta : 1;
      const int64_t u0 = before * a.ht_count + (int64_t)ht * n;
      const int64_t c0 = u0 / q;
      nitems = n > 0 ? (int)((u0 + n - 1) / q - c0 + 1) : 0;
      first = (int64_t)(seg + c0) * a.rows + row;   // partial row of the first split
    }
    float mx = -INFINITY;
    for (int c = lane; c < nitems; c += 32) mx = fmaxf(mx, a.part_lse[first + (int64_t)c * a.rows]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    float den = 0.f;
    for (int c = lane; c < nitems; c += 32) {
      const float ls = a.part_lse[first + (int64_t)c * a.rows];
      const float e = (mx == -INFINITY) ? 0.f : __expf(ls - mx);
      wsm[c] = e;
      den += e;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
    const float inv = den > 0.f ? 1.f / den : 0.f;
    __syncwarp();
    for (int c = lane; c < nitems; c += 32) wsm[c] *= inv;
    if (lane == 0) {
      first_s = first;
      nitems_s = nitems;
      lse_s = (mx == -INFINITY) ? -INFINITY : mx + logf(den);
    }
  }
  __syncthreads();
  const int nitems = nitems_s;
  const int64_t orow = (int64_t)b * qrows + rho;
  T* out = static_cast<T*>(a.out) + orow * a.r;
  const int nvec = a.r / 4;
  const int64_t stride = (int64_t)a.rows * a.r / 4;        // float4s between consecutive splits of this row
  for (int v = threadIdx.x; v < nvec; v += kCombThreads) {
    const float4* src = reinterpret_cast<const float4*>(a.part_o + first_s * a.r) + v;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    int c = 0;
    for (; c + 8 <= nitems; c += 8) {
      float4 x[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) x[u] = src[(int64_t)(c + u) * stride];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const float w = wsm[c + u];
        acc.x = fmaf(w, x[u].x, acc.x);
        acc.y = fmaf(w, x[u].y, acc.y);
        acc.z = fmaf(w, x[u].z, acc.z);
        acc.w = fmaf(w, x[u].w, acc.w);
      }
    }
    for (; c < nitems; ++c) {
      const float4 x = src[(int64_t)c * stride];
      const float w = wsm[c];
      acc.x = fmaf(w, x.x, acc.x);
      acc.y = fmaf(w, x.y, acc.y);
      acc.z = fmaf(w, x.z, acc.z);
      acc.w = fmaf(w, x.w, acc.w);
    }
    store4<T>(out + v * 4, acc);
  }
  if (threadIdx.x == 0) a.lse[orow] = lse_s;
}

cudaError_t launch_combine(const CombineArgs& a, bool bf16, cudaStream_t st) {
  const int64_t rows = (int64_t)a.batch * a.ht_count * a.rows;
  const size_t smem = (size_t)a.max_items * sizeof(float);
  if (bf16) return launch_chained(combine_kernel<__nv_bfloat16>, dim3((unsigned)rows), dim3(kCombThreads), smem, st, a);
  return launch_chained(combine_kernel<float>, dim3((unsigned)rows), dim3(kCombThreads), smem, st, a);
}

}  // namespace qkn
