// Split-KV combine: merge the per-split partial results of one decode step.
// Each split s of a query row carries a normalised partial output o_s and its
// log-sum-exp lse_s; the row's result is
//   lse = log sum_s exp(lse_s),   o = sum_s exp(lse_s - lse) * o_s,
// which is exactly the softmax over the union of the splits' tokens.
// One CTA per query row.  Every thread owns 16 bytes of the row and loads
// them from the first eight splits while warp 0 turns the splits' lse values
// into weights (shared memory); then the threads combine, streaming any
// further splits eight at a time.
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
  // the row's splits: from the segment descriptor the tcgen05 decode wrote (every thread reads it,
  // so that the partials' loads go out at once), else from the schedule, recomputed by warp 0
  int64_t first;
  int nitems;
  if (a.seg_desc) {
    const int2 d = a.seg_desc[seg];
    // a sequence with a rejected length has no splits: the tcgen05 kernel wrote its rows itself
    if (d.y <= 0) return;
    first = (int64_t)d.x * a.rows + row;
    nitems = d.y;
  } else {
    if (warp == 0) {
      SchedParams sp{a.seq_lens, a.batch, a.s_q, a.max_blocks, a.ht_count, a.ncta, a.item_cost};
      const int64_t total = sched_total_units(sp);
      const int32_t n = pages_of(a.seq_lens[b], sp);
      if (n == 0 && ht == 0 && row == 0 && lane == 0) record_status(a.status, QKN_ERR_BOUNDS);
      const int64_t q = total > 0 ? (total + a.ncta - 1) / a.ncta : 1;
      const int64_t u0 = sched_units_before(sp, b) + (int64_t)ht * seg_units(n, sp);
      const SegSplit sg = seg_split(u0, n, q, sp.item_cost);
      if (lane == 0) {
        nitems_s = n > 0 ? sg.nitems : 0;
        first_s = (int64_t)(seg + sg.c0) * a.rows + row;   // partial row of the first split
      }
    }
    __syncthreads();
    first = first_s;
    nitems = nitems_s;
  }
  // this thread's 16 bytes of the row from the first kHead splits, loaded beside the lse values
  constexpr int kHead = 8;
  const int nvec = a.r / 4;
  const int64_t stride = (int64_t)a.rows * a.r / 4;        // float4s between consecutive splits of this row
  const float4* src0 = reinterpret_cast<const float4*>(a.part_o + first * a.r);
  float4 head[kHead];
  const int v0 = threadIdx.x;
#pragma unroll
  for (int u = 0; u < kHead; ++u)
    head[u] = (u < nitems && v0 < nvec) ? src0[(int64_t)u * stride + v0] : make_float4(0.f, 0.f, 0.f, 0.f);
  if (warp == 0) {
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
    if (lane == 0) lse_s = (mx == -INFINITY) ? -INFINITY : mx + logf(den);
  }
  __syncthreads();
  const int64_t orow = (int64_t)b * qrows + rho;
  T* out = static_cast<T*>(a.out) + orow * a.r;
  for (int v = v0; v < nvec; v += kCombThreads) {
    const float4* src = src0 + v;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    int c = 0;
    if (v == v0) {
#pragma unroll
      for (int u = 0; u < kHead; ++u) {
        const float w = u < nitems ? wsm[u] : 0.f;
        acc.x = fmaf(w, head[u].x, acc.x);
        acc.y = fmaf(w, head[u].y, acc.y);
        acc.z = fmaf(w, head[u].z, acc.z);
        acc.w = fmaf(w, head[u].w, acc.w);
      }
      c = kHead;
    }
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
