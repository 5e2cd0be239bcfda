// Split-KV combine: merge the per-split partial results of one decode step.
// Each split s of a query row carries a normalised partial output o_s and its
// log-sum-exp lse_s; the row's result is
//   lse = log sum_s exp(lse_s),   o = sum_s exp(lse_s - lse) * o_s,
// which is exactly the softmax over the union of the splits' tokens.
// One CTA per query row.  Every thread owns 16 bytes of the row and merges
// the splits for them on its own: it loads the splits' lse values together
// with its 16 bytes of their partials, four splits at a time, and keeps a
// running maximum.  After the segment descriptor, one round of memory latency
// per four splits; no shared memory and no barrier (few registers, so that
// many rows are in flight at once).
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

// kDesc: the splits come from the segment descriptors the tcgen05 decode wrote; else from the
// schedule, recomputed (one instantiation each keeps the descriptor path small)
template <typename T, bool kDesc>
__global__ void __launch_bounds__(kCombThreads, kDesc ? 12 : 8) combine_kernel(CombineArgs a) {
  __shared__ int64_t first_s;
  __shared__ int nitems_s;
  pdl_trigger();
  pdl_wait();
  const int grow = blockIdx.x;                            // (segment, row)
  const int seg = grow / a.rows, row = grow - seg * a.rows;
  const int b = seg / a.ht_count, ht = seg - b * a.ht_count;
  const int qrows = a.s_q * a.heads;
  const int rho = ht * a.rows + row;
  if (b >= a.batch || rho >= qrows) return;
  // the row's splits: from the segment descriptor the tcgen05 decode wrote, else from the
  // schedule, recomputed by warp 0
  int64_t first;
  int nitems;
  if constexpr (kDesc) {
    const int2 d = a.seg_desc[seg];
    // a sequence with a rejected length has no splits: the tcgen05 kernel wrote its rows itself
    if (d.y <= 0) return;
    // A decode that stopped early (a bounded wait ran out) leaves some descriptors unwritten, i.e.
    // holding a previous call's values or nothing meaningful.  Every descriptor is checked against
    // this launch's slots before a partial is read; a bad one gives zero rows, lse = -inf.
    if (d.x < 0 || d.y > a.max_items || (int64_t)d.x + (int64_t)(d.y - 1) * a.ht_count >= a.nslots) {
      if (threadIdx.x == 0) record_status(a.status, QKN_ERR_BOUNDS);
      const int64_t orow = (int64_t)b * qrows + rho;
      T* out = static_cast<T*>(a.out) + orow * a.r;
      for (int v = threadIdx.x; v < a.r / 4; v += kCombThreads) store4<T>(out + v * 4, make_float4(0.f, 0.f, 0.f, 0.f));
      if (threadIdx.x == 0) a.lse[orow] = -INFINITY;
      return;
    }
    first = (int64_t)d.x * a.rows + row;
    nitems = d.y;
  } else {
    if (threadIdx.x < 32) {
      const int lane = threadIdx.x;
      SchedParams sp{a.seq_lens, a.batch, a.s_q, a.max_blocks, a.ht_count, a.ncta, a.item_cost};
      const int64_t total = sched_total_units(sp);
      const int32_t n = pages_of(a.seq_lens[b], sp);
      if (n == 0 && ht == 0 && row == 0 && lane == 0) record_status(a.status, QKN_ERR_BOUNDS);
      const int32_t ng = sched_groups(sp);
      const int64_t q = total > 0 ? (total + ng - 1) / ng : 1;
      const SegSplit sg = seg_split(sched_units_before(sp, b), n, q, sp.item_cost);
      if (lane == 0) {
        nitems_s = n > 0 ? sg.nitems : 0;
        first_s = ((int64_t)(b + sg.c0) * a.ht_count + ht) * a.rows + row;   // partial row of the first split
      }
    }
    __syncthreads();
    first = first_s;
    nitems = nitems_s;
  }
  // Every thread owns 16 bytes of the row and merges the splits on its own, with a running
  // maximum of their lse values: acc = sum_s exp(lse_s - m) o_s, den = sum_s exp(lse_s - m).
  // The lse values and the partials of kDepth splits are loaded together.
  constexpr int kDepth = 4;
  const int nvec = a.r / 4;
  // consecutive splits of a segment sit ht_count slots apart
  const int64_t lstride = (int64_t)a.rows * a.ht_count;
  const int64_t stride = lstride * a.r / 4;                 // float4s between consecutive splits of this row
  const float4* src0 = reinterpret_cast<const float4*>(a.part_o + first * a.r);
  const float* lsrc = a.part_lse + first;
  const int64_t orow = (int64_t)b * qrows + rho;
  T* out = static_cast<T*>(a.out) + orow * a.r;
  for (int v = threadIdx.x; v < nvec; v += kCombThreads) {
    float m = -INFINITY, den = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int c = 0; c < nitems; c += kDepth) {
      float ls[kDepth];
      float4 x[kDepth];
#pragma unroll
      for (int u = 0; u < kDepth; ++u) {
        const bool in = c + u < nitems;
        ls[u] = in ? lsrc[(int64_t)(c + u) * lstride] : -INFINITY;
        x[u] = in ? src0[(int64_t)(c + u) * stride + v] : make_float4(0.f, 0.f, 0.f, 0.f);
      }
      float mc = m;
#pragma unroll
      for (int u = 0; u < kDepth; ++u) mc = fmaxf(mc, ls[u]);
      if (mc == -INFINITY) continue;                    // nothing visible so far
      const float sc = __expf(m - mc);                  // m == -inf gives 0
      acc.x *= sc; acc.y *= sc; acc.z *= sc; acc.w *= sc;
      den *= sc;
#pragma unroll
      for (int u = 0; u < kDepth; ++u) {
        const float w = __expf(ls[u] - mc);             // ls == -inf gives 0
        den += w;
        acc.x = fmaf(w, x[u].x, acc.x);
        acc.y = fmaf(w, x[u].y, acc.y);
        acc.z = fmaf(w, x[u].z, acc.z);
        acc.w = fmaf(w, x[u].w, acc.w);
      }
      m = mc;
    }
    const float inv = den > 0.f ? 1.f / den : 0.f;
    store4<T>(out + v * 4, make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv));
    if (v == 0) a.lse[orow] = den > 0.f ? m + logf(den) : -INFINITY;
  }
}

cudaError_t launch_combine(const CombineArgs& a, bool bf16, cudaStream_t st) {
  const int64_t rows = (int64_t)a.batch * a.ht_count * a.rows;
  const size_t smem = 0;
  const dim3 grid((unsigned)rows), block(kCombThreads);
  if (a.seg_desc)
    return bf16 ? launch_chained(combine_kernel<__nv_bfloat16, true>, grid, block, smem, st, a)
                : launch_chained(combine_kernel<float, true>, grid, block, smem, st, a);
  return bf16 ? launch_chained(combine_kernel<__nv_bfloat16, false>, grid, block, smem, st, a)
              : launch_chained(combine_kernel<float, false>, grid, block, smem, st, a);
}

}  // namespace qkn
