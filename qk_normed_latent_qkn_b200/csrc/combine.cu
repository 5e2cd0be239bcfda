// Split-KV combine: merge the per-split partial results of one decode step.
// Each split s of a query row carries a normalised partial output o_s and its
// log-sum-exp lse_s; the row's result is
//   lse = log sum_s exp(lse_s),   o = sum_s exp(lse_s - lse) * o_s,
// which is exactly the softmax over the union of the splits' tokens.
// One CTA per query row, or per four rows of a segment when there are many
// rows.  Every thread owns the same 16 bytes of each of its rows and merges the
// splits for them on its own: it loads the splits' lse values together with
// its 16 bytes of their partials (four splits at a time for one row, two for
// four rows) and keeps a running maximum per row.  After the segment
// descriptor, one round of memory latency per group of splits; no shared
// memory and no barrier.
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
// schedule, recomputed (one instantiation each keeps the descriptor path small).  RPC: query rows
// per CTA; every thread owns the same 16 bytes of each of them, and the rows' loads are issued
// together, so that a CTA keeps RPC times as many loads in flight and the grid fits in fewer waves.
// The RPC rows of a CTA lie in one segment (RPC divides the tile's row count).
// kGroup: the GQA route's row tiles, each holding one KV group's query rows (CombineArgs.group_heads);
// the RPC rows of a CTA then belong to one query token (RPC divides n_g), so that they are
// consecutive rows of the output as well.
template <typename T, bool kDesc, int RPC, bool kGroup = false>
__global__ void __launch_bounds__(kCombThreads) combine_kernel(CombineArgs a) {
  __shared__ int64_t first_s;
  __shared__ int nitems_s;
  pdl_trigger();
  pdl_wait();
  const int grow0 = blockIdx.x * RPC;                     // first (segment, row) of this CTA
  const int seg = grow0 / a.rows, row0 = grow0 - seg * a.rows;
  const int b = seg / a.ht_count, ht = seg - b * a.ht_count;
  const int qrows = a.s_q * a.heads;
  int rho0, nrows;                                        // first query row, rows of this CTA
  if constexpr (kGroup) {
    const int g = ht / a.tiles_per_group, rb = ht - g * a.tiles_per_group;
    const int u = rb * a.rows + row0;                     // u = j * n_g + m
    const int span = a.s_q * a.group_heads;
    if (b >= a.batch || u >= span) return;
    const int j = u / a.group_heads, m = u - j * a.group_heads;
    rho0 = j * a.heads + g * a.group_heads + m;
    nrows = min(RPC, span - u);
  } else {
    rho0 = ht * a.rows + row0;
    if (b >= a.batch || rho0 >= qrows) return;
    nrows = min(RPC, qrows - rho0);                       // rows of this CTA inside the sequence
  }
  const int64_t orow0 = (int64_t)b * qrows + rho0;
  const int nvec = a.r / 4;
  // the splits of the segment: from the descriptor the tcgen05 decode wrote, else from the
  // schedule, recomputed by warp 0.  first: partial row of row0 in the first split.
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
      for (int i = 0; i < nrows; ++i) {
        T* out = static_cast<T*>(a.out) + (orow0 + i) * a.r;
        for (int v = threadIdx.x; v < nvec; v += kCombThreads) store4<T>(out + v * 4, make_float4(0.f, 0.f, 0.f, 0.f));
        if (threadIdx.x == 0) a.lse[orow0 + i] = -INFINITY;
      }
      return;
    }
    first = (int64_t)d.x * a.rows + row0;
    nitems = d.y;
  } else {
    if (threadIdx.x < 32) {
      const int lane = threadIdx.x;
      SchedParams sp{a.seq_lens, a.batch, a.s_q, a.max_blocks, a.ht_count, a.ncta, a.item_cost};
      const int64_t total = sched_total_units(sp);
      const int32_t n = pages_of(a.seq_lens[b], sp);
      if (n == 0 && ht == 0 && row0 == 0 && lane == 0) record_status(a.status, QKN_ERR_BOUNDS);
      const int32_t ng = sched_groups(sp);
      const int64_t q = total > 0 ? (total + ng - 1) / ng : 1;
      const SegSplit sg = seg_split(sched_units_before(sp, b), n, q, sp.item_cost);
      if (lane == 0) {
        nitems_s = n > 0 ? sg.nitems : 0;
        first_s = ((int64_t)(b + sg.c0) * a.ht_count + ht) * a.rows + row0;
      }
    }
    __syncthreads();
    first = first_s;
    nitems = nitems_s;
  }
  // Every thread owns 16 bytes of each row and merges the splits for them on its own, with a
  // running maximum of their lse values: acc = sum_s exp(lse_s - m) o_s, den = sum_s exp(lse_s - m).
  // The lse values and the partials of kDepth splits of all the CTA's rows are loaded together.
  constexpr int kDepth = RPC == 1 ? 4 : 2;
  // consecutive splits of a segment sit ht_count slots apart
  const int64_t lstride = (int64_t)a.rows * a.ht_count;
  const int64_t stride = lstride * a.r / 4;                 // float4s between consecutive splits of a row
  const float4* src0 = reinterpret_cast<const float4*>(a.part_o + first * a.r);
  const float* lsrc = a.part_lse + first;
  for (int v = threadIdx.x; v < nvec; v += kCombThreads) {
    float m[RPC], den[RPC];
    float4 acc[RPC];
#pragma unroll
    for (int i = 0; i < RPC; ++i) {
      m[i] = -INFINITY;
      den[i] = 0.f;
      acc[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    for (int c = 0; c < nitems; c += kDepth) {
      float ls[RPC][kDepth];
      float4 x[RPC][kDepth];
#pragma unroll
      for (int u = 0; u < kDepth; ++u) {
#pragma unroll
        for (int i = 0; i < RPC; ++i) {
          const bool in = c + u < nitems && i < nrows;
          ls[i][u] = in ? lsrc[(int64_t)(c + u) * lstride + i] : -INFINITY;
          x[i][u] = in ? src0[(int64_t)(c + u) * stride + (int64_t)i * nvec + v] : make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
#pragma unroll
      for (int i = 0; i < RPC; ++i) {
        float mc = m[i];
#pragma unroll
        for (int u = 0; u < kDepth; ++u) mc = fmaxf(mc, ls[i][u]);
        if (mc == -INFINITY) continue;                  // nothing visible so far
        const float sc = __expf(m[i] - mc);             // m == -inf gives 0
        acc[i].x *= sc; acc[i].y *= sc; acc[i].z *= sc; acc[i].w *= sc;
        den[i] *= sc;
#pragma unroll
        for (int u = 0; u < kDepth; ++u) {
          const float w = __expf(ls[i][u] - mc);        // ls == -inf gives 0
          den[i] += w;
          acc[i].x = fmaf(w, x[i][u].x, acc[i].x);
          acc[i].y = fmaf(w, x[i][u].y, acc[i].y);
          acc[i].z = fmaf(w, x[i][u].z, acc[i].z);
          acc[i].w = fmaf(w, x[i][u].w, acc[i].w);
        }
        m[i] = mc;
      }
    }
#pragma unroll
    for (int i = 0; i < RPC; ++i) {
      if (i >= nrows) break;
      const float inv = den[i] > 0.f ? 1.f / den[i] : 0.f;
      T* out = static_cast<T*>(a.out) + (orow0 + i) * a.r;
      store4<T>(out + v * 4, make_float4(acc[i].x * inv, acc[i].y * inv, acc[i].z * inv, acc[i].w * inv));
      if (v == 0) a.lse[orow0 + i] = den[i] > 0.f ? m[i] + logf(den[i]) : -INFINITY;
    }
  }
}

cudaError_t launch_combine(const CombineArgs& a, bool bf16, cudaStream_t st) {
  // rows per CTA: four when one row per CTA would take more than about two waves of the GPU
  // (4,096 rows of 128 threads), one otherwise (more CTAs, four splits loaded at a time)
  const int64_t rows = (int64_t)a.batch * a.ht_count * a.rows;
  const size_t smem = 0;
  const dim3 block(kCombThreads);
  if (a.rows % 4 == 0 && rows >= 4096) {
    const dim3 grid((unsigned)(rows / 4));
    if (a.seg_desc)
      return bf16 ? launch_chained(combine_kernel<__nv_bfloat16, true, 4>, grid, block, smem, st, a)
                  : launch_chained(combine_kernel<float, true, 4>, grid, block, smem, st, a);
    return bf16 ? launch_chained(combine_kernel<__nv_bfloat16, false, 4>, grid, block, smem, st, a)
                : launch_chained(combine_kernel<float, false, 4>, grid, block, smem, st, a);
  }
  const dim3 grid((unsigned)rows);
  if (a.seg_desc)
    return bf16 ? launch_chained(combine_kernel<__nv_bfloat16, true, 1>, grid, block, smem, st, a)
                : launch_chained(combine_kernel<float, true, 1>, grid, block, smem, st, a);
  return bf16 ? launch_chained(combine_kernel<__nv_bfloat16, false, 1>, grid, block, smem, st, a)
              : launch_chained(combine_kernel<float, false, 1>, grid, block, smem, st, a);
}

cudaError_t launch_combine_grouped(const CombineArgs& a, cudaStream_t st) {
  // four rows per CTA when they never straddle two query tokens (n_g and the tile's rows multiples of 4)
  const int64_t rows = (int64_t)a.batch * a.ht_count * a.rows;
  const dim3 block(kCombThreads);
  if (a.rows % 4 == 0 && a.group_heads % 4 == 0 && rows >= 4096)
    return launch_chained(combine_kernel<__nv_bfloat16, false, 4, true>, dim3((unsigned)(rows / 4)), block, 0, st, a);
  return launch_chained(combine_kernel<__nv_bfloat16, false, 1, true>, dim3((unsigned)rows), block, 0, st, a);
}

}  // namespace qkn
