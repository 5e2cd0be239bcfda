// Split-KV combine: merge the per-split partial results of one decode step.
// Each split s of a query row carries a normalised partial output o_s and its
// log-sum-exp lse_s; the row's result is
//   lse = log sum_s exp(lse_s),   o = sum_s exp(lse_s - lse) * o_s,
// which is exactly the softmax over the union of the splits' tokens.
// One CTA per segment (sequence, query-row tile); one warp per query row,
// lanes striding over the latent dimension.
#include "common.cuh"
#include "kernels.h"

namespace qkn {

template <typename T>
__global__ void __launch_bounds__(256) combine_kernel(CombineArgs a) {
  __shared__ int64_t seg_u0_s, quota_s;
  __shared__ int32_t n_s;
  const int seg = blockIdx.x;
  const int b = seg / a.ht_count, ht = seg - b * a.ht_count;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp == 0) {
    SchedParams sp{a.seq_lens, a.batch, a.s_q, a.max_blocks, a.ht_count, a.ncta};
    const int64_t total = sched_total_units(sp);
    const int64_t before = sched_pages_before(sp, b);
    const int32_t n = pages_of(a.seq_lens[b], sp);
    if (lane == 0) {
      if (n == 0 && ht == 0) record_status(a.status, QKN_ERR_BOUNDS);
      quota_s = (total + a.ncta - 1) / a.ncta;
      n_s = n;
      seg_u0_s = before * a.ht_count + (int64_t)ht * n;
    }
  }
  __syncthreads();
  const int32_t n = n_s;
  const int64_t q = quota_s > 0 ? quota_s : 1;
  const int64_t c0 = seg_u0_s / q;
  const int64_t c1 = n > 0 ? (seg_u0_s + n - 1) / q : c0 - 1;
  const int qrows = a.s_q * a.heads;
  T* out = static_cast<T*>(a.out);
  for (int row = warp; row < a.rows; row += blockDim.x >> 5) {
    const int rho = ht * a.rows + row;
    if (rho >= qrows) break;
    const int64_t orow = (int64_t)b * qrows + rho;
    float mx = -INFINITY;
    for (int64_t c = c0; c <= c1; ++c) mx = fmaxf(mx, a.part_lse[(seg + c) * a.rows + row]);
    float den = 0.f;
    if (mx != -INFINITY)
      for (int64_t c = c0; c <= c1; ++c) den += __expf(a.part_lse[(seg + c) * a.rows + row] - mx);
    const float lse = (mx == -INFINITY) ? -INFINITY : mx + logf(den);
    for (int k = lane; k < a.r; k += 32) {
      float acc = 0.f;
      if (mx != -INFINITY)
        for (int64_t c = c0; c <= c1; ++c) {
          const float ls = a.part_lse[(seg + c) * a.rows + row];
          if (ls != -INFINITY)
            acc = fmaf(__expf(ls - lse), a.part_o[((seg + c) * a.rows + row) * a.r + k], acc);
        }
      out[orow * a.r + k] = from_f32<T>(acc);
    }
    if (lane == 0) a.lse[orow] = lse;
  }
}

cudaError_t launch_combine(const CombineArgs& a, bool bf16, cudaStream_t st) {
  const int segs = a.batch * a.ht_count;
  if (bf16)
    combine_kernel<__nv_bfloat16><<<segs, 256, 0, st>>>(a);
  else
    combine_kernel<float><<<segs, 256, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace qkn
