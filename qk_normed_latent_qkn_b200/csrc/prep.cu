// qkn_append_absorb: a decode step's cache append and query absorption in
// one launch.  The two are independent ("QK-Normed MLA: QK normalization
// without full key caching", technical summary, Metodología items 1-4: the
// key statistic is computed at append time, the norm weights are folded into
// the query), so one grid hosts CTAs of both kinds: first the append CTAs of
// the one-launch append (key-statistic column blocks plus the copy column),
// then the absorption CTAs.  A step then needs no fork and join of two
// streams, and the decode that follows chains onto one kernel.
#include "prep_blocks.cuh"

namespace qkn {

namespace {

constexpr int kPrepThreads = kRmsCols * kRmsSlices;     // 512
constexpr int kPrepTT = 16;                             // append token tile

struct PrepArgs {
  AppendArgs ap;
  AbsorbArgs ab;
  int32_t append_x, append_y, append_ctas;              // append grid (x, y, groups), flattened
  int32_t absorb_y;                                     // absorption grid (H, absorb_y), flattened after it
};

template <typename T>
__global__ void __launch_bounds__(kPrepThreads, 2) prep_kernel(const __grid_constant__ PrepArgs p) {
  extern __shared__ float4 smem4[];
  float* smem = reinterpret_cast<float*>(smem4);
  // dependents may launch only once everything before this kernel is complete: a decode that
  // streams old cache pages before its own wait (step_writes_only) relies on it
  pdl_wait();
  pdl_trigger();
  int bid = blockIdx.x;
  if (bid < p.append_ctas) {
    const int x = bid % p.append_x;
    bid /= p.append_x;
    keyrms_block<T, kPrepTT, true>(p.ap, x, bid % p.append_y, bid / p.append_y, smem);
  } else {
    bid -= p.append_ctas;
    absorb_block<T, kPrepThreads / 32>(p.ab, bid / p.absorb_y, bid % p.absorb_y, smem);
  }
}

}  // namespace

bool prep_fusable(const AppendArgs& ap, const AbsorbArgs& ab) {
  return ap.ak_scratch != nullptr && ap.n_tok <= 256 && ap.n_tok > 0 && ab.n_q > 0;
}

cudaError_t launch_prep(const AppendArgs& ap, const AbsorbArgs& ab, bool bf16, cudaStream_t st) {
  PrepArgs p;
  p.ap = ap;
  p.ab = ab;
  p.append_x = (ap.ncols + kRmsCols - 1) / kRmsCols + 1;
  p.append_y = (ap.n_tok + kPrepTT - 1) / kPrepTT;
  p.append_ctas = p.append_x * p.append_y * ap.groups;
  constexpr int kAbsRows = absorb_rows<kPrepThreads / 32>();
  p.absorb_y = (ab.r + kAbsRows - 1) / kAbsRows + 1;
  const int64_t ctas = (int64_t)p.append_ctas + (int64_t)ab.heads * p.absorb_y;
  const size_t smem_append = ((size_t)kPrepTT * ap.r + (size_t)kRmsSlices * kPrepTT * kRmsCols) * sizeof(float);
  const size_t smem_absorb = absorb_smem_bytes(kAbsRows, ab.d_h);
  const size_t smem = smem_append > smem_absorb ? smem_append : smem_absorb;
  auto kernel = bf16 ? prep_kernel<__nv_bfloat16> : prep_kernel<float>;
  static PerDeviceOnce attrs[2];
  cudaError_t e = once_per_device(attrs[bf16 ? 1 : 0], [&] { return set_smem_attrs(kernel, 200 * 1024); });
  if (e != cudaSuccess) return e;
  return launch_chained(kernel, dim3((unsigned)ctas), dim3(kPrepThreads), smem, st, p);
}

}  // namespace qkn
