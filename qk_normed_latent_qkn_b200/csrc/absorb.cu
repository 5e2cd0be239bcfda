// qkn_absorb_query kernels: fold the static norm weights into the query
// ("QK-Normed MLA: QK normalization without full key caching", technical
// summary, Metodología item 1 and the decode-logit equation).
//
//   q~[i,h]  = W^K_{g,h} (gamma_q[h] * gamma_k[h] * q[i,h])        (absorb_qtilde)
//   a_q[i,h] = sigma / S(q[i,h])                                   (absorb_row)
//   q^R^[i,h] = sigma * RoPE_pos(gamma_qR[h] * q^R / S(q^R))        (absorb_row)
// One launch: one extra CTA per head does the per-row work beside the q~ CTAs.
#include "prep_blocks.cuh"

namespace qkn {

// grid (H, ceil(r / 64) + 1); block 256 (see absorb_block).
template <typename T>
__global__ void __launch_bounds__(256) absorb_qtilde_kernel(const __grid_constant__ AbsorbArgs a) {
  extern __shared__ float4 smem4[];
  pdl_trigger();
  pdl_wait();
  absorb_block<T, 8>(a, blockIdx.x, blockIdx.y, reinterpret_cast<float*>(smem4));
}

template <typename T>
static cudaError_t launch_absorb_t(const AbsorbArgs& a, cudaStream_t st) {
  const size_t smem = absorb_smem_bytes(absorb_rows<8>(), a.d_h);
  static PerDeviceOnce attrs;
  cudaError_t e = once_per_device(attrs, [] { return set_smem_attrs(absorb_qtilde_kernel<T>, 200 * 1024); });
  if (e != cudaSuccess) return e;
  dim3 grid(a.heads, (a.r + absorb_rows<8>() - 1) / absorb_rows<8>() + 1);
  return launch_chained(absorb_qtilde_kernel<T>, grid, dim3(256), smem, st, a);
}

cudaError_t launch_absorb(const AbsorbArgs& a, bool bf16, cudaStream_t st) {
  return bf16 ? launch_absorb_t<__nv_bfloat16>(a, st) : launch_absorb_t<float>(a, st);
}

}  // namespace qkn
