// qkn_append_absorb: a decode step's cache append and query absorption in
// one launch.  The two are independent ("QK-Normed MLA: QK normalization
// without full key caching", technical summary, Metodología items 1-4: the
// key statistic is computed at append time, the norm weights are folded into
// the query), so one grid hosts CTAs of three kinds, two CTAs per SM: the
// append CTAs of the one-launch append (key-statistic column blocks plus the
// copy column), one CTA per head for a_q and the RoPE query, then the
// absorption CTAs (head, latent-row block), each of which copies its W^K
// slice with cp.async.  A step then needs no fork and join of two streams,
// and the decode that follows chains onto one kernel.
#include "prep_blocks.cuh"

namespace qkn {

namespace {

constexpr int kPrepThreads = kRmsCols * kRmsSlices;     // 512
constexpr int kPrepWarps = kPrepThreads / 32;
constexpr int kPrepTT = 16;                             // append token tile

struct PrepArgs {
  AppendArgs ap;
  AbsorbArgs ab;
  int32_t append_x, append_y, append_ctas;              // append grid (x, y, groups), flattened
};

// shared memory (floats): [row buffers kPrepWarps x 128 | append scratch or absorption buffers]
template <typename T>
__global__ void __launch_bounds__(kPrepThreads, 2) prep_kernel(const __grid_constant__ PrepArgs p) {
  extern __shared__ float4 smem4[];
  float* smem = reinterpret_cast<float*>(smem4);
  float (*rows)[128] = reinterpret_cast<float (*)[128]>(smem);
  float* work = smem + kPrepWarps * 128;
  // dependents may launch only once everything before this kernel is complete: a decode that
  // streams old cache pages before its own wait (step_writes_only) relies on it
  pdl_wait();
  pdl_trigger();
  int bid = blockIdx.x;
  if (bid < p.append_ctas) {
    const int x = bid % p.append_x;
    bid /= p.append_x;
    keyrms_block<T, kPrepTT, true>(p.ap, x, bid % p.append_y, bid / p.append_y, work, rows);
    return;
  }
  bid -= p.append_ctas;
  if (bid < p.ab.heads) {
    absorb_head_rows<T, kPrepWarps>(p.ab, bid, rows);
    return;
  }
  bid -= p.ab.heads;
  constexpr int KB = absorb_unit_rows<kPrepWarps>();
  const int pitch = absorb_pitch(p.ab.d_h);
  float* sv = work + KB * pitch;
  absorb_zero_pads<kPrepWarps>(p.ab, work, 1);
  absorb_load_w<kPrepWarps>(p.ab, bid, work);
  absorb_unit<T, kPrepWarps>(p.ab, bid, work, sv, sv + kAbsQ * pitch, 0, rows, false);
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
  const int64_t ctas = (int64_t)p.append_ctas + ab.heads + absorb_units<kPrepWarps>(ab.heads, ab.r, ab.n_q);
  const size_t app = (size_t)kPrepTT * ap.r + (size_t)kRmsSlices * kPrepTT * kRmsCols;
  const size_t abs1 = absorb_unit_floats<kPrepWarps>(ab.d_h, 1);
  const size_t smem = ((size_t)kPrepWarps * 128 + (app > abs1 ? app : abs1)) * sizeof(float);
  auto kernel = bf16 ? prep_kernel<__nv_bfloat16> : prep_kernel<float>;
  static PerDeviceOnce attrs[2];
  cudaError_t e = once_per_device(attrs[bf16 ? 1 : 0], [&] { return set_smem_attrs(kernel, 227 * 1024); });
  if (e != cudaSuccess) return e;
  return launch_chained(kernel, dim3((unsigned)ctas), dim3(kPrepThreads), smem, st, p);
}

}  // namespace qkn
