// qkn_absorb_query kernel: fold the static norm weights into the query
// ("QK-Normed MLA: QK normalization without full key caching", technical
// summary, Metodología item 1 and the decode-logit equation).
//
//   q~[i,h]  = W^K_{g,h} (gamma_q[h] * gamma_k[h] * q[i,h])        (absorption units)
//   a_q[i,h] = sigma / S(q[i,h])                                   (absorb_row)
//   q^R^[i,h] = sigma * RoPE_pos(gamma_qR[h] * q^R / S(q^R))        (absorb_row)
// Persistent CTAs, one per SM, over the absorption units (head, latent-row block); the W^K slice
// of a CTA's next unit is in flight while it works on the current one (prep_blocks.cuh).
#include "prep_blocks.cuh"

namespace qkn {

namespace {

constexpr int kAbsWarps = 16;
constexpr int kAbsSmemMax = 227 * 1024;

struct AbsorbLaunch {
  AbsorbArgs a;
  int32_t units, nbuf;
};

template <typename T>
__global__ void __launch_bounds__(kAbsWarps * 32, 1) absorb_kernel(const __grid_constant__ AbsorbLaunch p) {
  extern __shared__ float4 smem4[];
  pdl_trigger();
  pdl_wait();
  constexpr int KB = absorb_unit_rows<kAbsWarps>();
  float* smem = reinterpret_cast<float*>(smem4);
  float (*rows)[128] = reinterpret_cast<float (*)[128]>(smem);
  float* absm = smem + kAbsWarps * 128;
  const int pitch = absorb_pitch(p.a.d_h);
  const int wstride = (p.nbuf - 1) * KB * pitch;        // second W buffer (the first when nbuf == 1)
  float* sv = absm + p.nbuf * KB * pitch;
  float* g2 = sv + kAbsQ * pitch;
  absorb_zero_pads<kAbsWarps>(p.a, absm, p.nbuf);
  const int G = gridDim.x;
  int cur = 0;
  bool loaded = false;
  for (int u = blockIdx.x; u < p.units; u += G) {
    if (!loaded) absorb_load_w<kAbsWarps>(p.a, u, absm + cur * wstride);
    const int nxt = u + G;
    int pending = 0;
    if (p.nbuf == 2 && nxt < p.units) {
      absorb_load_w<kAbsWarps>(p.a, nxt, absm + (cur ^ 1) * wstride);
      pending = 1;
    }
    absorb_unit<T, kAbsWarps>(p.a, u, absm + cur * wstride, sv, g2, pending, rows, true);
    loaded = pending != 0;
    if (p.nbuf == 2) cur ^= 1;
  }
}

template <typename T>
cudaError_t launch_absorb_t(const AbsorbArgs& a, cudaStream_t st) {
  AbsorbLaunch p;
  p.a = a;
  p.units = absorb_units<kAbsWarps>(a.heads, a.r, a.n_q);
  const size_t rows_floats = (size_t)kAbsWarps * 128;
  size_t floats = rows_floats + absorb_unit_floats<kAbsWarps>(a.d_h, 2);
  p.nbuf = 2;
  if (floats * 4 > kAbsSmemMax) {
    floats = rows_floats + absorb_unit_floats<kAbsWarps>(a.d_h, 1);
    p.nbuf = 1;
  }
  if (floats * 4 > kAbsSmemMax) return cudaErrorNotSupported;
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  const int ctas = p.units < sms ? p.units : sms;
  static PerDeviceOnce attrs;
  e = once_per_device(attrs, [] { return set_smem_attrs(absorb_kernel<T>, kAbsSmemMax); });
  if (e != cudaSuccess) return e;
  return launch_chained(absorb_kernel<T>, dim3((unsigned)ctas), dim3(kAbsWarps * 32), floats * 4, st, p);
}

}  // namespace

cudaError_t launch_absorb(const AbsorbArgs& a, bool bf16, cudaStream_t st) {
  return bf16 ? launch_absorb_t<__nv_bfloat16>(a, st) : launch_absorb_t<float>(a, st);
}

}  // namespace qkn
