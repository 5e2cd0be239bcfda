// Split-KV merge fused with the per-head value up-projection.
//
// On the absorbed route the values are the latents c_t, so the attention
// output o_lat[i, h] lives in latent space (width r), and each head's value
// up-projection W^UV_h (r x d_v) is applied once to that output instead of to
// every cached token (GQLA summary, section 2, absorbed MQA route: the
// up-projections move into the query and output projections).  This kernel
// merges the split-KV partials of a row (as the plain merge does) and
// multiplies the merged row by W^UV_h in the same CTA, so o_lat never goes to
// global memory:
//   o_lat[i, h] = sum_s exp(lse_s - lse) o_s,  lse[i, h] = log sum_s exp(lse_s),
//   o_v[i, h] = o_lat[i, h] W^UV_h.
// One CTA per (head h, kRows query rows i = b s_q + j, group of d_v / G output columns); G > 1
// only when heads x row blocks would leave SMs idle (each column group merges the same rows, the
// repeated partial reads coming from L2, and loads only its columns of W^UV_h):
//   1. bf16 storage: W^UV_h goes to shared memory by cp.async while the merge
//      runs (issued before the wait for the decode, which never writes it);
//   2. the merge: each warp takes rows in turn, every lane owning 16-byte
//      pieces of the row, two splits loaded at a time; merged rows go to
//      shared memory in the storage type and lse to global memory;
//   3. the product [kRows x r] x [r x d_v]: bf16 mma.sync m16n8k16 with fp32
//      accumulation, fragments by ldmatrix (W^UV_h stays in its [r][d_v]
//      layout; the .trans form gives the K-pairs of a column), the result
//      rounded once to bf16.  fp32 storage takes fp32 FMAs, W^UV_h read from
//      global memory (test-sized shapes).
// The product is a small share of the work (kRows x d_v x r MACs per CTA
// against the W^UV_h and partial-row bytes it reads), so the warp-level MMA
// suffices.
#include <type_traits>

#include "common.cuh"
#include "kernels.h"
#include "mma_sync.cuh"
#include "sm100.cuh"

namespace qkn {

namespace {

using sm100::smem_u32;

constexpr int kUpThreads = 512;             // 16 warps
constexpr int kUpWarps = kUpThreads / 32;

template <typename S>
__device__ __forceinline__ void store_row4(S* p, float4 v);
template <>
__device__ __forceinline__ void store_row4<float>(float* p, float4 v) {
  *reinterpret_cast<float4*>(p) = v;
}
template <>
__device__ __forceinline__ void store_row4<__nv_bfloat16>(__nv_bfloat16* p, float4 v) {
  __nv_bfloat162 lo = __floats2bfloat162_rn(v.x, v.y), hi = __floats2bfloat162_rn(v.z, v.w);
  uint2 u;
  u.x = *reinterpret_cast<uint32_t*>(&lo);
  u.y = *reinterpret_cast<uint32_t*>(&hi);
  *reinterpret_cast<uint2*>(p) = u;
}

// Shared-memory layout: [W^UV_h (bf16 only)] [merged rows] [first split row, split count per row].
// bf16: W^UV_h as [r][d_v + 8] and rows as [kRows][r + 8]: 16-byte row starts for cp.async and
// ldmatrix, and the 8 rows of every 8x8 ldmatrix tile in distinct banks (a pitch of 4 mod 8 words).
struct UpLayout {
  size_t w_off, o_off, misc_off, total;
  int wpitch, opitch;                       // elements per stored row
};

__host__ __device__ inline UpLayout up_layout(bool bf16, int rows, int r, int dv) {
  UpLayout l;
  const size_t es = bf16 ? 2 : 4;
  l.wpitch = bf16 ? dv + 8 : 0;
  l.opitch = bf16 ? r + 8 : r;
  l.w_off = 0;
  l.o_off = bf16 ? (size_t)r * l.wpitch * es : 0;
  l.misc_off = l.o_off + (size_t)rows * l.opitch * es;
  l.total = l.misc_off + (size_t)rows * 16;
  return l;
}

template <typename T, int kRows>
__global__ void __launch_bounds__(kUpThreads, 1) combine_up_kernel(const CombineUpArgs u) {
  constexpr bool kTensor = std::is_same<T, __nv_bfloat16>::value;
  extern __shared__ __align__(16) unsigned char up_smem[];
  const CombineArgs& a = u.c;
  pdl_trigger();
  const int h = blockIdx.x;
  const int i0 = blockIdx.y * kRows;                      // first query row (b s_q + j) of the CTA
  const int n_q = a.batch * a.s_q;
  const int nrows = min(kRows, n_q - i0);                 // rows of this CTA that exist
  const int r = a.r, dv = u.d_v;
  const int dvc = dv / u.col_groups, n_lo = (int)blockIdx.z * dvc;   // this CTA's output columns
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const UpLayout L = up_layout(kTensor, kRows, r, dvc);
  T* ws = reinterpret_cast<T*>(up_smem + L.w_off);
  T* os = reinterpret_cast<T*>(up_smem + L.o_off);
  int64_t* first_s = reinterpret_cast<int64_t*>(up_smem + L.misc_off);
  int* nitems_s = reinterpret_cast<int*>(up_smem + L.misc_off + (size_t)kRows * 8);
  const T* w = static_cast<const T*>(u.w_uv) + (int64_t)h * r * dv + n_lo;   // column n_lo of W^UV_h

  // ---- 1. W^UV_h into shared memory, in flight during the merge
  if constexpr (kTensor) {
    const int cpr = dvc / 8;                              // 16-byte chunks per row of the columns
    const uint32_t wbase = smem_u32(ws);
    for (int c = threadIdx.x; c < r * cpr; c += kUpThreads) {
      const int k = c / cpr, n8 = c - k * cpr;
      cp_async16(wbase + (uint32_t)(k * L.wpitch + n8 * 8) * 2u, w + (int64_t)k * dv + n8 * 8);
    }
  }
  pdl_wait();                                             // the decode's partials are complete

  // ---- 2a. the splits of every row: (first partial row, count)
  if (a.seg_desc) {
    if (threadIdx.x < kRows) {
      const int rr = threadIdx.x, i = i0 + rr;
      int64_t first = 0;
      int nitems = 0;
      if (rr < nrows) {
        const int b = i / a.s_q, rho = (i - b * a.s_q) * a.heads + h;
        const int ht = rho / a.rows;
        const int2 d = a.seg_desc[b * a.ht_count + ht];
        // d.y <= 0: a sequence with a rejected length (no splits; the decode recorded the error).
        // A decode that stopped early leaves some descriptors unwritten: each is checked against
        // this launch's slots before a partial is read, and a bad one gives zero rows, lse = -inf.
        if (d.y > 0 && (d.x < 0 || d.y > a.max_items ||
                        (int64_t)d.x + (int64_t)(d.y - 1) * a.ht_count >= a.nslots)) {
          record_status(a.status, QKN_ERR_BOUNDS);
        } else if (d.y > 0) {
          first = (int64_t)d.x * a.rows + (rho - ht * a.rows);
          nitems = d.y;
        }
      }
      first_s[rr] = first;
      nitems_s[rr] = nitems;
    }
  } else {
    // recomputed from the schedule, one full warp per row (the unit scans are warp-wide)
    SchedParams sp{a.seq_lens, a.batch, a.s_q, a.max_blocks, a.ht_count, a.ncta, a.item_cost};
    const int64_t total = sched_total_units(sp);
    const int32_t ng = sched_groups(sp);
    const int64_t q = total > 0 ? (total + ng - 1) / ng : 1;
    for (int rr = warp; rr < kRows; rr += kUpWarps) {
      int64_t first = 0;
      int nitems = 0;
      if (rr < nrows) {
        const int i = i0 + rr;
        const int b = i / a.s_q, rho = (i - b * a.s_q) * a.heads + h;
        const int ht = rho / a.rows;
        const int32_t n = pages_of(a.seq_lens[b], sp);
        const SegSplit sg = seg_split(sched_units_before(sp, b), n, q, sp.item_cost);
        if (n == 0 && lane == 0) record_status(a.status, QKN_ERR_BOUNDS);
        nitems = n > 0 ? sg.nitems : 0;
        first = ((int64_t)(b + sg.c0) * a.ht_count + ht) * a.rows + (rho - ht * a.rows);
      }
      if (lane == 0) {
        first_s[rr] = first;
        nitems_s[rr] = nitems;
      }
    }
  }
  __syncthreads();

  // ---- 2b. merge: warp w takes rows w, w + 16, ...; lane l owns the 16-byte pieces v = l + 32 t
  const int nvec = r / 4;                                 // <= 128: four pieces per lane at most
  const int64_t lstride = (int64_t)a.rows * a.ht_count;   // consecutive splits sit ht_count slots apart
  const int64_t stride = lstride * nvec;
  for (int rr = warp; rr < kRows; rr += kUpWarps) {
    T* orow = os + (size_t)rr * L.opitch;
    const int nitems = nitems_s[rr];
    const float4* src0 = reinterpret_cast<const float4*>(a.part_o) + first_s[rr] * nvec;
    const float* lsrc = a.part_lse + first_s[rr];
    float m = -INFINITY, den = 0.f;
    float4 acc[4];
#pragma unroll
    for (int t = 0; t < 4; ++t) acc[t] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int c = 0; c < nitems; c += 2) {
      float ls[2];
      float4 x[2][4];
#pragma unroll
      for (int s = 0; s < 2; ++s) {
        const bool in = c + s < nitems;
        ls[s] = in ? lsrc[(int64_t)(c + s) * lstride] : -INFINITY;
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const int v = lane + 32 * t;
          x[s][t] = (in && v < nvec) ? src0[(int64_t)(c + s) * stride + v] : make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
      const float mc = fmaxf(m, fmaxf(ls[0], ls[1]));
      if (mc == -INFINITY) continue;                      // nothing visible so far
      const float sc = __expf(m - mc);                    // m == -inf gives 0
      den *= sc;
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        acc[t].x *= sc; acc[t].y *= sc; acc[t].z *= sc; acc[t].w *= sc;
      }
#pragma unroll
      for (int s = 0; s < 2; ++s) {
        const float wgt = __expf(ls[s] - mc);             // ls == -inf gives 0
        den += wgt;
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          acc[t].x = fmaf(wgt, x[s][t].x, acc[t].x);
          acc[t].y = fmaf(wgt, x[s][t].y, acc[t].y);
          acc[t].z = fmaf(wgt, x[s][t].z, acc[t].z);
          acc[t].w = fmaf(wgt, x[s][t].w, acc[t].w);
        }
      }
      m = mc;
    }
    // rows past the last query row and rows without splits come out as zeros, lse = -inf
    const float inv = den > 0.f ? 1.f / den : 0.f;
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const int v = lane + 32 * t;
      if (v < nvec)
        store_row4<T>(orow + v * 4, make_float4(acc[t].x * inv, acc[t].y * inv, acc[t].z * inv, acc[t].w * inv));
    }
    if (lane == 0 && rr < nrows && blockIdx.z == 0)
      a.lse[(int64_t)(i0 + rr) * a.heads + h] = den > 0.f ? m + logf(den) : -INFINITY;
  }
  if constexpr (kTensor) cp_async_wait_all();
  __syncthreads();

  // ---- 3. o_v = o_lat W^UV_h for the CTA's rows
  T* out = static_cast<T*>(u.out_v);
  const int64_t ostride = (int64_t)a.heads * dv;          // between consecutive query rows of o_v
  T* out0 = out + ((int64_t)i0 * a.heads + h) * dv + n_lo;
  if constexpr (kTensor) {
    // Task = (group of kMt m-tiles of 16 rows, pair of n-tiles of 8 columns); kRows / 16 / kMt = 2
    // groups, so 2 d_v / 16 tasks over the 16 warps.  Fragments (lane = 4 gid + tig): A rows gid and
    // gid + 8, k 2 tig, 2 tig + 1 and + 8; B k 2 tig, 2 tig + 1 and + 8, column gid; D rows gid and
    // gid + 8, columns 2 tig, 2 tig + 1.
    constexpr int kMt = kRows / 32;
    const int gid = lane >> 2, tig = lane & 3;
    const int npairs = dvc / 16;
    const uint32_t obase = smem_u32(os), wbase = smem_u32(ws);
    for (int task = warp; task < 2 * npairs; task += kUpWarps) {
      const int mg = task / npairs, np = task - mg * npairs;
      const int mt0 = mg * kMt;
      if (mt0 * 16 >= nrows) continue;                    // all rows of the group are padding
      float d[kMt][2][4] = {};
      // ldmatrix lane addresses: A rows (lane & 15), k + 8 (lane >> 4); B k rows (lane & 15),
      // columns + 8 (lane >> 4)
      const uint32_t a_addr = obase + (uint32_t)((mt0 * 16 + (lane & 15)) * L.opitch + (lane >> 4) * 8) * 2u;
      const uint32_t b_addr = wbase + (uint32_t)((lane & 15) * L.wpitch + np * 16 + (lane >> 4) * 8) * 2u;
      for (int k0 = 0; k0 < r; k0 += 16) {
        uint32_t bf[4];
        ldsm_x4_trans(b_addr + (uint32_t)(k0 * L.wpitch) * 2u, bf);
#pragma unroll
        for (int mt = 0; mt < kMt; ++mt) {
          uint32_t af[4];
          ldsm_x4(a_addr + (uint32_t)(mt * 16 * L.opitch + k0) * 2u, af);
          mma_bf16_m16n8k16(d[mt][0], af, bf[0], bf[1]);
          mma_bf16_m16n8k16(d[mt][1], af, bf[2], bf[3]);
        }
      }
#pragma unroll
      for (int mt = 0; mt < kMt; ++mt)
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {
            const int rr = (mt0 + mt) * 16 + gid + hf * 8;
            if (rr >= nrows) continue;
            const int n = np * 16 + nt * 8 + 2 * tig;
            *reinterpret_cast<__nv_bfloat162*>(out0 + rr * ostride + n) =
                __floats2bfloat162_rn(d[mt][nt][2 * hf], d[mt][nt][2 * hf + 1]);
          }
    }
  } else {
    // fp32: thread t takes outputs e = t, t + 512, ... as (row e / dvc, column e % dvc)
    for (int e = threadIdx.x; e < nrows * dvc; e += kUpThreads) {
      const int rr = e / dvc, n = e - rr * dvc;
      const float* orow = reinterpret_cast<const float*>(os) + (size_t)rr * L.opitch;
      const float* wc = reinterpret_cast<const float*>(w) + n;
      float acc = 0.f;
      for (int k = 0; k < r; ++k) acc = fmaf(orow[k], __ldg(wc + (int64_t)k * dv), acc);
      reinterpret_cast<float*>(out0)[rr * ostride + n] = acc;
    }
  }
}

constexpr int kMaxUpSmem = 227 * 1024;

template <typename T, int kRows>
cudaError_t launch_up_t(CombineUpArgs u, cudaStream_t st) {
  static PerDeviceOnce attrs;
  cudaError_t e = once_per_device(attrs, [] { return set_smem_attrs(combine_up_kernel<T, kRows>, kMaxUpSmem); });
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0;
  e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  const int n_q = u.c.batch * u.c.s_q;
  const int ctas = u.c.heads * ((n_q + kRows - 1) / kRows);
  // column groups repeat the merge of the CTA's rows (from L2) for every group, which costs more
  // than it gains unless the grid leaves most SMs idle: below a quarter of the SMs, the fewest
  // groups (a divisor of d_v / 16) that reach half of them (measured: 16 heads x 16 rows 14.4 ->
  // 12.3 us; 64 and 128 heads slower with groups)
  const int pairs = u.d_v / 16;
  int g = 1;
  while (4 * ctas < sms && g < pairs && 2 * ctas * g < sms) {
    ++g;
    while (pairs % g) ++g;
  }
  u.col_groups = g;
  const UpLayout L = up_layout(std::is_same<T, __nv_bfloat16>::value, kRows, u.c.r, u.d_v / g);
  const dim3 grid((unsigned)u.c.heads, (unsigned)((n_q + kRows - 1) / kRows), (unsigned)g);
  return launch_chained(combine_up_kernel<T, kRows>, grid, dim3(kUpThreads), L.total, st, u);
}

// Rows per CTA: 64 (four m-tiles per load of W^UV_h) once a head has more than 32 query rows and
// they fit beside W^UV_h, else 32.
int up_rows(bool bf16, int r, int dv, int n_q) {
  return n_q > 32 && up_layout(bf16, 64, r, dv).total <= (size_t)kMaxUpSmem ? 64 : 32;
}

}  // namespace

bool combine_up_supported(bool bf16, int r, int dv, int n_q) {
  (void)n_q;
  if (dv <= 0 || dv % 16 || r <= 0 || r % 16 || r > 512) return false;
  return up_layout(bf16, 32, r, dv).total <= (size_t)kMaxUpSmem;
}

cudaError_t launch_combine_up(const CombineUpArgs& u, bool bf16, cudaStream_t st) {
  const int n_q = u.c.batch * u.c.s_q;
  if (!combine_up_supported(bf16, u.c.r, u.d_v, n_q)) return cudaErrorNotSupported;
  if (up_rows(bf16, u.c.r, u.d_v, n_q) == 64)
    return bf16 ? launch_up_t<__nv_bfloat16, 64>(u, st) : launch_up_t<float, 64>(u, st);
  return bf16 ? launch_up_t<__nv_bfloat16, 32>(u, st) : launch_up_t<float, 32>(u, st);
}

}  // namespace qkn
