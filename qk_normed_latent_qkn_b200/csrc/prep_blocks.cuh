// Device-side building blocks of the append and query-absorption kernels,
// shared by their own launches (append.cu, absorb.cu) and by the one-launch
// step preparation (prep.cu).  The functions take the CTA's block
// coordinates and shared memory as arguments, so that one kernel can host
// CTAs of both kinds.
#pragma once

#include <type_traits>

#include "common.cuh"
#include "kernels.h"

namespace qkn {

// Token i of the call, by one warp: the latent row copied, the RoPE key
// RMS-normalised, weighted and rotated.  `row` is the warp's 128-float
// shared-memory buffer (d_R <= 128).
template <typename T>
__device__ __forceinline__ void append_token(const AppendArgs& a, int i, int lane, float* row) {
  const int64_t slot = a.slot[i];
  if (slot < 0 || slot >= a.n_slots) return;        // outside the pool: the token is skipped
  const int32_t pos = a.pos[i];
  // latent row: 16-byte vectors (rows are a multiple of 16 bytes)
  const uint4* src = reinterpret_cast<const uint4*>(static_cast<const T*>(a.c_new) + (int64_t)i * a.r);
  uint4* dst = reinterpret_cast<uint4*>(static_cast<T*>(a.latent) + slot * a.r);
  const int nvec = a.r * (int)sizeof(T) / 16;
  uint4 cv[4];
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int k = lane + 32 * u;
    if (k < nvec) cv[u] = src[k];
  }
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int k = lane + 32 * u;
    if (k < nvec) dst[k] = cv[u];
  }
  for (int k = lane + 128; k < nvec; k += 32) dst[k] = src[k];

  // RoPE key: d_R <= 128, so each lane holds at most 4 elements.
  const T* kr = static_cast<const T*>(a.k_rope_raw) + (int64_t)i * a.d_rope;
  float x[4];
  float ss = 0.f;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int k = lane + 32 * q;
    x[q] = k < a.d_rope ? to_f32(kr[k]) : 0.f;
    ss += x[q] * x[q];
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const float inv = 1.0f / sqrtf(ss / (float)a.d_rope + a.eps);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int k = lane + 32 * q;
    if (k < a.d_rope) x[q] = x[q] * inv * a.gamma_kr[k];
  }
  // Pair element k (< d/2) with k + d/2, which sits in lane (k + d/2) % 32 of
  // slot (k + d/2) / 32.  Gather the partner through the warp's shared buffer.
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int k = lane + 32 * q;
    if (k < a.d_rope) row[k] = x[q];
  }
  __syncwarp();
  T* kout = static_cast<T*>(a.k_rope) + slot * a.d_rope;
  const int half = a.d_rope / 2;
  for (int k = lane; k < half; k += 32) {
    const float x1 = row[k], x2 = row[k + half];
    float sn, cs;
    rope_sincos(pos, a.freq.f[k], sn, cs);
    kout[k] = from_f32<T>(x1 * cs - x2 * sn);
    kout[k + half] = from_f32<T>(x2 * cs + x1 * sn);
  }
  __syncwarp();
}

// Key statistic sum(z^2) over the n_g d_h columns of z = c W^K_g.  Two forms
// of the same sum:
//   direct: sum_n z_n^2 with z = c W^K_g             (matrix W, width columns)
//   Gram:   sum_n (c G)_n c_n with G = W^K_g W^K_g^T  (matrix G, r columns)
// The Gram form (the identity |cW|^2 = c (W W^T) c^T) reads an r x r matrix
// instead of r x n_g d_h, a 32-fold cut at r = 512 and n_g d_h = 16384.
// CTA = (16 matrix columns, TT tokens, group); its 512 threads are 16 columns
// x 32 slices of the latent dimension, so a decode step's handful of tokens
// still spreads over several CTAs per group.  Every thread loads its slice of
// one matrix column in one batch of independent loads and applies it to the
// TT tokens held in shared memory; slices are summed in shared memory, turned
// into the column's term (z^2, or (cG)_n c_n), reduced over the CTA's 16
// columns and added into the token's a_k slot (zeroed by append_copy_kernel).
constexpr int kRmsCols = 16;
constexpr int kRmsSlices = 32;

// FUSED (the cache has ak_scratch): the whole append in this one launch.  One
// more CTA column (block x == number of column blocks) copies the tile's
// latents and RoPE keys; the column CTAs add their sums into the slot's
// accumulator in ak_scratch and count themselves in, and the CTA whose count
// completes a token writes a_k = 1 / sqrt(sum / width + eps) and returns the
// accumulator and the count to zero.
// `rows`: a 128-float buffer per warp (kRmsCols * kRmsSlices / 32 of them) for the copy column.
template <typename T, int TT, bool FUSED>
__device__ __forceinline__ void keyrms_block(const AppendArgs& a, int bx, int by, int bz, float* smem,
                                             float (*rows)[128]) {
  float* cs = smem;                                               // [TT][r]
  float* zp = cs + TT * a.r;                                      // [kRmsSlices][TT][kRmsCols]
  const int g = bz;
  const int t0 = by * TT;
  const int ntok = min(TT, a.n_tok - t0);
  const int ncols = a.ncols;
  const bool gram = a.key_gram != nullptr;
  const int col = threadIdx.x % kRmsCols, slice = threadIdx.x / kRmsCols;
  const int n = bx * kRmsCols + col;
  const int nblk = (ncols + kRmsCols - 1) / kRmsCols;
  if constexpr (FUSED) {
    if (bx == nblk) {
      const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
      if (bz == 0)
        for (int i = warp; i < ntok; i += kRmsCols * kRmsSlices / 32) append_token<T>(a, t0 + i, lane, rows[warp]);
      return;
    }
  }

  // latent rows [k0, k1) of this slice; W loads are issued before the token tile is staged
  const int k0 = (int)((int64_t)slice * a.r / kRmsSlices);
  const int k1 = (int)((int64_t)(slice + 1) * a.r / kRmsSlices);
  const float* w = (gram ? a.key_gram : a.w_k) + (int64_t)g * a.r * ncols + min(n, ncols - 1);
  constexpr int kBatch = 16;
  float wv[kBatch];
#pragma unroll
  for (int u = 0; u < kBatch; ++u) wv[u] = (k0 + u < k1) ? w[(int64_t)(k0 + u) * ncols] : 0.f;

  {   // stage the token tile as fp32, 16 bytes of input per load
    constexpr int kPer = 16 / (int)sizeof(T);          // elements per 16-byte load
    const uint4* c4 = reinterpret_cast<const uint4*>(static_cast<const T*>(a.c_new) + (int64_t)t0 * a.r);
    const int nvec = TT * a.r / kPer;
    for (int e0 = threadIdx.x; e0 < nvec; e0 += 4 * kRmsCols * kRmsSlices) {
      uint4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int e = e0 + u * kRmsCols * kRmsSlices;
        v[u] = (e < nvec && (e * kPer) / a.r < ntok) ? c4[e] : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int e = e0 + u * kRmsCols * kRmsSlices;
        if (e < nvec) {
          const T* x = reinterpret_cast<const T*>(&v[u]);
#pragma unroll
          for (int q = 0; q < kPer; ++q) cs[e * kPer + q] = to_f32(x[q]);
        }
      }
    }
  }
  __syncthreads();

  float acc[TT];
#pragma unroll
  for (int t = 0; t < TT; ++t) acc[t] = 0.f;
  for (int kb = k0;; ) {
    const int nk = min(kBatch, k1 - kb);
    if (nk == kBatch && (kb & 3) == 0 && (a.r & 3) == 0) {
      // 16-byte token reads: four FMAs per shared-memory load
#pragma unroll
      for (int t = 0; t < TT; ++t) {
        const float4* crow = reinterpret_cast<const float4*>(cs + t * a.r + kb);
#pragma unroll
        for (int u4 = 0; u4 < kBatch / 4; ++u4) {
          const float4 cv = crow[u4];
          acc[t] = fmaf(cv.x, wv[4 * u4 + 0], acc[t]);
          acc[t] = fmaf(cv.y, wv[4 * u4 + 1], acc[t]);
          acc[t] = fmaf(cv.z, wv[4 * u4 + 2], acc[t]);
          acc[t] = fmaf(cv.w, wv[4 * u4 + 3], acc[t]);
        }
      }
    } else {
#pragma unroll
      for (int t = 0; t < TT; ++t) {
        const float* crow = cs + t * a.r + kb;
#pragma unroll
        for (int u = 0; u < kBatch; ++u)
          if (u < nk) acc[t] = fmaf(crow[u], wv[u], acc[t]);
      }
    }
    kb += kBatch;
    if (kb >= k1) break;
#pragma unroll
    for (int u = 0; u < kBatch; ++u) wv[u] = (kb + u < k1) ? w[(int64_t)(kb + u) * ncols] : 0.f;
  }
#pragma unroll
  for (int t = 0; t < TT; ++t) zp[(slice * TT + t) * kRmsCols + col] = acc[t];
  __syncthreads();
  // thread (slice, col) finishes tokens slice, slice + 32, ...: z summed over slices, turned into
  // the column's term, then summed over the 16 columns of its half-warp
  for (int t = slice; t < TT; t += kRmsSlices) {
    float z = 0.f;
#pragma unroll
    for (int sl = 0; sl < kRmsSlices; ++sl) z += zp[(sl * TT + t) * kRmsCols + col];
    float v = (n < ncols) ? z * (gram ? cs[t * a.r + n] : z) : 0.f;
#pragma unroll
    for (int o = kRmsCols / 2; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    const int64_t s_t = t < ntok ? (int64_t)a.slot[t0 + t] : -1;
    if (col == 0 && t < ntok && s_t >= 0 && s_t < a.n_slots) {
      const int64_t i = s_t * a.groups + g;
      if constexpr (FUSED) {
        float* acc = reinterpret_cast<float*>(a.ak_scratch + 2 * i);
        unsigned int* cnt = a.ak_scratch + 2 * i + 1;
        atomicAdd(acc, v);
        __threadfence();
        if (atomicAdd(cnt, 1u) == (unsigned int)(nblk - 1)) {
          __threadfence();
          const float total = atomicExch(acc, 0.f);
          a.a_k[i] = 1.0f / sqrtf(total / (float)a.width + a.eps);
          atomicExch(cnt, 0u);
        }
      } else {
        atomicAdd(a.a_k + i, v);
      }
    }
  }
}

// a_q[i,h] and the rotated RoPE query of one (query row i, head h), by one warp.
template <typename T>
__device__ __forceinline__ void absorb_row(const AbsorbArgs& a, int i, int h, float* row, int lane) {
  const int64_t wid = (int64_t)i * a.heads + h;
  const T* q = static_cast<const T*>(a.q) + wid * a.d_h;
  float ss = 0.f;
  for (int d = lane; d < a.d_h; d += 32) {
    const float v = to_f32(q[d]);
    ss += v * v;
  }
  const T* qr = static_cast<const T*>(a.q_rope) + wid * a.d_rope;
  float sr = 0.f;
  for (int d = lane; d < a.d_rope; d += 32) {
    const float v = to_f32(qr[d]);
    row[d] = v;
    sr += v * v;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    ss += __shfl_xor_sync(0xffffffffu, ss, o);
    sr += __shfl_xor_sync(0xffffffffu, sr, o);
  }
  if (lane == 0) a.a_q[wid] = a.softmax_scale / sqrtf(ss / (float)a.d_h + a.eps);
  const float inv = a.softmax_scale / sqrtf(sr / (float)a.d_rope + a.eps);
  __syncwarp();
  const int half = a.d_rope / 2;
  const int32_t pos = a.pos[i];
  T* out = static_cast<T*>(a.q_rope_hat) + wid * a.d_rope;
  for (int d = lane; d < half; d += 32) {
    const float x1 = row[d] * inv * a.gamma_qr[h * a.d_rope + d];
    const float x2 = row[d + half] * inv * a.gamma_qr[h * a.d_rope + d + half];
    float sn, cs;
    rope_sincos(pos, a.freq.f[d], sn, cs);
    out[d] = from_f32<T>(x1 * cs - x2 * sn);
    out[d + half] = from_f32<T>(x2 * cs + x1 * sn);
  }
  __syncwarp();
}

constexpr int kAbsQ = 32;        // query rows per pass

// fp32 -> TF32 (round to nearest, ties away), kept in an fp32 register
__device__ __forceinline__ float round_tf32(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return __uint_as_float(r);
}
// D += A B, m16n8k8, TF32 inputs, fp32 accumulators (warp-wide)
__device__ __forceinline__ void mma_tf32_m16n8k8(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
  asm volatile(
      "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// a_q and the rotated RoPE query of every query row of head h, one warp per row.
template <typename T, int NW>
__device__ __forceinline__ void absorb_head_rows(const AbsorbArgs& a, int h, float (*rows)[128]) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = warp; i < a.n_q; i += NW) absorb_row<T>(a, i, h, rows[warp], lane);
}

// ---------------------------------------------------------------- absorption units
// The absorption q~[i, h] = W^K_{g,h} (gamma_q[h] gamma_k[h] q[i, h]) as units (head h, KB = 8 NW
// latent rows from kbase = kc KB, query rows [qb QB, (qb + 1) QB)), unit
// j = (h ceil(r / KB) + kc) ceil(n_q / QB) + qb, for CTAs of NW warps (the units that share a W
// slice are consecutive, so the later copies of it come from L2).  A unit's
// slice of W^K_{g,h} (KB rows of d_h contiguous fp32 values) is copied raw with 16-byte cp.async
// (no register staging) into a W buffer; gamma_q gamma_k is folded into the staged query rows
// instead of into W (the same products in another order).  For bf16 storage the products run on
// the tensor cores in TF32 (fp32 accumulation): the query rows are rounded to TF32, the raw W
// values are truncated to it by the MMA (relative error below 2^-10, beside the bf16 rounding of
// q~ at 2^-9); fp32 storage keeps fp32 FMAs.  a_q and the RoPE query of head h come from
// absorb_head_rows, or from the units of each query block.
//
// Shared memory (floats): nbuf W buffers [KB][pitch], the query rows [kAbsQ][pitch], gamma_q gamma_k
// [d_h].  The row pitch is the smallest p >= d_h + 4 with p = 8 (mod 32): the TF32 products read a
// fragment's two K values as one 8-byte pair (below), and with that pitch the 16 threads of each
// half-warp (rows gid < 4, pairs 2 tig) hit 32 distinct banks; the 4 pad columns stay zero.
__host__ __device__ inline int absorb_pitch(int d_h) { return d_h + 4 + (((8 - (d_h + 4)) % 32) + 32) % 32; }
template <int NW>
__host__ __device__ constexpr int absorb_unit_rows() { return NW * 8; }
template <int NW>
inline size_t absorb_unit_floats(int d_h, int nbuf) {
  return (size_t)(nbuf * absorb_unit_rows<NW>() + kAbsQ) * absorb_pitch(d_h) + d_h;
}
constexpr int kAbsQB = 128;      // query rows per absorption unit (in passes of kAbsQ)
template <int NW>
__host__ __device__ inline int absorb_units(int heads, int r, int n_q) {
  return heads * ((r + absorb_unit_rows<NW>() - 1) / absorb_unit_rows<NW>()) * ((n_q + kAbsQB - 1) / kAbsQB);
}

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"((uint32_t)__cvta_generic_to_shared(dst)), "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_pending(int n) {
  if (n > 0) asm volatile("cp.async.wait_group 1;" ::: "memory");
  else asm volatile("cp.async.wait_group 0;" ::: "memory");
}

// Issue the copies of unit j's slice of W^K into `wb` and commit them as one group (every thread
// commits, possibly an empty group).  Rows past r are not copied (their outputs are not stored).
template <int NW>
__device__ __forceinline__ void absorb_load_w(const AbsorbArgs& a, int j, float* wb) {
  constexpr int KB = absorb_unit_rows<NW>(), kT = NW * 32;
  const int nkc = (a.r + KB - 1) / KB, nqb = (a.n_q + kAbsQB - 1) / kAbsQB;
  const int hk = j / nqb;
  const int h = hk / nkc, kbase = (hk - h * nkc) * KB;
  const int ng = a.heads / a.groups, g = h / ng, m = h - g * ng;
  const int width = ng * a.d_h, pitch = absorb_pitch(a.d_h), dq = a.d_h / 4;
  const float* w = a.w_k + (int64_t)g * a.r * width + (int64_t)m * a.d_h;
  const int nrows = min(KB, a.r - kbase);
  if (kT % dq == 0) {
    // each thread keeps one 16-byte column of the slice and walks its rows
    const int d4 = threadIdx.x % dq, rstep = kT / dq;
    for (int rr = threadIdx.x / dq; rr < nrows; rr += rstep)
      cp_async16(wb + rr * pitch + d4 * 4, w + (int64_t)(kbase + rr) * width + d4 * 4);
  } else {
    for (int e = threadIdx.x; e < nrows * dq; e += kT) {
      const int rr = e / dq, d4 = e - rr * dq;
      cp_async16(wb + rr * pitch + d4 * 4, w + (int64_t)(kbase + rr) * width + d4 * 4);
    }
  }
  cp_async_commit();
}

// Zero the 4 pad columns of every W and query row once per kernel: the TF32 loop reads them when
// d_h % 8 == 4, and the copies never write them.
template <int NW>
__device__ __forceinline__ void absorb_zero_pads(const AbsorbArgs& a, float* abs_smem, int nbuf) {
  const int pitch = absorb_pitch(a.d_h);
  for (int rr = threadIdx.x; rr < nbuf * absorb_unit_rows<NW>() + kAbsQ; rr += NW * 32)
    *reinterpret_cast<float4*>(abs_smem + rr * pitch + a.d_h) = make_float4(0.f, 0.f, 0.f, 0.f);
}

// Unit j with its W slice in `wb` (its copies committed as the older of at most `pending` + 1
// outstanding groups of this thread).  Starts and ends with the CTA's query rows and gamma
// buffers free; ends with a barrier, after which `wb` may be refilled.
// `rows`: a 128-float buffer per warp, for the a_q / RoPE rows when the units do them (rows_too:
// the units of a query block share its rows, unit kc taking every ceil(r / KB)-th one); otherwise
// absorb_head_rows does them separately.
template <typename T, int NW>
__device__ __forceinline__ void absorb_unit(const AbsorbArgs& a, int j, const float* wb, float* sv, float* g2,
                                            int pending, float (*rows)[128], bool rows_too) {
  constexpr int kThreadsAbs = NW * 32;
  constexpr int KB = absorb_unit_rows<NW>();
  constexpr int kRowWarps = NW / 2;
  static_assert(kRowWarps * 16 == KB && kAbsQ == 32, "warp tiling of the absorption unit");
  constexpr bool kTensor = std::is_same<T, __nv_bfloat16>::value;
  const int pitch = absorb_pitch(a.d_h), dq = a.d_h / 4;
  const int nkc = (a.r + KB - 1) / KB, nqb = (a.n_q + kAbsQB - 1) / kAbsQB;
  const int hk = j / nqb, qb = j - hk * nqb;
  const int h = hk / nkc, kc = hk - h * nkc, kbase = kc * KB;
  const int q_lo = qb * kAbsQB, q_hi = min(a.n_q, q_lo + kAbsQB);   // this unit's query rows
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const T* q = static_cast<const T*>(a.q);
  T* out = static_cast<T*>(a.q_tilde);
  // stage query rows [i0, i0 + nq) of head h times gamma_q gamma_k (zeros past nq); g2 is ready
  auto stage_q = [&](int i0, int nq) {
    for (int e = threadIdx.x; e < kAbsQ * dq; e += kThreadsAbs) {
      const int qi = (dq == 32) ? (e >> 5) : e / dq, d4 = e - qi * dq;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (qi < nq) {
        const T* src = q + ((int64_t)(i0 + qi) * a.heads + h) * a.d_h + d4 * 4;
        const float4 gg = reinterpret_cast<const float4*>(g2)[d4];
        v = make_float4(to_f32(src[0]) * gg.x, to_f32(src[1]) * gg.y, to_f32(src[2]) * gg.z, to_f32(src[3]) * gg.w);
        if constexpr (kTensor) v = make_float4(round_tf32(v.x), round_tf32(v.y), round_tf32(v.z), round_tf32(v.w));
      }
      *reinterpret_cast<float4*>(sv + qi * pitch + d4 * 4) = v;
    }
  };
  if ((int)threadIdx.x < dq) {
    const float4 gq = *reinterpret_cast<const float4*>(a.gamma_q + h * a.d_h + threadIdx.x * 4);
    const float4 gk = *reinterpret_cast<const float4*>(a.gamma_k + h * a.d_h + threadIdx.x * 4);
    reinterpret_cast<float4*>(g2)[threadIdx.x] = make_float4(gq.x * gk.x, gq.y * gk.y, gq.z * gk.z, gq.w * gk.w);
  }
  __syncthreads();
  stage_q(q_lo, min(kAbsQ, q_hi - q_lo));
  cp_async_wait_pending(pending);                        // this unit's W slice has landed
  const int rw = warp % kRowWarps, qw = warp / kRowWarps;
  for (int i0 = q_lo; i0 < q_hi; i0 += kAbsQ) {
    const int nq = min(kAbsQ, q_hi - i0);
    if (i0 > q_lo) {
      __syncthreads();                                     // the previous pass is done with sv
      stage_q(i0, nq);
    }
    __syncthreads();
    if (qw * 16 >= nq) continue;                           // no query rows for this warp (warp-uniform)
    if constexpr (kTensor) {
      // m16n8k8 TF32 products: A = 16 rows of the slice, B = 8 query rows, per 8 columns of d_h.
      // Fragments (lane = 4 gid + tig): A holds (row gid | gid + 8, K index tig | tig + 4), B
      // (query row gid, K index tig | tig + 4), D (row gid | gid + 8, query row 2 tig | 2 tig + 1).
      // K index tig carries column d + 2 tig of d_h and K index tig + 4 column d + 2 tig + 1 (the same
      // map on A and B, so the 8 products of a step are those of columns d .. d + 7): each thread
      // reads a fragment's two values as one 8-byte pair.
      const int gid = lane >> 2, tig = lane & 3;
      const float* wa = wb + (rw * 16 + gid) * pitch + 2 * tig;
      const float* qb = sv + (qw * 16 + gid) * pitch + 2 * tig;
      float dacc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll 4
      for (int d = 0; d < a.d_h; d += 8) {
        const float2 w0 = *reinterpret_cast<const float2*>(wa + d);
        const float2 w1 = *reinterpret_cast<const float2*>(wa + 8 * pitch + d);
        const uint32_t af[4] = {__float_as_uint(w0.x), __float_as_uint(w1.x), __float_as_uint(w0.y),
                                __float_as_uint(w1.y)};
#pragma unroll
        for (int jj = 0; jj < 2; ++jj) {
          const float2 q2 = *reinterpret_cast<const float2*>(qb + jj * 8 * pitch + d);
          const uint32_t bf[2] = {__float_as_uint(q2.x), __float_as_uint(q2.y)};
          mma_tf32_m16n8k8(dacc[jj], af, bf);
        }
      }
#pragma unroll
      for (int jj = 0; jj < 2; ++jj) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int row = rw * 16 + gid + (e >> 1) * 8;
          const int qi = qw * 16 + jj * 8 + 2 * tig + (e & 1);
          if (qi < nq && kbase + row < a.r)
            out[((int64_t)(i0 + qi) * a.heads + h) * a.r + kbase + row] = from_f32<T>(dacc[jj][e]);
        }
      }
    } else {
      // fp32 FMAs: lane (rg, qg) = (lane % 8, lane / 8) takes rows rg, rg + 8 of the warp's 16 and
      // query rows qg, qg + 4, qg + 8, qg + 12: per 4 columns of d_h 2 W and 4 query vectors
      const int rg = lane & 7, qg = lane >> 3;
      const int k0 = rw * 16 + rg;
      const float* wrow0 = wb + k0 * pitch;
      const float* wrow1 = wrow0 + 8 * pitch;
      const float* qrow = sv + (qw * 16 + qg) * pitch;
      float acc0[4] = {0.f, 0.f, 0.f, 0.f}, acc1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
      for (int d = 0; d < a.d_h; d += 4) {
        const float4 w0 = *reinterpret_cast<const float4*>(wrow0 + d);
        const float4 w1 = *reinterpret_cast<const float4*>(wrow1 + d);
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          const float4 sq = *reinterpret_cast<const float4*>(qrow + 4 * v * pitch + d);
          acc0[v] = fmaf(w0.x, sq.x, fmaf(w0.y, sq.y, fmaf(w0.z, sq.z, fmaf(w0.w, sq.w, acc0[v]))));
          acc1[v] = fmaf(w1.x, sq.x, fmaf(w1.y, sq.y, fmaf(w1.z, sq.z, fmaf(w1.w, sq.w, acc1[v]))));
        }
      }
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        const int qi = qw * 16 + qg + 4 * v;
        if (qi < nq) {
          T* o = out + ((int64_t)(i0 + qi) * a.heads + h) * a.r + kbase;
          if (kbase + k0 < a.r) o[k0] = from_f32<T>(acc0[v]);
          if (kbase + k0 + 8 < a.r) o[k0 + 8] = from_f32<T>(acc1[v]);
        }
      }
    }
  }
  if (rows_too) {
    // a_q and the rotated RoPE query of head h, one warp per query row
    for (int i = q_lo + kc + warp * nkc; i < q_hi; i += NW * nkc) absorb_row<T>(a, i, h, rows[warp], lane);
  }
  __syncthreads();
}

}  // namespace qkn
