// The GQA route of GQLA ("GQLA", section 2, "Ruta GQA") on a cache of keys
// and values expanded per KV group, and its sparse form (section 2, "GQLA
// Disperso").  One key head and one value head per group: the up-projections
// W^UK_g, W^UV_g are indexed by group (section 2, Arquitectura).
//
// Append, for every new token t and group g:
//   k_{t,g} = RMSNorm(c_t W^UK_g) gamma_k[g]      (over the group's d_h columns)
//   v_{t,g} = c_t W^UV_g
// and the shared RoPE key RoPE_p(RMSNorm(k^R_t) gamma_kR): the cache of that
// route (2 g d_h values per token plus the RoPE key).  The key is normalised
// after its up-projection, as the QK-Normed key is ("QK-Normed MLA",
// technical summary, "Planteamiento del Problema"); on this route the key is
// stored, so the normalisation is applied once, at append time.
//
// Decode: grouped-query attention over that cache.  Query row (j, h) of
// sequence b, h in group g = h / n_g, at position L - s_q + j:
//   l[t] = sigma (RMSNorm(q_jh) gamma_q[h] . k_{t,g} + RoPE(RMSNorm(q^R_jh) gamma_qR[h]) . k^R_t)
// over the tokens t <= L - s_q + j (dense), or over the tokens listed for
// (j, g) among them (sparse); softmax; o = sum_t p_t v_{t,g}.  The queries
// are normalised and rotated inside the decode, per tile.
//
// The route reads (2 g d_h + d_R) * 2 bytes per token for 2 h_q s_q (d_h +
// d_R + d_v) FLOPs: 19 FLOP/B at h_q = 128, g = 8, s_q = 1, 39 at s_q = 2,
// far below the B200's ridge (about 250), so the decode is built around the
// cache stream: one persistent CTA per SM on the split-KV device schedule
// (common.cuh), a four-page cp.async ring, and a page's two products on the
// warp-level bf16 tensor-core path (mma.sync): with 16 or 32 query rows per
// tile they are too narrow to pay for tcgen05's tensor-memory round trips.
#include <float.h>

#include "common.cuh"
#include "kernels.h"
#include "mma_sync.cuh"
#include "sm100.cuh"

namespace qkn {

namespace {

using sm100::smem_u32;

__device__ __forceinline__ float4 bf16x4_to_f32(uint2 u) {
  const float2 lo = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
  const float2 hi = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
  return make_float4(lo.x, lo.y, hi.x, hi.y);
}

// ------------------------------------------------------------------ append
// CTA (token block of 32, group g, part): part 0 the group's keys, part 1 its
// values (an fp32 [32 x r] x [r x d] product, d <= 128, the latent and the
// weight staged through shared memory 32 latent columns at a time; warp w
// owns tokens 4 w .. 4 w + 3, lane l columns 4 l .. 4 l + 3, so that a key
// row's sum of squares is one warp reduction), part 2 the RoPE keys (group 0
// only, one warp per token).
constexpr int kAppTok = 32;
constexpr int kAppK = 32;
constexpr int kAppThreads = 256;
constexpr int kAppWarps = kAppThreads / 32;

__global__ void __launch_bounds__(kAppThreads) gqa_append_kernel(const GqaAppendArgs a) {
  __shared__ float c_s[kAppTok][kAppK + 1];
  __shared__ __align__(16) float w_s[kAppK][128];
  __shared__ float r_s[kAppWarps][128];
  pdl_trigger();
  pdl_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tok0 = blockIdx.x * kAppTok, g = blockIdx.y, part = blockIdx.z;
  const int tok_end = min(tok0 + kAppTok, a.n_tok);

  if (part == 2) {
    if (g != 0) return;
    for (int i = tok0 + warp; i < tok_end; i += kAppWarps) {
      const int32_t s = a.slot[i];
      if (s < 0 || (int64_t)s >= a.n_slots) continue;     // outside the pool: skipped (warp-uniform)
      const __nv_bfloat16* kr = static_cast<const __nv_bfloat16*>(a.k_rope_raw) + (int64_t)i * a.d_rope;
      float x[4];
      float ss = 0.f;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int k = lane + 32 * q;
        x[q] = k < a.d_rope ? __bfloat162float(kr[k]) : 0.f;
        ss += x[q] * x[q];
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      const float inv = 1.0f / sqrtf(ss / (float)a.d_rope + a.eps);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int k = lane + 32 * q;
        if (k < a.d_rope) r_s[warp][k] = x[q] * inv * a.gamma_kr[k];
      }
      __syncwarp();
      __nv_bfloat16* out = static_cast<__nv_bfloat16*>(a.k_rope) + (int64_t)s * a.d_rope;
      const int half = a.d_rope / 2;
      const int32_t pos = a.pos[i];
      for (int k = lane; k < half; k += 32) {
        const float x1 = r_s[warp][k], x2 = r_s[warp][k + half];
        float sn, cs;
        rope_sincos(pos, a.freq.f[k], sn, cs);
        out[k] = __float2bfloat16_rn(x1 * cs - x2 * sn);
        out[k + half] = __float2bfloat16_rn(x2 * cs + x1 * sn);
      }
      __syncwarp();
    }
    return;
  }

  const int ncol = part == 0 ? a.d_h : a.d_v;        // <= 128, a multiple of 4
  const bool colok = 4 * lane < ncol;
  float acc[4][4];
#pragma unroll
  for (int u = 0; u < 4; ++u)
#pragma unroll
    for (int v = 0; v < 4; ++v) acc[u][v] = 0.f;
  const __nv_bfloat16* cn = static_cast<const __nv_bfloat16*>(a.c_new);
  const int c4n = ncol / 4;
  for (int k0 = 0; k0 < a.r; k0 += kAppK) {
    __syncthreads();
    {   // latent chunk [32 tokens][32 columns], four values per thread
      const int e = threadIdx.x * 4, t = e / kAppK, kk = e - t * kAppK;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (tok0 + t < a.n_tok)
        v = bf16x4_to_f32(*reinterpret_cast<const uint2*>(cn + (int64_t)(tok0 + t) * a.r + k0 + kk));
      c_s[t][kk] = v.x;
      c_s[t][kk + 1] = v.y;
      c_s[t][kk + 2] = v.z;
      c_s[t][kk + 3] = v.w;
    }
    // weight chunk [32 rows][ncol]
    for (int e = threadIdx.x; e < kAppK * c4n; e += kAppThreads) {
      const int kk = e / c4n, c4 = e - kk * c4n;
      const int64_t off = ((int64_t)g * a.r + k0 + kk) * ncol + 4 * c4;
      float4 w;
      if (part == 0)
        w = *reinterpret_cast<const float4*>(a.w_uk + off);
      else
        w = bf16x4_to_f32(*reinterpret_cast<const uint2*>(static_cast<const __nv_bfloat16*>(a.w_uv) + off));
      *reinterpret_cast<float4*>(&w_s[kk][4 * c4]) = w;
    }
    __syncthreads();
    if (colok) {
#pragma unroll 8
      for (int kk = 0; kk < kAppK; ++kk) {
        const float4 w = *reinterpret_cast<const float4*>(&w_s[kk][4 * lane]);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float c = c_s[4 * warp + u][kk];
          acc[u][0] = fmaf(c, w.x, acc[u][0]);
          acc[u][1] = fmaf(c, w.y, acc[u][1]);
          acc[u][2] = fmaf(c, w.z, acc[u][2]);
          acc[u][3] = fmaf(c, w.w, acc[u][3]);
        }
      }
    }
  }
  __nv_bfloat16* cache = static_cast<__nv_bfloat16*>(part == 0 ? a.k_cache : a.v_cache);
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int i = tok0 + 4 * warp + u;
    float scale = 1.f;
    if (part == 0) {   // 1 / S(k) over the d_h columns: one warp holds the row
      float ss = acc[u][0] * acc[u][0] + acc[u][1] * acc[u][1] + acc[u][2] * acc[u][2] + acc[u][3] * acc[u][3];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      scale = 1.0f / sqrtf(ss / (float)a.d_h + a.eps);
    }
    if (i >= a.n_tok || !colok) continue;
    const int32_t s = a.slot[i];
    if (s < 0 || (int64_t)s >= a.n_slots) continue;        // outside the pool: skipped
    const int64_t row = ((int64_t)(s / kBlockSize) * a.groups + g) * kBlockSize + s % kBlockSize;
    float v[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) v[q] = acc[u][q] * (part == 0 ? scale * a.gamma_k[g * a.d_h + 4 * lane + q] : 1.f);
    uint2 pk;
    pk.x = pack_bf16x2(v[0], v[1]);
    pk.y = pack_bf16x2(v[2], v[3]);
    *reinterpret_cast<uint2*>(cache + row * ncol + 4 * lane) = pk;
  }
}

// ------------------------------------------------------------------ decode
constexpr int kGqaThreads = 256;
constexpr int kGqaWarps = kGqaThreads / 32;
constexpr int kGqaStages = 4;        // cache pages in the ring
constexpr int kTok = kBlockSize;     // tokens per page (64)

// Shared-memory plan of one instantiation.  Row pitches are the row widths
// plus 8 elements (4 mod 8 words): 16-byte row starts for cp.async and
// ldmatrix, and the 8 rows of every 8 x 8 ldmatrix tile in distinct banks.
template <int MT, int DH, int DR, int DV>
struct GqaShape {
  static constexpr int MP = 16 * MT;                   // query rows of a tile
  static constexpr int KS = (DH + DR) / 16;            // k-steps of the score product
  static constexpr int KSC = DH / 16;                  // ... of which over the content block
  static constexpr int KP = DH + 8, RP = DR + 8, VP = DV + 8, QP = DH + DR + 8, PP = kTok + 8;
  static constexpr int CPR = (DH + DR + DV) / 8;       // 16-byte pieces of a token's rows
  static constexpr int K_OFF = 0;
  static constexpr int R_OFF = kTok * KP * 2;
  static constexpr int V_OFF = R_OFF + kTok * RP * 2;
  static constexpr int STAGE = V_OFF + kTok * VP * 2;  // bytes per ring stage
  static constexpr int Q_OFF = kGqaStages * STAGE;     // the tile's queries, bf16 [MP][QP]
  static constexpr int P_OFF = Q_OFF + MP * QP * 2;    // the page's probabilities, bf16 [MP][PP]
  static constexpr int WMAX_OFF = P_OFF + MP * PP * 2; // per column-warp row maxima [8][MP]
  static constexpr int WSUM_OFF = WMAX_OFF + kGqaWarps * MP * 4;
  static constexpr int M_OFF = WSUM_OFF + kGqaWarps * MP * 4;   // running maxima, two buffers [2][MP]
  static constexpr int L_OFF = M_OFF + 2 * MP * 4;              // running sums [MP]
  static constexpr int OK_OFF = L_OFF + MP * 4;                 // sparse: listed-token flags [stages][64]
  static constexpr int SMEM = OK_OFF + kGqaStages * kTok * 4;
  static constexpr int CWN = kGqaWarps / MT;           // warps over one m-tile's columns (score product)
  static constexpr int NC = DV / 16;                   // 16-column slices of the output
  static constexpr int TPW = (MT * NC + kGqaWarps - 1) / kGqaWarps;   // output slices per warp
  static_assert(KSC % 2 == 0 && (KS - KSC) % 2 == 0, "k-steps are taken in pairs within one block");
  static_assert(CPR % 4 == 0, "four threads per token row");
  static_assert(MT * NC <= kGqaWarps || NC == kGqaWarps, "a warp's output slices share their columns");
  static_assert(STAGE % 16 == 0 && (MP * QP * 2) % 16 == 0 && (MP * PP * 2) % 16 == 0, "16-byte offsets");
};

// What one item works on.
struct GqaTile {
  int32_t b, g, rb;      // sequence, KV group, row block of the group's rows
  int32_t j;             // sparse: the query token of the tile; dense: -1 (rows over all query tokens)
  int32_t L;             // sequence length
  int32_t u0, u1;        // dense: pages [u0, u1); sparse: 64-entry chunks of the token list
  int64_t slot;          // dense: workspace slot of the partial result
};

// Query token j and head h of tile row i; false for a padding row.
__device__ __forceinline__ bool tile_row(const GqaDecodeArgs& a, const GqaTile& t, int ng, int mp, int i, int& j,
                                         int& h) {
  if (t.j >= 0) {
    const int m = t.rb * mp + i;
    j = t.j;
    h = t.g * ng + m;
    return m < ng;
  }
  const int u = t.rb * mp + i;
  j = u / ng;
  h = t.g * ng + (u - j * ng);
  return u < a.s_q * ng;
}

template <int MT, int DH, int DR, int DV, bool SPARSE>
__device__ __forceinline__ void gqa_run_tile(const GqaDecodeArgs& a, const GqaTile& t, unsigned char* smem) {
  using S = GqaShape<MT, DH, DR, DV>;
  constexpr int MP = S::MP;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gid = lane >> 2, tig = lane & 3;
  const int ng = a.heads / a.groups;
  const uint32_t sbase = smem_u32(smem);
  __nv_bfloat16* q_s = reinterpret_cast<__nv_bfloat16*>(smem + S::Q_OFF);
  float* wmax_s = reinterpret_cast<float*>(smem + S::WMAX_OFF);
  float* wsum_s = reinterpret_cast<float*>(smem + S::WSUM_OFF);
  float* m_s = reinterpret_cast<float*>(smem + S::M_OFF);
  float* l_s = reinterpret_cast<float*>(smem + S::L_OFF);
  int32_t* ok_s = reinterpret_cast<int32_t*>(smem + S::OK_OFF);

  // ---- 1. the tile's queries: RMS-normalised with gamma_q, the RoPE block also rotated to the
  // query's position; one warp per row
  for (int i = warp; i < MP; i += kGqaWarps) {
    int j, h;
    const bool valid = tile_row(a, t, ng, MP, i, j, h);
    __nv_bfloat16* qrow = q_s + i * S::QP;
    if (lane == 0) {
      m_s[i] = -INFINITY;
      l_s[i] = 0.f;
    }
    if (!valid) {
      for (int d = lane; d < DH + DR; d += 32) qrow[d] = __float2bfloat16_rn(0.f);
      continue;
    }
    const int64_t qr = ((int64_t)t.b * a.s_q + j) * a.heads + h;
    const __nv_bfloat16* qp = static_cast<const __nv_bfloat16*>(a.q) + qr * DH;
    float x[DH / 32];
    float ss = 0.f;
#pragma unroll
    for (int q = 0; q < DH / 32; ++q) {
      x[q] = __bfloat162float(qp[lane + 32 * q]);
      ss += x[q] * x[q];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float inv = 1.0f / sqrtf(ss / (float)DH + a.eps);
#pragma unroll
    for (int q = 0; q < DH / 32; ++q)
      qrow[lane + 32 * q] = __float2bfloat16_rn(x[q] * inv * a.gamma_q[h * DH + lane + 32 * q]);
    const __nv_bfloat16* rp = static_cast<const __nv_bfloat16*>(a.q_rope) + qr * DR;
    const float* gr = a.gamma_qr + h * DR;
    const int32_t pos = t.L - a.s_q + j;
    if constexpr (DR == 64) {            // pair (lane, lane + 32) sits in this lane
      const float y1 = __bfloat162float(rp[lane]), y2 = __bfloat162float(rp[lane + 32]);
      float sr = y1 * y1 + y2 * y2;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sr += __shfl_xor_sync(0xffffffffu, sr, o);
      const float ir = 1.0f / sqrtf(sr / (float)DR + a.eps);
      const float x1 = y1 * ir * gr[lane], x2 = y2 * ir * gr[lane + 32];
      float sn, cs;
      rope_sincos(pos, a.freq.f[lane], sn, cs);
      qrow[DH + lane] = __float2bfloat16_rn(x1 * cs - x2 * sn);
      qrow[DH + lane + 32] = __float2bfloat16_rn(x2 * cs + x1 * sn);
    } else {                             // DR == 32: pair (k, k + 16) across lanes k and k ^ 16
      const float y = __bfloat162float(rp[lane]);
      float sr = y * y;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sr += __shfl_xor_sync(0xffffffffu, sr, o);
      const float xn = y * (1.0f / sqrtf(sr / (float)DR + a.eps)) * gr[lane];
      const float other = __shfl_xor_sync(0xffffffffu, xn, 16);
      const int k = lane & 15;
      float sn, cs;
      rope_sincos(pos, a.freq.f[k], sn, cs);
      const float x1 = lane < 16 ? xn : other, x2 = lane < 16 ? other : xn;
      qrow[DH + lane] = __float2bfloat16_rn(lane < 16 ? x1 * cs - x2 * sn : x2 * cs + x1 * sn);
    }
  }
  __syncthreads();

  // ---- 2. this warp's query fragments (the score product's A operand), kept in registers
  const int mt_w = warp / S::CWN, cw = warp % S::CWN;
  uint32_t qa[S::KS][4];
#pragma unroll
  for (int ks = 0; ks < S::KS; ++ks)
    ldsm_x4(sbase + S::Q_OFF + (uint32_t)(((mt_w * 16 + (lane & 15)) * S::QP + ks * 16 + (lane >> 4) * 8) * 2), qa[ks]);
  // the last visible position of this lane's two rows (gid, gid + 8 of the warp's m-tile); -1 for padding
  int32_t lim[2];
#pragma unroll
  for (int hf = 0; hf < 2; ++hf) {
    int j, h;
    const bool valid = tile_row(a, t, ng, MP, mt_w * 16 + gid + 8 * hf, j, h);
    lim[hf] = valid ? t.L - a.s_q + j : -1;
  }

  // ---- 3. the page ring: thread tid copies 16-byte pieces q4, q4 + 4, ... of token row tid / 4
  const int npg = t.u1 - t.u0;
  auto issue = [&](int u, int st) {
    const int n = tid >> 2, q4 = tid & 3;
    bool ok;
    int32_t blk = 0, off = n;
    if constexpr (SPARSE) {
      const int e = u * kTok + n;
      const int32_t tok = e < a.sel_k
                              ? a.selection[(((int64_t)t.b * a.s_q + t.j) * a.groups + t.g) * a.sel_k + e]
                              : -1;
      ok = tok >= 0 && tok <= t.L - a.s_q + t.j;
      if (q4 == 0) ok_s[st * kTok + n] = ok ? 1 : 0;
      if (ok) {
        blk = a.block_table[(int64_t)t.b * a.max_blocks + tok / kTok];
        off = tok % kTok;
      }
    } else {
      ok = u * kTok + n < t.L;
      blk = a.block_table[(int64_t)t.b * a.max_blocks + u];
    }
    if (ok && (blk < 0 || blk >= a.num_blocks)) {
      record_status(a.status, QKN_ERR_BOUNDS);
      blk = 0;
    }
    const uint32_t dst = sbase + (uint32_t)(st * S::STAGE);
    const int64_t grow = ((int64_t)blk * a.groups + t.g) * kTok + off;   // row of the per-group caches
    const int64_t rrow = (int64_t)blk * kTok + off;                       // row of the RoPE key cache
#pragma unroll
    for (int k = 0; k < S::CPR / 4; ++k) {
      const int c = q4 + 4 * k;
      uint32_t d;
      const __nv_bfloat16* src;
      if (c < DH / 8) {
        d = dst + S::K_OFF + (uint32_t)((n * S::KP + 8 * c) * 2);
        src = static_cast<const __nv_bfloat16*>(a.k_cache) + grow * DH + 8 * c;
      } else if (c < (DH + DR) / 8) {
        const int cr = c - DH / 8;
        d = dst + S::R_OFF + (uint32_t)((n * S::RP + 8 * cr) * 2);
        src = static_cast<const __nv_bfloat16*>(a.k_rope) + rrow * DR + 8 * cr;
      } else {
        const int cv = c - (DH + DR) / 8;
        d = dst + S::V_OFF + (uint32_t)((n * S::VP + 8 * cv) * 2);
        src = static_cast<const __nv_bfloat16*>(a.v_cache) + grow * DV + 8 * cv;
      }
      if (ok)
        cp_async16(d, src);
      else   // a token past the sequence's end or not listed: zeros, so that p = 0 never meets a NaN
        asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(d), "r"(0u), "r"(0u), "r"(0u), "r"(0u)
                     : "memory");
    }
  };
#pragma unroll
  for (int s = 0; s < kGqaStages - 1; ++s) {
    if (s < npg) issue(t.u0 + s, s);
    cp_async_commit();
  }

  float o[S::TPW][2][4];
#pragma unroll
  for (int u = 0; u < S::TPW; ++u)
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) o[u][nt][e] = 0.f;
  const int nc_w = warp % S::NC;                 // the output columns of this warp's slices

  for (int it = 0; it < npg; ++it) {
    cp_async_wait_group<kGqaStages - 2>();       // this page's copies (this thread's) have landed
    __syncthreads();                             // ... everyone's; and the page before is consumed
    if (it + kGqaStages - 1 < npg) issue(t.u0 + it + kGqaStages - 1, (it + kGqaStages - 1) % kGqaStages);
    cp_async_commit();
    const int st = it % kGqaStages;
    const int cur = it & 1, nxt = cur ^ 1;
    const uint32_t stage = sbase + (uint32_t)(st * S::STAGE);
    const int unit = t.u0 + it;

    // ---- scores of this warp's MT n-tiles (tokens tok0 .. tok0 + 8 MT - 1), two accumulators
    // (even and odd k-steps) to halve the dependent chain
    const int tok0 = cw * 8 * MT;
    float sa[MT][4], sb[MT][4];
#pragma unroll
    for (int nt = 0; nt < MT; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) sa[nt][e] = sb[nt][e] = 0.f;
#pragma unroll
    for (int ks = 0; ks < S::KS; ks += 2) {
#pragma unroll
      for (int nt = 0; nt < MT; ++nt) {
        const int row = tok0 + nt * 8 + (lane & 7);
        uint32_t addr;
        if (ks < S::KSC)
          addr = stage + S::K_OFF + (uint32_t)((row * S::KP + ks * 16 + (lane >> 3) * 8) * 2);
        else
          addr = stage + S::R_OFF + (uint32_t)((row * S::RP + (ks - S::KSC) * 16 + (lane >> 3) * 8) * 2);
        uint32_t bq[4];
        ldsm_x4(addr, bq);
        mma_bf16_m16n8k16(sa[nt], qa[ks], bq[0], bq[1]);
        mma_bf16_m16n8k16(sb[nt], qa[ks + 1], bq[2], bq[3]);
      }
    }
    float rmax[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int nt = 0; nt < MT; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int hf = e >> 1, col = tok0 + nt * 8 + 2 * tig + (e & 1);
        bool vis;
        if constexpr (SPARSE)
          vis = lim[hf] >= 0 && ok_s[st * kTok + col] != 0;
        else
          vis = unit * kTok + col <= lim[hf];
        sa[nt][e] = vis ? (sa[nt][e] + sb[nt][e]) * a.score_scale : -INFINITY;
        rmax[hf] = fmaxf(rmax[hf], sa[nt][e]);
      }
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      rmax[hf] = fmaxf(rmax[hf], __shfl_xor_sync(0xffffffffu, rmax[hf], 1));
      rmax[hf] = fmaxf(rmax[hf], __shfl_xor_sync(0xffffffffu, rmax[hf], 2));
    }
    if (tig == 0) {
      wmax_s[cw * MP + mt_w * 16 + gid] = rmax[0];
      wmax_s[cw * MP + mt_w * 16 + gid + 8] = rmax[1];
    }
    __syncthreads();

    // ---- softmax over the page: the row's new maximum, p = 2^(s - m) rounded to bf16 into P, and
    // the partial sums of the rounded values
    float psum[2] = {0.f, 0.f}, base[2];
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      const int row = mt_w * 16 + gid + 8 * hf;
      float mx = m_s[cur * MP + row];
#pragma unroll
      for (int c = 0; c < S::CWN; ++c) mx = fmaxf(mx, wmax_s[c * MP + row]);
      base[hf] = mx == -INFINITY ? 0.f : mx;
      if (cw == 0 && tig == 0) m_s[nxt * MP + row] = mx;
    }
#pragma unroll
    for (int nt = 0; nt < MT; ++nt)
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        const int row = mt_w * 16 + gid + 8 * hf, col = tok0 + nt * 8 + 2 * tig;
        const __nv_bfloat162 pv = __floats2bfloat162_rn(exp2f(sa[nt][2 * hf] - base[hf]),
                                                        exp2f(sa[nt][2 * hf + 1] - base[hf]));
        psum[hf] += __low2float(pv) + __high2float(pv);
        *reinterpret_cast<__nv_bfloat162*>(smem + S::P_OFF + (row * S::PP + col) * 2) = pv;
      }
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      psum[hf] += __shfl_xor_sync(0xffffffffu, psum[hf], 1);
      psum[hf] += __shfl_xor_sync(0xffffffffu, psum[hf], 2);
      if (tig == 0) wsum_s[cw * MP + mt_w * 16 + gid + 8 * hf] = psum[hf];
    }
    __syncthreads();

    // ---- running sums (one thread per row), then o = o * 2^(m_old - m_new) + P V
    if (tid < MP) {
      const float mo = m_s[cur * MP + tid], mn = m_s[nxt * MP + tid];
      float add = 0.f;
#pragma unroll
      for (int c = 0; c < S::CWN; ++c) add += wsum_s[c * MP + tid];
      l_s[tid] = l_s[tid] * (mo == -INFINITY ? 0.f : exp2f(mo - mn)) + add;
    }
#pragma unroll
    for (int u = 0; u < S::TPW; ++u) {
      const int task = warp + kGqaWarps * u;
      if (task >= MT * S::NC) continue;
      const int mt_t = task / S::NC;
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        const int row = mt_t * 16 + gid + 8 * hf;
        const float mo = m_s[cur * MP + row], mn = m_s[nxt * MP + row];
        const float corr = mo == -INFINITY ? 0.f : exp2f(mo - mn);
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          o[u][nt][2 * hf] *= corr;
          o[u][nt][2 * hf + 1] *= corr;
        }
      }
    }
    if (warp < MT * S::NC) {
#pragma unroll
      for (int ks = 0; ks < kTok / 16; ++ks) {
        uint32_t bv[4];
        ldsm_x4_trans(stage + S::V_OFF + (uint32_t)(((ks * 16 + (lane & 15)) * S::VP + nc_w * 16 + (lane >> 4) * 8) * 2),
                      bv);
#pragma unroll
        for (int u = 0; u < S::TPW; ++u) {
          const int task = warp + kGqaWarps * u;
          if (task >= MT * S::NC) continue;
          const int mt_t = task / S::NC;
          uint32_t ap[4];
          ldsm_x4(sbase + S::P_OFF + (uint32_t)(((mt_t * 16 + (lane & 15)) * S::PP + ks * 16 + (lane >> 4) * 8) * 2),
                  ap);
          mma_bf16_m16n8k16(o[u][0], ap, bv[0], bv[1]);
          mma_bf16_m16n8k16(o[u][1], ap, bv[2], bv[3]);
        }
      }
    }
  }
  cp_async_wait_group<0>();                      // only empty groups can remain
  __syncthreads();                               // the last running sums

  // ---- 4. normalised output: the partial result of a split (dense) or the row's result (sparse)
  const int fin = npg & 1;                       // buffer of the final maxima
#pragma unroll
  for (int u = 0; u < S::TPW; ++u) {
    const int task = warp + kGqaWarps * u;
    if (task >= MT * S::NC) continue;
    const int mt_t = task / S::NC, nc_t = task % S::NC;
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      const int row = mt_t * 16 + gid + 8 * hf;
      int j, h;
      if (!tile_row(a, t, ng, MP, row, j, h)) continue;
      const float l = l_s[row];
      const float inv = l > 0.f ? 1.0f / l : 0.f;
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        const int col = nc_t * 16 + nt * 8 + 2 * tig;
        const float v0 = o[u][nt][2 * hf] * inv, v1 = o[u][nt][2 * hf + 1] * inv;
        if constexpr (SPARSE) {
          __nv_bfloat16* out = static_cast<__nv_bfloat16*>(a.out) + (((int64_t)t.b * a.s_q + j) * a.heads + h) * DV;
          *reinterpret_cast<uint32_t*>(out + col) = pack_bf16x2(v0, v1);
        } else {
          *reinterpret_cast<float2*>(a.part_o + (t.slot * MP + row) * DV + col) = make_float2(v0, v1);
        }
      }
    }
  }
  if (tid < MP) {
    const float l = l_s[tid];
    const float lse = l > 0.f ? (m_s[fin * MP + tid] + log2f(l)) * 0.6931471805599453f : -INFINITY;
    if constexpr (SPARSE) {
      int j, h;
      if (tile_row(a, t, ng, MP, tid, j, h)) a.lse[((int64_t)t.b * a.s_q + j) * a.heads + h] = lse;
    } else {
      a.part_lse[t.slot * MP + tid] = lse;
    }
  }
  __syncthreads();                               // before the next tile's queries and running state
}

template <int MT, int DH, int DR, int DV, bool SPARSE>
__global__ void __launch_bounds__(kGqaThreads, 1) gqa_decode_kernel(const GqaDecodeArgs a) {
  using S = GqaShape<MT, DH, DR, DV>;
  extern __shared__ __align__(128) unsigned char gqa_smem[];
  __shared__ Cursor cur_s;
  pdl_trigger();
  pdl_wait();
  if constexpr (SPARSE) {
    // one tile per (sequence, query token, group, row block), all of its list's chunks
    const int per_b = a.s_q * a.groups * a.tpg;
    const int64_t tiles = (int64_t)a.batch * per_b;
    for (int64_t x = blockIdx.x; x < tiles; x += gridDim.x) {
      GqaTile t;
      t.b = (int32_t)(x / per_b);
      int rem = (int)(x - (int64_t)t.b * per_b);
      t.j = rem / (a.groups * a.tpg);
      rem -= t.j * (a.groups * a.tpg);
      t.g = rem / a.tpg;
      t.rb = rem - t.g * a.tpg;
      t.L = a.seq_lens[t.b];
      t.u0 = 0;
      t.u1 = (a.sel_k + kTok - 1) / kTok;
      t.slot = 0;
      if (t.L < a.s_q || t.L > a.max_blocks * kTok) {
        // rejected length: zero rows, lse = -inf (CTA-uniform)
        if (threadIdx.x == 0) record_status(a.status, QKN_ERR_BOUNDS);
        const int ng = a.heads / a.groups;
        for (int e = threadIdx.x; e < S::MP * DV; e += kGqaThreads) {
          int j, h;
          const int i = e / DV, col = e - i * DV;
          if (!tile_row(a, t, ng, S::MP, i, j, h)) continue;
          const int64_t row = ((int64_t)t.b * a.s_q + j) * a.heads + h;
          static_cast<__nv_bfloat16*>(a.out)[row * DV + col] = __float2bfloat16_rn(0.f);
          if (col == 0) a.lse[row] = -INFINITY;
        }
        continue;
      }
      gqa_run_tile<MT, DH, DR, DV, true>(a, t, gqa_smem);
    }
  } else {
    SchedParams sp{a.seq_lens, a.batch, a.s_q, a.max_blocks, a.ht_count, a.ncta, a.item_cost};
    if (threadIdx.x < 32) {
      Cursor c = sched_begin(sp, blockIdx.x);
      if (threadIdx.x == 0) cur_s = c;
    }
    __syncthreads();
    Cursor cur = cur_s;
    Item it;
    while (sched_next(cur, sp, blockIdx.x, it)) {
      GqaTile t;
      t.b = it.b;
      t.g = it.ht / a.tpg;
      t.rb = it.ht - t.g * a.tpg;
      t.j = -1;
      t.L = it.L;
      t.u0 = it.p0;
      t.u1 = it.p1;
      t.slot = it.slot;
      gqa_run_tile<MT, DH, DR, DV, false>(a, t, gqa_smem);
    }
  }
}

template <int MT, int DH, int DR, int DV>
cudaError_t launch_gqa_shape(const GqaDecodeArgs& a, cudaStream_t st) {
  using S = GqaShape<MT, DH, DR, DV>;
  static PerDeviceOnce attrs;
  cudaError_t e = once_per_device(attrs, [] {
    cudaError_t r = set_smem_attrs(gqa_decode_kernel<MT, DH, DR, DV, false>, S::SMEM);
    return r != cudaSuccess ? r : set_smem_attrs(gqa_decode_kernel<MT, DH, DR, DV, true>, S::SMEM);
  });
  if (e != cudaSuccess) return e;
  if (a.selection) {
    const int64_t tiles = (int64_t)a.batch * a.s_q * a.groups * a.tpg;
    const unsigned grid = (unsigned)(tiles < (1LL << 30) ? tiles : (1LL << 30));
    return launch_chained(gqa_decode_kernel<MT, DH, DR, DV, true>, dim3(grid), dim3(kGqaThreads), (size_t)S::SMEM,
                          st, a);
  }
  return launch_chained(gqa_decode_kernel<MT, DH, DR, DV, false>, dim3(a.ncta), dim3(kGqaThreads), (size_t)S::SMEM,
                        st, a);
}

}  // namespace

bool gqa_supported(int d_h, int d_rope, int d_v) {
  return (d_h == 128 && d_rope == 64 && d_v == 128) || (d_h == 64 && d_rope == 32 && d_v == 64);
}

cudaError_t launch_gqa_append(const GqaAppendArgs& a, cudaStream_t st) {
  const dim3 grid((unsigned)((a.n_tok + kAppTok - 1) / kAppTok), (unsigned)a.groups, 3);
  return launch_chained(gqa_append_kernel, grid, dim3(kAppThreads), 0, st, a);
}

cudaError_t launch_gqa_decode(const GqaDecodeArgs& a, cudaStream_t st) {
  if (a.rows != 16 && a.rows != 32) return cudaErrorInvalidValue;
  const bool two = a.rows == 32;
  if (a.d_h == 128 && a.d_rope == 64 && a.d_v == 128)
    return two ? launch_gqa_shape<2, 128, 64, 128>(a, st) : launch_gqa_shape<1, 128, 64, 128>(a, st);
  if (a.d_h == 64 && a.d_rope == 32 && a.d_v == 64)
    return two ? launch_gqa_shape<2, 64, 32, 64>(a, st) : launch_gqa_shape<1, 64, 32, 64>(a, st);
  return cudaErrorNotSupported;
}

}  // namespace qkn
