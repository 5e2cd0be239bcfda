// Split-KV QK-Normed MLA decode on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// What it computes ("QK-Normed MLA: QK normalization without full key
// caching", technical summary, Metodología, decode-logit equation; the
// scalar factors are fused into the attention kernel as the summary's
// caveats ask): for every query row rho of a tile and every cached token t
//   l[t, rho] = a_q[rho] * a_k[t, g(rho)] * (c_t . q~[rho]) + k^R^_t . q^R^[rho]
// then an online softmax over the CTA's token range and O = sum_t p * c_t.
//
// Orientation ("swap AB"): tokens are the MMA M dimension and query rows are
// N (R = 16, 32 or 64).  A tile is one 64-token cache page:
//   S^T[64 x R]   = C[64 x 512] . Q~^T            (K = latent, 32 MMAs, M = 64)
//   S_R^T[64 x R] = K^R[64 x 64] . Q^R^T          (K = RoPE,   4 MMAs, M = 64)
//   O^T[512 x R] += C^T[512 x 64] . P^T[64 x R]   (4 latent blocks x 4 MMAs, M = 128)
// with the page's latent staged once in shared memory and read by both
// products (as K-major A for S, as MN-major A for O).  One page (72 KB with
// its RoPE key) is small enough that two to three pages stay resident, so
// the loads of the next pages run while the softmax and the output product
// of the current page hold theirs.
//
// Tensor memory: O^T takes 4R columns over all 128 lanes; S^T and S_R^T take
// R columns each in the 64-row layout (token m in lane (m % 16) + 32 (m / 16))
// and are double buffered, so that the scores of page i+1 are computed while
// the softmax and the output product of page i run.
//
// Warp roles (352 threads, one CTA per SM):
//   warps 0-7  softmax + epilogue, two groups of four warps that split the
//              query rows of the tile: group h takes columns [hR/2, (h+1)R/2)
//              of S^T and O^T.  Within a group, warp w (mod 4) reads TMEM lanes
//              32w..32w+31, so lane i < 16 of it owns token 16w + i of a page
//              and thread t owns latent row t of each O^T block; column maxima
//              and sums are reduced across the group's 128 threads.  A column
//              never leaves its group, so the groups synchronise only through
//              the tile barriers;
//   warp 8     TMA producer: query tiles per item, then per page four 16 KB
//              latent slots, the RoPE-key chunk and the a_k rows; the whole
//              warp reads the block table 32 entries at a time;
//   warp 9     TMEM allocator and issuer of the score MMAs (S^T, S_R^T);
//   warp 10    issuer of the output MMAs (O^T).
// A single thread issues tcgen05.mma at a bounded rate, so the two products
// have one issuing thread each, and every shared-memory descriptor is built
// once: a K step or a ring slot only moves its start-address field.
// Every mbarrier wait is bounded; a wait that runs out records
// QKN_ERR_TIMEOUT in the workspace status word and the CTA winds down.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace qkn {
using namespace sm100;

namespace {

constexpr int kPage = 64;                   // tokens per tile (one cache page; MMA M of the score product)
constexpr int kRkv = 512;                   // latent width this kernel takes
constexpr int kChunks = kRkv / 64;          // 64-column (128-byte) chunks of the latent
constexpr int kDrope = 64;                  // RoPE width this kernel takes
constexpr int kChunkBytes = kPage * 128;    // one 64-column chunk of one page: 8 KB
constexpr int kSlotBytes = 2 * kChunkBytes; // a ring slot holds one 128-column latent block of a page: 16 KB
constexpr int kSlotsPerTile = kChunks / 2;
constexpr int kKrBytes = kPage * kDrope * 2;            // RoPE keys of one page: 8 KB
constexpr int kMaxGroups = 8;
constexpr int kAkSlotBytes = kPage * kMaxGroups * 4;    // a_k rows of one page: up to 2 KB
constexpr int kSoftWarps = 8;               // two groups of four
constexpr int kSoftThreads = kSoftWarps * 32;
constexpr int kGroupThreads = 128;
constexpr int kProducerWarp = kSoftWarps;   // then the two MMA issuers
constexpr int kScoreWarp = kSoftWarps + 1;
constexpr int kOutWarp = kSoftWarps + 2;
constexpr int kThreads = (kSoftWarps + 3) * 32;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleLog2 = 8.0f;        // rescale O only when a column max grows by > 2^8
constexpr int64_t kDrainLimit = 4000000000LL;
constexpr int kEarlyPages = 2;            // pages the producer may issue before the query tile (ring holds >= 2)

template <int R>
struct Cfg {
  // RoPE-key / a_k / P^T slots: a page holds one from its load until its output MMAs finish; at R = 64
  // two suffice (the latent ring holds two pages), which leaves room for an eighth latent slot
  static constexpr int NKR = (R == 64) ? 2 : 4;
  static constexpr int TMEM_COLS = (8 * R <= 128) ? 128 : (8 * R <= 256 ? 256 : 512);
  static constexpr int Q_OFF = 0;                                    // R x 512 bf16, 8 chunks
  static constexpr int QR_OFF = Q_OFF + R * 1024;                    // R x 64 bf16
  static constexpr int KR_OFF = QR_OFF + ((R * 128 + 1023) / 1024) * 1024;
  static constexpr int AK_OFF = KR_OFF + NKR * kKrBytes;
  static constexpr int MISC_OFF = AK_OFF + NKR * kAkSlotBytes;
  static constexpr int MISC_BYTES = 4096;
  static constexpr int C_OFF = MISC_OFF + MISC_BYTES;                // 1024-aligned: every term above is
  static constexpr int kBudget = 232448 - 1024;                      // opt-in maximum less alignment slack
  static constexpr int NS = (kBudget - C_OFF) / kSlotBytes;          // latent ring slots (one block of a page each)
  static constexpr int SMEM = C_OFF + NS * kSlotBytes + 1024;
  static_assert(C_OFF % 1024 == 0, "swizzle atoms need 1024-byte alignment");
  static_assert(NS >= kSlotsPerTile + 2, "the ring must hold more than one page");
  static_assert(SMEM <= 232448, "shared memory budget");
  static_assert(4 * R + 2 * 2 * R <= TMEM_COLS, "tensor memory budget");
};

template <int R, int NS, int NKR>
struct Misc {
  uint64_t full[NS], empty[NS], krfull[NKR], krempty[NKR];
  uint64_t akfull[NKR];           // the page's a_k rows landed (read by the softmax only)
  uint64_t s_full[2], s_empty[2];
  // Per-tile handshakes alternate between two barriers by tile parity (tile n: barrier n & 1,
  // phase n >> 1): the softmax may run two tiles ahead of the output issuer, and a parity wait
  // needs the barrier to be at most one phase past the phase waited for.
  uint64_t p_full[2];             // P^T of tile n written
  uint64_t pv_done[2];            // output MMAs of tile n complete
  uint64_t q_full, q_empty, o_empty, drain;
  uint32_t tmem_base;
  int32_t abort_flag;
  Cursor cursor;
  alignas(16) float aq2[R];      // a_q * log2(e) per column (query row)
  alignas(16) int32_t grp[R];    // KV group per column
  alignas(16) int32_t qlim[R];   // last visible token position per column (-1: padding column)
  alignas(16) float mu[R];       // running max (log2 units) used for the exponentials
  alignas(16) float corr[R];     // rescale factor of the current tile
  alignas(16) float linv[R];
  alignas(16) float red[4][R];   // partial column reductions of the four warps of each group
};

}  // namespace

struct TcMaps {
  CUtensorMap latent;   // [8 chunks][num_blocks*64 rows][64] bf16 view of the latent, box 2 x 64 x 64
  CUtensorMap krope;    // [num_blocks*64, 64]  bf16, box 64 x 64
  CUtensorMap qt;       // [n_q*H, 512]         bf16, box 64 x R
  CUtensorMap qr;       // [n_q*H, 64]          bf16, box 64 x R
};

// Column reduction across the 32 lanes of a warp: on entry each lane holds R
// values (one per column); on exit lane L holds the reduction over the warp's
// 32 rows of columns [L*R/32, (L+1)*R/32) (R >= 32) or of column L*R/32
// (R < 32; neighbouring lanes hold the same column).  Each step hands half of
// the remaining columns to the partner lane, so the whole reduction takes
// R-1 shuffles (plus plain butterflies once one column is left).
template <int R, bool MAX>
__device__ __forceinline__ void warp_col_reduce(float (&v)[R], int lane) {
#pragma unroll
  for (int s = 0; s < 5; ++s) {
    const int len = R >> s;
    const int bit = 16 >> s;
    const bool upper = (lane & bit) != 0;
    if (len >= 2) {
      const int half = len / 2;
#pragma unroll
      for (int c = 0; c < half; ++c) {
        const float send = upper ? v[c] : v[c + half];
        const float keep = upper ? v[c + half] : v[c];
        const float got = __shfl_xor_sync(0xffffffffu, send, bit);
        v[c] = MAX ? fmaxf(keep, got) : keep + got;
      }
    } else {
      const float got = __shfl_xor_sync(0xffffffffu, v[0], bit);
      v[0] = MAX ? fmaxf(v[0], got) : v[0] + got;
    }
  }
}

// Write the warp-reduced columns of this lane into red[warp][...].
template <int R>
__device__ __forceinline__ void store_reduced(float* red_w, const float (&v)[R], int lane) {
  if constexpr (R >= 32) {
    constexpr int per = R / 32;
#pragma unroll
    for (int i = 0; i < per; ++i) red_w[lane * per + i] = v[i];
  } else {
    constexpr int share = 32 / R;
    if ((lane % share) == 0) red_w[lane / share] = v[0];
  }
}

// Votes over the 128 threads that share named barrier `bar` (one barrier per softmax group).
__device__ __forceinline__ bool group_all(bool ok, uint32_t bar) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, %2, 128, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)ok), "r"(bar)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ bool group_any(bool v, uint32_t bar) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, 128, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v), "r"(bar)
      : "memory");
  return r != 0;
}

// SKIP: long chunks of queries (a prefill): an item ends at the last page its tile's rows can see,
// so an item may have no pages (separate instantiation, so that the decode's code is unchanged).
template <int R, bool AK_ONE, bool SKIP>
__global__ void __launch_bounds__(kThreads, 1) decode_tc_kernel(const DecodeArgs a, const __grid_constant__ TcMaps maps) {
  using C = Cfg<R>;
  constexpr int NS = C::NS, NKR = C::NKR;
  using MiscT = Misc<R, NS, NKR>;
  static_assert(sizeof(MiscT) <= C::MISC_BYTES, "misc shared-memory block");
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte alignment for the 128-byte swizzle atoms, by pointer arithmetic on the shared
  // array so that every access below stays a shared-memory (not generic) access
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  MiscT& ms = *reinterpret_cast<MiscT*>(smem + C::MISC_OFF);
  const uint32_t sb = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const SchedParams sp{a.seq_lens, a.batch, a.s_q, a.max_blocks, a.ht_count, a.ncta, a.item_cost,
                       SKIP ? a.heads : 0, a.rows, a.vis_end};
  const int qrows = a.s_q * a.heads;
  const int G = a.groups;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(smem_u32(&ms.full[s]), 1);
      mbar_init(smem_u32(&ms.empty[s]), 1);
    }
    for (int s = 0; s < NKR; ++s) {
      mbar_init(smem_u32(&ms.krfull[s]), 1);
      mbar_init(smem_u32(&ms.akfull[s]), 1);
      mbar_init(smem_u32(&ms.krempty[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&ms.s_full[b]), 1);
      mbar_init(smem_u32(&ms.s_empty[b]), kSoftThreads);
      mbar_init(smem_u32(&ms.pv_done[b]), 1);
      mbar_init(smem_u32(&ms.p_full[b]), kSoftThreads);
    }
    mbar_init(smem_u32(&ms.q_full), 1);
    mbar_init(smem_u32(&ms.q_empty), 1);
    mbar_init(smem_u32(&ms.o_empty), kSoftThreads);
    mbar_init(smem_u32(&ms.drain), 2);     // one commit from each MMA issuer
    ms.abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == kProducerWarp && lane == 0) {
    prefetch_tmap(&maps.latent);
    prefetch_tmap(&maps.krope);
    prefetch_tmap(&maps.qt);
    prefetch_tmap(&maps.qr);
  }
  if (warp == kScoreWarp) {
    tmem_alloc(smem_u32(&ms.tmem_base), C::TMEM_COLS);
    tmem_relinquish();
  }
  // everything above touches only this CTA's own memory.  By default every input is read after the
  // wait for the preceding kernel; with step_writes_only the lengths, the block table and the cache
  // pages without new tokens are not written by it, so the schedule and the producer start at once
  // and only the query tile, the pages with new tokens and the softmax (a_q) wait.
  pdl_trigger();
  if (!a.step_writes_only) pdl_wait();
  if (warp == 0) {
    Cursor c = sched_begin(sp, blockIdx.x);
    if (lane == 0) ms.cursor = c;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ms.tmem_base;
  Cursor cur = ms.cursor;
  Item it;

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------ producer (whole warp, elected issue)
    RingPos<NS> cw;
    RingPos<NKR> kw;
    int64_t c_issued = 0, k_issued = 0;
    int n_item = 0;
    bool ok = true;
    const uint32_t akpage = (uint32_t)kPage * (uint32_t)G * 4u;
    bool waited = !a.step_writes_only;
    int early_pages = 0;                  // pages issued before the first query tile
    int q_last = -1;                      // item whose query tile was issued last
    while (ok && sched_next(cur, sp, blockIdx.x, it)) {
      const int32_t* row = a.block_table + (int64_t)it.b * a.max_blocks;
      // the first 32 block-table entries of the item are read before the query tile is issued, so
      // that the two memory latencies overlap
      int32_t mine = (it.p0 + lane < it.p1) ? row[it.p0 + lane] : 0;
      // The query tile is issued at once unless the first pages may stream before the wait: then it
      // goes out before the first page with new tokens or once the ring holds kEarlyPages pages
      // (the score MMAs, which free the ring, need it).
      bool q_pending = true;
      auto issue_q = [&]() -> bool {
        if (!waited) {
          pdl_wait();
          waited = true;
        }
        if (!mbar_wait_warp(smem_u32(&ms.q_empty), (n_item & 1) ^ 1, a.wait_limit)) return false;
        const int qrow0 = it.b * qrows + it.ht * R;
        const uint32_t qf = smem_u32(&ms.q_full);
        mbar_arrive_expect_tx_elect(qf, R * 1024 + R * 128);
#pragma unroll
        for (int k = 0; k < kChunks; ++k) tma_load_2d_elect(sb + C::Q_OFF + k * R * 128, &maps.qt, k * 64, qrow0, qf);
        tma_load_2d_elect(sb + C::QR_OFF, &maps.qr, 0, qrow0, qf);
        q_pending = false;
        q_last = n_item;
        return true;
      };
      if (waited && !issue_q()) { ok = false; break; }
      // pages from here on hold this step's tokens
      const int first_new_page = ((a.vis_end ? a.vis_end[it.b] : it.L) - a.s_q) / kPage;
      for (int pb = it.p0; pb < it.p1 && ok; pb += 32) {
        // 32 block-table entries per warp-wide load
        if (pb > it.p0) mine = (pb + lane < it.p1) ? row[pb + lane] : 0;
        if (mine < 0 || mine >= a.num_blocks) {
          record_status(a.status, QKN_ERR_BOUNDS);
          mine = 0;
        }
        const int cnt = min(32, it.p1 - pb);
        for (int k = 0; k < cnt && ok; ++k) {
          const int32_t blk = __shfl_sync(0xffffffffu, mine, k);
          if (q_pending && (pb + k >= first_new_page || early_pages >= kEarlyPages)) {
            if (!issue_q()) { ok = false; break; }
          }
          if (q_pending) ++early_pages;
          for (int m = 0; m < kSlotsPerTile; ++m) {
            if (!mbar_wait_warp(smem_u32(&ms.empty[cw.slot]), cw.phase ^ 1u, a.wait_limit)) { ok = false; break; }
            const uint32_t fb = smem_u32(&ms.full[cw.slot]);
            mbar_arrive_expect_tx_elect(fb, kSlotBytes);
            const uint32_t dst = sb + C::C_OFF + cw.slot * kSlotBytes;
            tma_load_3d_elect(dst, &maps.latent, 0, blk * kPage, 2 * m, fb);   // chunks 2m, 2m+1 of the page
            cw.next();
            ++c_issued;
          }
          if (!ok) break;
          if (!mbar_wait_warp(smem_u32(&ms.krempty[kw.slot]), kw.phase ^ 1u, a.wait_limit)) { ok = false; break; }
          // the RoPE keys feed the score MMAs; the a_k rows only the softmax, so they get their own
          // barrier and their latency stays off the score path
          const uint32_t kb = smem_u32(&ms.krfull[kw.slot]);
          mbar_arrive_expect_tx_elect(kb, kKrBytes);
          tma_load_2d_elect(sb + C::KR_OFF + kw.slot * kKrBytes, &maps.krope, 0, blk * kPage, kb);
          // (a test of the timeout path withholds the first page's a_k copy: nothing else completes
          // that barrier phase, so the softmax's bounded wait for it runs out)
          if (!AK_ONE && !(a.withhold_ak && k_issued == 0)) {
            const uint32_t akb = smem_u32(&ms.akfull[kw.slot]);
            mbar_arrive_expect_tx_elect(akb, akpage);
            bulk_load_elect(sb + C::AK_OFF + kw.slot * kAkSlotBytes, a.a_k + (int64_t)blk * kPage * G, akpage, akb);
          }
          kw.next();
          ++k_issued;
        }
      }
      if (ok && q_pending && !issue_q()) ok = false;
      ++n_item;
    }
    if (!waited) pdl_wait();
    if (!ok && lane == 0) {
      record_status(a.status, QKN_ERR_TIMEOUT);
      ms.abort_flag = 1;
      // let the copies already in flight land before the CTA's memory is released
      const int64_t first = c_issued > NS ? c_issued - NS : 0;
      for (int64_t i = first; i < c_issued; ++i)
        mbar_wait(smem_u32(&ms.full[i % NS]), (i / NS) & 1, kDrainLimit);
      const int64_t kfirst = k_issued > NKR ? k_issued - NKR : 0;
      for (int64_t i = kfirst; i < k_issued; ++i) {
        mbar_wait(smem_u32(&ms.krfull[i % NKR]), (i / NKR) & 1, kDrainLimit);
        if (!AK_ONE && !(a.withhold_ak && i == 0))
          mbar_wait(smem_u32(&ms.akfull[i % NKR]), (i / NKR) & 1, kDrainLimit);
      }
      // and the last query tile (the one before it was complete when its q_empty wait returned)
      if (q_last >= 0) mbar_wait(smem_u32(&ms.q_full), (uint32_t)(q_last & 1), kDrainLimit);
    }
  } else if (warp == kScoreWarp) {
    // ------------------------------------------------------------ score MMA issuer (whole warp)
    constexpr uint32_t idS = idesc_bf16(kPage, R, false, false);
    const uint64_t dC = smem_desc(sb + C::C_OFF, 16, 1024);
    const uint64_t dQ = smem_desc(sb + C::Q_OFF, 16, 1024);
    const uint64_t dKR = smem_desc(sb + C::KR_OFF, 16, 1024);
    const uint64_t dQR = smem_desc(sb + C::QR_OFF, 16, 1024);
    RingPos<NS> cr;
    RingPos<NKR> kr;
    RingPos<2> sbuf;          // S buffer of the tile, and the phase of its use
    int n_item = 0;
    bool ok = true;
    while (ok && sched_next(cur, sp, blockIdx.x, it)) {
      if (!mbar_wait_warp(smem_u32(&ms.q_full), n_item & 1, a.wait_limit)) { ok = false; break; }
      tc_fence_after();
      for (int p = it.p0; p < it.p1 && ok; ++p) {
        // S buffer b was last read by the softmax of the tile two back
        const int b = sbuf.slot;
        if (!mbar_wait_warp(smem_u32(&ms.s_empty[b]), sbuf.phase ^ 1u, a.wait_limit)) { ok = false; break; }
        tc_fence_after();
        const uint32_t tS = tmem + 4 * R + b * 2 * R;
        // S^T = C . Q~^T over the 8 latent chunks, two chunks per ring slot
        for (int m = 0; m < kSlotsPerTile; ++m) {
          if (!mbar_wait_warp(smem_u32(&ms.full[cr.slot]), cr.phase, a.wait_limit)) { ok = false; break; }
          tc_fence_after();
          const uint64_t a0 = dC + (uint64_t)(cr.slot * (kSlotBytes >> 4));
          const uint64_t b0 = dQ + (uint64_t)(m * ((2 * R * 128) >> 4));
#pragma unroll
          for (int u = 0; u < 8; ++u) {   // chunk u / 4 of the slot, K step u % 4 (32 bytes) inside it
            const uint32_t aoff = (uint32_t)(((u >> 2) * kChunkBytes + (u & 3) * 32) >> 4);
            const uint32_t boff = (uint32_t)(((u >> 2) * R * 128 + (u & 3) * 32) >> 4);
            mma_bf16_elect(tS, a0 + aoff, b0 + boff, idS, (m | u) != 0 ? 1u : 0u);
          }
          cr.next();
        }
        if (!ok) break;
        // S_R^T = K^R . Q^R^T
        if (!mbar_wait_warp(smem_u32(&ms.krfull[kr.slot]), kr.phase, a.wait_limit)) { ok = false; break; }
        tc_fence_after();
        const uint64_t akr = dKR + (uint64_t)(kr.slot * (kKrBytes >> 4));
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) mma_bf16_elect(tS + R, akr + 2 * kk, dQR + 2 * kk, idS, kk != 0 ? 1u : 0u);
        mma_commit_elect(smem_u32(&ms.s_full[b]));
        kr.next();
        sbuf.next();
      }
      if (!ok) break;
      mma_commit_elect(smem_u32(&ms.q_empty));
      ++n_item;
    }
    if (!ok && lane == 0) {
      record_status(a.status, QKN_ERR_TIMEOUT);
      ms.abort_flag = 1;
    }
    // every MMA issued so far must finish before the tensor memory is freed
    mma_commit_elect(smem_u32(&ms.drain));
    mbar_wait_warp(smem_u32(&ms.drain), 0, kDrainLimit);
  } else if (warp == kOutWarp) {
    // ------------------------------------------------------------ output MMA issuer (whole warp)
    constexpr uint32_t idPV = idesc_bf16(128, R, true, true);
    // P^T is stored token-major (MN-major B): rows of 2R bytes, swizzled with the matching width
    constexpr uint32_t kPswz = (R == 16) ? 6u : (R == 32) ? 4u : 2u;   // 32 / 64 / 128-byte swizzle
    // A = C^T of one latent block (MN-major: the two chunks of a slot are LBO apart, 8-token groups SBO apart)
    const uint64_t dCt = smem_desc(sb + C::C_OFF, kChunkBytes, 1024);
    // B = P^T (MN-major, 2R-byte rows, SBO = eight rows)
    const uint64_t dP = smem_desc_sw(sb + C::KR_OFF, 16, 16 * R, kPswz);
    RingPos<NS> cr;
    RingPos<NKR> kr;
    RingPos<2> pb;            // P / output handshake barrier of the tile, and the phase of its use
    int n_item = 0;
    bool ok = true;
    while (ok && sched_next(cur, sp, blockIdx.x, it)) {
      // O^T of the previous item must have been read out before it is overwritten; with empty items
      // possible it is waited once per item, pages or not, so that the barrier is never more than one
      // phase ahead
      if (SKIP && !mbar_wait_warp(smem_u32(&ms.o_empty), (n_item & 1) ^ 1, a.wait_limit)) { ok = false; break; }
      for (int p = it.p0; p < it.p1 && ok; ++p) {
        if (!SKIP && p == it.p0 && !mbar_wait_warp(smem_u32(&ms.o_empty), (n_item & 1) ^ 1, a.wait_limit)) {
          ok = false;
          break;
        }
        if (!mbar_wait_warp(smem_u32(&ms.p_full[pb.slot]), pb.phase, a.wait_limit)) { ok = false; break; }
        tc_fence_after();
        const uint64_t bP = dP + (uint64_t)(kr.slot * (kKrBytes >> 4));
        const uint32_t acc0 = p > it.p0 ? 1u : 0u;
        for (int m = 0; m < kSlotsPerTile; ++m) {
          const uint64_t a0 = dCt + (uint64_t)(cr.slot * (kSlotBytes >> 4));
#pragma unroll
          for (int kk = 0; kk < kPage / 16; ++kk)
            mma_bf16_elect(tmem + m * R, a0 + (uint64_t)((kk * 2048) >> 4), bP + (uint64_t)((kk * 32 * R) >> 4), idPV,
                           kk > 0 ? 1u : acc0);
          mma_commit_elect(smem_u32(&ms.empty[cr.slot]));
          cr.next();
        }
        mma_commit_elect(smem_u32(&ms.krempty[kr.slot]));
        mma_commit_elect(smem_u32(&ms.pv_done[pb.slot]));
        kr.next();
        pb.next();
      }
      if (!ok) break;
      ++n_item;
    }
    if (!ok && lane == 0) {
      record_status(a.status, QKN_ERR_TIMEOUT);
      ms.abort_flag = 1;
    }
    mma_commit_elect(smem_u32(&ms.drain));
    mbar_wait_warp(smem_u32(&ms.drain), 0, kDrainLimit);
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    // Group hg (warps 4hg .. 4hg + 3) owns the NH = R / 2 columns [hg NH, (hg + 1) NH) of the tile.
    // Thread t of the group's 128: in the 64-row score layout it holds token `tok` of the page (TMEM
    // lane tok % 16 of warp tok / 16 of the group) and the group's columns of parity `par`: local
    // column 2j + par in its slot j.  In the 128-row O^T layout it holds latent row t of each block.
    const int hg = warp >> 2;
    const int wq = warp & 3;
    const int t = threadIdx.x & (kGroupThreads - 1);
    const uint32_t gbar = 1u + (uint32_t)hg;           // the group's named barrier
    const uint32_t tl = tmem + ((uint32_t)(wq * 32) << 16);
    const int tok = wq * 16 + (lane >> 2) + 8 * (lane & 1);
    const int par = (lane >> 1) & 1;
    constexpr int NH = R / 2;                          // columns per group
    constexpr int NJ = R / 4;                          // columns per thread
    const int cb = hg * NH;                            // the group's first column
    // per-column values are stored group by group, parity-major inside a group: local column c of
    // group hg at cb + pm(c)
    auto pm = [](int c) { return (c & 1) * NJ + (c >> 1); };
    const float* aq_p = ms.aq2 + cb + par * NJ;
    const int32_t* ql_p = ms.qlim + cb + par * NJ;
    const int32_t* grp_p = ms.grp + cb + par * NJ;
    float* mu_p = ms.mu + cb + par * NJ;
    const float* corr_p = ms.corr + cb + par * NJ;
    // O^T columns per TMEM access in the rescale and the epilogue
    constexpr int kOcols = NH < 16 ? 8 : 16;
    auto tmem_ld_o = [](uint32_t addr, uint32_t (&v)[kOcols]) {
      if constexpr (kOcols == 8) tmem_ld8(addr, v); else tmem_ld16(addr, v);
    };
    auto tmem_st_o = [](uint32_t addr, const uint32_t (&v)[kOcols]) {
      if constexpr (kOcols == 8) tmem_st8(addr, v); else tmem_st16(addr, v);
    };
    auto pv_wait = [&](int64_t n) {
      return mbar_wait(smem_u32(&ms.pv_done[n & 1]), (uint32_t)((n >> 1) & 1), a.wait_limit);
    };
    // maximum (MAX) or sum over the 16 threads of the warp that hold the same columns (lane bits
    // 0, 2, 3, 4 vary); threads with lane 0 / 2 then store their parity's columns into red[wq]
    auto reduce_store = [&](float (&v)[NJ], bool is_max) {
#pragma unroll
      for (int j = 0; j < NJ; ++j) {
#pragma unroll
        for (int o : {1, 4, 8, 16}) {
          const float u = __shfl_xor_sync(0xffffffffu, v[j], o);
          v[j] = is_max ? fmaxf(v[j], u) : v[j] + u;
        }
      }
      if ((lane & ~2) == 0) {
#pragma unroll
        for (int j = 0; j < NJ; ++j) ms.red[wq][cb + par * NJ + j] = v[j];
      }
    };
    if (a.step_writes_only) pdl_wait();                // a_q is written by the preceding kernel
    const int ng = a.heads / G;
    RingPos<NKR> kr;
    int c_first = 0;          // ring slot of the tile's first latent block
    int64_t tile_n = 0;
    int n_item = 0;
    bool ok = true;
    // sequences b = blockIdx.x (mod gridDim.x) with a rejected length are this CTA's to report (checked
    // while the first scores are still being loaded)
    bool rejected = false;
    for (int b = blockIdx.x + t * gridDim.x; b < a.batch; b += kGroupThreads * gridDim.x)
      rejected |= pages_of(a.seq_lens[b], sp) == 0;
    rejected = group_any(rejected, gbar);
    while (ok && sched_next(cur, sp, blockIdx.x, it)) {
      if (t < NH) {
        const int rho = it.ht * R + cb + t;
        const bool valid = rho < qrows;
        const int j = valid ? rho / a.heads : 0;
        const int h = valid ? rho - j * a.heads : 0;
        const int sl = cb + pm(t);
        ms.aq2[sl] = valid ? a.a_q[(int64_t)it.b * qrows + rho] * kLog2e : 0.f;
        ms.grp[sl] = h / ng;
        ms.qlim[sl] = valid ? (a.vis_end ? a.vis_end[it.b] : it.L) - a.s_q + j : -1;
        ms.mu[sl] = -INFINITY;
      }
      named_bar_sync(gbar, kGroupThreads);
      float lpart[NJ];
#pragma unroll
      for (int j = 0; j < NJ; ++j) lpart[j] = 0.f;
      for (int p = it.p0; p < it.p1; ++p) {
        const int tok0 = p * kPage;
        const int nvalid = min(kPage, it.L - tok0);
        const int ks = kr.slot;
        const int sbuf = (int)(tile_n & 1);
        const uint32_t tSc = tl + 4 * R + sbuf * 2 * R;   // this tile's S^T columns; S_R^T follows at + R
        // every thread waits for the scores itself; the verdicts are pooled at the group vote below
        bool got = mbar_wait(smem_u32(&ms.s_full[sbuf]), (tile_n >> 1) & 1, a.wait_limit);
        // output MMAs of two tiles back (normally long complete).  Tile n signals barrier n & 1 in its
        // phase n >> 1; waiting for every tile two back keeps each barrier at most one phase ahead of
        // the phase waited for, which a parity wait needs.
        if (t == 0 && tile_n > 1) got = pv_wait(tile_n - 2) && got;
        tc_fence_after();
        const bool row_ok = tok < nvalid;
        const int tpos = tok0 + tok;
        const float* akrow = reinterpret_cast<const float*>(smem + C::AK_OFF + ks * kAkSlotBytes) + tok * G;
        float ak0 = 1.f;
        // this token's scaled logits, log2 units, of this thread's columns (-inf where not visible)
        float x[NJ];
        {
          constexpr int NL = NJ < 16 ? NJ : 16;        // registers per 16x64b load
#pragma unroll
          for (int b0 = 0; b0 < NJ; b0 += NL) {
            uint32_t sc[NL], sr[NL];
            if constexpr (NL == 4) {
              tmem_ld16x64_x4(tSc + cb + 2 * b0, sc);
              tmem_ld16x64_x4(tSc + R + cb + 2 * b0, sr);
            } else if constexpr (NL == 8) {
              tmem_ld16x64_x8(tSc + cb + 2 * b0, sc);
              tmem_ld16x64_x8(tSc + R + cb + 2 * b0, sr);
            } else {
              tmem_ld16x64_x16(tSc + cb + 2 * b0, sc);
              tmem_ld16x64_x16(tSc + R + cb + 2 * b0, sr);
            }
            if (!AK_ONE && b0 == 0) {
              // the a_k rows: their barrier and load overlap the TMEM loads' latency
              got = mbar_wait(smem_u32(&ms.akfull[ks]), kr.phase, a.wait_limit) && got;
              ak0 = akrow[0];
            }
            tmem_wait_ld();
            reg_tie(sc);
            reg_tie(sr);
#pragma unroll
            for (int q = 0; q < NL; q += 4) {
              const float4 aq4 = *reinterpret_cast<const float4*>(aq_p + b0 + q);
              const int4 ql4 = *reinterpret_cast<const int4*>(ql_p + b0 + q);
              const float aqv[4] = {aq4.x, aq4.y, aq4.z, aq4.w};
              const int qlv[4] = {ql4.x, ql4.y, ql4.z, ql4.w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                float akc = ak0;
                if (!AK_ONE && G > 1) akc = akrow[grp_p[b0 + q + e]];
                const float v = aqv[e] * akc * __uint_as_float(sc[q + e]) + kLog2e * __uint_as_float(sr[q + e]);
                x[b0 + q + e] = (row_ok && tpos <= qlv[e]) ? v : -INFINITY;
              }
            }
          }
        }
        // Fast path: the exponentials are taken against the running reference mu, which only has
        // to stay within 2^8 of the true column maximum.  One group vote finds out whether any
        // logit of the tile passed mu + 8; only then are the column maxima reduced.
        bool over = false;
#pragma unroll
        for (int j = 0; j < NJ; j += 4) {
          const float4 m4 = *reinterpret_cast<const float4*>(mu_p + j);
          over |= (x[j] > m4.x + kRescaleLog2) | (x[j + 1] > m4.y + kRescaleLog2) |
                  (x[j + 2] > m4.z + kRescaleLog2) | (x[j + 3] > m4.w + kRescaleLog2);
        }
        if (group_any(over || !got, gbar)) {
          if (group_any(!got, gbar)) { ok = false; break; }
          float v[NJ];
#pragma unroll
          for (int j = 0; j < NJ; ++j) v[j] = x[j];
          reduce_store(v, true);
          named_bar_sync(gbar, kGroupThreads);
          bool mine = false;
          if (t < NH) {
            // thread t < NH updates the group's column slot cb + t
            const int sl = cb + t;
            const float mt = fmaxf(fmaxf(ms.red[0][sl], ms.red[1][sl]), fmaxf(ms.red[2][sl], ms.red[3][sl]));
            const float mo = ms.mu[sl];
            float cr = 1.f;
            if (mt > mo + kRescaleLog2) {
              cr = (mo == -INFINITY) ? 0.f : ex2(mo - mt);
              ms.mu[sl] = mt;
              mine = true;
            }
            ms.corr[sl] = cr;
          }
          if (group_any(mine, gbar) && p > it.p0) {
            // O^T holds this item's earlier tiles: rescale it once the previous tile's output
            // MMAs are complete
            bool done = true;
            if (t == 0) done = pv_wait(tile_n - 1);
            if (!group_all(done, gbar)) { ok = false; break; }
            tc_fence_after();
#pragma unroll
            for (int m = 0; m < 4; ++m) {
#pragma unroll
              for (int c0 = 0; c0 < NH; c0 += kOcols) {
                uint32_t ov[kOcols];
                tmem_ld_o(tl + m * R + cb + c0, ov);
                tmem_wait_ld();
                reg_tie(ov);
#pragma unroll
                for (int e = 0; e < kOcols; ++e)
                  ov[e] = __float_as_uint(__uint_as_float(ov[e]) * ms.corr[cb + pm(c0 + e)]);
                tmem_st_o(tl + m * R + cb + c0, ov);
                tmem_wait_st();
              }
            }
          }
#pragma unroll
          for (int j = 0; j < NJ; ++j) lpart[j] *= corr_p[j];
        }
        // probabilities, running column sums, and P^T into the RoPE-key slot, token-major: row `tok`
        // holds the token's R probabilities (2R bytes), 16-byte units swizzled by row.  The two threads
        // of a token in a group swap half of their values (shuffle with lane ^ 2), so that each holds
        // complete column pairs: parity 0 the group's local columns 0 .. NH/2 - 1, parity 1 the rest.
        {
          float pr[NJ];
#pragma unroll
          for (int j = 0; j < NJ; j += 4) {
            const float4 m4 = *reinterpret_cast<const float4*>(mu_p + j);
            const float mv[4] = {m4.x, m4.y, m4.z, m4.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              pr[j + e] = x[j + e] == -INFINITY ? 0.f : ex2(x[j + e] - mv[e]);
              lpart[j + e] += pr[j + e];
            }
          }
          constexpr int NP = NJ / 2;                     // column pairs each thread writes
          uint32_t words[NP];
#pragma unroll
          for (int j = 0; j < NP; ++j) {
            const float send = par == 0 ? pr[j + NP] : pr[j];
            const float got2 = __shfl_xor_sync(0xffffffffu, send, 2);
            // parity 0: local columns (2j, 2j + 1) = (mine, partner's); parity 1: local columns
            // (2(j + NP), 2(j + NP) + 1) = (partner's, mine)
            const __nv_bfloat162 b2 = par == 0 ? __floats2bfloat162_rn(pr[j], got2)
                                               : __floats2bfloat162_rn(got2, pr[j + NP]);
            words[j] = *reinterpret_cast<const uint32_t*>(&b2);
          }
          uint8_t* prow = smem + C::KR_OFF + ks * kKrBytes + tok * (2 * R);
          const int swz = (R == 16) ? ((tok >> 2) & 1) : (R == 32) ? ((tok >> 1) & 3) : (tok & 7);
          // this thread's NP words start at byte 2 (cb + par NH / 2) of the row
          const int byte0 = 2 * (cb + par * (NH / 2));
          if constexpr (NP == 2) {                       // R = 16: half of a 16-byte unit
            const int unit = byte0 >> 4;
            *reinterpret_cast<uint2*>(prow + ((unit ^ swz) << 4) + (byte0 & 15)) = make_uint2(words[0], words[1]);
          } else {
#pragma unroll
            for (int u = 0; u < NP / 4; ++u) {
              const int unit = (byte0 >> 4) + u;         // 16-byte unit of the row
              *reinterpret_cast<uint4*>(prow + ((unit ^ swz) << 4)) =
                  make_uint4(words[4 * u], words[4 * u + 1], words[4 * u + 2], words[4 * u + 3]);
            }
          }
        }
        // the S buffer is free for the tile after next
        tc_fence_before();
        mbar_arrive(smem_u32(&ms.s_empty[sbuf]));
        // rows of the page past the context: zero them so that 0 * garbage cannot reach O (the four
        // threads of a token take two of its eight chunks each)
        if (!row_ok) {
#pragma unroll
          for (int k = (2 * hg + par) * 2; k < (2 * hg + par) * 2 + 2; ++k) {
            const int sl = c_first + k / 2 < NS ? c_first + k / 2 : c_first + k / 2 - NS;
            uint4* rowp = reinterpret_cast<uint4*>(smem + C::C_OFF + sl * kSlotBytes + (k & 1) * kChunkBytes + tok * 128);
#pragma unroll
            for (int q = 0; q < 8; ++q) rowp[q] = make_uint4(0, 0, 0, 0);
          }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(smem_u32(&ms.p_full[tile_n & 1]));
        c_first = c_first + kSlotsPerTile < NS ? c_first + kSlotsPerTile : c_first + kSlotsPerTile - NS;
        kr.next();
        ++tile_n;
      }
      if (!ok) break;
      // ---------------- epilogue: O / l and lse for this item
      bool got = true;
      if (t == 0) {
        if (tile_n > 1) got = pv_wait(tile_n - 2);
        if (!SKIP || tile_n > 0) got = got && pv_wait(tile_n - 1);   // (an empty first item has no tiles)
      }
      if (!group_all(got, gbar)) { ok = false; break; }
      tc_fence_after();
      // A query chunk's segment that one CTA holds whole (long chunks: every CTA group covers whole
      // sequences) is written straight to the output, and its descriptor says "no splits" so that the
      // merge leaves it alone; not when the merge applies the value up-projection (no output here).
      bool direct = false;
      if constexpr (SKIP) {
        if (a.out != nullptr && it.p0 == 0)
          direct = seg_split(it.seg_u0, pages_of(it.L, sp), cur.quota, sp.item_cost).nitems == 1;
      }
      reduce_store(lpart, false);
      named_bar_sync(gbar, kGroupThreads);
      if (t < NH) {
        const int c = cb + t;                            // the column (query row of the tile)
        const int sl = cb + pm(t);
        const float l = ms.red[0][sl] + ms.red[1][sl] + ms.red[2][sl] + ms.red[3][sl];
        ms.linv[c] = l > 0.f ? 1.f / l : 0.f;
        const float lse_c = l > 0.f ? (ms.mu[sl] + log2f(l)) * kLn2 : -INFINITY;
        if (!direct) {
          a.part_lse[(int64_t)it.slot * R + c] = lse_c;
        } else if (it.ht * R + c < qrows) {
          a.lse[(int64_t)it.b * qrows + it.ht * R + c] = lse_c;
        }
      }
      named_bar_sync(gbar, kGroupThreads);
      float* po = a.part_o + (int64_t)it.slot * R * kRkv;
      __nv_bfloat16* pd = static_cast<__nv_bfloat16*>(a.out) + ((int64_t)it.b * qrows + it.ht * R) * kRkv;
#pragma unroll
      for (int m = 0; m < 4; ++m) {
#pragma unroll
        for (int c0 = cb; c0 < cb + NH; c0 += kOcols) {
          uint32_t ov[kOcols];
          tmem_ld_o(tl + m * R + c0, ov);
          tmem_wait_ld();
          reg_tie(ov);
#pragma unroll
          for (int e = 0; e < kOcols; ++e)
            // (with empty items, a row with no visible token writes zeros, whatever the TMEM holds)
            if constexpr (SKIP) {
              const float v = ms.linv[c0 + e] > 0.f ? __uint_as_float(ov[e]) * ms.linv[c0 + e] : 0.f;
              if (!direct)
                po[(int64_t)(c0 + e) * kRkv + m * 128 + t] = v;
              else if (it.ht * R + c0 + e < qrows)
                pd[(int64_t)(c0 + e) * kRkv + m * 128 + t] = __float2bfloat16_rn(v);
            } else {
              po[(int64_t)(c0 + e) * kRkv + m * 128 + t] = __uint_as_float(ov[e]) * ms.linv[c0 + e];
            }
        }
      }
      tc_fence_before();
      mbar_arrive(smem_u32(&ms.o_empty));
      // the CTA holding a segment's first split tells the merge kernel where its splits are
      if (threadIdx.x == 0 && it.p0 == 0) {
        const SegSplit sg = seg_split(it.seg_u0, pages_of(it.L, sp), cur.quota, sp.item_cost);
        a.seg_desc[it.b * a.ht_count + it.ht] =
            direct ? make_int2(0, 0) : make_int2((it.b + sg.c0) * a.ht_count + it.ht, sg.nitems);
      }
      ++n_item;
    }
    if (!ok && t == 0) {
      record_status(a.status, QKN_ERR_TIMEOUT);
      ms.abort_flag = 1;
    }
    // A sequence whose length was rejected (outside [s_q, max_blocks * 64]) has no units: its rows
    // are written as zero with lse = -inf, and the status records QKN_ERR_BOUNDS.
    const int ts = threadIdx.x;                        // 0 .. kSoftThreads - 1 over both groups
    for (int b = blockIdx.x; rejected && b < a.batch; b += gridDim.x) {
      if (pages_of(a.seq_lens[b], sp) != 0) continue;
      if (ts == 0) record_status(a.status, QKN_ERR_BOUNDS);
      for (int ht = ts; ht < a.ht_count; ht += kSoftThreads) a.seg_desc[b * a.ht_count + ht] = make_int2(0, 0);
      // (no latent output when the merge applies the value up-projection: it writes those rows)
      uint4* ob = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.out) + (int64_t)b * qrows * kRkv);
      for (int64_t e = ts; a.out && e < (int64_t)qrows * kRkv / 8; e += kSoftThreads) ob[e] = make_uint4(0, 0, 0, 0);
      for (int e = ts; e < qrows; e += kSoftThreads) a.lse[(int64_t)b * qrows + e] = -INFINITY;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kScoreWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// ---------------------------------------------------------------- host side
namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// 2-D bf16 row-major tensor [rows, inner], 128-byte swizzled boxes [box_rows, box_inner].
bool make_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint32_t box_inner,
              uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {inner * 2};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D view of the latent cache [rows, 512] as [8 chunks][rows][64]: dimension 0 is the 64 columns
// of a chunk, dimension 1 the token row (stride 1024 bytes), dimension 2 the chunk (stride 128
// bytes).  A box of 2 chunks x 64 rows lands as two consecutive 8 KB swizzled chunk tiles.
bool make_latent_map(CUtensorMap* m, const void* base, uint64_t rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {64, rows, 8};
  cuuint64_t strides[2] = {512 * 2, 128};
  cuuint32_t box[3] = {64, 64, 2};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Encoded tensor maps, cached by what they encode (base address, extents and box), so that an
// eager decode does not pay four host-side encodings per call.  A map holds only an address and a
// geometry, so an entry stays valid for any buffer later placed at the same address with the same
// extents.  A small table with least-recently-used replacement, under a mutex.
class TmapCache {
 public:
  template <typename Encode>
  bool get(const void* base, uint64_t inner, uint64_t rows, uint32_t box_rows, int kind, CUtensorMap* out,
           Encode&& encode) {
    std::lock_guard<std::mutex> lock(mu_);
    ++tick_;
    int victim = 0;
    for (int i = 0; i < kEntries; ++i) {
      Entry& e = e_[i];
      if (e.used && e.base == base && e.inner == inner && e.rows == rows && e.box_rows == box_rows &&
          e.kind == kind) {
        e.used = tick_;
        *out = e.map;
        return true;
      }
      if (e.used < e_[victim].used) victim = i;
    }
    if (!encode(out)) return false;
    e_[victim] = Entry{base, inner, rows, box_rows, kind, tick_, *out};
    return true;
  }

 private:
  static constexpr int kEntries = 32;
  struct Entry {
    const void* base;
    uint64_t inner, rows;
    uint32_t box_rows;
    int kind;
    uint64_t used;   // 0: empty
    CUtensorMap map;
  };
  std::mutex mu_;
  uint64_t tick_ = 0;
  Entry e_[kEntries] = {};
};

TmapCache& tmap_cache() {
  static TmapCache c;
  return c;
}

template <int R, bool AK_ONE, bool SKIP>
cudaError_t launch_tc3(const DecodeArgs& a, const TcMaps& maps, cudaStream_t st) {
  static PerDeviceOnce attrs;
  cudaError_t e = once_per_device(attrs, [] {
    return cudaFuncSetAttribute(decode_tc_kernel<R, AK_ONE, SKIP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                Cfg<R>::SMEM);
  });
  if (e != cudaSuccess) return e;
  return launch_chained(decode_tc_kernel<R, AK_ONE, SKIP>, dim3(a.ncta), dim3(kThreads), Cfg<R>::SMEM, st, a, maps);
}

// Page skipping pays only when a tile's rows span many query positions: more query rows per
// sequence than two tiles (s_q > 2 at 64 heads per tile) is a chunk of a prefill.
template <int R, bool AK_ONE>
cudaError_t launch_tc(const DecodeArgs& a, const TcMaps& maps, cudaStream_t st) {
  return a.s_q * a.heads > 2 * R ? launch_tc3<R, AK_ONE, true>(a, maps, st) : launch_tc3<R, AK_ONE, false>(a, maps, st);
}

}  // namespace

bool decode_tc_supported(int r, int d_rope, int rows, int groups) {
  return r == kRkv && d_rope == kDrope && (rows == 16 || rows == 32 || rows == 64) && groups >= 1 &&
         groups <= kMaxGroups;
}

cudaError_t launch_decode_tc(const DecodeArgs& a, cudaStream_t st) {
  if (!decode_tc_supported(a.r, a.d_rope, a.rows, a.groups)) return cudaErrorNotSupported;
  TcMaps maps;
  const uint64_t cache_rows = (uint64_t)a.num_blocks * 64;
  const uint64_t q_rows = (uint64_t)a.batch * a.s_q * a.heads;
  TmapCache& tc = tmap_cache();
  if (!tc.get(a.latent, kRkv, cache_rows, 64, 0, &maps.latent,
              [&](CUtensorMap* m) { return make_latent_map(m, a.latent, cache_rows); }) ||
      !tc.get(a.k_rope, kDrope, cache_rows, 64, 1, &maps.krope,
              [&](CUtensorMap* m) { return make_map(m, a.k_rope, kDrope, cache_rows, 64, 64); }) ||
      !tc.get(a.q_tilde, kRkv, q_rows, a.rows, 1, &maps.qt,
              [&](CUtensorMap* m) { return make_map(m, a.q_tilde, kRkv, q_rows, 64, a.rows); }) ||
      !tc.get(a.q_rope_hat, kDrope, q_rows, a.rows, 1, &maps.qr,
              [&](CUtensorMap* m) { return make_map(m, a.q_rope_hat, kDrope, q_rows, 64, a.rows); }))
    return cudaErrorInvalidValue;
  switch (a.rows * 2 + (a.ak_one ? 1 : 0)) {
    case 32: return launch_tc<16, false>(a, maps, st);
    case 33: return launch_tc<16, true>(a, maps, st);
    case 64: return launch_tc<32, false>(a, maps, st);
    case 65: return launch_tc<32, true>(a, maps, st);
    case 128: return launch_tc<64, false>(a, maps, st);
    case 129: return launch_tc<64, true>(a, maps, st);
  }
  return cudaErrorNotSupported;
}

}  // namespace qkn
