// Split-KV QK-Normed MLA decode for tiles of 128 query rows, on a pair of CTAs
// (a thread-block cluster of two) that split the latent width between them.
//
// What it computes ("QK-Normed MLA: QK normalization without full key
// caching", technical summary, Metodología, decode-logit equation; the scalar
// factors are fused into the attention kernel as the summary's caveats ask):
// for query row rho of the tile and cached token t
//   l[rho, t] = a_q[rho] * a_k[t, g(rho)] * (q~[rho] . c_t) + q^R^[rho] . k^R^_t
// then an online softmax over the pair's token range and O = sum_t p * c_t.
//
// Why a pair.  With 128 query rows as the MMA's M dimension every product runs
// on the whole tensor datapath, but the fp32 accumulator O[128 x 512] alone
// would fill one SM's tensor memory.  So CTA c of the pair keeps latent
// columns [256c, 256c + 256): it loads only that half of each 64-token cache
// page, holds O[128 x 256], and computes a partial score over its half:
//   S_c[128 x 64] = Q~[:, half] . C[:, half]^T      (K = 256: 16 MMAs, M = 128, N = 64)
//   S_R[128 x 64] = Q^R^[:, half] . K^R[:, half]^T  (K = 32: the RoPE block is split the same way)
// The softmax is split by tokens: CTA c finishes the logits of tokens
// [32c, 32c + 32) of each page for all 128 rows.  Each CTA sends its partial
// logits a_q a_k S_c + S_R of the other token half to the peer through
// distributed shared memory (st.async into the peer's exchange buffer), adds
// the peer's part to its own half, and the two exchange their row maxima, so
// that both keep the same running reference per row (and rescale O by the
// same factors without exchanging them).  Each CTA writes the probabilities of
// its token half into its P tile and copies the tile into the peer with one
// bulk copy; both then run
//   O[128 x 256] += P[128 x 64] . C[64 x 256 of its half]   (4 MMAs, M = 128, N = 256)
// Each cache byte is read once, by one CTA of the pair.  No load with cluster
// multicast is used; the tensor core's commit signals both CTAs' P barrier.
//
// Tensor memory (512 columns): O at [0, 256); S_c and S_R of two tiles at
// [256 + 128 b, 256 + 128 b + 128), b = tile parity.
//
// Warp roles (352 threads, one CTA per SM):
//   warps 0-7  math: warp w takes TMEM lanes 32 (w % 4) + 16 (w / 4) .. + 15 (16 query rows) in
//              the 16x64b layout: two threads per row, one per column parity, so that a row's
//              values meet by one shuffle.  Every math warp does the same work on all four
//              SM sub-partitions (the lane quadrant of TMEM a warp can read is fixed by its
//              sub-partition);
//   warp 8     TMA producer (query tile per item; per page the latent half, the RoPE-key half and
//              the a_k rows);
//   warp 9     TMEM allocator and issuer of the score MMAs;
//   warp 10    issuer of the output MMAs.
// Every mbarrier wait is bounded; a wait that runs out records QKN_ERR_TIMEOUT
// and the CTA winds down.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace qkn {
using namespace sm100;

namespace {

constexpr int kPage = 64;                   // tokens per tile (one cache page; MMA N of the score product)
constexpr int kRkv = 512;                   // latent width this kernel takes
constexpr int kHalf = 256;                  // latent columns per CTA
constexpr int kDrope = 64;                  // RoPE width this kernel takes
constexpr int kRopeHalf = 32;               // RoPE columns per CTA
constexpr int kRows = 128;                  // query rows per tile (MMA M)
constexpr int kMaxGroups = 4;
constexpr int kMathWarps = 8;
constexpr int kProducerWarp = kMathWarps;
constexpr int kScoreWarp = kMathWarps + 1;
constexpr int kOutWarp = kMathWarps + 2;
constexpr int kThreads = (kMathWarps + 3) * 32;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescale = 5.545177444479562f;   // rescale O only when a row maximum grows by > ln 256
constexpr int64_t kDrainLimit = 4000000000LL;
constexpr int64_t kSettleCycles = 400000;   // after an abort: time for exchanges in flight to land
constexpr int kEarlyPages = 2;              // pages the producer may issue before the query tile

// shared-memory layout (offsets from a 1024-byte aligned base)
constexpr int kQChunk = kRows * 128;                     // 64 latent columns of 128 rows: 16 KB
constexpr int Q_OFF = 0;                                 // Q~ half: 4 chunks, 128-byte swizzle
constexpr int QR_OFF = Q_OFF + 4 * kQChunk;              // Q^R^ half: [128 rows][64 B], 64-byte swizzle
constexpr int kPHalf = kRows * 64;                       // P of one token half: [128 rows][32 tokens] bf16
constexpr int P_OFF = QR_OFF + kRows * 64;               // P tiles of token halves 0 and 1, 64-byte swizzle
constexpr int kXBytes = kRows * 32 * 4;                  // the peer's partial logits of this CTA's token half
constexpr int X_OFF = P_OFF + 2 * kPHalf;
constexpr int MISC_OFF = X_OFF + kXBytes;
constexpr int MISC_BYTES = 3072;
constexpr int RING_OFF = MISC_OFF + MISC_BYTES;
constexpr int kLatBytes = kPage * kHalf * 2;             // the page's latent half: 32 KB (4 chunks of 8 KB)
constexpr int kKrBytes = kPage * kRopeHalf * 2;          // the page's RoPE-key half: 4 KB
constexpr int kAkBytes = kPage * kMaxGroups * 4;         // the page's a_k rows: up to 1 KB
constexpr int SLOT_BYTES = kLatBytes + kKrBytes + kAkBytes;
constexpr int KR_IN_SLOT = kLatBytes;
constexpr int AK_IN_SLOT = kLatBytes + kKrBytes;
constexpr int NS = 3;                                    // ring slots (pages)
constexpr int SMEM = RING_OFF + NS * SLOT_BYTES + 1024;
static_assert(P_OFF % 1024 == 0 && RING_OFF % 1024 == 0 && SLOT_BYTES % 1024 == 0, "swizzle atom alignment");
static_assert(SMEM <= 232448, "shared memory budget");

struct PairMisc {
  uint64_t full[NS], empty[NS];   // ring: page landed / page's last reader (output MMAs) done
  uint64_t s_full[2], s_empty[2]; // score accumulators of a tile parity: written / read out (8 warps)
  uint64_t x_full;                // the peer's partial logits of this CTA's token half landed (1 arm + 16 KB)
  uint64_t x_free;                // the peer's math warps have read this CTA's partial logits (8 remote)
  uint64_t m_full[2], m_free[2];  // row maxima of a tile parity: the peer's landed (1 arm + 512 B) / read (8)
  uint64_t pr_full;               // the peer's P half landed (1 arm + 8 KB)
  uint64_t p_ready;               // P tile complete and O rescaled: the output MMAs may run (8 warps)
  uint64_t p_free;                // output MMAs of the tile done in both CTAs (2 commits)
  uint64_t l_full, l_free;        // the peer's row sums of an item landed (1 arm + 512 B) / read (8 remote)
  uint64_t q_full, q_empty, o_empty, drain;
  uint32_t tmem_base;
  int32_t abort_flag;             // a role of this CTA stopped early
  int32_t abort_any;              // either CTA of the pair did (set by both, read after a cluster barrier)
  Cursor cursor;
  alignas(16) float mx_recv[2][kRows];   // the peer's row maxima over its token half, per tile parity
  alignas(16) float l_recv[kRows];       // the peer's row sums over its token half
  alignas(16) float linv[kRows];         // 1 / l per row, for the epilogue's 32x32b read-out
};
static_assert(sizeof(PairMisc) <= MISC_BYTES, "misc shared-memory block");

// 64-byte swizzle of a [rows][64 B] tile: 16-byte unit u of row r sits at unit u ^ ((r >> 1) & 3).
__device__ __forceinline__ uint32_t sw64(int row, int unit) { return (uint32_t)(row * 64 + ((unit ^ ((row >> 1) & 3)) << 4)); }
// The exchange buffer holds a 128-byte row per query row: 16 fp32 per column parity.  Its 16-byte
// units are swizzled by row so that 8 consecutive rows hit distinct banks.
__device__ __forceinline__ uint32_t xoff(int row, int unit) { return (uint32_t)(row * 128 + ((unit ^ (row & 7)) << 4)); }

}  // namespace

struct PairMaps {
  CUtensorMap latent;   // [8 chunks][num_blocks*64 rows][64] bf16 view of the latent, box 4 x 64 x 64
  CUtensorMap krope;    // [num_blocks*64, 64] bf16, box 32 x 64, 64-byte swizzle
  CUtensorMap qt;       // [n_q*H, 512] bf16, box 64 x 128
  CUtensorMap qr;       // [n_q*H, 64] bf16, box 32 x 128, 64-byte swizzle
};

template <bool AK_ONE>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    decode_pair_kernel(const DecodeArgs a, const __grid_constant__ PairMaps maps) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  PairMisc& ms = *reinterpret_cast<PairMisc*>(smem + MISC_OFF);
  const uint32_t sb = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t crank = cluster_ctarank();            // c: this CTA's latent half and row half
  const uint32_t prank = crank ^ 1u;
  const int pair = blockIdx.x >> 1;                    // the schedule's unit of work is the pair
  const SchedParams sp{a.seq_lens, a.batch, a.s_q, a.max_blocks, a.ht_count, a.ncta, a.item_cost,
                       a.heads, a.rows, a.vis_end};
  const int qrows = a.s_q * a.heads;
  const int G = a.groups;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(smem_u32(&ms.full[s]), 1);
      mbar_init(smem_u32(&ms.empty[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&ms.s_full[b]), 1);
      mbar_init(smem_u32(&ms.s_empty[b]), kMathWarps);
    }
    mbar_init(smem_u32(&ms.x_full), 1);
    mbar_init(smem_u32(&ms.x_free), kMathWarps);
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&ms.m_full[b]), 1);
      mbar_init(smem_u32(&ms.m_free[b]), kMathWarps);
    }
    mbar_init(smem_u32(&ms.pr_full), 1);
    mbar_init(smem_u32(&ms.p_ready), kMathWarps);
    mbar_init(smem_u32(&ms.p_free), 2);
    mbar_init(smem_u32(&ms.l_full), 1);
    mbar_init(smem_u32(&ms.l_free), kMathWarps);
    mbar_init(smem_u32(&ms.q_full), 1);
    mbar_init(smem_u32(&ms.q_empty), 1);
    mbar_init(smem_u32(&ms.o_empty), kMathWarps);
    mbar_init(smem_u32(&ms.drain), 2);
    ms.abort_flag = 0;
    ms.abort_any = 0;
    mbar_fence_init();
  }
  if (warp == kProducerWarp && lane == 0) {
    prefetch_tmap(&maps.latent);
    prefetch_tmap(&maps.krope);
    prefetch_tmap(&maps.qt);
    prefetch_tmap(&maps.qr);
  }
  if (warp == kScoreWarp) {
    tmem_alloc(smem_u32(&ms.tmem_base), 512);
    tmem_relinquish();
  }
  pdl_trigger();
  if (!a.step_writes_only) pdl_wait();
  if (warp == 0) {
    Cursor c = sched_begin(sp, pair);
    if (lane == 0) ms.cursor = c;
  }
  // both CTAs' barriers are initialised before either touches the other's shared memory
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem = ms.tmem_base;
  Cursor cur = ms.cursor;
  Item it;
  bool ok = true;

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------ producer (whole warp, elected issue)
    RingPos<NS> cw;
    int64_t issued = 0;
    int n_item = 0;
    const uint32_t akpage = AK_ONE ? 0u : (uint32_t)kPage * (uint32_t)G * 4u;
    bool waited = !a.step_writes_only;
    int early_pages = 0;
    int q_last = -1;
    int64_t withheld = -1;                // page whose a_k copy a timeout test withholds
    while (ok && sched_next(cur, sp, pair, it)) {
      const int32_t* row = a.block_table + (int64_t)it.b * a.max_blocks;
      int32_t mine = (it.p0 + lane < it.p1) ? row[it.p0 + lane] : 0;
      bool q_pending = true;
      auto issue_q = [&]() -> bool {
        if (!waited) {
          pdl_wait();
          waited = true;
        }
        if (!mbar_wait_warp(smem_u32(&ms.q_empty), (n_item & 1) ^ 1, a.wait_limit)) return false;
        const int qrow0 = it.b * qrows + it.ht * kRows;
        const uint32_t qf = smem_u32(&ms.q_full);
        mbar_arrive_expect_tx_elect(qf, 4 * kQChunk + kRows * 64);
#pragma unroll
        for (int k = 0; k < 4; ++k)
          tma_load_2d_elect(sb + Q_OFF + k * kQChunk, &maps.qt, (int)crank * kHalf + k * 64, qrow0, qf);
        tma_load_2d_elect(sb + QR_OFF, &maps.qr, (int)crank * kRopeHalf, qrow0, qf);
        q_pending = false;
        q_last = n_item;
        return true;
      };
      if (waited && !issue_q()) { ok = false; break; }
      const int first_new_page = ((a.vis_end ? a.vis_end[it.b] : it.L) - a.s_q) / kPage;
      for (int pb = it.p0; pb < it.p1 && ok; pb += 32) {
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
          if (!mbar_wait_warp(smem_u32(&ms.empty[cw.slot]), cw.phase ^ 1u, a.wait_limit)) { ok = false; break; }
          const uint32_t fb = smem_u32(&ms.full[cw.slot]);
          const uint32_t dst = sb + RING_OFF + cw.slot * SLOT_BYTES;
          mbar_arrive_expect_tx_elect(fb, kLatBytes + kKrBytes + akpage);
          // latent chunks 4c .. 4c + 3 of the page (one box), the RoPE-key half, the a_k rows
          tma_load_3d_elect(dst, &maps.latent, 0, blk * kPage, (int)crank * 4, fb);
          tma_load_2d_elect(dst + KR_IN_SLOT, &maps.krope, (int)crank * kRopeHalf, blk * kPage, fb);
          if (!AK_ONE) {
            // (a test of the timeout path withholds the first page's a_k rows: that page's barrier
            // phase then never completes, and the waits for it run out)
            if (a.withhold_ak && issued == 0)
              withheld = issued;
            else
              bulk_load_elect(dst + AK_IN_SLOT, a.a_k + (int64_t)blk * kPage * G, akpage, fb);
          }
          cw.next();
          ++issued;
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
      const int64_t first = issued > NS ? issued - NS : 0;
      for (int64_t i = first; i < issued; ++i)
        if (i != withheld) mbar_wait(smem_u32(&ms.full[i % NS]), (uint32_t)((i / NS) & 1), kDrainLimit);
      if (q_last >= 0) mbar_wait(smem_u32(&ms.q_full), (uint32_t)(q_last & 1), kDrainLimit);
    }
  } else if (warp == kScoreWarp) {
    // ------------------------------------------------------------ score MMA issuer (whole warp)
    constexpr uint32_t idS = idesc_bf16(kRows, kPage, false, false);
    const uint64_t dQ = smem_desc(sb + Q_OFF, 16, 1024);                 // A: Q~ half, K-major, 128 B rows
    const uint64_t dQR = smem_desc_sw(sb + QR_OFF, 16, 512, 4);          // A: Q^R^ half, K-major, 64 B rows
    const uint64_t dC = smem_desc(sb + RING_OFF, 16, 1024);              // B: latent chunk [64 tok][128 B]
    const uint64_t dKR = smem_desc_sw(sb + RING_OFF + KR_IN_SLOT, 16, 512, 4);   // B: K^R half [64 tok][64 B]
    RingPos<NS> cr;
    RingPos<2> sbuf;
    int n_item = 0;
    while (ok && sched_next(cur, sp, pair, it)) {
      if (!mbar_wait_warp(smem_u32(&ms.q_full), n_item & 1, a.wait_limit)) { ok = false; break; }
      tc_fence_after();
      for (int p = it.p0; p < it.p1 && ok; ++p) {
        const int b = sbuf.slot;
        if (!mbar_wait_warp(smem_u32(&ms.s_empty[b]), sbuf.phase ^ 1u, a.wait_limit)) { ok = false; break; }
        if (!mbar_wait_warp(smem_u32(&ms.full[cr.slot]), cr.phase, a.wait_limit)) { ok = false; break; }
        tc_fence_after();
        const uint32_t tS = tmem + kHalf + b * 128;
        const uint64_t slot = (uint64_t)((cr.slot * SLOT_BYTES) >> 4);
#pragma unroll
        for (int u = 0; u < 16; ++u) {   // chunk u / 4 of the half, K step u % 4 (32 bytes) inside it
          const uint32_t aoff = (uint32_t)(((u >> 2) * kQChunk + (u & 3) * 32) >> 4);
          const uint32_t boff = (uint32_t)(((u >> 2) * (kPage * 128) + (u & 3) * 32) >> 4);
          mma_bf16_elect(tS, dQ + aoff, dC + slot + boff, idS, u != 0 ? 1u : 0u);
        }
#pragma unroll
        for (int u = 0; u < 2; ++u)
          mma_bf16_elect(tS + 64, dQR + (uint32_t)((u * 32) >> 4), dKR + slot + (uint32_t)((u * 32) >> 4), idS,
                         u != 0 ? 1u : 0u);
        mma_commit_elect(smem_u32(&ms.s_full[b]));
        cr.next();
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
    mma_commit_elect(smem_u32(&ms.drain));
    mbar_wait_warp(smem_u32(&ms.drain), 0, kDrainLimit);
  } else if (warp == kOutWarp) {
    // ------------------------------------------------------------ output MMA issuer (whole warp)
    constexpr uint32_t idPV = idesc_bf16(kRows, kHalf, false, true);
    // A: P as two K-major [128 rows][32 tokens] tiles (token halves), 64-byte swizzle
    const uint64_t dP = smem_desc_sw(sb + P_OFF, 16, 512, 4);
    // B: the page's latent half, MN-major: 64-column chunks LBO = 8 KB apart, 8-token groups SBO = 1 KB apart
    const uint64_t dCt = smem_desc(sb + RING_OFF, kPage * 128, 1024);
    RingPos<NS> cr;
    int64_t tile_n = 0;
    int n_item = 0;
    while (ok && sched_next(cur, sp, pair, it)) {
      // once per item, pages or not, so that the barrier is never more than one phase ahead
      if (!mbar_wait_warp(smem_u32(&ms.o_empty), (n_item & 1) ^ 1, a.wait_limit)) { ok = false; break; }
      for (int p = it.p0; p < it.p1 && ok; ++p) {
        if (!mbar_wait_warp(smem_u32(&ms.p_ready), (uint32_t)(tile_n & 1), a.wait_limit)) { ok = false; break; }
        tc_fence_after();
        const uint64_t slot = (uint64_t)((cr.slot * SLOT_BYTES) >> 4);
        const uint32_t acc0 = p > it.p0 ? 1u : 0u;
#pragma unroll
        for (int kk = 0; kk < kPage / 16; ++kk)   // tokens 16 kk .. + 15: tile kk / 2, 32-byte step kk % 2
          mma_bf16_elect(tmem, dP + (uint32_t)(((kk >> 1) * kPHalf + (kk & 1) * 32) >> 4),
                         dCt + slot + (uint32_t)((kk * 2048) >> 4), idPV, kk > 0 ? 1u : acc0);
        mma_commit_elect(smem_u32(&ms.empty[cr.slot]));
        mma_commit_pair_elect(smem_u32(&ms.p_free), (uint16_t)0x3);
        cr.next();
        ++tile_n;
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
    // ------------------------------------------------------------ math warps
    const int quad = warp & 3;                         // TMEM lane quadrant (= the warp's sub-partition)
    const int half = warp >> 2;
    // 16x64b layout: thread t holds lane (t >> 2) + 8 (t & 1) of the warp's 16 and the columns of
    // parity (t >> 1) & 1; the row's other thread is t ^ 2
    const int rho = quad * 32 + half * 16 + (lane >> 2) + 8 * (lane & 1);
    const int par = (lane >> 1) & 1;
    const uint32_t tq = tmem + ((uint32_t)(quad * 32 + half * 16) << 16);
    const uint32_t tl32 = tmem + ((uint32_t)(quad * 32) << 16);     // 32x32b: the whole quadrant
    const int own0 = (int)crank * 32, peer0 = (int)prank * 32;    // first token of each half of a page
    const bool leader = threadIdx.x == 0;
    const uint32_t peer_x_full = mapa_shared(smem_u32(&ms.x_full), prank);
    const uint32_t peer_x_free = mapa_shared(smem_u32(&ms.x_free), prank);
    const uint32_t peer_m_full = mapa_shared(smem_u32(&ms.m_full[0]), prank);     // + 8 b for parity b
    const uint32_t peer_m_free = mapa_shared(smem_u32(&ms.m_free[0]), prank);
    const uint32_t peer_pr_full = mapa_shared(smem_u32(&ms.pr_full), prank);
    const uint32_t peer_l_full = mapa_shared(smem_u32(&ms.l_full), prank);
    const uint32_t peer_l_free = mapa_shared(smem_u32(&ms.l_free), prank);
    const uint32_t peer_x = mapa_shared(sb + X_OFF, prank);
    const uint32_t peer_mx = mapa_shared(smem_u32(&ms.mx_recv[0][0]), prank);
    const uint32_t peer_l = mapa_shared(smem_u32(&ms.l_recv[0]), prank);
    const uint32_t peer_p = mapa_shared(sb + P_OFF, prank);
    if (a.step_writes_only) pdl_wait();                // a_q is written by the preceding kernel
    const int ng = a.heads / G;
    RingPos<NS> cr;
    int64_t tile_n = 0;
    int n_item = 0;
    // sequences b = pair (mod pairs) with a rejected length are this pair's to report (CTA 0)
    bool rejected = false;
    if (crank == 0)
      for (int b = pair; b < a.batch; b += a.ncta) rejected |= pages_of(a.seq_lens[b], sp) == 0;
    while (ok && sched_next(cur, sp, pair, it)) {
      // this row's scalars
      const int rg = it.ht * kRows + rho;
      const bool valid = rg < qrows;
      const int j = valid ? rg / a.heads : 0;
      const int grp = (valid ? rg - j * a.heads : 0) / ng;
      const float aq = valid ? a.a_q[(int64_t)it.b * qrows + rg] : 0.f;
      const int qlim = valid ? (a.vis_end ? a.vis_end[it.b] : it.L) - a.s_q + j : -1;
      float mu = -INFINITY, lsum = 0.f;               // reference and this thread's part of the row sum
      // A wait that runs out makes `got` false; the math warps leave together, at the next vote
      // over all 256 of them (every named barrier of the loop is such a vote), never at a barrier
      // that some of them would not reach.  `carry` takes the last wait of a tile to the next vote.
      bool carry = true;
      for (int p = it.p0; p < it.p1; ++p) {
        const int sbi = (int)(tile_n & 1);             // score buffer of the tile and its phase parity
        const uint32_t sph = (uint32_t)((tile_n >> 1) & 1);
        const uint32_t tph = (uint32_t)(tile_n & 1);   // phase parity of the once-per-tile barriers
        const uint32_t tS = tq + kHalf + sbi * 128;
        // scores of this row: S_c and S_R of this thread's parity in both token halves
        bool got = mbar_wait(smem_u32(&ms.s_full[sbi]), sph, a.wait_limit) && carry;
        tc_fence_after();
        uint32_t so[16], sp_[16], ro[16], rp[16];
        tmem_ld16x64_x16(tS + own0, so);
        tmem_ld16x64_x16(tS + peer0, sp_);
        tmem_ld16x64_x16(tS + 64 + own0, ro);
        tmem_ld16x64_x16(tS + 64 + peer0, rp);
        tmem_wait_ld();
        reg_tie(so);
        reg_tie(sp_);
        reg_tie(ro);
        reg_tie(rp);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&ms.s_empty[sbi]));
        // the page's a_k rows (the ring barrier also covers them; normally complete long before)
        const float* akp = reinterpret_cast<const float*>(smem + RING_OFF + cr.slot * SLOT_BYTES + AK_IN_SLOT);
        if (!AK_ONE) got = mbar_wait(smem_u32(&ms.full[cr.slot]), cr.phase, a.wait_limit) && got;
        // this CTA's part of the logits a_q a_k S_c + S_R (its latent and RoPE halves), token 2r + par
        // of each half
        float x[16], y[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) {
          const float ako = AK_ONE ? 1.f : akp[(own0 + 2 * r + par) * G + grp];
          const float akq = AK_ONE ? 1.f : akp[(peer0 + 2 * r + par) * G + grp];
          x[r] = fmaf(aq * ako, __uint_as_float(so[r]), __uint_as_float(ro[r]));
          y[r] = fmaf(aq * akq, __uint_as_float(sp_[r]), __uint_as_float(rp[r]));
        }
        // the peer's token half goes to the peer (once it has read the previous tile's)
        got = mbar_wait_cl(smem_u32(&ms.x_free), tph ^ 1u, a.wait_limit) && got;
        if (got) {
#pragma unroll
          for (int u = 0; u < 4; ++u)
            st_async_v4(peer_x + xoff(rho, par * 4 + u), __float_as_uint(y[4 * u]), __float_as_uint(y[4 * u + 1]),
                        __float_as_uint(y[4 * u + 2]), __float_as_uint(y[4 * u + 3]), peer_x_full);
        }
        // and the peer's part of this CTA's half comes back
        if (leader) mbar_arrive_expect_tx(smem_u32(&ms.x_full), kXBytes);
        got = mbar_wait_cl(smem_u32(&ms.x_full), tph, a.wait_limit) && got;
        if (got) {
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const float4 v = *reinterpret_cast<const float4*>(smem + X_OFF + xoff(rho, par * 4 + u));
            x[4 * u] += v.x;
            x[4 * u + 1] += v.y;
            x[4 * u + 2] += v.z;
            x[4 * u + 3] += v.w;
          }
        }
        __syncwarp();
        if (lane == 0 && got) mbar_arrive_remote(peer_x_free);
        // tokens past the context or after the row's query position get no weight (only the pages
        // that hold such tokens need the test)
        const int tok0 = p * kPage;
        const int nvalid = min(kPage, it.L - tok0);
        if (__any_sync(0xffffffffu, nvalid < kPage || tok0 + kPage - 1 > qlim)) {
#pragma unroll
          for (int r = 0; r < 16; ++r) {
            const int tok = own0 + 2 * r + par;
            if (tok >= nvalid || tok0 + tok > qlim) x[r] = -INFINITY;
          }
        }
        // row maximum over this CTA's token half, then over both: the peer gets this half's
        float m = x[0];
#pragma unroll
        for (int r = 1; r < 16; ++r) m = fmaxf(m, x[r]);
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
        got = mbar_wait_cl(smem_u32(&ms.m_free[sbi]), sph ^ 1u, a.wait_limit) && got;
        if (par == 0 && got) st_async_b32(peer_mx + (sbi * kRows + rho) * 4, __float_as_uint(m), peer_m_full + 8 * sbi);
        if (leader) mbar_arrive_expect_tx(smem_u32(&ms.m_full[sbi]), kRows * 4);
        got = mbar_wait_cl(smem_u32(&ms.m_full[sbi]), sph, a.wait_limit) && got;
        const float mt = fmaxf(m, ms.mx_recv[sbi][rho]);
        __syncwarp();
        if (lane == 0 && got) mbar_arrive_remote(peer_m_free + 8 * sbi);
        // The exponentials use a running reference mu per row that only has to stay within e^kR of
        // the true maximum; both CTAs see the same maxima, so they raise mu together.
        float corr = 1.f;
        if (mt > mu + kRescale) {
          corr = (mu == -INFINITY) ? 0.f : ex2((mu - mt) * kLog2e);
          mu = mt;
        }
        // O holds this item's earlier tiles: rescale this warp's rows (tcgen05.ld / st are
        // warp-collective, so the whole warp takes part, rows that did not change by 1) once the
        // previous tile's output MMAs are done
        const bool resc = __any_sync(0xffffffffu, corr != 1.f) && p > it.p0;   // warp-uniform
        if (resc) got = mbar_wait_cl(smem_u32(&ms.p_free), tph ^ 1u, a.wait_limit) && got;
        const bool warp_got = __all_sync(0xffffffffu, got);
        if (resc && warp_got) {
          tc_fence_after();
#pragma unroll
          for (int c0 = 0; c0 < kHalf; c0 += 32) {
            uint32_t ov[16];
            tmem_ld16x64_x16(tq + c0, ov);
            tmem_wait_ld();
            reg_tie(ov);
#pragma unroll
            for (int e = 0; e < 16; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * corr);
            tmem_st16x64_x16(tq + c0, ov);
          }
          tmem_wait_st();
        }
        lsum *= corr;
        // probabilities and this thread's part of the row sum; a row with no visible token so far
        // (mu = -inf) has only -inf logits, whose exponentials are 0 against any mu2
        const float mu2 = mu == -INFINITY ? 0.f : mu * kLog2e;
        float pr[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) {
          pr[r] = ex2(fmaf(x[r], kLog2e, -mu2));
          lsum += pr[r];
        }
        // bf16 pairs of consecutive tokens: the row's two threads swap half of their values, so that
        // parity 0 holds tokens 0 .. 15 of the half and parity 1 tokens 16 .. 31
        uint32_t w[8];
#pragma unroll
        for (int r = 0; r < 8; ++r) {
          const float send = par == 0 ? pr[r + 8] : pr[r];
          const float got2 = __shfl_xor_sync(0xffffffffu, send, 2);
          const __nv_bfloat162 b2 = par == 0 ? __floats2bfloat162_rn(pr[r], got2) : __floats2bfloat162_rn(got2, pr[r + 8]);
          w[r] = *reinterpret_cast<const uint32_t*>(&b2);
        }
        // the P tile is free once the previous tile's output MMAs are done in both CTAs
        got = mbar_wait_cl(smem_u32(&ms.p_free), tph ^ 1u, a.wait_limit) && got;
        if (got) {
          uint8_t* pt = smem + P_OFF + crank * kPHalf;
          *reinterpret_cast<uint4*>(pt + sw64(rho, par * 2)) = make_uint4(w[0], w[1], w[2], w[3]);
          *reinterpret_cast<uint4*>(pt + sw64(rho, par * 2 + 1)) = make_uint4(w[4], w[5], w[6], w[7]);
        }
        // rows of the page past the context: zero this CTA's latent half of them, so that 0 * (stale
        // bits, possibly NaN) cannot reach O through the output MMAs (the score MMAs are done with
        // the page: its s_full phase completed above)
        if (nvalid < kPage) {
          uint8_t* lat = smem + RING_OFF + cr.slot * SLOT_BYTES;
          for (int e = threadIdx.x; e < (kPage - nvalid) * 32; e += kMathWarps * 32) {
            const int tok = nvalid + (e >> 5), chunk = (e >> 3) & 3, unit = e & 7;
            *reinterpret_cast<uint4*>(lat + chunk * (kPage * 128) + tok * 128 + (unit << 4)) = make_uint4(0, 0, 0, 0);
          }
        }
        fence_proxy_async_smem();
        if (bar_any(!got, 1, kMathWarps * 32)) { ok = false; break; }
        if (leader) {
          // this CTA's P half into the peer's tile; and the arm for the peer's half
          mbar_arrive_expect_tx(smem_u32(&ms.pr_full), kPHalf);
          bulk_copy_to_peer(peer_p + crank * kPHalf, sb + P_OFF + crank * kPHalf, kPHalf, peer_pr_full);
        }
        // the output MMAs also need the peer's half
        carry = mbar_wait_cl(smem_u32(&ms.pr_full), tph, a.wait_limit);
        tc_fence_before();
        const bool warp_carry = __all_sync(0xffffffffu, carry);
        if (lane == 0 && warp_carry) mbar_arrive(smem_u32(&ms.p_ready));
        cr.next();
        ++tile_n;
      }
      if (!ok) break;
      // ---------------- epilogue of the item: O / l for every lane, lse
      bool got = (tile_n == 0 || mbar_wait_cl(smem_u32(&ms.p_free), (uint32_t)((tile_n - 1) & 1), a.wait_limit)) && carry;
      const float lh = lsum + __shfl_xor_sync(0xffffffffu, lsum, 2);   // this CTA's token half of the row
      got = mbar_wait_cl(smem_u32(&ms.l_free), (uint32_t)((n_item & 1) ^ 1), a.wait_limit) && got;
      if (par == 0 && got) st_async_b32(peer_l + rho * 4, __float_as_uint(lh), peer_l_full);
      if (leader) mbar_arrive_expect_tx(smem_u32(&ms.l_full), kRows * 4);
      got = mbar_wait_cl(smem_u32(&ms.l_full), (uint32_t)(n_item & 1), a.wait_limit) && got;
      const float l = lh + ms.l_recv[rho];
      __syncwarp();
      if (lane == 0 && got) mbar_arrive_remote(peer_l_free);
      if (par == 0) {
        ms.linv[rho] = l > 0.f ? 1.f / l : 0.f;
        if (crank == 0) a.part_lse[(int64_t)it.slot * kRows + rho] = l > 0.f ? mu + logf(l) : -INFINITY;
      }
      if (bar_any(!got, 1, kMathWarps * 32)) { ok = false; break; }
      tc_fence_after();
      // read-out in the 32x32b layout: this warp takes every row of its quadrant, O columns
      // [128 half, 128 half + 128)
      const int orow = quad * 32 + lane;
      const float linv = ms.linv[orow];
      float* po = a.part_o + ((int64_t)it.slot * kRows + orow) * kRkv + crank * kHalf + half * 128;
#pragma unroll
      for (int c0 = 0; c0 < 128; c0 += 16) {
        uint32_t ov[16];
        tmem_ld16(tl32 + half * 128 + c0, ov);
        tmem_wait_ld();
        reg_tie(ov);
        // a row with no visible token in the item writes zeros, whatever the TMEM holds
#pragma unroll
        for (int e = 0; e < 16; e += 4)
          *reinterpret_cast<float4*>(po + c0 + e) =
              linv > 0.f ? make_float4(__uint_as_float(ov[e]) * linv, __uint_as_float(ov[e + 1]) * linv,
                                       __uint_as_float(ov[e + 2]) * linv, __uint_as_float(ov[e + 3]) * linv)
                         : make_float4(0.f, 0.f, 0.f, 0.f);
      }
      tc_fence_before();
      named_bar_sync(1, kMathWarps * 32);              // ms.linv is read before the next item writes it
      if (lane == 0) mbar_arrive(smem_u32(&ms.o_empty));
      // the pair holding a segment's first split tells the merge kernel where its splits are
      if (crank == 0 && threadIdx.x == 0 && it.p0 == 0) {
        const SegSplit sg = seg_split(it.seg_u0, pages_of(it.L, sp), cur.quota, sp.item_cost);
        a.seg_desc[it.b * a.ht_count + it.ht] = make_int2((it.b + sg.c0) * a.ht_count + it.ht, sg.nitems);
      }
      ++n_item;
    }
    if (!ok && lane == 0) {
      record_status(a.status, QKN_ERR_TIMEOUT);
      ms.abort_flag = 1;
    }
    // A sequence whose length was rejected (outside [s_q, max_blocks * 64]) has no units: its rows
    // are written as zero with lse = -inf, and the status records QKN_ERR_BOUNDS (CTA 0 of the pair).
    const int ts = threadIdx.x;                        // 0 .. 255 over the math warps
    for (int b = pair; rejected && b < a.batch; b += a.ncta) {
      if (pages_of(a.seq_lens[b], sp) != 0) continue;
      if (ts == 0) record_status(a.status, QKN_ERR_BOUNDS);
      for (int ht = ts; ht < a.ht_count; ht += kMathWarps * 32) a.seg_desc[b * a.ht_count + ht] = make_int2(0, 0);
      // (no latent output when the merge applies the value up-projection: it writes those rows)
      uint4* ob = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.out) + (int64_t)b * qrows * kRkv);
      for (int64_t e = ts; a.out && e < (int64_t)qrows * kRkv / 8; e += kMathWarps * 32) ob[e] = make_uint4(0, 0, 0, 0);
      for (int e = ts; e < qrows; e += kMathWarps * 32) a.lse[(int64_t)b * qrows + e] = -INFINITY;
    }
  }

  tc_fence_before();
  __syncthreads();
  // Neither CTA leaves while the other may still write into its shared memory or arrive on its
  // barriers.  On the normal path every exchange has been consumed by now; after a timeout some
  // may still be in flight, so both CTAs then wait a little for them to land.  The two take the
  // same decision: each tells the other that it stopped early before the cluster barrier.
  if (threadIdx.x == 0 && ms.abort_flag) {
    ms.abort_any = 1;
    st_shared_remote_u32(mapa_shared(smem_u32(&ms.abort_any), prank), 1u);
  }
  cluster_sync();
  if (*reinterpret_cast<volatile int32_t*>(&ms.abort_any)) {
    const long long t0 = clock64();
    while (clock64() - t0 < kSettleCycles) {
    }
    cluster_sync();
  }
  if (warp == kScoreWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------- host side
namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D bf16 row-major tensor [rows, inner], boxes [box_rows, box_inner] with the given swizzle.
bool make_map2(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint32_t box_inner,
               uint32_t box_rows, CUtensorMapSwizzle swz) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {inner * 2};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D view of the latent cache [rows, 512] as [8 chunks][rows][64]; a box of 4 chunks x 64 rows lands
// as four consecutive 8 KB swizzled chunk tiles (one latent half of one page).
bool make_latent_map4(CUtensorMap* m, const void* base, uint64_t rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {64, rows, 8};
  cuuint64_t strides[2] = {512 * 2, 128};
  cuuint32_t box[3] = {64, 64, 4};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Encoded tensor maps cached by what they encode (see the single-CTA decode's cache).
class PairMapCache {
 public:
  template <typename Encode>
  bool get(const void* base, uint64_t rows, int kind, CUtensorMap* out, Encode&& encode) {
    std::lock_guard<std::mutex> lock(mu_);
    ++tick_;
    int victim = 0;
    for (int i = 0; i < kEntries; ++i) {
      Entry& e = e_[i];
      if (e.used && e.base == base && e.rows == rows && e.kind == kind) {
        e.used = tick_;
        *out = e.map;
        return true;
      }
      if (e.used < e_[victim].used) victim = i;
    }
    if (!encode(out)) return false;
    e_[victim] = Entry{base, rows, kind, tick_, *out};
    return true;
  }

 private:
  static constexpr int kEntries = 32;
  struct Entry {
    const void* base;
    uint64_t rows;
    int kind;
    uint64_t used;
    CUtensorMap map;
  };
  std::mutex mu_;
  uint64_t tick_ = 0;
  Entry e_[kEntries] = {};
};

PairMapCache& pair_maps() {
  static PairMapCache c;
  return c;
}

template <bool AK_ONE>
cudaError_t launch_pair(const DecodeArgs& a, const PairMaps& maps, cudaStream_t st) {
  static PerDeviceOnce attrs;
  cudaError_t e = once_per_device(attrs, [] {
    return cudaFuncSetAttribute(decode_pair_kernel<AK_ONE>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
  });
  if (e != cudaSuccess) return e;
  return launch_chained(decode_pair_kernel<AK_ONE>, dim3(2 * a.ncta), dim3(kThreads), SMEM, st, a, maps);
}

}  // namespace

bool decode_pair_supported(int r, int d_rope, int groups) {
  return r == kRkv && d_rope == kDrope && groups >= 1 && groups <= kMaxGroups;
}

int decode_pair_max_pairs(int sms) {
  static PerDeviceOnce once;
  static int cached[PerDeviceOnce::kTracked] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return sms / 2;
  auto query = [&]() -> cudaError_t {
    cudaError_t e = cudaFuncSetAttribute(decode_pair_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(sms);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = SMEM;
    int n = 0;
    e = cudaOccupancyMaxActiveClusters(&n, decode_pair_kernel<false>, &cfg);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < PerDeviceOnce::kTracked) cached[dev] = n;
    return cudaSuccess;
  };
  if (once.run(dev, cudaSuccess, query) != cudaSuccess) return sms / 2;
  const int n = (dev >= 0 && dev < PerDeviceOnce::kTracked) ? cached[dev] : 0;
  return n > 0 ? (n < sms / 2 ? n : sms / 2) : sms / 2;
}

cudaError_t launch_decode_pair(const DecodeArgs& a, cudaStream_t st) {
  if (!decode_pair_supported(a.r, a.d_rope, a.groups) || a.rows != kRows) return cudaErrorNotSupported;
  PairMaps maps;
  const uint64_t cache_rows = (uint64_t)a.num_blocks * 64;
  const uint64_t q_rows = (uint64_t)a.batch * a.s_q * a.heads;
  PairMapCache& c = pair_maps();
  if (!c.get(a.latent, cache_rows, 0, &maps.latent,
             [&](CUtensorMap* m) { return make_latent_map4(m, a.latent, cache_rows); }) ||
      !c.get(a.k_rope, cache_rows, 1, &maps.krope,
             [&](CUtensorMap* m) {
               return make_map2(m, a.k_rope, kDrope, cache_rows, kRopeHalf, 64, CU_TENSOR_MAP_SWIZZLE_64B);
             }) ||
      !c.get(a.q_tilde, q_rows, 2, &maps.qt,
             [&](CUtensorMap* m) {
               return make_map2(m, a.q_tilde, kRkv, q_rows, 64, kRows, CU_TENSOR_MAP_SWIZZLE_128B);
             }) ||
      !c.get(a.q_rope_hat, q_rows, 3, &maps.qr, [&](CUtensorMap* m) {
        return make_map2(m, a.q_rope_hat, kDrope, q_rows, kRopeHalf, kRows, CU_TENSOR_MAP_SWIZZLE_64B);
      }))
    return cudaErrorInvalidValue;
  return a.ak_one ? launch_pair<true>(a, maps, st) : launch_pair<false>(a, maps, st);
}

}  // namespace qkn
