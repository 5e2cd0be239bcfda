// Shared device helpers for libqkn: element types, the device status word,
// and the split-KV work schedule used by the decode and combine kernels.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include <utility>

#include "per_device.h"
#include "qkn.h"

namespace qkn {

constexpr int kBlockSize = 64;          // tokens per cache page
constexpr int kStatusBytes = 256;       // workspace header holding the status word

// ---------------------------------------------------------------- elements
__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// ---------------------------------------------------------------- launch chaining
// Kernels are launched with programmatic stream serialisation: each one lets
// its successor start launching at once (pdl_trigger) and waits for its
// predecessor's completion and memory flush (pdl_wait) before it reads
// anything an earlier launch may have written.  Without a programmatic
// predecessor pdl_wait returns immediately.
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Launch `kernel` on `st` with programmatic stream serialisation.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_chained(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                                  Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Opt a kernel into large dynamic shared memory and ask for the largest
// shared-memory carveout, so that several of its CTAs fit on one SM (the
// default carveout can hold the SM to one CTA of a kernel that uses 64 KB).
template <typename... KArgs>
inline cudaError_t set_smem_attrs(void (*kernel)(KArgs...), int max_dynamic_bytes) {
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, max_dynamic_bytes);
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                              (int)cudaSharedmemCarveoutMaxShared);
}

// Run a kernel's one-time attribute set-up on the current device: attributes
// are per device, so each device of the process gets its own (per_device.h).
template <typename F>
inline cudaError_t once_per_device(PerDeviceOnce& once, F&& setup) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  return once.run(dev, cudaSuccess, std::forward<F>(setup));
}

// ---------------------------------------------------------------- RoPE
// sin and cos of pos * freq.  The angle is formed and reduced to [-pi, pi] in
// fp64 (one-constant reduction by 2*pi is exact to ~1e-11 here, positions stay
// below 2^31), so that positions in the hundreds of thousands keep fp32
// accuracy; the reduced angle then goes through fp32 sincosf.
__device__ __forceinline__ void rope_sincos(int32_t pos, double freq, float& s, float& c) {
  const double ang = (double)pos * freq;
  const double k = rint(ang * 0.15915494309189535);            // 1 / (2 pi)
  const double red = fma(-k, 6.283185307179586, ang);          // ang - k * 2 pi
  sincosf((float)red, &s, &c);
}

// ---------------------------------------------------------------- status word
// The first int32 of the decode workspace.  Kernels record the first error
// they see (compare-and-swap from QKN_OK); the host reads it after a sync.
__device__ __forceinline__ void record_status(int32_t* status, int32_t code) {
  if (status) atomicCAS(status, (int32_t)QKN_OK, code);
}

// ---------------------------------------------------------------- schedule
// The decode work of one step: every sequence b has n(b) cache pages of 64
// tokens and HT query-row tiles; a segment is (sequence b, row tile ht).
// The CTAs form groups of HC = min(HT, ncta) CTAs, G = floor(ncta / HC) of
// them; CTA c is member c mod HC of group c / HC and takes the row tiles ht
// with ht mod HC = c mod HC.  The pages are laid out in "units", sequence by
// sequence; group g takes the contiguous unit range [g*Q, (g+1)*Q),
// Q = ceil(total / G), and every member works on the same pages for its own
// row tiles.  So the CTAs that read a page for different row tiles read it at
// about the same time, and the second read comes from L2 rather than HBM.
// Every sequence starts with `item_cost` units that carry no page: starting
// an item (loading its query tile, refilling the pipeline, writing the
// previous item's result) costs about that many pages of time, so a group
// whose range holds a sequence start gets that many pages fewer.  Sequence b
// is X + n(b) units (X = item_cost), its pages the last n(b) of them.
// The piece of segment (b, ht) that a CTA of group g works on is an "item";
// its partial result goes to workspace slot (b + g) * HT + ht, unique because
// sequences and groups advance together.
struct SchedParams {
  const int32_t* seq_lens;
  int32_t batch;
  int32_t s_q;
  int32_t max_blocks;
  int32_t ht_count;     // query-row tiles per sequence (HT)
  int32_t ncta;
  int32_t item_cost;    // units without pages at the start of every sequence
  // Decode kernels only (0 / null elsewhere): with heads and the rows per tile known, an item ends at
  // the last page its tile's rows can see (the causal limit of the tile's last query row), so that
  // the row tiles of a long chunk of queries (a prefill) skip the pages past their limit.  Such an
  // item may have no pages at all; it still takes its slot (zero output, lse = -inf).
  int32_t heads = 0;
  int32_t rows = 0;
  const int32_t* vis_end = nullptr;
};

__device__ __forceinline__ int32_t pages_of(int32_t L, const SchedParams& p) {
  if (L < p.s_q || L > p.max_blocks * kBlockSize) return 0;   // rejected length
  return (L + kBlockSize - 1) / kBlockSize;
}

// Units of a sequence with n pages (none for a rejected length).
__device__ __forceinline__ int64_t seq_units(int32_t n, const SchedParams& p) {
  return n > 0 ? (int64_t)n + p.item_cost : 0;
}

// CTAs per group (HC) and groups (G).
__device__ __forceinline__ int32_t sched_group_size(const SchedParams& p) {
  return p.ht_count < p.ncta ? p.ht_count : (p.ncta > 0 ? p.ncta : 1);
}
__device__ __forceinline__ int32_t sched_groups(const SchedParams& p) {
  const int32_t g = p.ncta / sched_group_size(p);
  return g > 0 ? g : 1;
}

// Units of sequences [0, b_end), computed by one full warp (all lanes get the result).
__device__ __forceinline__ int64_t sched_units_before(const SchedParams& p, int32_t b_end) {
  const int lane = threadIdx.x & 31;
  int64_t acc = 0;
  for (int b0 = 0; b0 < b_end; b0 += 32) {
    int b = b0 + lane;
    int64_t n = (b < b_end) ? seq_units(pages_of(p.seq_lens[b], p), p) : 0;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) n += __shfl_xor_sync(0xffffffffu, n, o);
    acc += n;
  }
  return acc;
}

// Total units, computed by one full warp.
__device__ __forceinline__ int64_t sched_total_units(const SchedParams& p) {
  return sched_units_before(p, p.batch);
}

// Cursor over the items of one CTA.  Start it with sched_begin (one full
// warp), copy it to every role, then step with sched_next (any thread).
struct Cursor {
  int64_t begin, end;    // the group's unit range
  int64_t seq_u0;        // first unit of the current sequence
  int32_t b, ht;         // current sequence and row tile
  int32_t n;             // pages of sequence b
  int32_t group;         // g
  int32_t ht0, hstep;    // this CTA's first row tile and the step between its row tiles (HC)
  int64_t quota;         // Q
};

// Item handed to the roles: pages [p0, p1) of sequence b, row tile ht; the
// sequence's units are [seg_u0, seg_u0 + item_cost + (pages of b)).
struct Item {
  int32_t b, ht, p0, p1, L, slot;
  int64_t seg_u0;
};

__device__ __forceinline__ Cursor sched_begin(const SchedParams& p, int32_t cta) {
  Cursor cur;
  const int lane = threadIdx.x & 31;
  const int64_t total = sched_total_units(p);
  const int32_t hc = sched_group_size(p), ng = sched_groups(p);
  const int64_t q = (total + ng - 1) / ng;
  cur.quota = q > 0 ? q : 1;
  cur.group = cta / hc;
  cur.ht0 = cta - cur.group * hc;
  cur.hstep = hc;
  cur.ht = cur.ht0;
  cur.begin = (int64_t)cur.group * cur.quota;
  cur.end = cur.begin + cur.quota < total ? cur.begin + cur.quota : total;
  cur.b = p.batch;
  cur.n = 0;
  cur.seq_u0 = total;
  if (cur.group >= ng || cur.ht0 >= p.ht_count || cur.begin >= cur.end) {
    cur.begin = cur.end = total;                     // no work
    return cur;
  }
  // Find the sequence holding unit `begin`: scan with a warp prefix sum.
  int64_t base = 0;
  for (int b0 = 0; b0 < p.batch; b0 += 32) {
    int b = b0 + lane;
    int64_t n = (b < p.batch) ? seq_units(pages_of(p.seq_lens[b], p), p) : 0;
    int64_t incl = n;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int64_t v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    const int64_t lo = base + incl - n, hi = base + incl;
    const unsigned hit = __ballot_sync(0xffffffffu, b < p.batch && n > 0 && cur.begin >= lo && cur.begin < hi);
    if (hit) {
      const int src = __ffs(hit) - 1;
      cur.seq_u0 = __shfl_sync(0xffffffffu, lo, src);
      cur.b = b0 + src;
      cur.n = pages_of(p.seq_lens[cur.b], p);
      return cur;
    }
    base += __shfl_sync(0xffffffffu, incl, 31);
  }
  return cur;
}

// Returns false when the CTA has no further item.  Any single thread.
__device__ __forceinline__ bool sched_next(Cursor& cur, const SchedParams& p, int32_t cta, Item& it) {
  (void)cta;
  while (cur.b < p.batch && cur.seq_u0 < cur.end) {
    // the sequence's pages are units [s0 + item_cost, s1)
    const int64_t s0 = cur.seq_u0, s1 = s0 + seq_units(cur.n, p);
    const int64_t pg0 = s0 + p.item_cost;
    const int64_t lo = cur.begin > pg0 ? cur.begin : pg0, hi = cur.end < s1 ? cur.end : s1;
    const bool overlaps = cur.n > 0 && lo < hi && cur.ht < p.ht_count;
    if (overlaps) {
      it.b = cur.b;
      it.ht = cur.ht;
      it.p0 = (int32_t)(lo - pg0);
      it.p1 = (int32_t)(hi - pg0);
      it.L = p.seq_lens[cur.b];
      it.slot = (cur.b + cur.group) * p.ht_count + cur.ht;
      it.seg_u0 = s0;
      if (p.heads > 0) {
        const int32_t jmax = min(p.s_q - 1, (cur.ht * p.rows + p.rows - 1) / p.heads);
        const int32_t last = (p.vis_end ? p.vis_end[cur.b] : it.L) - p.s_q + jmax;   // last visible token
        const int32_t lim = last >= 0 ? last / kBlockSize + 1 : 0;
        if (it.p1 > lim) it.p1 = lim > it.p0 ? lim : it.p0;
      }
      cur.ht += cur.hstep;                       // this CTA's next row tile of the same pages
      if (cur.ht < p.ht_count) return true;
    }
    // advance to the next sequence
    cur.ht = cur.ht0;
    cur.seq_u0 = s1;
    ++cur.b;
    cur.n = cur.b < p.batch ? pages_of(p.seq_lens[cur.b], p) : 0;
    if (overlaps) return true;
  }
  return false;
}

// The groups that share a sequence: its pages, units [u0 + item_cost, u0 +
// item_cost + n), are split over groups g0 .. g0 + nitems - 1 (quota q units
// each); the partial results of segment (b, ht) sit in workspace slots
// (b + g) * HT + ht for those groups: first slot (b + g0) * HT + ht, then
// every HT-th slot.
struct SegSplit {
  int32_t c0, nitems;   // first group, number of splits
};
__device__ __forceinline__ SegSplit seg_split(int64_t u0, int32_t n, int64_t q, int32_t item_cost) {
  SegSplit s;
  const int64_t pg0 = u0 + item_cost;
  s.c0 = (int32_t)(pg0 / q);
  s.nitems = (int32_t)((pg0 + n - 1) / q) - s.c0 + 1;
  return s;
}

// Workspace slots needed: one per (segment, CTA) pair that can meet.
inline int64_t sched_slots(int64_t batch, int64_t ht_count, int64_t ncta) {
  return batch * ht_count + ncta;
}

}  // namespace qkn
