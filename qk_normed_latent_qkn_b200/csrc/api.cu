// The C ABI of libqkn (declared in include/qkn.h): host-side argument checks,
// kernel selection, the decode workspace layout and kernel launches.  Every
// entry point validates before it enqueues anything, and none allocates.
#include <math.h>
#include <stdio.h>
#include <string.h>

#include "common.cuh"
#include "kernels.h"

using namespace qkn;

namespace {

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

size_t elem_size(qkn_dtype t) { return t == QKN_BF16 ? 2 : 4; }

qkn_status check_dims(const qkn_dims* d) {
  if (!d) return QKN_ERR_INVALID_ARG;
  if (d->dtype != QKN_F32 && d->dtype != QKN_BF16) return QKN_ERR_INVALID_ARG;
  if (d->num_heads <= 0 || d->num_groups <= 0 || d->num_heads % d->num_groups) return QKN_ERR_INVALID_ARG;
  if (d->block_size != kBlockSize) return QKN_ERR_INVALID_ARG;
  if (d->d_h <= 0 || d->d_h > 1024) return QKN_ERR_INVALID_ARG;
  // 16-byte rows for every token-major array (vector loads, TMA rows).
  if (d->r_kv <= 0 || d->r_kv > 1024 || (d->r_kv * elem_size(d->dtype)) % 16) return QKN_ERR_INVALID_ARG;
  if (d->d_rope <= 0 || d->d_rope > 128 || (d->d_rope % 2) ||
      (d->d_rope * elem_size(d->dtype)) % 16)
    return QKN_ERR_INVALID_ARG;
  if (!(d->eps >= 0.f) || !(d->softmax_scale >= 0.f) || !(d->rope_theta > 0.f)) return QKN_ERR_INVALID_ARG;
  const int64_t width = (int64_t)(d->num_heads / d->num_groups) * d->d_h;
  if (width > (1 << 24)) return QKN_ERR_INVALID_ARG;
  return QKN_OK;
}

qkn_status check_cache(const qkn_dims* d, const qkn_cache* c) {
  if (!c || !c->latent || !c->k_rope || !c->a_k || c->num_blocks <= 0) return QKN_ERR_INVALID_ARG;
  if (!aligned(c->latent, 16) || !aligned(c->k_rope, 16) || !aligned(c->a_k, 16) || !aligned(c->ak_scratch, 8))
    return QKN_ERR_INVALID_ARG;
  if ((int64_t)c->num_blocks * kBlockSize > INT32_MAX) return QKN_ERR_INVALID_ARG;
  (void)d;
  return QKN_OK;
}

int sm_count(int* out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  static int cached[64] = {0};
  if (dev >= 0 && dev < 64 && cached[dev] > 0) {
    *out = cached[dev];
    return 0;
  }
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return -1;
  if (dev >= 0 && dev < 64) cached[dev] = n;
  *out = n;
  return 0;
}

int ceil_div(int a, int b) { return (a + b - 1) / b; }

// sigma: the caller's, or 1 / sqrt(d_h + d_R) when the caller passes 0 (the usual scale for a
// logit whose dot products span the content and the RoPE block).
float softmax_scale_of(const qkn_dims* d) {
  return d->softmax_scale > 0.f ? d->softmax_scale : (float)(1.0 / sqrt((double)(d->d_h + d->d_rope)));
}

// RoPE pair frequencies theta^(-2i/d_R) in fp64 (constants of the dims).
RopeFreqs rope_freqs(const qkn_dims* d) {
  RopeFreqs r;
  for (int i = 0; i < 64; ++i) r.f[i] = i < d->d_rope / 2 ? pow((double)d->rope_theta, -2.0 * i / d->d_rope) : 0.0;
  return r;
}

// Rows per tile for the tcgen05 kernels: the smallest supported single-CTA
// tile that covers the per-sequence query rows, at most 64 (the fp32
// accumulator of a 64-row tile already fills an SM's tensor memory).  Tiles of
// 128 rows on CTA pairs that split the latent width (every MMA with 128 rows)
// are taken only when asked for (head_tile = 128): on this build they are
// slower than two 64-row tiles, because every page costs three exchanges
// between the two SMs in series.
int tc_rows(const qkn_dims* d, int s_q, const qkn_decode_opts* o) {
  if (o && o->head_tile) return o->head_tile;
  const int qrows = s_q * d->num_heads;
  if (qrows <= 16) return 16;
  if (qrows <= 32) return 32;
  return 64;
}

bool tc_supported(const qkn_dims* d, int rows) {
  if (rows == kPairRows) return decode_pair_supported(d->r_kv, d->d_rope, d->num_groups);
  return decode_tc_supported(d->r_kv, d->d_rope, rows, d->num_groups);
}

int pick_kernel(const qkn_dims* d, int s_q, const qkn_decode_opts* o) {
  const qkn_kernel want = o ? o->kernel : QKN_KERNEL_AUTO;
  const bool tc_ok = d->dtype == QKN_BF16 && tc_supported(d, tc_rows(d, s_q, o));
  if (want == QKN_KERNEL_SIMT) return QKN_KERNEL_SIMT;
  if (want == QKN_KERNEL_TCGEN05) return tc_ok ? QKN_KERNEL_TCGEN05 : -1;
  if (want != QKN_KERNEL_AUTO) return -1;
  return tc_ok ? QKN_KERNEL_TCGEN05 : QKN_KERNEL_SIMT;
}

struct WsLayout {
  size_t desc_off, lse_off, o_off, total;   // status word | segment descriptors | split lse | split outputs
};

WsLayout ws_layout(const qkn_dims* d, int batch, int s_q, int ncta) {
  // Size for the largest row tile any kernel may use, so that one workspace
  // serves every kernel choice.
  int64_t slot_rows = 0, segments = 0;
  const int qrows = s_q * d->num_heads;
  for (int rows : {kSimtRows, 16, 32, 64, kPairRows}) {
    const int64_t ht = ceil_div(qrows, rows);
    // the CTA-pair kernel's schedule counts pairs: at most half the CTAs
    const int64_t sr = sched_slots(batch, ht, rows == kPairRows ? ncta / 2 : ncta) * rows;
    if (sr > slot_rows) slot_rows = sr;
    if (batch * ht > segments) segments = batch * ht;
  }
  WsLayout w;
  w.desc_off = kStatusBytes;
  w.lse_off = w.desc_off + ((size_t)segments * 8 + 255) / 256 * 256;
  const size_t lse_bytes = ((size_t)slot_rows * 4 + 255) / 256 * 256;
  w.o_off = w.lse_off + lse_bytes;
  w.total = w.o_off + (size_t)slot_rows * d->r_kv * 4;
  return w;
}

}  // namespace

extern "C" {

const char* qkn_status_string(qkn_status s) {
  switch (s) {
    case QKN_OK: return "ok";
    case QKN_ERR_INVALID_ARG: return "invalid argument";
    case QKN_ERR_UNSUPPORTED: return "unsupported configuration";
    case QKN_ERR_CUDA: return "CUDA error";
    case QKN_ERR_TIMEOUT: return "device wait timed out";
    case QKN_ERR_BOUNDS: return "sequence length or block id out of range";
  }
  return "unknown status";
}

int32_t qkn_version(void) { return QKN_VERSION; }

}  // extern "C"

namespace {

// Validated launch arguments of an append (n_tok > 0) or QKN_OK with *empty for n_tok == 0.
qkn_status append_args(const qkn_dims* dims, const qkn_cache* cache, const void* c_new, const void* k_rope_raw,
                       const int32_t* slot, const int32_t* pos, int32_t n_tok, const float* w_k,
                       const float* key_gram, const float* gamma_kr, AppendArgs* a, bool* empty) {
  qkn_status st = check_dims(dims);
  if (st != QKN_OK) return st;
  if (n_tok < 0) return QKN_ERR_INVALID_ARG;
  *empty = n_tok == 0;
  if (*empty) return QKN_OK;
  if ((st = check_cache(dims, cache)) != QKN_OK) return st;
  if (!c_new || !k_rope_raw || !slot || !pos || !(w_k || key_gram) || !gamma_kr) return QKN_ERR_INVALID_ARG;
  if (!aligned(key_gram, 4)) return QKN_ERR_INVALID_ARG;
  if (!aligned(c_new, 16) || !aligned(k_rope_raw, 16)) return QKN_ERR_INVALID_ARG;
  a->latent = cache->latent;
  a->k_rope = cache->k_rope;
  a->a_k = cache->a_k;
  a->ak_scratch = cache->ak_scratch;
  a->c_new = c_new;
  a->k_rope_raw = k_rope_raw;
  a->slot = slot;
  a->pos = pos;
  a->w_k = w_k;
  a->key_gram = key_gram;
  a->gamma_kr = gamma_kr;
  a->n_tok = n_tok;
  a->r = dims->r_kv;
  a->d_rope = dims->d_rope;
  a->groups = dims->num_groups;
  a->width = (dims->num_heads / dims->num_groups) * dims->d_h;
  a->ncols = key_gram ? dims->r_kv : a->width;
  a->n_slots = (int64_t)cache->num_blocks * kBlockSize;
  a->eps = dims->eps;
  a->rope_theta = dims->rope_theta;
  a->freq = rope_freqs(dims);
  return QKN_OK;
}

// Validated launch arguments of a query absorption (n_q > 0) or QKN_OK with *empty for n_q == 0.
qkn_status absorb_args(const qkn_dims* dims, const void* q, const void* q_rope, const int32_t* pos, int32_t n_q,
                       const float* w_k, const float* gamma_q, const float* gamma_k, const float* gamma_qr,
                       void* q_tilde, float* a_q, void* q_rope_hat, AbsorbArgs* a, bool* empty) {
  qkn_status st = check_dims(dims);
  if (st != QKN_OK) return st;
  if (n_q < 0) return QKN_ERR_INVALID_ARG;
  *empty = n_q == 0;
  if (*empty) return QKN_OK;
  if (!q || !q_rope || !pos || !w_k || !gamma_q || !gamma_k || !gamma_qr || !q_tilde || !a_q || !q_rope_hat)
    return QKN_ERR_INVALID_ARG;
  if (dims->d_h > 256 || dims->d_h % 4) return QKN_ERR_UNSUPPORTED;
  if (!aligned(w_k, 16) || !aligned(gamma_q, 16) || !aligned(gamma_k, 16)) return QKN_ERR_INVALID_ARG;
  a->q = q;
  a->q_rope = q_rope;
  a->pos = pos;
  a->w_k = w_k;
  a->gamma_q = gamma_q;
  a->gamma_k = gamma_k;
  a->gamma_qr = gamma_qr;
  a->q_tilde = q_tilde;
  a->a_q = a_q;
  a->q_rope_hat = q_rope_hat;
  a->n_q = n_q;
  a->heads = dims->num_heads;
  a->groups = dims->num_groups;
  a->r = dims->r_kv;
  a->d_h = dims->d_h;
  a->d_rope = dims->d_rope;
  a->eps = dims->eps;
  a->softmax_scale = softmax_scale_of(dims);
  a->rope_theta = dims->rope_theta;
  a->freq = rope_freqs(dims);
  return QKN_OK;
}

}  // namespace

extern "C" {

qkn_status qkn_key_gram(const qkn_dims* dims, const float* w_k, float* key_gram, void* stream) {
  qkn_status st = check_dims(dims);
  if (st != QKN_OK) return st;
  if (!w_k || !key_gram) return QKN_ERR_INVALID_ARG;
  const int width = (dims->num_heads / dims->num_groups) * dims->d_h;
  cudaError_t e = launch_key_gram(w_k, key_gram, dims->num_groups, dims->r_kv, width,
                                  static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? QKN_OK : QKN_ERR_CUDA;
}

qkn_status qkn_append(const qkn_dims* dims, const qkn_cache* cache, const void* c_new,
                      const void* k_rope_raw, const int32_t* slot, const int32_t* pos, int32_t n_tok,
                      const float* w_k, const float* key_gram, const float* gamma_kr, void* stream) {
  AppendArgs a;
  bool empty = false;
  qkn_status st = append_args(dims, cache, c_new, k_rope_raw, slot, pos, n_tok, w_k, key_gram, gamma_kr, &a,
                              &empty);
  if (st != QKN_OK || empty) return st;
  cudaError_t e = launch_append(a, dims->dtype == QKN_BF16, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? QKN_OK : QKN_ERR_CUDA;
}

qkn_status qkn_absorb_query(const qkn_dims* dims, const void* q, const void* q_rope, const int32_t* pos,
                            int32_t n_q, const float* w_k, const float* gamma_q, const float* gamma_k,
                            const float* gamma_qr, void* q_tilde, float* a_q, void* q_rope_hat,
                            void* stream) {
  AbsorbArgs a;
  bool empty = false;
  qkn_status st = absorb_args(dims, q, q_rope, pos, n_q, w_k, gamma_q, gamma_k, gamma_qr, q_tilde, a_q,
                              q_rope_hat, &a, &empty);
  if (st != QKN_OK || empty) return st;
  cudaError_t e = launch_absorb(a, dims->dtype == QKN_BF16, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? QKN_OK : QKN_ERR_CUDA;
}

qkn_status qkn_append_absorb(const qkn_dims* dims, const qkn_cache* cache, const void* c_new,
                             const void* k_rope_raw, const int32_t* slot, const int32_t* pos, int32_t n_tok,
                             const void* q, const void* q_rope, const int32_t* qpos, int32_t n_q,
                             const float* w_k, const float* key_gram, const float* gamma_q, const float* gamma_k,
                             const float* gamma_qr, const float* gamma_kr, void* q_tilde, float* a_q,
                             void* q_rope_hat, void* stream) {
  AppendArgs ap;
  AbsorbArgs ab;
  bool no_append = false, no_absorb = false;
  qkn_status st = append_args(dims, cache, c_new, k_rope_raw, slot, pos, n_tok, w_k, key_gram, gamma_kr, &ap,
                              &no_append);
  if (st != QKN_OK) return st;
  st = absorb_args(dims, q, q_rope, qpos, n_q, w_k, gamma_q, gamma_k, gamma_qr, q_tilde, a_q, q_rope_hat, &ab,
                   &no_absorb);
  if (st != QKN_OK) return st;
  const bool bf16 = dims->dtype == QKN_BF16;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaSuccess;
  if (!no_append && !no_absorb && prep_fusable(ap, ab)) {
    e = launch_prep(ap, ab, bf16, cs);
  } else {
    if (!no_append) e = launch_append(ap, bf16, cs);
    if (e == cudaSuccess && !no_absorb) e = launch_absorb(ab, bf16, cs);
  }
  return e == cudaSuccess ? QKN_OK : QKN_ERR_CUDA;
}

qkn_status qkn_decode_workspace_size(const qkn_dims* dims, int32_t batch, int32_t s_q, int32_t num_sms,
                                     size_t* bytes) {
  qkn_status st = check_dims(dims);
  if (st != QKN_OK) return st;
  if (!bytes || batch < 0 || s_q < 1 || num_sms < 0) return QKN_ERR_INVALID_ARG;
  int n = num_sms;
  if (n == 0 && sm_count(&n) != 0) return QKN_ERR_CUDA;
  *bytes = ws_layout(dims, batch, s_q, n).total;
  return QKN_OK;
}

qkn_status qkn_workspace_init(void* workspace, size_t ws_bytes, void* stream) {
  if (!workspace || ws_bytes < (size_t)kStatusBytes || !aligned(workspace, 256)) return QKN_ERR_INVALID_ARG;
  cudaError_t e = cudaMemsetAsync(workspace, 0, kStatusBytes, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? QKN_OK : QKN_ERR_CUDA;
}

int32_t qkn_decode_kernel_for(const qkn_dims* dims, int32_t s_q, const qkn_decode_opts* opts) {
  if (check_dims(dims) != QKN_OK || s_q < 1) return -1;
  return pick_kernel(dims, s_q, opts);
}

}  // extern "C"

namespace {

// The value up-projection fused into the merge (qkn_decode_up), or none (qkn_decode).
struct UpProj {
  const void* w_uv;
  int32_t d_v;
  void* out_v;
};

// qkn_decode and qkn_decode_up: `out` is the latent output, or null when `up` is given.
qkn_status decode_impl(const qkn_dims* dims, const qkn_cache* cache, qkn_ak_mode ak_mode, const void* q_tilde,
                       const float* a_q, const void* q_rope_hat, const int32_t* block_table, int32_t max_blocks,
                       const int32_t* seq_lens, int32_t batch, int32_t s_q, void* workspace, size_t ws_bytes,
                       void* out, float* lse, const UpProj* up, const qkn_decode_opts* opts, void* stream) {
  qkn_status st = check_dims(dims);
  if (st != QKN_OK) return st;
  if ((st = check_cache(dims, cache)) != QKN_OK) return st;
  if (ak_mode != QKN_AK_CACHE && ak_mode != QKN_AK_ONE) return QKN_ERR_INVALID_ARG;
  if (batch < 0 || s_q < 1 || max_blocks < 1) return QKN_ERR_INVALID_ARG;
  if (up && (up->d_v <= 0 || up->d_v % 16)) return QKN_ERR_INVALID_ARG;
  if (batch == 0) return QKN_OK;
  if (!q_tilde || !a_q || !q_rope_hat || !block_table || !seq_lens || !workspace || !lse)
    return QKN_ERR_INVALID_ARG;
  if (up ? (!up->w_uv || !up->out_v || !aligned(up->w_uv, 16) || !aligned(up->out_v, 16))
         : (!out || !aligned(out, 16)))
    return QKN_ERR_INVALID_ARG;
  if (!aligned(q_tilde, 16) || !aligned(q_rope_hat, 16) || !aligned(workspace, 256)) return QKN_ERR_INVALID_ARG;
  if (up && !combine_up_supported(dims->dtype == QKN_BF16, dims->r_kv, up->d_v, batch * s_q))
    return QKN_ERR_UNSUPPORTED;
  if (opts && (opts->max_ctas < 0 || opts->wait_limit < 0 ||
               (opts->head_tile && opts->head_tile != 16 && opts->head_tile != 32 && opts->head_tile != 64 &&
                opts->head_tile != kPairRows)))
    return QKN_ERR_INVALID_ARG;
  const int kernel = pick_kernel(dims, s_q, opts);
  if (kernel < 0) return QKN_ERR_UNSUPPORTED;

  int nsm = 0;
  if (sm_count(&nsm) != 0) return QKN_ERR_CUDA;
  const WsLayout w = ws_layout(dims, batch, s_q, nsm);
  if (ws_bytes < w.total) return QKN_ERR_INVALID_ARG;
  int ncta = nsm;
  if (opts && opts->max_ctas > 0 && opts->max_ctas < ncta) ncta = opts->max_ctas;
  const bool pair = kernel == QKN_KERNEL_TCGEN05 && tc_rows(dims, s_q, opts) == kPairRows;
  if (pair) {
    // the schedule's unit is a CTA pair: as many as fit at once, within the CTA cap
    const int most = decode_pair_max_pairs(nsm);
    ncta = ncta / 2 < most ? ncta / 2 : most;
    if (ncta < 1) ncta = 1;
  }

  char* ws = static_cast<char*>(workspace);
  DecodeArgs a;
  a.latent = cache->latent;
  a.k_rope = cache->k_rope;
  a.a_k = cache->a_k;
  a.num_blocks = cache->num_blocks;
  a.q_tilde = q_tilde;
  a.a_q = a_q;
  a.q_rope_hat = q_rope_hat;
  a.block_table = block_table;
  a.max_blocks = max_blocks;
  a.seq_lens = seq_lens;
  a.batch = batch;
  a.s_q = s_q;
  a.heads = dims->num_heads;
  a.groups = dims->num_groups;
  a.r = dims->r_kv;
  a.d_rope = dims->d_rope;
  a.ak_one = ak_mode == QKN_AK_ONE;
  a.rows = kernel == QKN_KERNEL_TCGEN05 ? tc_rows(dims, s_q, opts) : kSimtRows;
  a.ht_count = ceil_div(s_q * dims->num_heads, a.rows);
  a.ncta = ncta;
  // starting an item costs about one page of time per 16 query rows of the tile (query tile,
  // pipeline refill, the previous item's epilogue), measured on the tcgen05 kernel
  a.item_cost = kernel == QKN_KERNEL_TCGEN05 ? (a.rows >= 64 ? 3 : a.rows / 16) : 1;
  a.part_lse = reinterpret_cast<float*>(ws + w.lse_off);
  a.part_o = reinterpret_cast<float*>(ws + w.o_off);
  a.status = reinterpret_cast<int32_t*>(ws);
  a.wait_limit = (opts && opts->wait_limit > 0) ? opts->wait_limit : (int64_t)4000000000LL;
  a.out = out;
  a.lse = lse;
  a.seg_desc = reinterpret_cast<int2*>(ws + w.desc_off);
  a.step_writes_only = (opts && opts->step_writes_only) ? 1 : 0;
  a.withhold_ak = (opts && opts->test_withhold_ak) ? 1 : 0;
  a.vis_end = opts ? opts->vis_end : nullptr;

  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  const bool bf16 = dims->dtype == QKN_BF16;
  cudaError_t e = pair ? launch_decode_pair(a, cs)
                  : kernel == QKN_KERNEL_TCGEN05 ? launch_decode_tc(a, cs) : launch_decode_simt(a, bf16, cs);
  if (e != cudaSuccess) return QKN_ERR_CUDA;
  if (opts && opts->split_event &&
      cudaEventRecordWithFlags(static_cast<cudaEvent_t>(opts->split_event), cs, cudaEventRecordExternal) !=
          cudaSuccess)
    return QKN_ERR_CUDA;

  CombineArgs c;
  c.seq_lens = seq_lens;
  c.batch = batch;
  c.s_q = s_q;
  c.heads = dims->num_heads;
  c.r = dims->r_kv;
  c.rows = a.rows;
  c.ht_count = a.ht_count;
  c.ncta = ncta;
  c.item_cost = a.item_cost;
  c.max_blocks = max_blocks;
  c.max_items = ncta + 1;
  c.nslots = sched_slots(batch, a.ht_count, ncta);
  c.part_o = a.part_o;
  c.part_lse = a.part_lse;
  c.out = out;
  c.lse = lse;
  c.status = a.status;
  c.seg_desc = kernel == QKN_KERNEL_TCGEN05 ? a.seg_desc : nullptr;
  if (up) {
    CombineUpArgs u;
    u.c = c;
    u.w_uv = up->w_uv;
    u.d_v = up->d_v;
    u.out_v = up->out_v;
    e = launch_combine_up(u, bf16, cs);
  } else {
    e = launch_combine(c, bf16, cs);
  }
  return e == cudaSuccess ? QKN_OK : QKN_ERR_CUDA;
}

}  // namespace

extern "C" {

qkn_status qkn_decode(const qkn_dims* dims, const qkn_cache* cache, qkn_ak_mode ak_mode, const void* q_tilde,
                      const float* a_q, const void* q_rope_hat, const int32_t* block_table, int32_t max_blocks,
                      const int32_t* seq_lens, int32_t batch, int32_t s_q, void* workspace, size_t ws_bytes,
                      void* out, float* lse, const qkn_decode_opts* opts, void* stream) {
  return decode_impl(dims, cache, ak_mode, q_tilde, a_q, q_rope_hat, block_table, max_blocks, seq_lens, batch, s_q,
                     workspace, ws_bytes, out, lse, nullptr, opts, stream);
}

qkn_status qkn_decode_up(const qkn_dims* dims, const qkn_cache* cache, qkn_ak_mode ak_mode, const void* q_tilde,
                         const float* a_q, const void* q_rope_hat, const int32_t* block_table, int32_t max_blocks,
                         const int32_t* seq_lens, int32_t batch, int32_t s_q, const void* w_uv, int32_t d_v,
                         void* workspace, size_t ws_bytes, void* out_v, float* lse, const qkn_decode_opts* opts,
                         void* stream) {
  const UpProj up{w_uv, d_v, out_v};
  return decode_impl(dims, cache, ak_mode, q_tilde, a_q, q_rope_hat, block_table, max_blocks, seq_lens, batch, s_q,
                     workspace, ws_bytes, nullptr, lse, &up, opts, stream);
}

qkn_status qkn_merge_partials(const qkn_dims* dims, int32_t n_parts, int64_t rows, const void* parts,
                              const float* lse_parts, void* out, float* lse, void* stream) {
  qkn_status st = check_dims(dims);
  if (st != QKN_OK) return st;
  if (n_parts < 1 || rows < 0) return QKN_ERR_INVALID_ARG;
  if (rows == 0) return QKN_OK;
  if (rows > INT32_MAX) return QKN_ERR_INVALID_ARG;   // grid x of row groups
  if (!parts || !lse_parts || !out || !lse || !aligned(parts, 16) || !aligned(out, 16)) return QKN_ERR_INVALID_ARG;
  cudaError_t e = launch_merge_parts(parts, lse_parts, n_parts, rows, dims->r_kv, out, lse, dims->dtype == QKN_BF16,
                                     static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? QKN_OK : QKN_ERR_CUDA;
}

qkn_status qkn_read_device_status(const void* workspace, void* stream, int32_t* device_status) {
  if (!workspace || !device_status) return QKN_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return QKN_ERR_CUDA;
  int32_t v = 0;
  if (cudaMemcpy(&v, workspace, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return QKN_ERR_CUDA;
  *device_status = v;
  return QKN_OK;
}

}  // extern "C"

// ---------------------------------------------------------------- the GQA route

namespace {

qkn_status check_gqa_cache(const qkn_gqa_cache* c) {
  if (!c || !c->k || !c->v || !c->k_rope || c->num_blocks <= 0 || c->d_v <= 0) return QKN_ERR_INVALID_ARG;
  if (!aligned(c->k, 16) || !aligned(c->v, 16) || !aligned(c->k_rope, 16)) return QKN_ERR_INVALID_ARG;
  if ((int64_t)c->num_blocks * kBlockSize > INT32_MAX) return QKN_ERR_INVALID_ARG;
  return QKN_OK;
}

// Query rows per tile and tiles per group: a dense tile holds the group's rows of every query token
// of the step (s_q n_g of them), a sparse one those of one query token (n_g), in tiles of 16 or 32.
void gqa_tiling(const qkn_dims* d, int s_q, bool sparse, int* rows, int* tpg) {
  const int ng = d->num_heads / d->num_groups;
  const int span = sparse ? ng : s_q * ng;
  *rows = span <= 16 ? 16 : 32;
  *tpg = ceil_div(span, *rows);
}

// Dense decode CTAs: one per SM (capped), whole groups of the schedule's row tiles where they fit.
int gqa_ncta(int nsm, int ht, int max_ctas) {
  int n = nsm;
  if (max_ctas > 0 && max_ctas < n) n = max_ctas;
  if (n >= ht) n = n / ht * ht;
  return n;
}

struct GqaWs {
  size_t lse_off, o_off, total;   // status word | split lse | split outputs
};

GqaWs gqa_ws_layout(const qkn_dims* d, int d_v, int batch, int s_q, int nsm) {
  int rows = 0, tpg = 0;
  gqa_tiling(d, s_q, false, &rows, &tpg);
  const int64_t ht = (int64_t)d->num_groups * tpg;
  // any CTA cap gives at most nsm CTAs, so nsm bounds the slots
  const int64_t slot_rows = sched_slots(batch, ht, nsm) * rows;
  GqaWs w;
  w.lse_off = kStatusBytes;
  w.o_off = w.lse_off + ((size_t)slot_rows * 4 + 255) / 256 * 256;
  w.total = w.o_off + (size_t)slot_rows * d_v * 4;
  return w;
}

}  // namespace

extern "C" {

qkn_status qkn_gqa_append(const qkn_dims* dims, const qkn_gqa_cache* cache, const void* c_new,
                          const void* k_rope_raw, const int32_t* slot, const int32_t* pos, int32_t n_tok,
                          const float* w_uk, const float* gamma_k, const void* w_uv, const float* gamma_kr,
                          void* stream) {
  qkn_status st = check_dims(dims);
  if (st != QKN_OK) return st;
  if (n_tok < 0) return QKN_ERR_INVALID_ARG;
  if ((st = check_gqa_cache(cache)) != QKN_OK) return st;
  if (dims->dtype != QKN_BF16 || !gqa_supported(dims->d_h, dims->d_rope, cache->d_v)) return QKN_ERR_UNSUPPORTED;
  // the expansion stages the latent 32 columns at a time; one grid row per group
  if (dims->r_kv % 32 || dims->num_groups > 65535) return QKN_ERR_UNSUPPORTED;
  if (n_tok == 0) return QKN_OK;
  if (!c_new || !k_rope_raw || !slot || !pos || !w_uk || !gamma_k || !w_uv || !gamma_kr) return QKN_ERR_INVALID_ARG;
  if (!aligned(c_new, 16) || !aligned(k_rope_raw, 16) || !aligned(w_uk, 16) || !aligned(w_uv, 16) ||
      !aligned(gamma_k, 4) || !aligned(gamma_kr, 4))
    return QKN_ERR_INVALID_ARG;
  GqaAppendArgs a;
  a.k_cache = cache->k;
  a.v_cache = cache->v;
  a.k_rope = cache->k_rope;
  a.c_new = c_new;
  a.k_rope_raw = k_rope_raw;
  a.slot = slot;
  a.pos = pos;
  a.w_uk = w_uk;
  a.gamma_k = gamma_k;
  a.w_uv = w_uv;
  a.gamma_kr = gamma_kr;
  a.n_tok = n_tok;
  a.r = dims->r_kv;
  a.d_h = dims->d_h;
  a.d_v = cache->d_v;
  a.d_rope = dims->d_rope;
  a.groups = dims->num_groups;
  a.n_slots = (int64_t)cache->num_blocks * kBlockSize;
  a.eps = dims->eps;
  a.freq = rope_freqs(dims);
  cudaError_t e = launch_gqa_append(a, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? QKN_OK : QKN_ERR_CUDA;
}

qkn_status qkn_gqa_workspace_size(const qkn_dims* dims, int32_t d_v, int32_t batch, int32_t s_q, int32_t num_sms,
                                  size_t* bytes) {
  qkn_status st = check_dims(dims);
  if (st != QKN_OK) return st;
  if (!bytes || d_v <= 0 || batch < 0 || s_q < 1 || num_sms < 0) return QKN_ERR_INVALID_ARG;
  int n = num_sms;
  if (n == 0 && sm_count(&n) != 0) return QKN_ERR_CUDA;
  *bytes = gqa_ws_layout(dims, d_v, batch, s_q, n).total;
  return QKN_OK;
}

qkn_status qkn_gqa_decode(const qkn_dims* dims, const qkn_gqa_cache* cache, const void* q, const void* q_rope,
                          const float* gamma_q, const float* gamma_qr, const int32_t* block_table,
                          int32_t max_blocks, const int32_t* seq_lens, int32_t batch, int32_t s_q,
                          const int32_t* selection, int32_t sel_k, void* workspace, size_t ws_bytes, void* out_v,
                          float* lse, int32_t max_ctas, void* stream) {
  qkn_status st = check_dims(dims);
  if (st != QKN_OK) return st;
  if ((st = check_gqa_cache(cache)) != QKN_OK) return st;
  if (dims->dtype != QKN_BF16 || !gqa_supported(dims->d_h, dims->d_rope, cache->d_v)) return QKN_ERR_UNSUPPORTED;
  if (batch < 0 || s_q < 1 || max_blocks < 1 || max_ctas < 0 || (selection && sel_k < 1)) return QKN_ERR_INVALID_ARG;
  if (batch == 0) return QKN_OK;
  if (!q || !q_rope || !gamma_q || !gamma_qr || !block_table || !seq_lens || !workspace || !out_v || !lse)
    return QKN_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(q_rope, 16) || !aligned(out_v, 16) || !aligned(workspace, 256) ||
      !aligned(gamma_q, 4) || !aligned(gamma_qr, 4))
    return QKN_ERR_INVALID_ARG;
  int nsm = 0;
  if (sm_count(&nsm) != 0) return QKN_ERR_CUDA;
  const bool sparse = selection != nullptr;
  const GqaWs w = gqa_ws_layout(dims, cache->d_v, batch, s_q, nsm);
  if (ws_bytes < (sparse ? (size_t)kStatusBytes : w.total)) return QKN_ERR_INVALID_ARG;

  char* ws = static_cast<char*>(workspace);
  GqaDecodeArgs a;
  a.k_cache = cache->k;
  a.v_cache = cache->v;
  a.k_rope = cache->k_rope;
  a.num_blocks = cache->num_blocks;
  a.q = q;
  a.q_rope = q_rope;
  a.gamma_q = gamma_q;
  a.gamma_qr = gamma_qr;
  a.block_table = block_table;
  a.max_blocks = max_blocks;
  a.seq_lens = seq_lens;
  a.batch = batch;
  a.s_q = s_q;
  a.heads = dims->num_heads;
  a.groups = dims->num_groups;
  a.d_h = dims->d_h;
  a.d_rope = dims->d_rope;
  a.d_v = cache->d_v;
  gqa_tiling(dims, s_q, sparse, &a.rows, &a.tpg);
  a.ht_count = dims->num_groups * a.tpg;
  a.ncta = gqa_ncta(nsm, a.ht_count, max_ctas);
  // starting an item (the tile's queries, filling the ring) is taken as two pages of time, an
  // estimate from the ring's depth that no measurement has tuned yet
  a.item_cost = 2;
  a.selection = selection;
  a.sel_k = sparse ? sel_k : 0;
  a.part_o = reinterpret_cast<float*>(ws + w.o_off);
  a.part_lse = reinterpret_cast<float*>(ws + w.lse_off);
  a.out = out_v;
  a.lse = lse;
  a.status = reinterpret_cast<int32_t*>(ws);
  a.eps = dims->eps;
  a.score_scale = softmax_scale_of(dims) * 1.4426950408889634f;   // sigma * log2(e)
  a.freq = rope_freqs(dims);
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  cudaError_t e = launch_gqa_decode(a, cs);
  if (e == cudaErrorNotSupported) return QKN_ERR_UNSUPPORTED;
  if (e != cudaSuccess) return QKN_ERR_CUDA;
  if (sparse) return QKN_OK;

  CombineArgs c;
  c.seq_lens = seq_lens;
  c.batch = batch;
  c.s_q = s_q;
  c.heads = dims->num_heads;
  c.r = cache->d_v;
  c.rows = a.rows;
  c.ht_count = a.ht_count;
  c.ncta = a.ncta;
  c.item_cost = a.item_cost;
  c.max_blocks = max_blocks;
  c.max_items = a.ncta + 1;
  c.nslots = sched_slots(batch, a.ht_count, a.ncta);
  c.part_o = a.part_o;
  c.part_lse = a.part_lse;
  c.out = out_v;
  c.lse = lse;
  c.status = a.status;
  c.seg_desc = nullptr;
  c.group_heads = dims->num_heads / dims->num_groups;
  c.tiles_per_group = a.tpg;
  e = launch_combine_grouped(c, cs);
  return e == cudaSuccess ? QKN_OK : QKN_ERR_CUDA;
}

}  // extern "C"
