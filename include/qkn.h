/*
 * qkn.h — C ABI of libqkn: QK-Normed MLA absorbed latent decode attention
 * for NVIDIA B200 (sm_100a).
 *
 * The method ("QK-Normed MLA: QK normalization without full key caching",
 * technical summary, Metodología items 1–4 and the decode-logit equation;
 * arXiv abstract) keeps MLA's latent cache and adds post-projection QK
 * RMSNorm without ever materialising a key:
 *   - RMSNorm(z) = z * gamma / S(z) splits into a static weight gamma and a
 *     dynamic scalar S(z);
 *   - the static key weight gamma_k (and gamma_q) are folded into the query
 *     side: q~[i,h] = W^K_{g(h),h} (gamma_q[h] * gamma_k[h] * q[i,h]);
 *   - the dynamic key statistic becomes one inverse-RMS scalar per token and
 *     KV group, a_k[t,g] = 1 / S(c_t W^K_g), cached next to the latent c_t;
 *   - content and RoPE blocks are normalised separately; the RoPE block uses
 *     ordinary materialised vectors;
 *   - decode logits are l[i,t,h] = (q~[i,h] . c_t) * a_q[i,h] * a_k[t,g(h)]
 *     + q^R^[i,h] . k^R^_t, a row/column rescale applied before the softmax;
 *     the output is the softmax-weighted sum of the latents c_t.
 *
 * Conventions shared by every call
 *   - All tensor arguments are DEVICE pointers to caller-owned memory,
 *     row-major, densely packed in the order the comments give.  The library
 *     allocates nothing (the decode workspace is caller-allocated too).
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Every call
 *     only validates host-side arguments and enqueues kernels; it returns
 *     before the GPU work runs.
 *   - Argument errors are found on the host before anything is launched and
 *     return QKN_ERR_INVALID_ARG or QKN_ERR_UNSUPPORTED; nothing is enqueued
 *     then.  A failed launch returns QKN_ERR_CUDA.  Problems only the device
 *     can see (a sequence length out of range, a bounded wait that ran out)
 *     are recorded in the workspace's status word; read it with
 *     qkn_read_device_status.
 *   - dtype QKN_BF16 means activations (c, k^R, q, q^R), the cache, q~, q^R^
 *     and the output are bf16; QKN_F32 means they are fp32.  Weights, norm
 *     weights, a_k, a_q and lse are always fp32.
 */
#ifndef QKN_H_
#define QKN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define QKN_VERSION 1

#if defined(__GNUC__)
#define QKN_EXPORT __attribute__((visibility("default")))
#else
#define QKN_EXPORT
#endif

typedef enum {
  QKN_OK = 0,
  QKN_ERR_INVALID_ARG = 1,   /* bad pointer, size, alignment or shape */
  QKN_ERR_UNSUPPORTED = 2,   /* valid but not implemented (e.g. a forced kernel that cannot take these dims) */
  QKN_ERR_CUDA = 3,          /* a CUDA runtime call or launch failed */
  QKN_ERR_TIMEOUT = 4,       /* device: a bounded wait inside a kernel ran out */
  QKN_ERR_BOUNDS = 5         /* device: a sequence length or block id outside its stated range */
} qkn_status;

typedef enum { QKN_F32 = 0, QKN_BF16 = 1 } qkn_dtype;

/* Column scale used by qkn_decode.  QKN_AK_ONE treats every a_k as 1 and does
 * not read the a_k cache: that is plain absorbed MLA on the same cache, the
 * baseline for the method's overhead. */
typedef enum { QKN_AK_CACHE = 0, QKN_AK_ONE = 1 } qkn_ak_mode;

/* Decode kernel choice.  AUTO takes the tcgen05 kernel whenever the dims
 * allow it and the CUDA-core kernel otherwise. */
typedef enum { QKN_KERNEL_AUTO = 0, QKN_KERNEL_SIMT = 1, QKN_KERNEL_TCGEN05 = 2 } qkn_kernel;

/* Model dimensions.  num_heads query heads form num_groups KV groups of
 * n_g = num_heads / num_groups consecutive heads; head h belongs to group
 * h / n_g and is slot h % n_g inside it.  W^K_g has n_g * d_h output columns,
 * head h's key slice being columns [(h % n_g) * d_h, (h % n_g + 1) * d_h). */
typedef struct {
  int32_t num_heads;
  int32_t num_groups;
  int32_t r_kv;          /* latent width r */
  int32_t d_h;           /* per-head content dimension */
  int32_t d_rope;        /* RoPE dimension d_R (even) */
  int32_t block_size;    /* cache page size in tokens; must be 64 */
  float eps;             /* RMSNorm: S(z) = sqrt(mean(z^2) + eps), all four norms */
  float softmax_scale;   /* sigma, applied to the whole logit (content + RoPE); 0 = 1/sqrt(d_h + d_rope) */
  float rope_theta;      /* RoPE base; pairs (i, i + d_R/2), angle pos * theta^(-2i/d_R) */
  qkn_dtype dtype;
} qkn_dims;

/* The decode cache (technical summary, Metodología item 3: the latent c_t is
 * the dominant state plus a small scalar cache of inverse RMS values; no
 * normalised key is stored).  Caller-allocated device memory:
 *   latent [num_blocks, block_size, r_kv]   dtype
 *   k_rope [num_blocks, block_size, d_rope] dtype, RMS-normalised and rotated
 *   a_k    [num_blocks, block_size, num_groups] fp32
 * Slot s of the pool is token s % block_size of block s / block_size.
 * Slots that no qkn_append has written may hold anything; decode never lets
 * them reach its output.
 *   ak_scratch [num_blocks, block_size, num_groups, 2] 32-bit words, optional:
 *     zero when allocated (e.g. cudaMemset); every qkn_append that completes
 *     leaves it zero again.  With it, qkn_append runs as one launch (a key
 *     statistic accumulator and an arrival count per slot and group); with
 *     NULL it runs as three.  After an append that did not complete (a
 *     sticky CUDA error), clear it again before the next append.  Decode
 *     does not read it. */
typedef struct {
  void* latent;
  void* k_rope;
  float* a_k;
  int32_t num_blocks;
  uint32_t* ak_scratch;
} qkn_cache;

/* Optional decode knobs (pass NULL for defaults). */
typedef struct {
  qkn_kernel kernel;       /* default QKN_KERNEL_AUTO */
  int32_t max_ctas;        /* cap on decode CTAs (split-KV width; CTA pairs take max_ctas / 2);
                              0 = one per SM */
  int32_t head_tile;       /* tcgen05: query rows per tile (16, 32 or 64 on one CTA; 128 on a pair of
                              CTAs that split the latent width, r_kv = 512, d_rope = 64, at most 4
                              groups); 0 = automatic (the smallest of 16, 32, 64 that covers a
                              sequence's query rows, 64 beyond that) */
  int64_t wait_limit;      /* bounded-wait limit in clock cycles for the mbarrier waits; 0 = default (~2 s) */
  void* split_event;       /* optional cudaEvent_t recorded between the split-KV kernel and the combine
                              kernel (external record, so it also works inside stream capture) */
  int32_t step_writes_only;/* 1: the caller guarantees that the work enqueued on `stream` since the
                              previous decode of these sequences wrote, of everything the decode reads,
                              only the queries (q_tilde, a_q, q_rope_hat) and the cache slots of each
                              sequence's last s_q tokens, and that it is complete or is one launch of
                              qkn_append_absorb or qkn_append made just before the decode (as in a
                              decode step; those kernels let the decode launch only once everything
                              enqueued before them is complete).  The tcgen05 decode then reads the lengths and the block
                              table and streams the other cache pages while that kernel is still
                              running, and waits for it only before the queries and the pages that hold
                              new tokens.  0 (default): it waits before reading anything. */
  int32_t test_withhold_ak;/* tests only: 1 makes the tcgen05 decode's producer skip the a_k copy of
                              every CTA's first cache page, so that the softmax's bounded wait for it
                              runs out: the decode records QKN_ERR_TIMEOUT, winds down (copies and
                              MMAs in flight are waited for, tensor memory is freed) and the merge
                              writes no partial it cannot vouch for.  It exercises the timeout path
                              without faulting or hanging the GPU.  Ignored with QKN_AK_ONE.  0 in use. */
  const int32_t* vis_end;  /* optional DEVICE array [batch]: where each sequence ends for the causal
                              limit, in this call's token numbering (token t of sequence b is the
                              t-th token of the pages block_table[b] lists).  Query j of sequence b
                              sees the tokens t <= vis_end[b] - s_q + j among the seq_lens[b] tokens
                              the call covers.  For a call that covers only part of a sequence's
                              pages (context parallelism: block_table[b] starts at the slice's first
                              page and seq_lens[b] counts the slice's tokens), vis_end[b] is the
                              sequence's length counted from that first page, so the limit stays the
                              whole sequence's.  NULL (default): vis_end = seq_lens. */
} qkn_decode_opts;

/* qkn_key_gram — G_g = W^K_g (W^K_g)^T for every group g, the r_kv x r_kv
 * matrix with which qkn_append computes the key statistic without forming
 * the key: sum over the n_g * d_h columns of (c W^K_g)^2 equals c G_g c^T.
 * The pages define the statistic on the up-projected key (technical summary,
 * Metodología items 2-4); the Gram form is the same sum, reached through
 * r_kv x r_kv products instead of r_kv x n_g d_h, and is this library's.
 * Accumulated in fp64, stored in fp32.  Compute it once per weight set.
 *   w_k      [num_groups, r_kv, n_g * d_h] fp32
 *   key_gram [num_groups, r_kv, r_kv] fp32 (out), symmetric
 * Returns QKN_ERR_INVALID_ARG for bad dims or NULL pointers. */
QKN_EXPORT qkn_status qkn_key_gram(const qkn_dims* dims, const float* w_k, float* key_gram, void* stream);

/* qkn_append — write n_tok new tokens into the cache.
 * For token i with slot s = slot[i] and position p = pos[i]:
 *   latent[s]  = c_new[i]                                    (copied as is)
 *   k_rope[s]  = RoPE_p(gamma_kr * k_rope_raw[i] / S(k_rope_raw[i]))
 *   a_k[s, g]  = 1 / S(c_new[i] W^K_g)   for every group g,
 * S(z) = sqrt(mean(z^2) + eps) over the full n_g * d_h width of c W^K_g.
 * This is the dynamic key statistic reduced to one scalar per token and KV
 * group, computed once at append time (technical summary, Metodología items
 * 2 and 4).  No key is stored.
 *   c_new      [n_tok, r_kv]   dtype
 *   k_rope_raw [n_tok, d_rope] dtype
 *   slot, pos  [n_tok] int32; every slot in [0, num_blocks * block_size)
 *   w_k        [num_groups, r_kv, n_g * d_h] fp32
 *   key_gram   [num_groups, r_kv, r_kv] fp32 from qkn_key_gram(w_k), or NULL.
 *              Given, the statistic is summed as c G_g c^T and w_k is not read
 *              (it may be NULL); NULL, as sum((c W^K_g)^2) from w_k.  The two
 *              agree up to fp32 rounding.
 *   gamma_kr   [d_rope] fp32 (shared by all heads)
 * n_tok == 0 is a no-op.  Slots must be distinct within one call.  Returns
 * QKN_ERR_INVALID_ARG when both w_k and key_gram are NULL. */
QKN_EXPORT qkn_status qkn_append(const qkn_dims* dims, const qkn_cache* cache,
                      const void* c_new, const void* k_rope_raw,
                      const int32_t* slot, const int32_t* pos, int32_t n_tok,
                      const float* w_k, const float* key_gram, const float* gamma_kr,
                      void* stream);
/* (qkn_append, qkn_append_absorb: a token whose slot id lies outside
 * [0, num_blocks * block_size) is skipped: nothing of it is written, so that a
 * bad id cannot write outside the pool.) */

/* qkn_absorb_query — fold the static norm weights into the query
 * (technical summary, Metodología item 1 and the decode-logit equation).
 * For query row i and head h (group g = h / n_g, slot m = h % n_g):
 *   q_tilde[i,h]    = W^K_g[:, m*d_h:(m+1)*d_h] (gamma_q[h] * gamma_k[h] * q[i,h])   in R^r
 *   a_q[i,h]        = softmax_scale / S(q[i,h])            (row scale, sigma folded in)
 *   q_rope_hat[i,h] = softmax_scale * RoPE_{pos[i]}(gamma_qr[h] * q_rope[i,h] / S(q_rope[i,h]))
 *   q          [n_q, H, d_h]    dtype       gamma_q, gamma_k [H, d_h] fp32
 *   q_rope     [n_q, H, d_rope] dtype       gamma_qr [H, d_rope] fp32
 *   pos        [n_q] int32 RoPE positions of the query rows
 *   w_k        [num_groups, r_kv, n_g * d_h] fp32
 *   q_tilde    [n_q, H, r_kv] dtype (out), a_q [n_q, H] fp32 (out),
 *   q_rope_hat [n_q, H, d_rope] dtype (out).
 * w_k, gamma_q and gamma_k must be 16-byte aligned (QKN_ERR_INVALID_ARG otherwise);
 * d_h must be a multiple of 4 and at most 256 (QKN_ERR_UNSUPPORTED otherwise).
 * n_q == 0 is a no-op. */
QKN_EXPORT qkn_status qkn_absorb_query(const qkn_dims* dims, const void* q, const void* q_rope,
                            const int32_t* pos, int32_t n_q, const float* w_k,
                            const float* gamma_q, const float* gamma_k, const float* gamma_qr,
                            void* q_tilde, float* a_q, void* q_rope_hat, void* stream);

/* qkn_append_absorb — qkn_append followed by qkn_absorb_query, in one launch
 * where possible.  The two steps are independent (technical summary,
 * Metodología items 1-4): the append writes the cache's new tokens and their
 * key statistic, the absorption folds the norm weights into the step's
 * queries; neither reads what the other writes.  Arguments are those of the
 * two calls (qpos are the query rows' RoPE positions; w_k is shared; key_gram
 * is the append's and may be NULL), with
 * the same layouts, validation and results.  One launch is used when the
 * cache carries ak_scratch, 0 < n_tok <= 256 and n_q > 0; otherwise the two
 * steps run as their own launches, in this order, on `stream`.  It exists so
 * that a decode step can prepare its inputs without forking two streams;
 * the pages have no counterpart. */
QKN_EXPORT qkn_status qkn_append_absorb(const qkn_dims* dims, const qkn_cache* cache,
                      const void* c_new, const void* k_rope_raw,
                      const int32_t* slot, const int32_t* pos, int32_t n_tok,
                      const void* q, const void* q_rope, const int32_t* qpos, int32_t n_q,
                      const float* w_k, const float* key_gram, const float* gamma_q,
                      const float* gamma_k, const float* gamma_qr, const float* gamma_kr,
                      void* q_tilde, float* a_q, void* q_rope_hat, void* stream);

/* Bytes of decode workspace needed for `batch` sequences of `s_q` query
 * tokens on a GPU with `num_sms` SMs (0 = ask the current device).  The
 * workspace holds a status word and the per-split partial results of the
 * split-KV decode.  Returns QKN_ERR_INVALID_ARG for bad dims. */
QKN_EXPORT qkn_status qkn_decode_workspace_size(const qkn_dims* dims, int32_t batch, int32_t s_q,
                                     int32_t num_sms, size_t* bytes);

/* Zero the workspace's status word (once, after allocating the workspace,
 * and after handling a reported device error).  Enqueued on `stream`. */
QKN_EXPORT qkn_status qkn_workspace_init(void* workspace, size_t ws_bytes, void* stream);

/* qkn_decode — one decode step of QK-Normed MLA attention over the cache.
 * Query row i = b * s_q + j is query token j of sequence b, at position
 * L_b - s_q + j; it attends to the tokens t of sequence b with t <= that
 * position (causal within the step).  For head h in group g:
 *   l[t]  = a_q[i,h] * a_k[t,g] * (q_tilde[i,h] . c_t) + q_rope_hat[i,h] . k^R^_t
 *   out[i,h] = sum_t softmax(l)[t] * c_t,   lse[i,h] = log sum_t exp(l[t])
 * (technical summary, Metodología, decode-logit equation: scalar factors as
 * a row/column rescale before the softmax).  The context is split across
 * CTAs (split-KV) and the partial results are merged by a combine kernel.
 *   q_tilde    [batch*s_q, H, r_kv] dtype; a_q [batch*s_q, H] fp32
 *   q_rope_hat [batch*s_q, H, d_rope] dtype
 *   block_table [batch, max_blocks] int32: block j of sequence b holds its
 *              tokens [64j, 64j+64); only the first ceil(L_b/64) entries of
 *              a row are read
 *   seq_lens   [batch] int32 on the device, s_q <= L_b <= max_blocks * 64
 *   workspace  >= qkn_decode_workspace_size(...) bytes, 256-byte aligned,
 *              initialised once with qkn_workspace_init
 *   out        [batch, s_q, H, r_kv] dtype; lse [batch, s_q, H] fp32
 * A sequence whose length breaks its bound is recorded as QKN_ERR_BOUNDS in
 * the status word and its rows are written as zeros with lse = -inf. */
QKN_EXPORT qkn_status qkn_decode(const qkn_dims* dims, const qkn_cache* cache, qkn_ak_mode ak_mode,
                      const void* q_tilde, const float* a_q, const void* q_rope_hat,
                      const int32_t* block_table, int32_t max_blocks,
                      const int32_t* seq_lens, int32_t batch, int32_t s_q,
                      void* workspace, size_t ws_bytes, void* out, float* lse,
                      const qkn_decode_opts* opts, void* stream);

/* qkn_decode_up — qkn_decode with the per-head value up-projection fused
 * into the merge of the split-KV partials (GQLA summary, section 2, absorbed
 * MQA route: on the absorbed path the values are the latents, and each head's
 * up-projection W^UV_h is applied once to the latent attention output instead
 * of to every cached token).  For query row i and head h:
 *   out_v[i,h] = o_lat[i,h] W^UV_h,   lse[i,h] as in qkn_decode,
 * o_lat[i,h] being qkn_decode's out[i,h]; o_lat is never written to memory.
 *   Arguments are those of qkn_decode with out replaced by
 *   w_uv   [H, r_kv, d_v] dtype, 16-byte aligned: W^UV_h = w_uv[h]
 *   d_v    value head width: a multiple of 16
 *   out_v  [batch, s_q, H, d_v] dtype (out), 16-byte aligned.
 * The same workspace serves (qkn_decode_workspace_size).  The merged latent
 * row is rounded to dtype before the product, as qkn_decode's out is; the
 * product accumulates in fp32 and is rounded once.  A sequence whose length
 * breaks its bound gets zero rows of out_v and lse = -inf, recorded as
 * QKN_ERR_BOUNDS in the status word.
 * Returns QKN_ERR_INVALID_ARG for a bad d_v or pointer, and
 * QKN_ERR_UNSUPPORTED when r_kv > 512 or, in bf16, a head's W^UV_h and 32
 * merged rows do not fit one CTA's shared memory
 * (r_kv * (d_v + 8) * 2 + 32 * (r_kv + 8) * 2 + 512 bytes <= 227 KB, i.e.
 * d_v <= 176 at r_kv = 512), before enqueuing anything. */
QKN_EXPORT qkn_status qkn_decode_up(const qkn_dims* dims, const qkn_cache* cache, qkn_ak_mode ak_mode,
                      const void* q_tilde, const float* a_q, const void* q_rope_hat,
                      const int32_t* block_table, int32_t max_blocks,
                      const int32_t* seq_lens, int32_t batch, int32_t s_q,
                      const void* w_uv, int32_t d_v,
                      void* workspace, size_t ws_bytes, void* out_v, float* lse,
                      const qkn_decode_opts* opts, void* stream);

/* Size of the scratch array that qkn_decode_noalloc uses in place of a
 * caller-allocated workspace.  Every GPU that loads libqkn holds this much
 * device memory for the scratch until the process exits. */
#define QKN_NOALLOC_SCRATCH_BYTES (32u << 20)

/* qkn_decode_noalloc — qkn_decode for callers that cannot allocate device
 * memory (an operator inside another engine that only hands over input and
 * output pointers, a serving loop whose pool already owns the whole GPU, a
 * latency-critical loop that must not pay cudaMalloc's implicit
 * synchronisation).  The paper has no counterpart: this is a deployment
 * variant of the same decode step.
 *   Arguments are those of qkn_decode without the workspace.  The split-KV
 *   partial results go to a fixed QKN_NOALLOC_SCRATCH_BYTES array inside the
 *   library instead; nothing is allocated and no allocating routine is called.
 *   device_status: optional DEVICE pointer to one int32; whenever the call
 *   returns QKN_OK, the decode's status word (a qkn_status) is written there on
 *   `stream` after the decode (QKN_OK for batch == 0).  When the call returns
 *   an error it is not written: the return value is then the status.
 *   Returns QKN_ERR_UNSUPPORTED, before enqueuing anything, when the problem
 *   needs more scratch than QKN_NOALLOC_SCRATCH_BYTES (that is, when
 *   qkn_decode_workspace_size for these dims, batch and s_q exceeds it).
 *   The first call on a device looks up the array's device address on that
 *   device (the calling thread's current device); make that first call before
 *   any stream capture.  All calls share the one array: calls whose GPU work
 *   overlaps (on different streams, or from different threads) race on it and
 *   must be serialised by the caller.  The status word is cleared at the start
 *   of every call. */
QKN_EXPORT qkn_status qkn_decode_noalloc(const qkn_dims* dims, const qkn_cache* cache, qkn_ak_mode ak_mode,
                      const void* q_tilde, const float* a_q, const void* q_rope_hat,
                      const int32_t* block_table, int32_t max_blocks,
                      const int32_t* seq_lens, int32_t batch, int32_t s_q,
                      void* out, float* lse, int32_t* device_status,
                      const qkn_decode_opts* opts, void* stream);

/* qkn_merge_partials — merge partial decode results of the same query rows.
 * For context-parallel decoding (each rank decodes a slice of every
 * sequence's pages, with qkn_decode_opts.vis_end, and the ranks' outputs
 * are all-gathered) the slices' results combine by the same identity as the
 * split-KV merge: for every row
 *   lse = log sum_p exp(lse_p),   out = sum_p exp(lse_p - lse) parts[p]
 * (the softmax over the union of the slices' tokens; QKN summary, decode-logit
 * equation, whose softmax runs over all cached tokens).
 *   parts     [n_parts, rows, r_kv] dtype, 16-byte aligned (each part as
 *             qkn_decode writes out: normalised over the part's tokens)
 *   lse_parts [n_parts, rows] fp32 (-inf: the part saw no token of the row)
 *   out       [rows, r_kv] dtype, 16-byte aligned; lse [rows] fp32
 * rows = batch * s_q * num_heads.  A row with no visible token in any part
 * gets zeros and lse = -inf.  Returns QKN_ERR_INVALID_ARG for n_parts < 1,
 * rows < 0 or a missing or misaligned pointer; rows == 0 is a no-op. */
QKN_EXPORT qkn_status qkn_merge_partials(const qkn_dims* dims, int32_t n_parts, int64_t rows, const void* parts,
                      const float* lse_parts, void* out, float* lse, void* stream);

/* ---------------------------------------------------------------------------
 * The GQA route of GQLA ("GQLA", section 2, "Ruta GQA") and its sparse form
 * ("GQLA Disperso").  Under GQLA's parameterisation the up-projections are
 * indexed by KV group: one key head W^UK_g [r_kv, d_h] with its norm weight
 * gamma_k[g] and one value head W^UV_g [r_kv, d_v] per group, shared by the
 * group's n_g = num_heads / num_groups query heads.  This route caches the
 * latent expanded into per-group keys and values (2 g d_h values per token)
 * plus the shared RoPE key, and decodes with ordinary grouped-query
 * attention over them.  Over the same weights it is algebraically equal to
 * the absorbed route (qkn_decode_up with W^UV_h = W^UV_{g(h)}, and W^K_g made
 * of n_g copies of W^UK_g): it trades cache bytes for FLOPs per byte.
 * bf16 storage only; (d_h, d_rope, d_v) = (128, 64, 128) or (64, 32, 64).
 * ------------------------------------------------------------------------- */

/* The GQA route's cache, caller-allocated device memory, bf16, 16-byte aligned:
 *   k      [num_blocks, num_groups, block_size, d_h]   normalised keys
 *   v      [num_blocks, num_groups, block_size, d_v]   values
 *   k_rope [num_blocks, block_size, d_rope]            as qkn_cache.k_rope
 * Slot s of the pool is token s % block_size of block s / block_size.  Slots
 * that no qkn_gqa_append has written may hold anything; the decode reads no
 * slot past a sequence's length. */
typedef struct {
  void* k;
  void* v;
  void* k_rope;
  int32_t num_blocks;
  int32_t d_v;
} qkn_gqa_cache;

/* qkn_gqa_append — expand n_tok new tokens into the GQA route's cache.
 * For token i with slot s = slot[i], position p = pos[i] and every group g:
 *   k[s, g] = gamma_k[g] * z / S(z),  z = c_new[i] W^UK_g   (S over the d_h columns)
 *   v[s, g] = c_new[i] W^UV_g
 *   k_rope[s] = RoPE_p(gamma_kr * k_rope_raw[i] / S(k_rope_raw[i]))
 * (GQLA summary, section 2, "Ruta GQA": the latent expanded into g groups of
 * keys and values; the key RMS-normalised after its up-projection as in the
 * QK-Normed summary, "Planteamiento del Problema").  fp32 products.
 *   c_new      [n_tok, r_kv] bf16, 16-byte aligned;  k_rope_raw [n_tok, d_rope] bf16, 16-byte aligned
 *   slot, pos  [n_tok] int32 device arrays; a token whose slot is outside
 *              [0, num_blocks * block_size) is skipped
 *   w_uk       [num_groups, r_kv, d_h] fp32, 16-byte aligned;  gamma_k [num_groups, d_h] fp32
 *   w_uv       [num_groups, r_kv, d_v] bf16, 16-byte aligned;  gamma_kr [d_rope] fp32
 * n_tok == 0 is a no-op.  Returns QKN_ERR_UNSUPPORTED for fp32 storage,
 * other head widths, r_kv not a multiple of 32 or more than 65535 groups,
 * QKN_ERR_INVALID_ARG for bad dims or a missing or misaligned pointer. */
QKN_EXPORT qkn_status qkn_gqa_append(const qkn_dims* dims, const qkn_gqa_cache* cache, const void* c_new,
                      const void* k_rope_raw, const int32_t* slot, const int32_t* pos, int32_t n_tok,
                      const float* w_uk, const float* gamma_k, const void* w_uv, const float* gamma_kr,
                      void* stream);

/* Bytes of device workspace qkn_gqa_decode needs for `batch` sequences of
 * s_q query tokens on a GPU of num_sms SMs (0 = the current device's).  The
 * sparse form needs only its first 256 bytes (the status word).  Initialise
 * it with qkn_workspace_init. */
QKN_EXPORT qkn_status qkn_gqa_workspace_size(const qkn_dims* dims, int32_t d_v, int32_t batch, int32_t s_q,
                      int32_t num_sms, size_t* bytes);

/* qkn_gqa_decode — one decode step of the GQA route.  Query row (j, h) of
 * sequence b, head h in group g = h / n_g, sits at position L_b - s_q + j and
 * gets
 *   l[t] = sigma (RMSNorm(q_jh) gamma_q[h] . k[t, g]
 *                 + RoPE_pos(RMSNorm(q^R_jh) gamma_qr[h]) . k_rope[t]),
 *   o_v[b, j, h] = sum_t softmax(l)[t] v[t, g],  lse[b, j, h] = log sum_t exp(l[t]),
 * over the tokens t <= L_b - s_q + j of the sequence (dense), or, with a
 * selection, over the tokens selection[b, j, g, :] lists among them (sparse
 * GQLA: the n_g heads of a group share the query token's list).  sigma is
 * dims->softmax_scale (0 = 1/sqrt(d_h + d_rope)); the queries are normalised
 * and rotated inside the call.
 *   q          [batch, s_q, num_heads, d_h] bf16 (raw queries)
 *   q_rope     [batch, s_q, num_heads, d_rope] bf16 (raw)
 *   gamma_q    [num_heads, d_h] fp32;  gamma_qr [num_heads, d_rope] fp32
 *   block_table [batch, max_blocks] int32, seq_lens [batch] int32 (device)
 *   selection  NULL (dense) or [batch, s_q, num_groups, sel_k] int32 token
 *              positions, -1 for none; a listed position after the query's
 *              is not attended; the positions of one list should be distinct
 *   out_v      [batch, s_q, num_heads, d_v] bf16, 16-byte aligned;  lse [batch, s_q, num_heads] fp32
 *   max_ctas   cap on the dense decode's CTAs (0 = one per SM)
 * Dense: a split-KV decode on a device schedule, then the merge of the
 * splits, on `stream`.  Sparse: one CTA per (sequence, query token, group).
 * A sequence whose length is below s_q or past its block table, and a block
 * id outside the pool, are recorded in the workspace status word
 * (QKN_ERR_BOUNDS); the former's rows come out as zeros with lse = -inf, the
 * latter reads block 0 instead.  A row with no token (an empty selection)
 * gets zeros and lse = -inf.  Returns QKN_ERR_UNSUPPORTED for fp32 storage or
 * other head widths, QKN_ERR_INVALID_ARG for bad arguments or a workspace
 * smaller than qkn_gqa_workspace_size says; batch == 0 is a no-op. */
QKN_EXPORT qkn_status qkn_gqa_decode(const qkn_dims* dims, const qkn_gqa_cache* cache, const void* q,
                      const void* q_rope, const float* gamma_q, const float* gamma_qr,
                      const int32_t* block_table, int32_t max_blocks, const int32_t* seq_lens, int32_t batch,
                      int32_t s_q, const int32_t* selection, int32_t sel_k, void* workspace, size_t ws_bytes,
                      void* out_v, float* lse, int32_t max_ctas, void* stream);

/* Synchronise `stream`, then read the workspace status word into *device_status
 * (a qkn_status value; QKN_OK if no kernel recorded an error).  The word is
 * sticky until qkn_workspace_init clears it. */
QKN_EXPORT qkn_status qkn_read_device_status(const void* workspace, void* stream, int32_t* device_status);

/* Which decode kernel qkn_decode would run for these dims and options
 * (QKN_KERNEL_SIMT or QKN_KERNEL_TCGEN05), or -1 if none can. */
QKN_EXPORT int32_t qkn_decode_kernel_for(const qkn_dims* dims, int32_t s_q, const qkn_decode_opts* opts);

QKN_EXPORT const char* qkn_status_string(qkn_status status);
QKN_EXPORT int32_t qkn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* QKN_H_ */
