// Host-side launch interfaces between the C ABI layer (api.cu) and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "qkn.h"

namespace qkn {

// RoPE frequencies theta^(-2i/d_R), i < d_R/2 (d_R <= 128), formed in fp64 on
// the host from the dims and passed by value with the launch.
struct RopeFreqs {
  double f[64];
};

struct AppendArgs {
  void* latent;            // cache pool
  void* k_rope;
  float* a_k;
  uint32_t* ak_scratch;    // [slots, groups, 2]: key statistic accumulator, arrival count; or null
  const void* c_new;       // [n_tok, r]
  const void* k_rope_raw;  // [n_tok, d_rope]
  const int32_t* slot;
  const int32_t* pos;
  const float* w_k;        // [groups, r, width]
  const float* key_gram;   // [groups, r, r] = W W^T per group, or null (then w_k)
  const float* gamma_kr;   // [d_rope]
  int32_t n_tok, r, d_rope, groups, width;   // width = n_g * d_h
  int32_t ncols;           // columns of the key-statistic matrix: r with key_gram, else width
  int64_t n_slots;         // cache slots (num_blocks * block_size): a token whose slot is outside is skipped
  float eps, rope_theta;
  RopeFreqs freq;
};

struct AbsorbArgs {
  const void* q;           // [n_q, H, d_h]
  const void* q_rope;      // [n_q, H, d_rope]
  const int32_t* pos;      // [n_q]
  const float* w_k;        // [groups, r, n_g * d_h]
  const float* gamma_q;    // [H, d_h]
  const float* gamma_k;    // [H, d_h]
  const float* gamma_qr;   // [H, d_rope]
  void* q_tilde;           // [n_q, H, r]
  float* a_q;              // [n_q, H]
  void* q_rope_hat;        // [n_q, H, d_rope]
  int32_t n_q, heads, groups, r, d_h, d_rope;
  float eps, softmax_scale, rope_theta;
  RopeFreqs freq;
};

struct DecodeArgs {
  const void* latent;        // [num_blocks, 64, r]
  const void* k_rope;        // [num_blocks, 64, d_rope]
  const float* a_k;          // [num_blocks, 64, groups]
  int32_t num_blocks;
  const void* q_tilde;       // [batch*s_q, H, r]
  const float* a_q;          // [batch*s_q, H]
  const void* q_rope_hat;    // [batch*s_q, H, d_rope]
  const int32_t* block_table;
  int32_t max_blocks;
  const int32_t* seq_lens;
  int32_t batch, s_q, heads, groups, r, d_rope;
  int32_t ak_one;            // 1: plain MLA (a_k treated as 1)
  int32_t rows;              // query rows per tile (R)
  int32_t ht_count;          // tiles per sequence = ceil(s_q*H / R)
  int32_t ncta;
  int32_t item_cost;         // schedule units without pages at the start of every segment
  float* part_o;             // [slots, R, r] fp32
  float* part_lse;           // [slots, R] fp32
  int32_t* status;           // workspace status word
  int64_t wait_limit;        // bounded-wait cycles (tcgen05 kernel)
  // tcgen05 kernel only: the rows of a sequence with a rejected length are written to out / lse
  // directly (zeros, -inf), and seg_desc[segment] = (first split slot, number of splits; the
  // splits sit ht_count slots apart) tells the merge kernel where the partials are
  void* out;                 // [batch, s_q, H, r] bf16
  float* lse;                // [batch, s_q, H]
  int2* seg_desc;            // [batch * ht_count]
  int32_t step_writes_only;  // qkn_decode_opts.step_writes_only: read inputs and old pages before the wait
  int32_t withhold_ak;       // qkn_decode_opts.test_withhold_ak (tests of the timeout path)
  const int32_t* vis_end;    // qkn_decode_opts.vis_end: per sequence, the causal limit's end (null: seq_lens)
};

struct CombineArgs {
  const int32_t* seq_lens;
  int32_t batch, s_q, heads, r, rows, ht_count, ncta, max_blocks;
  int32_t item_cost;         // as in DecodeArgs
  int32_t max_items;         // upper bound on splits per row (ncta + 1)
  int64_t nslots;            // workspace slots of this launch (batch * ht_count + ncta), each `rows` rows
  const float* part_o;
  const float* part_lse;
  void* out;                 // [batch, s_q, H, r]
  float* lse;                // [batch, s_q, H]
  int32_t* status;           // workspace status word
  const int2* seg_desc;      // per-segment (first slot, splits) from the tcgen05 kernel, or null
  // GQA route (gqa.cu) only; 0 elsewhere.  Row tiles hold one KV group's query rows: tile ht is
  // row block ht % tiles_per_group of group ht / tiles_per_group, whose rows u = (j, m), u = j * n_g + m
  // (query token j, head g * n_g + m) are laid out u = block * rows + row.
  int32_t group_heads = 0;   // n_g
  int32_t tiles_per_group = 0;
};

// Merge fused with the per-head value up-projection (combine_up.cu): c.out is not used; the merged
// latent row of (query row i, head h) is multiplied by W^UV_h and written to out_v.
struct CombineUpArgs {
  CombineArgs c;
  const void* w_uv;          // [H, r, d_v] in the storage type
  int32_t d_v;
  void* out_v;               // [batch, s_q, H, d_v] in the storage type
  int32_t col_groups;        // output column groups per (head, row block); set by the launcher
};

// GQA route of GQLA (gqa.cu): keys and values expanded per KV group, one key head and one value
// head per group.  bf16 storage.
struct GqaAppendArgs {
  void* k_cache;           // [num_blocks, groups, 64, d_h]   normalised keys
  void* v_cache;           // [num_blocks, groups, 64, d_v]
  void* k_rope;            // [num_blocks, 64, d_rope]        normalised, rotated RoPE keys
  const void* c_new;       // [n_tok, r]
  const void* k_rope_raw;  // [n_tok, d_rope]
  const int32_t* slot;
  const int32_t* pos;
  const float* w_uk;       // [groups, r, d_h] fp32
  const float* gamma_k;    // [groups, d_h]
  const void* w_uv;        // [groups, r, d_v] storage type
  const float* gamma_kr;   // [d_rope]
  int32_t n_tok, r, d_h, d_v, d_rope, groups;
  int64_t n_slots;         // a token whose slot is outside [0, n_slots) is skipped
  float eps;
  RopeFreqs freq;
};

struct GqaDecodeArgs {
  const void* k_cache;       // as in GqaAppendArgs
  const void* v_cache;
  const void* k_rope;
  int32_t num_blocks;
  const void* q;             // [batch, s_q, H, d_h]     raw queries
  const void* q_rope;        // [batch, s_q, H, d_rope]
  const float* gamma_q;      // [H, d_h]
  const float* gamma_qr;     // [H, d_rope]
  const int32_t* block_table;
  int32_t max_blocks;
  const int32_t* seq_lens;
  int32_t batch, s_q, heads, groups;
  int32_t d_h, d_rope, d_v;
  int32_t rows;              // query rows per tile: 16 or 32
  int32_t tpg;               // tiles per group (dense) or per (query token, group) (sparse)
  int32_t ht_count;          // dense: tiles per sequence (groups * tpg)
  int32_t ncta, item_cost;   // dense: the device schedule's CTAs and item start cost
  const int32_t* selection;  // sparse: [batch, s_q, groups, sel_k] token positions (-1: none); null = dense
  int32_t sel_k;
  float* part_o;             // dense: [slots, rows, d_v] normalised partial outputs
  float* part_lse;           // dense: [slots, rows]
  void* out;                 // sparse: [batch, s_q, H, d_v]
  float* lse;                // sparse: [batch, s_q, H]
  int32_t* status;
  float eps;
  float score_scale;         // sigma * log2(e): logits in base-2 units
  RopeFreqs freq;
};

bool gqa_supported(int d_h, int d_rope, int d_v);
cudaError_t launch_gqa_append(const GqaAppendArgs& a, cudaStream_t st);
cudaError_t launch_gqa_decode(const GqaDecodeArgs& a, cudaStream_t st);
// The merge of the GQA route's split partials (combine.cu, grouped row tiles).
cudaError_t launch_combine_grouped(const CombineArgs& a, cudaStream_t st);

cudaError_t launch_append(const AppendArgs& a, bool bf16, cudaStream_t st);
cudaError_t launch_key_gram(const float* w_k, float* gram, int groups, int r, int width, cudaStream_t st);
// One launch for both (prep.cu) when the append can run as one launch and is a decode step's size.
bool prep_fusable(const AppendArgs& ap, const AbsorbArgs& ab);
cudaError_t launch_prep(const AppendArgs& ap, const AbsorbArgs& ab, bool bf16, cudaStream_t st);
cudaError_t launch_absorb(const AbsorbArgs& a, bool bf16, cudaStream_t st);
cudaError_t launch_decode_simt(const DecodeArgs& a, bool bf16, cudaStream_t st);
cudaError_t launch_combine(const CombineArgs& a, bool bf16, cudaStream_t st);
// Merge n_parts normalised partial outputs of the same rows (merge_parts.cu).
cudaError_t launch_merge_parts(const void* parts, const float* lse_parts, int n_parts, int64_t rows, int r,
                               void* out, float* lse, bool bf16, cudaStream_t st);
bool combine_up_supported(bool bf16, int r, int d_v, int n_q);
cudaError_t launch_combine_up(const CombineUpArgs& u, bool bf16, cudaStream_t st);

// tcgen05 decode (bf16 only).  Returns cudaErrorNotSupported for dims it
// cannot take.
bool decode_tc_supported(int r, int d_rope, int rows, int groups);
cudaError_t launch_decode_tc(const DecodeArgs& a, cudaStream_t st);

// tcgen05 decode of 128-row tiles on CTA pairs that split the latent width (decode_pair.cu);
// DecodeArgs.ncta counts pairs there.  Returns cudaErrorNotSupported for dims it cannot take.
bool decode_pair_supported(int r, int d_rope, int groups);
int decode_pair_max_pairs(int sms);    // pairs resident at once on the current device (<= sms / 2)
cudaError_t launch_decode_pair(const DecodeArgs& a, cudaStream_t st);

constexpr int kSimtRows = 8;   // query rows per CTA of the CUDA-core decode
constexpr int kPairRows = 128; // query rows per tile of the CTA-pair decode

}  // namespace qkn
