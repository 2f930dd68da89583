// Launch descriptors of the CUDA kernels of libsegpaged.so (host <-> .cu glue).
#pragma once

#include <cuda_runtime.h>

#include "sp_internal.h"

namespace sp {

struct PackLaunch {
  const HeadDesc* heads;
  const PageDesc* pages;
  int32_t n_pages;
  int32_t D, P;
  bool bf16;
  bool fp8;      // E4M3 pages (dense side bf16 for pack, 1-byte codes for gather)
  float k_inv, v_inv;  // quantisation multipliers 1 / scale (fp8 pack)
  bool inverse;  // gather (pool -> dense) instead of pack
  int64_t stride_seq, stride_head, stride_tok, page_bytes;
  const void* kdense_in;
  const void* vdense_in;
  void* kpool_out;
  void* vpool_out;
  const void* kpool_in;
  const void* vpool_in;
  void* kdense_out;
  void* vdense_out;
};
void launch_pack(const PackLaunch& L, cudaStream_t s);
// Zero-fill the pages ids[0 .. n) of both pools (a ring plan's spare pool, at build).
cudaError_t launch_zero_pages(const int32_t* ids, int32_t n, int64_t page_bytes, void* kpool, void* vpool,
                              cudaStream_t s);

// Pack of several layers in one launch (kernel parameter, passed by value).
constexpr int kMaxPackLayers = 128;
struct PackLayersArgs {
  int32_t n_layers;
  int32_t page_begin[kMaxPackLayers + 1];  // prefix sums of the layers' page counts
  const HeadDesc* heads[kMaxPackLayers];
  const PageDesc* pages[kMaxPackLayers];
  const void* kd[kMaxPackLayers];
  const void* vd[kMaxPackLayers];
  float k_inv[kMaxPackLayers], v_inv[kMaxPackLayers];  // E4M3 pages: 1 / scale per layer
  int64_t stride_seq, stride_head, stride_tok, page_bytes;
};
cudaError_t launch_pack_layers(const PackLayersArgs& la, bool bf16, bool fp8, int D, int P, void* kpool, void* vpool,
                               cudaStream_t s);

struct DecodeLaunch {
  const HeadDesc* heads;
  const PageDesc* pages;
  const DecodeItem* items;
  const int32_t* cta_begin;
  const CombineItem* combine;
  int32_t n_ctas, n_combine;
  int32_t D, P, group, num_q_heads;
  bool bf16;
  int64_t page_bytes;
  int64_t pool_pages;  // pages a pool must hold; a table page id outside [0, pool_pages) is reported
  const void* kpool;
  const void* vpool;
  const void* q;  // [B, Hq, D]
  void* out;      // [B, Hq, D]
  float* lse;     // [B, Hq] or null
  float scale_log2;  // softmax scale * log2(e) (* k_scale for E4M3 pages)
  bool fp8;          // E4M3 pages
  float v_scale;     // E4M3 pages: value scale, applied to the normalised output
  float* partial;    // workspace partial slots
  int32_t* counters; // workspace arrival counters of split heads (zero between calls)
  int32_t* status;
  // Fused decode step of a ring plan (bf16 / E4M3 pages): before attending, each
  // CTA appends the new token of the heads whose target or evicted page lies in
  // its page range, and the CTA that finishes a head advances its context.
  bool append;
  const void* k_new;   // [B, Hkv, D] bf16 rows, strides in elements
  const void* v_new;
  int64_t new_stride_seq, new_stride_head;
  float k_inv, v_inv;  // E4M3 pages: 1 / k_scale, 1 / v_scale
  int32_t* free_pool;  // table's spare pool section (count, then ids)
};
cudaError_t launch_decode(const DecodeLaunch& L, cudaStream_t s);

// Argument checks and launch set-up shared by the attention entry points
// (segpaged_attention and the allocation-free decode), so that both refuse
// exactly the same arguments.
sp_status check_table(const sp_plan* plan, const void* d_table);
sp_status check_attention_args(const sp_plan* plan, const void* d_table, const void* k_pool, const void* v_pool,
                               const void* q, const void* out, const float* lse, float softmax_scale);
float softmax_scale_of(const sp_plan* plan, float softmax_scale);  // <= 0 selects 1 / sqrt(head_dim)
// Decode launch of a plan whose scratch (status block, counters, partials) starts at `scratch`.
DecodeLaunch decode_launch_of(const sp_plan* plan, const void* d_table, const void* k_pool, const void* v_pool,
                              const void* q, void* out, float* lse, float softmax_scale, void* scratch,
                              int32_t* status);

struct PrefillLaunch {
  const HeadDesc* heads;
  const PageDesc* pages;
  const PrefillItem* items;
  int32_t n_items;
  int32_t D, P, group, num_q_heads, total_rows;
  bool bf16;
  int64_t page_bytes;
  int64_t pool_pages;  // pages a pool must hold; a table page id outside [0, pool_pages) is reported
  const void* kpool;
  const void* vpool;
  const void* q;  // [rows, Hq, D]
  void* out;
  float* lse;
  float scale_log2;
  int32_t* status;
};
cudaError_t launch_prefill(const PrefillLaunch& L, cudaStream_t s);

struct AppendLaunch {
  HeadDesc* heads;  // device table, updated in place
  PageDesc* pages;
  int32_t n_heads;
  int32_t D, P;
  bool bf16;
  bool fp8;            // E4M3 pages: the new bf16 rows are quantised on the way in
  float k_inv, v_inv;  // 1 / k_scale, 1 / v_scale
  int64_t stride_seq, stride_head, page_bytes;
  int64_t pool_pages;
  const void* k_new;  // [B, Hkv, D] with the given strides (elements)
  const void* v_new;
  void* kpool;
  void* vpool;
  int32_t* status;
  int32_t* free_pool;  // table's spare pool section (count, then ids)
};
cudaError_t launch_append(const AppendLaunch& a, cudaStream_t s);

// Attention mass per page-size block (segpaged_block_mass): the importance a
// retrieval head's top-p selection reads.  Passed by value (__grid_constant__),
// the per-sequence context lengths included.
constexpr int kMassMaxBatch = 2048;
constexpr int kMassBlock = 64;  // positions per block (the bf16 page size)
struct BlockMassLaunch {
  const void* k;  // dense bf16 keys, element strides below, head_dim contiguous
  int64_t stride_seq, stride_head, stride_tok;
  const void* q;  // [B, Hq, D] bf16: each sequence's query at its last position
  float scale_log2;
  int32_t B, Hq, Hkv, G, D;
  int32_t nb_max;          // blocks of the longest sequence: the workspace's row pitch
  int32_t blocks_per_cta;  // grid.x = ceil(nb_max / blocks_per_cta), grid.y = B * Hkv
  float* ws_m;             // [B * Hq][nb_max]: a block's score maximum (log2 units)
  float* ws_s;             // [B * Hq][nb_max]: its sum of 2^(score - maximum)
  float* mass;             // [B * Hkv][mass_stride]
  int64_t mass_stride;
  int32_t L[kMassMaxBatch];
};
cudaError_t launch_block_mass(const BlockMassLaunch& a, cudaStream_t s);

}  // namespace sp
