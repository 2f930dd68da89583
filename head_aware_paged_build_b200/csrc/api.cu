// Device entry points of libsegpaged.so (the C ABI of segpaged.h).
//
// Each call validates its arguments on the host, before any launch, then
// enqueues kernels on the caller's stream.  There is no host or library
// fallback: a dtype / shape without a kernel returns SP_ERR_UNSUPPORTED.
#include <cmath>
#include <cstdint>
#include <limits>
#include <string>

#include "kernels.h"
#include "sp_internal.h"

namespace sp {
cudaError_t launch_prefill_f32(const PrefillLaunch& a, cudaStream_t s);
cudaError_t launch_prefill_bf16(const PrefillLaunch& a, cudaStream_t s);

sp_status check_table(const sp_plan* plan, const void* d_table) {
  if (!plan) return fail(SP_ERR_INVALID_ARG, "plan is NULL");
  if (!d_table || (reinterpret_cast<uintptr_t>(d_table) % 16) != 0)
    return fail(SP_ERR_INVALID_ARG, "d_table must be a 16-byte aligned device pointer");
  return SP_OK;
}

sp_status check_attention_args(const sp_plan* plan, const void* d_table, const void* k_pool, const void* v_pool,
                            const void* q, const void* out, const float* lse, float softmax_scale) {
  sp_status st = check_table(plan, d_table);
  if (st != SP_OK) return st;
  auto aligned_to = [](const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; };
  if (!k_pool || !v_pool || !q || !out) return fail(SP_ERR_INVALID_ARG, "pool, q and out must be non-NULL");
  if (!aligned_to(k_pool, 16) || !aligned_to(v_pool, 16) || !aligned_to(q, 16) || !aligned_to(out, 16))
    return fail(SP_ERR_INVALID_ARG, "pools, q and out must be 16-byte aligned");
  if (lse && !aligned_to(lse, 4)) return fail(SP_ERR_INVALID_ARG, "lse must be 4-byte aligned");
  if (!std::isfinite(softmax_scale)) return fail(SP_ERR_INVALID_ARG, "softmax_scale must be finite");
  return SP_OK;
}

float softmax_scale_of(const sp_plan* plan, float softmax_scale) {
  return softmax_scale > 0.f ? softmax_scale : 1.0f / std::sqrt(float(plan->prob.head_dim));
}

DecodeLaunch decode_launch_of(const sp_plan* plan, const void* d_table, const void* k_pool, const void* v_pool,
                              const void* q, void* out, float* lse, float softmax_scale, void* scratch,
                              int32_t* status) {
  const float scale_log2 = softmax_scale_of(plan, softmax_scale) * 1.4426950408889634f;
  const uint8_t* tbl = static_cast<const uint8_t*>(d_table);
  DecodeLaunch L{};
  L.heads = reinterpret_cast<const HeadDesc*>(tbl + plan->hdr.off_heads);
  L.pages = reinterpret_cast<const PageDesc*>(tbl + plan->hdr.off_pages);
  L.items = reinterpret_cast<const DecodeItem*>(tbl + plan->hdr.off_decode_items);
  L.cta_begin = reinterpret_cast<const int32_t*>(tbl + plan->hdr.off_decode_cta);
  L.combine = reinterpret_cast<const CombineItem*>(tbl + plan->hdr.off_combine);
  L.n_ctas = plan->hdr.n_decode_ctas;
  L.n_combine = plan->hdr.n_combine;
  L.D = plan->prob.head_dim;
  L.P = plan->prob.page_size;
  L.group = plan->group;
  L.num_q_heads = plan->prob.num_q_heads;
  L.bf16 = plan->prob.dtype == SP_BF16;
  L.page_bytes = plan->sizes.page_bytes;
  L.pool_pages = plan->sizes.pool_pages;
  L.kpool = k_pool, L.vpool = v_pool, L.q = q, L.out = out, L.lse = lse;
  L.scale_log2 = plan->fp8 ? scale_log2 * plan->k_scale : scale_log2;
  L.fp8 = plan->fp8;
  L.v_scale = plan->fp8 ? plan->v_scale : 1.f;
  L.partial = reinterpret_cast<float*>(static_cast<uint8_t*>(scratch) + plan->partial_offset);
  L.counters = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(scratch) + kStatusBytes);
  L.status = status;
  return L;
}

namespace {

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

template <typename T>
const T* section(const void* d_table, int64_t off) {
  return reinterpret_cast<const T*>(static_cast<const uint8_t*>(d_table) + off);
}

sp_status cuda_fail(cudaError_t e, const char* what) {
  return fail(SP_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
}


sp_status pack_common(const sp_plan* plan, const void* d_table, const void* k_in, const void* v_in, void* k_out,
                      void* v_out, bool inverse, int64_t stride_seq, int64_t stride_head, int64_t stride_tok,
                      void* stream) {
  sp_status st = check_table(plan, d_table);
  if (st != SP_OK) return st;
  if (!k_in || !v_in || !k_out || !v_out) return fail(SP_ERR_INVALID_ARG, "K/V pointers must be non-NULL");
  if (!aligned(k_in, 16) || !aligned(v_in, 16) || !aligned(k_out, 16) || !aligned(v_out, 16))
    return fail(SP_ERR_INVALID_ARG, "K/V pointers must be 16-byte aligned");
  // dense element size: the problem dtype, except the 1-byte codes a gather of E4M3 pages writes
  const int64_t eb = (inverse && plan->fp8) ? 1 : plan->elem_bytes;
  if (stride_head < 0 || stride_tok < 0 || (stride_seq < 0 && stride_seq != SP_VARLEN))
    return fail(SP_ERR_INVALID_ARG, "strides must be >= 0 (stride_seq may be SP_VARLEN)");
  if ((stride_head * eb) % 16 || (stride_tok * eb) % 16 || (stride_seq > 0 && (stride_seq * eb) % 16))
    return fail(SP_ERR_INVALID_ARG, "strides must give 16-byte aligned rows");
  PackLaunch L{};
  L.heads = section<HeadDesc>(d_table, plan->hdr.off_heads);
  L.pages = section<PageDesc>(d_table, plan->hdr.off_pages);
  L.n_pages = plan->hdr.n_vpages;
  L.D = plan->prob.head_dim;
  L.P = plan->prob.page_size;
  L.bf16 = plan->prob.dtype == SP_BF16;
  L.fp8 = plan->fp8;
  L.k_inv = 1.0f / plan->k_scale;
  L.v_inv = 1.0f / plan->v_scale;
  L.inverse = inverse;
  L.stride_seq = stride_seq;
  L.stride_head = stride_head;
  L.stride_tok = stride_tok;
  L.page_bytes = plan->sizes.page_bytes;
  if (inverse) {
    L.kpool_in = k_in, L.vpool_in = v_in, L.kdense_out = k_out, L.vdense_out = v_out;
  } else {
    L.kdense_in = k_in, L.vdense_in = v_in, L.kpool_out = k_out, L.vpool_out = v_out;
  }
  launch_pack(L, static_cast<cudaStream_t>(stream));
  cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess && !inverse && plan->hdr.n_spare > 0)  // the spare pool starts zero-filled
    e = launch_zero_pages(section<int32_t>(d_table, plan->hdr.off_free) + kFreeIdsOffset, plan->hdr.n_spare,
                          plan->sizes.page_bytes, k_out, v_out, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SP_OK : cuda_fail(e, inverse ? "segpaged_gather launch" : "build_segpaged_cache launch");
}

}  // namespace
}  // namespace sp

extern "C" {

sp_status segpaged_table_write(const sp_plan* plan, void* d_table, size_t bytes, void* stream) {
  if (!plan) return sp::fail(SP_ERR_INVALID_ARG, "plan is NULL");
  if (!d_table || !sp::aligned(d_table, 16)) return sp::fail(SP_ERR_INVALID_ARG, "d_table must be 16-byte aligned");
  if (bytes < plan->blob.size()) return sp::fail(SP_ERR_WORKSPACE, "table buffer smaller than table_bytes");
  const cudaError_t e = cudaMemcpyAsync(d_table, plan->blob.data(), plan->blob.size(), cudaMemcpyHostToDevice,
                                        static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SP_OK : sp::cuda_fail(e, "segpaged_table_write");
}

sp_status build_segpaged_cache(const sp_plan* plan, const void* d_table, const void* k_dense, const void* v_dense,
                               int64_t stride_seq, int64_t stride_head, int64_t stride_tok, void* k_pool,
                               void* v_pool, void* stream) {
  return sp::pack_common(plan, d_table, k_dense, v_dense, k_pool, v_pool, false, stride_seq, stride_head,
                         stride_tok, stream);
}

sp_status build_segpaged_cache_layers(int32_t n_layers, const sp_plan* const* plans, const void* const* d_tables,
                                      const void* const* k_dense, const void* const* v_dense, int64_t stride_seq,
                                      int64_t stride_head, int64_t stride_tok, void* k_pool, void* v_pool,
                                      void* stream) {
  using namespace sp;
  if (n_layers < 1 || n_layers > kMaxPackLayers)
    return fail(SP_ERR_INVALID_ARG, "n_layers must be in [1, " + std::to_string(kMaxPackLayers) + "]");
  if (!plans || !d_tables || !k_dense || !v_dense) return fail(SP_ERR_INVALID_ARG, "arrays must be non-NULL");
  if (!k_pool || !v_pool || !aligned(k_pool, 16) || !aligned(v_pool, 16))
    return fail(SP_ERR_INVALID_ARG, "pools must be non-NULL and 16-byte aligned");
  const sp_plan* p0 = plans[0];
  if (!p0) return fail(SP_ERR_INVALID_ARG, "plans[0] is NULL");
  const int64_t eb = p0->elem_bytes;
  if (stride_head < 0 || stride_tok < 0 || (stride_seq < 0 && stride_seq != SP_VARLEN))
    return fail(SP_ERR_INVALID_ARG, "strides must be >= 0 (stride_seq may be SP_VARLEN)");
  if ((stride_head * eb) % 16 || (stride_tok * eb) % 16 || (stride_seq > 0 && (stride_seq * eb) % 16))
    return fail(SP_ERR_INVALID_ARG, "strides must give 16-byte aligned rows");
  PackLayersArgs la{};
  la.n_layers = n_layers;
  la.stride_seq = stride_seq, la.stride_head = stride_head, la.stride_tok = stride_tok;
  la.page_bytes = p0->sizes.page_bytes;
  int64_t total = 0;
  for (int32_t i = 0; i < n_layers; ++i) {
    const sp_plan* p = plans[i];
    sp_status st = check_table(p, d_tables[i]);
    if (st != SP_OK) return st;
    if (p->prob.dtype != p0->prob.dtype || p->prob.head_dim != p0->prob.head_dim ||
        p->prob.page_size != p0->prob.page_size || p->fp8 != p0->fp8)
      return fail(SP_ERR_INVALID_ARG, "every layer needs the same dtype, head_dim, page_size and page type");
    if (p->hdr.n_spare > 0)
      return fail(SP_ERR_UNSUPPORTED, "plans with a spare pool are packed by build_segpaged_cache");
    if (!k_dense[i] || !v_dense[i] || !aligned(k_dense[i], 16) || !aligned(v_dense[i], 16))
      return fail(SP_ERR_INVALID_ARG, "dense K/V pointers must be non-NULL and 16-byte aligned");
    la.page_begin[i] = int32_t(total);
    la.heads[i] = section<HeadDesc>(d_tables[i], p->hdr.off_heads);
    la.pages[i] = section<PageDesc>(d_tables[i], p->hdr.off_pages);
    la.kd[i] = k_dense[i], la.vd[i] = v_dense[i];
    la.k_inv[i] = 1.0f / p->k_scale, la.v_inv[i] = 1.0f / p->v_scale;
    total += p->hdr.n_vpages;
    if (total > std::numeric_limits<int32_t>::max()) return fail(SP_ERR_UNSUPPORTED, "more than 2^31 pages");
  }
  la.page_begin[n_layers] = int32_t(total);
  const cudaError_t e = launch_pack_layers(la, p0->prob.dtype == SP_BF16, p0->fp8, p0->prob.head_dim,
                                           p0->prob.page_size, k_pool, v_pool, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SP_OK : cuda_fail(e, "build_segpaged_cache_layers launch");
}

sp_status segpaged_gather(const sp_plan* plan, const void* d_table, const void* k_pool, const void* v_pool,
                          void* k_out, void* v_out, int64_t stride_seq, int64_t stride_head, int64_t stride_tok,
                          void* stream) {
  return sp::pack_common(plan, d_table, k_pool, v_pool, k_out, v_out, true, stride_seq, stride_head, stride_tok,
                         stream);
}

sp_status segpaged_attention(const sp_plan* plan, const void* d_table, const void* k_pool, const void* v_pool,
                             const void* q, void* out, float* lse, float softmax_scale, void* workspace,
                             size_t workspace_bytes, void* stream) {
  using namespace sp;
  sp_status st = check_attention_args(plan, d_table, k_pool, v_pool, q, out, lse, softmax_scale);
  if (st != SP_OK) return st;
  if (!workspace || !aligned(workspace, 256)) return fail(SP_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  if (int64_t(workspace_bytes) < plan->sizes.workspace_bytes)
    return fail(SP_ERR_WORKSPACE, "workspace smaller than workspace_bytes");
  const float scale_log2 = softmax_scale_of(plan, softmax_scale) * 1.4426950408889634f;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  int32_t* status = static_cast<int32_t*>(workspace);
  cudaError_t e;
  if (plan->sizes.is_decode) {
    e = launch_decode(decode_launch_of(plan, d_table, k_pool, v_pool, q, out, lse, softmax_scale, workspace, status),
                      s);
  } else {
    PrefillLaunch L{};
    L.heads = section<HeadDesc>(d_table, plan->hdr.off_heads);
    L.pages = section<PageDesc>(d_table, plan->hdr.off_pages);
    L.items = section<PrefillItem>(d_table, plan->hdr.off_prefill);
    L.n_items = plan->hdr.n_prefill_items;
    L.D = plan->prob.head_dim;
    L.P = plan->prob.page_size;
    L.group = plan->group;
    L.num_q_heads = plan->prob.num_q_heads;
    L.total_rows = int32_t(plan->sizes.num_queries);
    L.bf16 = plan->prob.dtype == SP_BF16;
    L.page_bytes = plan->sizes.page_bytes;
    L.pool_pages = plan->sizes.pool_pages;
    L.kpool = k_pool, L.vpool = v_pool, L.q = q, L.out = out, L.lse = lse;
    L.scale_log2 = scale_log2;
    L.status = status;
    e = L.bf16 ? launch_prefill_bf16(L, s) : launch_prefill_f32(L, s);
    if (e == cudaErrorNotSupported) return fail(SP_ERR_UNSUPPORTED, "no prefill kernel for this configuration");
  }
  return e == cudaSuccess ? SP_OK : cuda_fail(e, "segpaged_attention launch");
}

sp_status segpaged_decode_append(const sp_plan* plan, void* d_table, const void* k_new, const void* v_new,
                                 int64_t stride_seq, int64_t stride_head, void* k_pool, void* v_pool, void* workspace,
                                 void* stream) {
  using namespace sp;
  sp_status st = check_table(plan, d_table);
  if (st != SP_OK) return st;
  if (!(plan->prob.flags & SP_FLAG_RING)) return fail(SP_ERR_INVALID_ARG, "segpaged_decode_append needs a ring plan");
  if (!k_new || !v_new || !k_pool || !v_pool || !workspace)
    return fail(SP_ERR_INVALID_ARG, "k_new, v_new, pools and workspace must be non-NULL");
  if (!aligned(k_new, 16) || !aligned(v_new, 16) || !aligned(k_pool, 16) || !aligned(v_pool, 16) ||
      !aligned(workspace, 256))
    return fail(SP_ERR_INVALID_ARG, "new rows and pools must be 16-byte aligned, workspace 256-byte aligned");
  const int64_t eb = plan->elem_bytes;
  if (stride_seq < 0 || stride_head < 0 || (stride_seq * eb) % 16 || (stride_head * eb) % 16)
    return fail(SP_ERR_INVALID_ARG, "strides must be >= 0 and give 16-byte aligned rows");
  AppendLaunch L{};
  L.heads = const_cast<HeadDesc*>(section<HeadDesc>(d_table, plan->hdr.off_heads));
  L.pages = const_cast<PageDesc*>(section<PageDesc>(d_table, plan->hdr.off_pages));
  L.n_heads = plan->hdr.n_heads;
  L.D = plan->prob.head_dim;
  L.P = plan->prob.page_size;
  L.bf16 = plan->prob.dtype == SP_BF16;
  L.fp8 = plan->fp8;
  L.k_inv = 1.0f / plan->k_scale;
  L.v_inv = 1.0f / plan->v_scale;
  L.stride_seq = stride_seq;
  L.stride_head = stride_head;
  L.page_bytes = plan->sizes.page_bytes;
  L.pool_pages = plan->sizes.pool_pages;
  L.k_new = k_new, L.v_new = v_new, L.kpool = k_pool, L.vpool = v_pool;
  L.status = static_cast<int32_t*>(workspace);
  L.free_pool = const_cast<int32_t*>(section<int32_t>(d_table, plan->hdr.off_free));
  const cudaError_t e = launch_append(L, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SP_OK : cuda_fail(e, "segpaged_decode_append launch");
}

sp_status segpaged_decode_step(const sp_plan* plan, void* d_table, const void* k_new, const void* v_new,
                               int64_t stride_seq, int64_t stride_head, void* k_pool, void* v_pool, const void* q,
                               void* out, float* lse, float softmax_scale, void* workspace, size_t workspace_bytes,
                               void* stream) {
  using namespace sp;
  sp_status st = check_attention_args(plan, d_table, k_pool, v_pool, q, out, lse, softmax_scale);
  if (st != SP_OK) return st;
  if (!(plan->prob.flags & SP_FLAG_RING)) return fail(SP_ERR_INVALID_ARG, "segpaged_decode_step needs a ring plan");
  if (!k_new || !v_new || !aligned(k_new, 16) || !aligned(v_new, 16))
    return fail(SP_ERR_INVALID_ARG, "k_new and v_new must be non-NULL and 16-byte aligned");
  const int64_t eb = plan->elem_bytes;
  if (stride_seq < 0 || stride_head < 0 || (stride_seq * eb) % 16 || (stride_head * eb) % 16)
    return fail(SP_ERR_INVALID_ARG, "strides must be >= 0 and give 16-byte aligned rows");
  if (!workspace || !aligned(workspace, 256)) return fail(SP_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  if (int64_t(workspace_bytes) < plan->sizes.workspace_bytes)
    return fail(SP_ERR_WORKSPACE, "workspace smaller than workspace_bytes");
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (plan->prob.dtype != SP_BF16) {  // fp32 pages: the append kernel, then the decode kernels
    st = segpaged_decode_append(plan, d_table, k_new, v_new, stride_seq, stride_head, k_pool, v_pool, workspace,
                                stream);
    if (st != SP_OK) return st;
    return segpaged_attention(plan, d_table, k_pool, v_pool, q, out, lse, softmax_scale, workspace,
                              workspace_bytes, stream);
  }
  DecodeLaunch L = decode_launch_of(plan, d_table, k_pool, v_pool, q, out, lse, softmax_scale, workspace,
                                    static_cast<int32_t*>(workspace));
  L.append = true;
  L.k_new = k_new, L.v_new = v_new;
  L.new_stride_seq = stride_seq, L.new_stride_head = stride_head;
  L.k_inv = 1.0f / plan->k_scale, L.v_inv = 1.0f / plan->v_scale;
  L.free_pool = const_cast<int32_t*>(section<int32_t>(d_table, plan->hdr.off_free));
  const cudaError_t e = launch_decode(L, s);
  return e == cudaSuccess ? SP_OK : cuda_fail(e, "segpaged_decode_step launch");
}

sp_status segpaged_read_device_status(const void* workspace, int32_t* code, void* stream) {
  if (!workspace || !code) return sp::fail(SP_ERR_INVALID_ARG, "workspace and code must be non-NULL");
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return sp::cuda_fail(e, "segpaged_read_device_status sync");
  e = cudaMemcpy(code, workspace, sizeof(int32_t), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return sp::cuda_fail(e, "segpaged_read_device_status copy");
  if (*code != 0) return sp::fail(SP_ERR_DEVICE_CHECK, "device status code " + std::to_string(*code));
  return SP_OK;
}

sp_status segpaged_clear_device_status(void* workspace, void* stream) {
  if (!workspace) return sp::fail(SP_ERR_INVALID_ARG, "workspace must be non-NULL");
  const cudaError_t e = cudaMemsetAsync(workspace, 0, sp::kStatusBytes, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SP_OK : sp::cuda_fail(e, "segpaged_clear_device_status");
}

}  // extern "C"
