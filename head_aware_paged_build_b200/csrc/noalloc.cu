// segpaged_attention_decode_noalloc: the decode attention call for callers
// that cannot allocate device memory.
//
// segpaged_attention needs a caller-provided workspace for the partial
// results of heads split across CTAs.  Some callers cannot provide one: an
// engine whose device memory is carved into a fixed arena before serving
// starts (no byte is left for a library's scratch), or a latency-critical loop
// that must not call cudaMalloc, which can synchronise the whole device.  This
// entry point takes its scratch from a fixed-size array in the library's own
// device image instead, and allocates nothing: no cudaMalloc, no cudaFree, no
// allocating library call.
//
// The array lives for as long as the library is loaded, once on every GPU that
// loads it, and is shared by every call on that GPU.  It keeps the last call's
// contents; the parts that must start at zero (the status word and the split
// heads' arrival counters) are cleared by each call.  Calls whose kernels overlap on the GPU (different
// streams, or different host threads, same device) race on the array and
// corrupt each other's partial results: serialise them.
#include <cmath>
#include <mutex>
#include <string>

#include "kernels.h"
#include "sp_internal.h"

namespace sp {
namespace {

// Upper bound of the scratch a decode plan may need (status word + partials).
constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;  // 4 MiB per GPU

static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
void* g_scratch_addr[kMaxDevices] = {};
cudaError_t g_scratch_err[kMaxDevices] = {};
std::once_flag g_scratch_once[kMaxDevices];

// Host code cannot use &g_noalloc_scratch as a device address (it is a host
// stand-in).  Resolve the real address once per device, with that device
// current.
cudaError_t scratch_address(int dev, void** out) {
  std::call_once(g_scratch_once[dev], [dev] {
    void* p = nullptr;
    g_scratch_err[dev] = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    g_scratch_addr[dev] = p;
  });
  *out = g_scratch_addr[dev];
  return g_scratch_err[dev];
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

}  // namespace
}  // namespace sp

extern "C" sp_status segpaged_attention_decode_noalloc(const sp_plan* plan, const void* d_table, const void* k_pool,
                                                        const void* v_pool, const void* q, void* out, float* lse,
                                                        float softmax_scale, int32_t* d_status, void* stream) {
  using namespace sp;
  if (!plan) return fail(SP_ERR_INVALID_ARG, "plan is NULL");
  if (!plan->sizes.is_decode)
    return fail(SP_ERR_UNSUPPORTED, "segpaged_attention_decode_noalloc takes decode plans only");
  if (!d_table || !k_pool || !v_pool || !q || !out)
    return fail(SP_ERR_INVALID_ARG, "table, pools, q and out must be non-NULL");
  if (!aligned16(d_table) || !aligned16(k_pool) || !aligned16(v_pool) || !aligned16(q) || !aligned16(out))
    return fail(SP_ERR_INVALID_ARG, "table, pools, q and out must be 16-byte aligned");
  if ((lse && (reinterpret_cast<uintptr_t>(lse) & 3)) || (d_status && (reinterpret_cast<uintptr_t>(d_status) & 3)))
    return fail(SP_ERR_INVALID_ARG, "lse and d_status must be 4-byte aligned");
  if (!(softmax_scale == softmax_scale) || softmax_scale > 3.0e38f || softmax_scale < -3.0e38f)
    return fail(SP_ERR_INVALID_ARG, "softmax_scale must be finite");
  if (size_t(plan->sizes.workspace_bytes) > kNoAllocScratchBytes)
    return fail(SP_ERR_WORKSPACE, "this decode plan needs " + std::to_string(plan->sizes.workspace_bytes) +
                                      " bytes of scratch; the built-in scratch holds " +
                                      std::to_string(kNoAllocScratchBytes) +
                                      " (use segpaged_attention with a caller workspace, or fewer target_ctas)");
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(SP_ERR_CUDA, std::string("cudaGetDevice: ") + cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return fail(SP_ERR_UNSUPPORTED, "device index above 63");
  void* scratch = nullptr;
  e = scratch_address(dev, &scratch);
  if (e != cudaSuccess || !scratch)
    return fail(SP_ERR_CUDA, std::string("cudaGetSymbolAddress of the built-in scratch: ") + cudaGetErrorString(e));

  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  int32_t* status = d_status ? d_status : static_cast<int32_t*>(scratch);
  // The status word and the split heads' arrival counters must start at zero
  // (the counters return to zero by themselves unless a call was cut short).
  e = cudaMemsetAsync(scratch, 0, size_t(plan->partial_offset), s);
  if (e != cudaSuccess) return fail(SP_ERR_CUDA, std::string("clearing the control block: ") + cudaGetErrorString(e));
  const float scale = softmax_scale > 0.f ? softmax_scale : 1.0f / std::sqrt(float(plan->prob.head_dim));
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
  L.scale_log2 = scale * 1.4426950408889634f * (plan->fp8 ? plan->k_scale : 1.f);
  L.fp8 = plan->fp8;
  L.v_scale = plan->fp8 ? plan->v_scale : 1.f;
  L.partial = reinterpret_cast<float*>(static_cast<uint8_t*>(scratch) + plan->partial_offset);
  L.counters = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(scratch) + kStatusBytes);
  L.status = status;
  e = launch_decode(L, s);
  return e == cudaSuccess ? SP_OK : fail(SP_ERR_CUDA, std::string("decode launch: ") + cudaGetErrorString(e));
}
