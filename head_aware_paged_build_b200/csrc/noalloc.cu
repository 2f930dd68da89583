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
// contents; the part that must start at zero (the split heads' arrival
// counters) is cleared by each call.  Device-side errors go to a status word
// the caller owns (d_status), so that the caller can read them.  Calls whose
// kernels overlap on the GPU (different streams, or different host threads,
// same device) race on the array and corrupt each other's partial results:
// serialise them.
#include <cstdint>
#include <mutex>
#include <string>

#include "kernels.h"
#include "sp_internal.h"

namespace sp {
namespace {

// Upper bound of the scratch a decode plan may need (control block + partials).
constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;  // 4 MiB per GPU

static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
void* g_scratch_addr[kMaxDevices] = {};
std::mutex g_scratch_mutex;

// Host code cannot use &g_noalloc_scratch as a device address (it is a host
// stand-in).  Resolve the real address with the device current, once per
// device: only a successful lookup is kept, so a lookup that failed (for
// example one attempted while the stream was being captured) is simply tried
// again by the next call.
cudaError_t scratch_address(int dev, void** out) {
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) {
      *out = nullptr;
      return e;
    }
    if (!p) {
      *out = nullptr;
      return cudaErrorInvalidSymbol;
    }
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

}  // namespace
}  // namespace sp

extern "C" sp_status segpaged_attention_decode_noalloc(const sp_plan* plan, const void* d_table, const void* k_pool,
                                                        const void* v_pool, const void* q, void* out, float* lse,
                                                        float softmax_scale, int32_t* d_status, void* stream) {
  using namespace sp;
  // the same argument checks as segpaged_attention, then this call's own
  sp_status st = check_attention_args(plan, d_table, k_pool, v_pool, q, out, lse, softmax_scale);
  if (st != SP_OK) return st;
  if (!plan->sizes.is_decode)
    return fail(SP_ERR_UNSUPPORTED, "segpaged_attention_decode_noalloc takes decode plans only");
  if (!d_status || (reinterpret_cast<uintptr_t>(d_status) & 3))
    return fail(SP_ERR_INVALID_ARG, "d_status must be a 4-byte aligned device int32 owned by the caller");
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
  if (e != cudaSuccess)
    return fail(SP_ERR_CUDA, std::string("cudaGetSymbolAddress of the built-in scratch: ") + cudaGetErrorString(e));

  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  // The split heads' arrival counters must start at zero (they return to zero
  // by themselves unless a call was cut short); the partial results need no
  // clearing.  The status block in front of them is cleared with them.
  e = cudaMemsetAsync(scratch, 0, size_t(plan->partial_offset), s);
  if (e != cudaSuccess) return fail(SP_ERR_CUDA, std::string("clearing the control block: ") + cudaGetErrorString(e));
  e = launch_decode(decode_launch_of(plan, d_table, k_pool, v_pool, q, out, lse, softmax_scale, scratch, d_status),
                    s);
  return e == cudaSuccess ? SP_OK : fail(SP_ERR_CUDA, std::string("decode launch: ") + cudaGetErrorString(e));
}
