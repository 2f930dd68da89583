// Decode-step append for ring plans: one new token per sequence, in place.
//
// One CTA per (sequence, kv-head).  The new token's position is the head's
// current context length L (read from the device table); append_common.cuh
// gives its page and slot, writes its K row and V column, and updates the
// table in place (the target page's valid range, the eviction of the token
// that leaves a LOCAL window, the context length).  E4M3 pages receive the
// codes of the new bf16 row, quantised as the pack does.
#include "append_common.cuh"
#include "kernels.h"

namespace sp {
namespace {

constexpr int kAppendThreads = 128;

template <typename T, int D, int P, bool FP8 = false>
__global__ void __launch_bounds__(kAppendThreads) append_kernel(AppendLaunch a) {
  HeadDesc* hd = a.heads + blockIdx.x;
  const HeadDesc h = *hd;
  const int L = h.ctx_len;
  int vp, slot;
  append_target<P>(h, vp, slot);
  if (vp >= h.n_vpages) {  // no reserved page left: report, change nothing
    if (threadIdx.x == 0) record_error(a.status, kDevAppendFull);
    return;
  }
  PageDesc* pg = a.pages + h.vpage_begin + vp;
  __shared__ int32_t s_phys;
  if (threadIdx.x == 0) s_phys = append_take_page(pg, a.free_pool, a.status);
  __syncthreads();
  const int64_t phys = s_phys;
  if (phys == kNoPage) return;  // the spare pool is empty: the append is skipped (reported)
  if (phys < 0 || phys >= a.pool_pages) {  // corrupted table: report, write nothing
    if (threadIdx.x == 0) record_error(a.status, kDevBadPage);
    return;
  }
  const T* kn = static_cast<const T*>(a.k_new) + int64_t(h.b) * a.stride_seq + int64_t(h.kv) * a.stride_head;
  const T* vn = static_cast<const T*>(a.v_new) + int64_t(h.b) * a.stride_seq + int64_t(h.kv) * a.stride_head;
  append_write_token<T, D, P, FP8>(kn, vn, static_cast<uint8_t*>(a.kpool) + phys * a.page_bytes,
                                   static_cast<uint8_t*>(a.vpool) + phys * a.page_bytes, slot, a.k_inv, a.v_inv,
                                   threadIdx.x, kAppendThreads);
  if (threadIdx.x != 0) return;
  append_update_target(pg, L, slot);
  int evp, eslot, epos;
  append_eviction<P>(h, evp, eslot, epos);
  if (evp >= 0) append_update_eviction(a.pages + h.vpage_begin + evp, epos, eslot);
  hd->ctx_len = L + 1;
  hd->q_start = L;
}

}  // namespace

cudaError_t launch_append(const AppendLaunch& a, cudaStream_t s) {
  if (a.n_heads == 0) return cudaSuccess;
  if (a.fp8) {
    if (a.D == 128) append_kernel<__nv_bfloat16, 128, 64, true><<<a.n_heads, kAppendThreads, 0, s>>>(a);
    else append_kernel<__nv_bfloat16, 64, 64, true><<<a.n_heads, kAppendThreads, 0, s>>>(a);
  } else if (a.bf16) {
    if (a.D == 128) append_kernel<__nv_bfloat16, 128, 64><<<a.n_heads, kAppendThreads, 0, s>>>(a);
    else append_kernel<__nv_bfloat16, 64, 64><<<a.n_heads, kAppendThreads, 0, s>>>(a);
  } else if (a.P == 16) {
    if (a.D == 128) append_kernel<float, 128, 16><<<a.n_heads, kAppendThreads, 0, s>>>(a);
    else append_kernel<float, 64, 16><<<a.n_heads, kAppendThreads, 0, s>>>(a);
  } else {
    if (a.D == 128) append_kernel<float, 128, 64><<<a.n_heads, kAppendThreads, 0, s>>>(a);
    else append_kernel<float, 64, 64><<<a.n_heads, kAppendThreads, 0, s>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace sp
