// Decode-step append for ring plans: one new token per sequence, in place.
//
// One CTA per (sequence, kv-head).  The new token's position is the head's
// current context length L (read from the device table).  Its K row and V
// column are written into the page slot the ring layout assigns:
//   GLOBAL: page L / P of the head (pages were reserved for the append
//           capacity), slot L % P;
//   LOCAL:  a sink page while L < sink, else ring slot L mod (R P) of the R
//           ring pages, R = ceil(window / P) + 1.
// Then the table is updated in place: the target page's valid range grows (or
// restarts when the ring wraps onto a page whose tokens all left the window),
// the token at L - window leaves a LOCAL head's window (its page's range
// shrinks from below: eviction), and the head's context grows by one.  No
// token ever moves ("SegPagedAttention runtime design", §3: a local head's
// occupancy does not depend on the context length).  E4M3 pages receive the
// codes of the new bf16 row, quantised as the pack does.
#include "device_common.cuh"
#include "kernels.h"

namespace sp {
namespace {

constexpr int kAppendThreads = 128;

template <typename T, int D, int P, bool FP8 = false>
__global__ void __launch_bounds__(kAppendThreads) append_kernel(AppendLaunch a) {
  HeadDesc* hd = a.heads + blockIdx.x;
  const int L = hd->ctx_len;
  const bool local = hd->kind == 1;
  const int nsink = local ? (hd->sink + P - 1) / P : 0;
  const int R = local ? (hd->window + P - 1) / P + 1 : 0;
  int vp, slot;
  if (!local || L < hd->sink) {
    vp = L / P, slot = L % P;
  } else {
    const int r = L % (R * P);
    vp = nsink + r / P, slot = r % P;
  }
  if (vp >= hd->n_vpages) {  // no reserved page left: report, change nothing
    if (threadIdx.x == 0) record_error(a.status, kDevAppendFull);
    return;
  }
  PageDesc* pg = a.pages + hd->vpage_begin + vp;
  const int64_t phys = pg->phys;
  if (phys < 0 || phys >= a.pool_pages) {  // corrupted table: report, write nothing
    if (threadIdx.x == 0) record_error(a.status, kDevBadPage);
    return;
  }
  const T* kn = static_cast<const T*>(a.k_new) + int64_t(hd->b) * a.stride_seq + int64_t(hd->kv) * a.stride_head;
  const T* vn = static_cast<const T*>(a.v_new) + int64_t(hd->b) * a.stride_seq + int64_t(hd->kv) * a.stride_head;
  uint8_t* kdst = static_cast<uint8_t*>(a.kpool) + phys * a.page_bytes;
  uint8_t* vdst = static_cast<uint8_t*>(a.vpool) + phys * a.page_bytes;
  constexpr int CR = D * int(sizeof(T)) / 16;
  if constexpr (FP8) {
    for (int c = threadIdx.x; c < CR; c += kAppendThreads) {  // 8 values -> 8 codes
      const uint4 v = reinterpret_cast<const uint4*>(kn)[c];
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
      uint32_t q[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const float x0 = __uint_as_float(w[2 * h] << 16) * a.k_inv, x1 = __uint_as_float(w[2 * h] & 0xffff0000u) * a.k_inv;
        const float x2 = __uint_as_float(w[2 * h + 1] << 16) * a.k_inv,
                    x3 = __uint_as_float(w[2 * h + 1] & 0xffff0000u) * a.k_inv;
        q[h] = uint32_t(pack_e4m3x2(x0, x1)) | (uint32_t(pack_e4m3x2(x2, x3)) << 16);
      }
      *reinterpret_cast<uint2*>(kdst + fp8_kpage_offset(slot, c * 8, D)) = make_uint2(q[0], q[1]);
    }
    for (int i = threadIdx.x; i < D; i += kAppendThreads) {
      const float x = __bfloat162float(vn[i]) * a.v_inv;
      vdst[fp8_vpage_offset(i, fp8_vtok_pos(slot))] = uint8_t(pack_e4m3x2(x, 0.f));
    }
  } else {
  for (int c = threadIdx.x; c < CR; c += kAppendThreads) {
    const uint4 v = reinterpret_cast<const uint4*>(kn)[c];
    if constexpr (sizeof(T) == 2)
      *reinterpret_cast<uint4*>(kdst + kpage_chunk_offset_bf16(slot, c, P)) = v;
    else
      *reinterpret_cast<uint4*>(kdst + (int64_t(slot) * D) * 4 + c * 16) = v;
  }
  for (int i = threadIdx.x; i < D; i += kAppendThreads) {
    // transposed V page: row i, token column `slot`
    int64_t off;
    if constexpr (sizeof(T) == 2)
      off = vpage_chunk_offset_bf16(i, slot >> 3) + (slot & 7) * 2;
    else
      off = (int64_t(i) * P + slot) * 4;
    *reinterpret_cast<T*>(vdst + off) = vn[i];
  }
  }
  if (threadIdx.x != 0) return;
  // the target page: a new run starts when the page held other positions
  int lo = slot_lo(*pg);
  if (slot_hi(*pg) <= lo || pg->abs_start != L - slot) {
    pg->abs_start = L - slot;
    lo = slot;
  }
  pg->span = make_span(lo, slot + 1) | (pg->span & kSpanCausal);
  // eviction: position L - window leaves the window [L + 1 - window, L]
  if (local) {
    const int e = L - hd->window;
    if (e >= hd->sink) {
      const int re = e % (R * P);
      PageDesc* pe = a.pages + hd->vpage_begin + nsink + re / P;
      const int se = re % P;
      if (pe->abs_start == e - se) {
        const int elo = max(slot_lo(*pe), se + 1), ehi = slot_hi(*pe);
        pe->span = elo < ehi ? (make_span(elo, ehi) | (pe->span & kSpanCausal)) : 0;
      }
    }
  }
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
