// The decode-step append of ring plans, as device helpers shared by the
// standalone append kernel and the fused append + decode kernel, so that both
// write the same bytes and make the same table changes.
//
// The new token sits at position L, the head's current context length:
//   GLOBAL: page L / P of the head (pages reserved for the append capacity),
//           slot L % P;
//   LOCAL:  a sink page while L < sink, else ring slot L mod (R P) of the R
//           ring pages after the sink pages, R = ceil(window / P) + 1.
// Its page's valid range grows (or restarts when the ring wraps onto a page
// whose tokens all left the window); for a LOCAL head the token at L - window
// leaves the window (its page's range shrinks from below); the context grows
// by one.  No token ever moves ("SegPagedAttention runtime design", §3: a
// local head's occupancy does not depend on the context length).
#pragma once

#include "device_common.cuh"

namespace sp {

// Page index (in the head's list) and slot of the new token of head hd.
template <int P>
__device__ __forceinline__ void append_target(const HeadDesc& hd, int& vp, int& slot) {
  const int L = hd.ctx_len;
  if (hd.kind != 1 || L < hd.sink) {
    vp = L / P, slot = L % P;
  } else {
    const int nsink = (hd.sink + P - 1) / P, R = (hd.window + P - 1) / P + 1;
    const int r = L % (R * P);
    vp = nsink + r / P, slot = r % P;
  }
}

// The page (index in the head's list, or -1) and slot of the token that leaves
// a LOCAL head's window when the token at L is appended.
template <int P>
__device__ __forceinline__ void append_eviction(const HeadDesc& hd, int& vp, int& slot, int& pos) {
  vp = -1, slot = 0, pos = hd.ctx_len - hd.window;
  if (hd.kind != 1 || pos < hd.sink) return;
  const int nsink = (hd.sink + P - 1) / P, R = (hd.window + P - 1) / P + 1;
  const int re = pos % (R * P);
  vp = nsink + re / P, slot = re % P;
}

// The physical page of the target record, taken from the ring plan's shared
// spare pool when the record has none yet (a GLOBAL head growing into a page
// it reserved as a record only).  Returns kNoPage, and records device code 7,
// when the pool is empty.  The pool only hands pages out during a table's
// life (segpaged_table_write refills it), so one atomic decrement per page is
// enough.  One thread.
__device__ __forceinline__ int32_t append_take_page(PageDesc* pg, int32_t* free_pool, int32_t* status) {
  int32_t phys = pg->phys;
  if (phys != kNoPage) return phys;
  if (free_pool) {
    const int32_t idx = atomicSub(free_pool, 1) - 1;
    if (idx >= 0) {
      phys = free_pool[kFreeIdsOffset + idx];
      pg->phys = phys;
      return phys;
    }
    atomicAdd(free_pool, 1);
  }
  record_error(status, kDevPoolEmpty);
  return kNoPage;
}

// The target page's new valid range (one thread).
__device__ __forceinline__ void append_update_target(PageDesc* pg, int L, int slot) {
  int lo = slot_lo(*pg);
  if (slot_hi(*pg) <= lo || pg->abs_start != L - slot) {
    pg->abs_start = L - slot;
    lo = slot;
  }
  pg->span = make_span(lo, slot + 1) | (pg->span & kSpanCausal);
}

// The evicted token's page loses it, if the page still holds that position's run (one thread).
__device__ __forceinline__ void append_update_eviction(PageDesc* pe, int pos, int slot) {
  if (pe->abs_start == pos - slot) {
    const int elo = max(slot_lo(*pe), slot + 1), ehi = slot_hi(*pe);
    pe->span = elo < ehi ? (make_span(elo, ehi) | (pe->span & kSpanCausal)) : 0;
  }
}

// Write the new token's K row and V column into page slot `slot` (threads
// t = first, first + stride, ... of the caller cooperate).  bf16 pages use the
// swizzled operand layouts, fp32 pages row-major K and transposed V, E4M3
// pages the codes of the bf16 values times 1 / scale (nearest even,
// saturating), as the pack writes them.  The new row never overlaps the page,
// so the loads need not wait for the stores.
template <typename T, int D, int P, bool FP8>
__device__ __forceinline__ void append_write_token(const T* __restrict__ kn, const T* __restrict__ vn,
                                                   uint8_t* __restrict__ kdst, uint8_t* __restrict__ vdst, int slot,
                                                   float k_inv, float v_inv, int first, int stride) {
  constexpr int CR = D * int(sizeof(T)) / 16;
  if constexpr (FP8) {
    for (int c = first; c < CR; c += stride) {  // 8 values -> 8 codes
      const uint4 v = reinterpret_cast<const uint4*>(kn)[c];
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
      uint32_t q[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const float x0 = __uint_as_float(w[2 * h] << 16) * k_inv, x1 = __uint_as_float(w[2 * h] & 0xffff0000u) * k_inv;
        const float x2 = __uint_as_float(w[2 * h + 1] << 16) * k_inv,
                    x3 = __uint_as_float(w[2 * h + 1] & 0xffff0000u) * k_inv;
        q[h] = uint32_t(pack_e4m3x2(x0, x1)) | (uint32_t(pack_e4m3x2(x2, x3)) << 16);
      }
      *reinterpret_cast<uint2*>(kdst + fp8_kpage_offset(slot, c * 8, D)) = make_uint2(q[0], q[1]);
    }
    for (int i = first; i < D; i += stride) {
      const float x = __bfloat162float(vn[i]) * v_inv;
      vdst[fp8_vpage_offset(i, fp8_vtok_pos(slot))] = uint8_t(pack_e4m3x2(x, 0.f));
    }
  } else {
    for (int c = first; c < CR; c += stride) {
      const uint4 v = reinterpret_cast<const uint4*>(kn)[c];
      if constexpr (sizeof(T) == 2)
        *reinterpret_cast<uint4*>(kdst + kpage_chunk_offset_bf16(slot, c, P)) = v;
      else
        *reinterpret_cast<uint4*>(kdst + (int64_t(slot) * D) * 4 + c * 16) = v;
    }
    for (int i = first; i < D; i += stride) {
      // transposed V page: row i, token column `slot`
      int64_t off;
      if constexpr (sizeof(T) == 2)
        off = vpage_chunk_offset_bf16(i, slot >> 3) + (slot & 7) * 2;
      else
        off = (int64_t(i) * P + slot) * 4;
      *reinterpret_cast<T*>(vdst + off) = vn[i];
    }
  }
}

}  // namespace sp
