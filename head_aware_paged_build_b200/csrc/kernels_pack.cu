// build_segpaged_cache (pack) and its inverse (gather).
//
// One CTA per page: it copies the page's stored rows of dense K/V (16-byte
// vector loads, consecutive threads on consecutive chunks of a row) into the
// pool's page layout.  K chunks move straight to their swizzled slot; V is
// transposed through shared memory.  Slots outside the page's valid range
// [lo, hi) are written as zeros so that every pool byte the attention kernels
// read is a finite number ("SegPagedAttention runtime design", §3:
// build_segpaged_cache packs dense KV and keeps only what a head can see).
#include "device_common.cuh"
#include "kernels.h"

namespace sp {
namespace {

constexpr int kPackThreads = 256;

struct PackArgs {
  const HeadDesc* heads;
  const PageDesc* pages;
  int64_t stride_seq, stride_head, stride_tok;  // stride_seq < 0: packed by context rows
  int64_t page_bytes;
};

// Shared-memory row pitch of the V staging tile: one extra 32-bit word per row
// makes column reads (the transpose) and row writes both bank-conflict free.
template <typename T>
__host__ __device__ constexpr int vstage_pitch_words(int D) {
  return D * int(sizeof(T)) / 4 + 1;
}

template <typename T>
__device__ __forceinline__ int64_t kpage_chunk(int t, int c16, int P, int D) {
  if constexpr (sizeof(T) == 2) {
    return kpage_chunk_offset_bf16(t, c16, P);
  } else {
    return (int64_t(t) * D) * 4 + c16 * 16;
  }
}

template <typename T>
__device__ __forceinline__ int64_t vpage_chunk(int i, int c16, int P) {
  if constexpr (sizeof(T) == 2) {
    return vpage_chunk_offset_bf16(i, c16);
  } else {
    return (int64_t(i) * P) * 4 + c16 * 16;
  }
}

template <typename T, int D, int P>
__device__ __forceinline__ void pack_page(const PackArgs& a, int page, const T* __restrict__ kd,
                                          const T* __restrict__ vd, uint8_t* __restrict__ kpool,
                                          uint8_t* __restrict__ vpool) {
  constexpr int CR = D * int(sizeof(T)) / 16;   // 16-byte chunks per dense row
  constexpr int EPC = 16 / int(sizeof(T));      // elements per chunk
  constexpr int PW = vstage_pitch_words<T>(D);  // staging pitch (32-bit words)
  constexpr int VR = P / EPC;                   // chunks per transposed V row
  __shared__ uint32_t stage[P * PW];

  const PageDesc pg = a.pages[page];
  if (pg.phys < 0) return;  // a record waiting for a page from the spare pool holds nothing
  const HeadDesc hd = a.heads[pg.head];
  const int64_t base = (a.stride_seq >= 0 ? int64_t(hd.b) * a.stride_seq : int64_t(hd.ctx_row0) * a.stride_tok) +
                       int64_t(hd.kv) * a.stride_head;
  uint8_t* kdst = kpool + int64_t(pg.phys) * a.page_bytes;
  uint8_t* vdst = vpool + int64_t(pg.phys) * a.page_bytes;

  for (int idx = threadIdx.x; idx < P * CR; idx += kPackThreads) {
    const int t = idx / CR, c = idx % CR;
    uint4 kv4 = make_uint4(0, 0, 0, 0), vv4 = make_uint4(0, 0, 0, 0);
    if (t >= slot_lo(pg) && t < slot_hi(pg)) {
      const int64_t row = base + int64_t(pg.abs_start + t) * a.stride_tok;
      kv4 = __ldg(reinterpret_cast<const uint4*>(kd + row) + c);
      vv4 = __ldg(reinterpret_cast<const uint4*>(vd + row) + c);
    }
    *reinterpret_cast<uint4*>(kdst + kpage_chunk<T>(t, c, P, D)) = kv4;
    uint32_t* s = stage + t * PW + c * 4;
    s[0] = vv4.x, s[1] = vv4.y, s[2] = vv4.z, s[3] = vv4.w;
  }
  __syncthreads();
  // transposed V: row i (dimension) holds the page's P tokens
  const T* st = reinterpret_cast<const T*>(stage);
  for (int idx = threadIdx.x; idx < D * VR; idx += kPackThreads) {
    const int i = idx / VR, c = idx % VR;
    alignas(16) T vals[EPC];
#pragma unroll
    for (int e = 0; e < EPC; ++e) vals[e] = st[(c * EPC + e) * (PW * 4 / int(sizeof(T))) + i];
    *reinterpret_cast<uint4*>(vdst + vpage_chunk<T>(i, c, P)) = *reinterpret_cast<const uint4*>(vals);
  }
}

template <typename T, int D, int P>
__global__ void __launch_bounds__(kPackThreads) pack_kernel(PackArgs a, const T* __restrict__ kd,
                                                            const T* __restrict__ vd, uint8_t* __restrict__ kpool,
                                                            uint8_t* __restrict__ vpool) {
  pack_page<T, D, P>(a, blockIdx.x, kd, vd, kpool, vpool);
}

template <typename T, int D, int P>
__global__ void __launch_bounds__(kPackThreads) gather_kernel(PackArgs a, const uint8_t* __restrict__ kpool,
                                                              const uint8_t* __restrict__ vpool, T* __restrict__ kd,
                                                              T* __restrict__ vd) {
  constexpr int CR = D * int(sizeof(T)) / 16;
  constexpr int EPC = 16 / int(sizeof(T));
  constexpr int PW = vstage_pitch_words<T>(D);
  constexpr int VR = P / EPC;
  __shared__ uint32_t stage[P * PW];

  const PageDesc pg = a.pages[blockIdx.x];
  if (pg.phys < 0) return;  // a record waiting for a page from the spare pool holds nothing
  const HeadDesc hd = a.heads[pg.head];
  const int64_t base = (a.stride_seq >= 0 ? int64_t(hd.b) * a.stride_seq : int64_t(hd.ctx_row0) * a.stride_tok) +
                       int64_t(hd.kv) * a.stride_head;
  const uint8_t* ksrc = kpool + int64_t(pg.phys) * a.page_bytes;
  const uint8_t* vsrc = vpool + int64_t(pg.phys) * a.page_bytes;

  T* st = reinterpret_cast<T*>(stage);
  for (int idx = threadIdx.x; idx < D * VR; idx += kPackThreads) {
    const int i = idx / VR, c = idx % VR;
    alignas(16) T vals[EPC];
    *reinterpret_cast<uint4*>(vals) = *reinterpret_cast<const uint4*>(vsrc + vpage_chunk<T>(i, c, P));
#pragma unroll
    for (int e = 0; e < EPC; ++e) st[(c * EPC + e) * (PW * 4 / int(sizeof(T))) + i] = vals[e];
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < P * CR; idx += kPackThreads) {
    const int t = idx / CR, c = idx % CR;
    if (t < slot_lo(pg) || t >= slot_hi(pg)) continue;
    const int64_t row = base + int64_t(pg.abs_start + t) * a.stride_tok;
    reinterpret_cast<uint4*>(kd + row)[c] = *reinterpret_cast<const uint4*>(ksrc + kpage_chunk<T>(t, c, P, D));
    const uint32_t* s = stage + t * PW + c * 4;
    reinterpret_cast<uint4*>(vd + row)[c] = make_uint4(s[0], s[1], s[2], s[3]);
  }
}

// ---------------------------------------------------------------------------
// E4M3 pages (page size 64): K page [64 tokens][D] codes, V page [D][64
// positions] codes at fp8_kpage_offset() / fp8_vpage_offset(); V positions order the tokens
// as fp8_vtok_pos() says.  Dense side: bf16 for pack, 1-byte codes for gather.
// Codes are E4M3(fp32(x) * (1 / scale)), nearest-even, saturating.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float bf16_bits_to_float(uint32_t bits16) { return __uint_as_float(bits16 << 16); }

__device__ __forceinline__ uint32_t quant4(uint32_t w0, uint32_t w1, float inv) {
  // four bf16 values (two words, low half first) -> four codes, first value in the low byte
  const uint16_t c0 = pack_e4m3x2(bf16_bits_to_float(w0 & 0xffff) * inv, bf16_bits_to_float(w0 >> 16) * inv);
  const uint16_t c1 = pack_e4m3x2(bf16_bits_to_float(w1 & 0xffff) * inv, bf16_bits_to_float(w1 >> 16) * inv);
  return uint32_t(c0) | (uint32_t(c1) << 16);
}

template <int D>
__device__ __forceinline__ void pack_fp8_page(const PackArgs& a, int page, float k_inv, float v_inv,
                                              const __nv_bfloat16* __restrict__ kd,
                                              const __nv_bfloat16* __restrict__ vd, uint8_t* __restrict__ kpool,
                                              uint8_t* __restrict__ vpool) {
  constexpr int P = 64;
  constexpr int CR = D * 2 / 16;                            // 16-byte bf16 chunks per dense row
  constexpr int PW = vstage_pitch_words<__nv_bfloat16>(D);  // staging pitch (32-bit words)
  __shared__ uint32_t stage[P * PW];
  const PageDesc pg = a.pages[page];
  if (pg.phys < 0) return;  // a record waiting for a page from the spare pool holds nothing
  const HeadDesc hd = a.heads[pg.head];
  const int64_t base = (a.stride_seq >= 0 ? int64_t(hd.b) * a.stride_seq : int64_t(hd.ctx_row0) * a.stride_tok) +
                       int64_t(hd.kv) * a.stride_head;
  uint8_t* kdst = kpool + int64_t(pg.phys) * a.page_bytes;
  uint8_t* vdst = vpool + int64_t(pg.phys) * a.page_bytes;
  for (int idx = threadIdx.x; idx < P * CR; idx += kPackThreads) {
    const int t = idx / CR, c = idx % CR;
    uint4 kv4 = make_uint4(0, 0, 0, 0), vv4 = make_uint4(0, 0, 0, 0);
    if (t >= slot_lo(pg) && t < slot_hi(pg)) {
      const int64_t row = base + int64_t(pg.abs_start + t) * a.stride_tok;
      kv4 = __ldg(reinterpret_cast<const uint4*>(kd + row) + c);
      vv4 = __ldg(reinterpret_cast<const uint4*>(vd + row) + c);
    }
    *reinterpret_cast<uint2*>(kdst + fp8_kpage_offset(t, c * 8, D)) =
        make_uint2(quant4(kv4.x, kv4.y, k_inv), quant4(kv4.z, kv4.w, k_inv));
    uint32_t* st = stage + t * PW + c * 4;
    st[0] = vv4.x, st[1] = vv4.y, st[2] = vv4.z, st[3] = vv4.w;
  }
  __syncthreads();
  const uint16_t* sv = reinterpret_cast<const uint16_t*>(stage);  // [token][dim] bf16, pitch 2 PW
  for (int idx = threadIdx.x; idx < D * 4; idx += kPackThreads) {
    const int i = idx / 4, c = idx % 4;  // row i (dimension), positions 16 c .. 16 c + 15
    uint32_t q[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      float x[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) x[u] = bf16_bits_to_float(sv[fp8_vpos_tok(c * 16 + e * 4 + u) * PW * 2 + i]) * v_inv;
      q[e] = uint32_t(pack_e4m3x2(x[0], x[1])) | (uint32_t(pack_e4m3x2(x[2], x[3])) << 16);
    }
    *reinterpret_cast<uint4*>(vdst + fp8_vpage_offset(i, c * 16)) = make_uint4(q[0], q[1], q[2], q[3]);
  }
}

template <int D>
__global__ void __launch_bounds__(kPackThreads) pack_fp8_kernel(PackArgs a, float k_inv, float v_inv,
                                                                const __nv_bfloat16* __restrict__ kd,
                                                                const __nv_bfloat16* __restrict__ vd,
                                                                uint8_t* __restrict__ kpool,
                                                                uint8_t* __restrict__ vpool) {
  pack_fp8_page<D>(a, blockIdx.x, k_inv, v_inv, kd, vd, kpool, vpool);
}

// Several layers in one launch: CTA i packs page i of the layers' concatenated
// page lists; the layer is found by a binary search of the page offsets.
template <typename T, int D, int P, bool FP8>
__global__ void __launch_bounds__(kPackThreads) pack_layers_kernel(PackLayersArgs la, uint8_t* __restrict__ kpool,
                                                                   uint8_t* __restrict__ vpool) {
  int lo = 0, hi = la.n_layers - 1;
  while (lo < hi) {  // last layer whose first page <= blockIdx.x
    const int mid = (lo + hi + 1) / 2;
    if (la.page_begin[mid] <= int(blockIdx.x)) lo = mid;
    else hi = mid - 1;
  }
  const PackArgs a{la.heads[lo], la.pages[lo], la.stride_seq, la.stride_head, la.stride_tok, la.page_bytes};
  const int page = int(blockIdx.x) - la.page_begin[lo];
  if constexpr (FP8)
    pack_fp8_page<D>(a, page, la.k_inv[lo], la.v_inv[lo], static_cast<const __nv_bfloat16*>(la.kd[lo]),
                     static_cast<const __nv_bfloat16*>(la.vd[lo]), kpool, vpool);
  else
    pack_page<T, D, P>(a, page, static_cast<const T*>(la.kd[lo]), static_cast<const T*>(la.vd[lo]), kpool, vpool);
}

template <int D>
__global__ void __launch_bounds__(kPackThreads) gather_fp8_kernel(PackArgs a, const uint8_t* __restrict__ kpool,
                                                                  const uint8_t* __restrict__ vpool,
                                                                  uint8_t* __restrict__ kd, uint8_t* __restrict__ vd) {
  constexpr int P = 64;
  constexpr int SP = P + 4;  // staging pitch (bytes) of the V codes [D][tokens]
  __shared__ uint8_t stage[D * SP];
  const PageDesc pg = a.pages[blockIdx.x];
  if (pg.phys < 0) return;  // a record waiting for a page from the spare pool holds nothing
  const HeadDesc hd = a.heads[pg.head];
  const int64_t base = (a.stride_seq >= 0 ? int64_t(hd.b) * a.stride_seq : int64_t(hd.ctx_row0) * a.stride_tok) +
                       int64_t(hd.kv) * a.stride_head;
  const uint8_t* ksrc = kpool + int64_t(pg.phys) * a.page_bytes;
  const uint8_t* vsrc = vpool + int64_t(pg.phys) * a.page_bytes;
  for (int idx = threadIdx.x; idx < D * P / 16; idx += kPackThreads) {
    const int i = idx / (P / 16), c = idx % (P / 16);
    alignas(16) uint8_t b[16];
    *reinterpret_cast<uint4*>(b) = *reinterpret_cast<const uint4*>(vsrc + fp8_vpage_offset(i, c * 16));
#pragma unroll
    for (int e = 0; e < 16; ++e) stage[i * SP + fp8_vpos_tok(c * 16 + e)] = b[e];
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < P * D / 16; idx += kPackThreads) {
    const int t = idx / (D / 16), c = idx % (D / 16);
    if (t < slot_lo(pg) || t >= slot_hi(pg)) continue;
    const int64_t row = base + int64_t(pg.abs_start + t) * a.stride_tok;
    reinterpret_cast<uint4*>(kd + row)[c] = *reinterpret_cast<const uint4*>(ksrc + fp8_kpage_offset(t, c * 16, D));
    alignas(16) uint8_t b[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) b[e] = stage[(c * 16 + e) * SP + t];
    reinterpret_cast<uint4*>(vd + row)[c] = *reinterpret_cast<const uint4*>(b);
  }
}

template <int D>
void launch_pack_fp8(const PackLaunch& L, cudaStream_t s) {
  PackArgs a{L.heads, L.pages, L.stride_seq, L.stride_head, L.stride_tok, L.page_bytes};
  if (L.inverse)
    gather_fp8_kernel<D><<<L.n_pages, kPackThreads, 0, s>>>(a, static_cast<const uint8_t*>(L.kpool_in),
                                                            static_cast<const uint8_t*>(L.vpool_in),
                                                            static_cast<uint8_t*>(L.kdense_out),
                                                            static_cast<uint8_t*>(L.vdense_out));
  else
    pack_fp8_kernel<D><<<L.n_pages, kPackThreads, 0, s>>>(a, L.k_inv, L.v_inv,
                                                          static_cast<const __nv_bfloat16*>(L.kdense_in),
                                                          static_cast<const __nv_bfloat16*>(L.vdense_in),
                                                          static_cast<uint8_t*>(L.kpool_out),
                                                          static_cast<uint8_t*>(L.vpool_out));
}

template <typename T, int D, int P>
void launch_pack_t(const PackLaunch& L, cudaStream_t s) {
  PackArgs a{L.heads, L.pages, L.stride_seq, L.stride_head, L.stride_tok, L.page_bytes};
  if (L.inverse)
    gather_kernel<T, D, P><<<L.n_pages, kPackThreads, 0, s>>>(a, static_cast<const uint8_t*>(L.kpool_in),
                                                              static_cast<const uint8_t*>(L.vpool_in),
                                                              static_cast<T*>(L.kdense_out),
                                                              static_cast<T*>(L.vdense_out));
  else
    pack_kernel<T, D, P><<<L.n_pages, kPackThreads, 0, s>>>(a, static_cast<const T*>(L.kdense_in),
                                                            static_cast<const T*>(L.vdense_in),
                                                            static_cast<uint8_t*>(L.kpool_out),
                                                            static_cast<uint8_t*>(L.vpool_out));
}

// Zero one page of each pool per block: the spare pool's pages, so that an
// append that takes one leaves only finite values in the slots it masks out.
__global__ void __launch_bounds__(kPackThreads) zero_pages_kernel(const int32_t* __restrict__ ids,
                                                                  int64_t page_bytes, uint8_t* __restrict__ kpool,
                                                                  uint8_t* __restrict__ vpool) {
  const int64_t phys = ids[blockIdx.x];
  uint4* k = reinterpret_cast<uint4*>(kpool + phys * page_bytes);
  uint4* v = reinterpret_cast<uint4*>(vpool + phys * page_bytes);
  for (int64_t i = threadIdx.x; i < page_bytes / 16; i += kPackThreads) {
    k[i] = make_uint4(0, 0, 0, 0);
    v[i] = make_uint4(0, 0, 0, 0);
  }
}

}  // namespace

cudaError_t launch_zero_pages(const int32_t* ids, int32_t n, int64_t page_bytes, void* kpool, void* vpool,
                              cudaStream_t s) {
  if (n == 0) return cudaSuccess;
  zero_pages_kernel<<<n, kPackThreads, 0, s>>>(ids, page_bytes, static_cast<uint8_t*>(kpool),
                                               static_cast<uint8_t*>(vpool));
  return cudaGetLastError();
}

cudaError_t launch_pack_layers(const PackLayersArgs& la, bool bf16, bool fp8, int D, int P, void* kpool, void* vpool,
                               cudaStream_t s) {
  const int n = la.page_begin[la.n_layers];
  if (n == 0) return cudaSuccess;
  uint8_t* kp = static_cast<uint8_t*>(kpool);
  uint8_t* vp = static_cast<uint8_t*>(vpool);
  if (fp8) {
    if (D == 128) pack_layers_kernel<__nv_bfloat16, 128, 64, true><<<n, kPackThreads, 0, s>>>(la, kp, vp);
    else pack_layers_kernel<__nv_bfloat16, 64, 64, true><<<n, kPackThreads, 0, s>>>(la, kp, vp);
  } else if (bf16) {
    if (D == 128) pack_layers_kernel<__nv_bfloat16, 128, 64, false><<<n, kPackThreads, 0, s>>>(la, kp, vp);
    else pack_layers_kernel<__nv_bfloat16, 64, 64, false><<<n, kPackThreads, 0, s>>>(la, kp, vp);
  } else if (P == 16) {
    if (D == 128) pack_layers_kernel<float, 128, 16, false><<<n, kPackThreads, 0, s>>>(la, kp, vp);
    else pack_layers_kernel<float, 64, 16, false><<<n, kPackThreads, 0, s>>>(la, kp, vp);
  } else {
    if (D == 128) pack_layers_kernel<float, 128, 64, false><<<n, kPackThreads, 0, s>>>(la, kp, vp);
    else pack_layers_kernel<float, 64, 64, false><<<n, kPackThreads, 0, s>>>(la, kp, vp);
  }
  return cudaGetLastError();
}

void launch_pack(const PackLaunch& L, cudaStream_t s) {
  if (L.n_pages == 0) return;
  if (L.fp8) {
    if (L.D == 128) launch_pack_fp8<128>(L, s);
    else launch_pack_fp8<64>(L, s);
  } else if (L.bf16) {
    if (L.D == 128) launch_pack_t<__nv_bfloat16, 128, 64>(L, s);
    else launch_pack_t<__nv_bfloat16, 64, 64>(L, s);
  } else if (L.P == 16) {
    if (L.D == 128) launch_pack_t<float, 128, 16>(L, s);
    else launch_pack_t<float, 64, 16>(L, s);
  } else {
    if (L.D == 128) launch_pack_t<float, 128, 64>(L, s);
    else launch_pack_t<float, 64, 64>(L, s);
  }
}

}  // namespace sp
