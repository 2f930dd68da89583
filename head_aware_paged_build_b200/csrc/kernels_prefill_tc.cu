// bf16 prefill on 5th-generation tensor cores (tcgen05, sm_100a).
//
// One CTA per (q-head, 128-row query tile).  It visits only the KV tiles of
// 128 tokens (two pages) that some row of the tile can see, in the head's
// stored order: the sink tiles and the recent-window tiles of a local head,
// the causal prefix of a global head ("SegPagedAttention runtime design", §4:
// each (query-head, kv-head) pair runs over its own true length, no mask over
// invisible KV).  Only tiles that cross a boundary (causal diagonal, window
// edge, sink page, a segment's partial last page) are masked per element.
//
// Warp roles (192 threads):
//   warp 0      producer: Q tile by TMA (128-byte swizzle), K and V pages by
//               1-D bulk copies (pool pages are stored in the tensor cores'
//               swizzled K-major operand layout, V transposed)
//   warp 1      TMEM owner and MMA issuer: S = Q K^T and O += P V as
//               tcgen05.mma kind::f16, fp32 accumulators in TMEM
//               (O: D columns, S: two buffers of 128 columns)
//   warps 2-5   softmax: one query row per thread, S read with tcgen05.ld,
//               online softmax in the log2 domain with a lazy rescale of O
//               (only when the row maximum grows by more than 2^8), P
//               written to shared memory as the bf16 A operand of P V;
//               then the epilogue (O / l, LSE).
// Every wait is bounded; a wait that runs out records a status code and the
// CTA drains its copies and MMAs, frees its TMEM and returns.
#include <cuda.h>

#include <mutex>

#include "device_common.cuh"
#include "kernels.h"
#include "tc_ptx.cuh"

namespace sp {
namespace {

constexpr int kTile = kPrefillTileTokensBf16;  // 128 query rows, 128 KV tokens
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleLog2 = 8.0f;  // rescale O only when the max grows by more than 2^8
constexpr float kLn2 = 0.6931471805599453f;

template <int D, int NS>
struct TcSmem {
  static constexpr int kQ = D / 64 * 16384;  // [D/64][128 rows][128 B]
  static constexpr int kK = D / 64 * 16384;  // [D/64][128 tokens][128 B]
  static constexpr int kV = 2 * D * 128;     // [2 pages][D rows][64 tokens * 2 B]
  static constexpr int kStage = kK + kV;
  static constexpr int kP = 2 * 16384;       // [2][128 rows][64 tokens * 2 B]
  static constexpr int kOffQ = 0;
  static constexpr int kOffStage = kOffQ + kQ;
  static constexpr int kOffP = kOffStage + NS * kStage;
  static constexpr int kOffBar = kOffP + kP;
  static constexpr int kBytes = kOffBar + 256 + 1024;  // barriers + 1 KB alignment slack
};

// Does every query row p in [p_first, p_last] see every slot of this page?
__device__ __forceinline__ bool page_fully_visible(const PageDesc& pg, bool exists, const HeadDesc& hd, int p_first,
                                                   int p_last) {
  if (!exists || pg.nvalid != 64) return false;
  const int a0 = pg.abs_start, a1 = pg.abs_start + 63;
  if (a1 > p_first) return false;
  if (hd.kind == 0) return true;
  return a1 < hd.sink || a0 > p_last - hd.window;
}

struct Bars {
  uint64_t q;
  uint64_t p_full;
  uint64_t o_done;
  uint64_t done;
  uint64_t s_full[2];
  uint64_t s_free[2];
};

template <int D, int NS>
__global__ void __launch_bounds__(kThreads, 1) prefill_tc_kernel(const __grid_constant__ CUtensorMap qmap,
                                                                  PrefillLaunch a) {
  using Sm = TcSmem<D, NS>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* q_s = smem + Sm::kOffQ;
  uint8_t* stage_s = smem + Sm::kOffStage;
  uint8_t* p_s = smem + Sm::kOffP;
  Bars* bars = reinterpret_cast<Bars*>(smem + Sm::kOffBar);
  uint64_t* kv_full = reinterpret_cast<uint64_t*>(bars + 1);
  uint64_t* kv_free = kv_full + NS;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(kv_free + NS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const PrefillItem it = a.items[blockIdx.x];
  const HeadDesc hd = a.heads[it.head];
  const int n1 = it.t1 - it.t0;
  const int n = n1 + (it.t3 - it.t2);

  if (threadIdx.x == 0) {
    mbar_init(&bars->q, 1);
    mbar_init(&bars->p_full, 128);
    mbar_init(&bars->o_done, 1);
    mbar_init(&bars->done, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars->s_full[b], 1);
      mbar_init(&bars->s_free[b], 128);
    }
    for (int s = 0; s < NS; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_free[s], 1);
    }
    *abort_flag = 0;
    fence_barrier_init();
    tc::prefetch_tensormap(&qmap);
  }
  if (warp == 1) {
    tc::tmem_alloc(tmem_slot, kTmemCols);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const uint32_t t_o = tmem;          // O: columns [0, D)
  const uint32_t t_s0 = tmem + 128;   // S buffers: [128, 256), [256, 384)

  auto fail = [&](int32_t code) {
    record_error(a.status, code);
    *abort_flag = 1;
  };

  if (warp == 0) {
    // ------------------------------ producer ------------------------------
    if (lane == 0) {
      const uint8_t* kpool = static_cast<const uint8_t*>(a.kpool);
      const uint8_t* vpool = static_cast<const uint8_t*>(a.vpool);
      mbar_arrive_expect_tx(&bars->q, Sm::kQ);
      for (int h = 0; h < D / 64; ++h) tc::tma_load_3d(q_s + h * 16384, &qmap, h * 64, it.qh, it.q_row, &bars->q);
      int issued = 0;
      for (int j = 0; j < n && !*abort_flag; ++j) {
        const int st = j % NS;
        if (j >= NS && !mbar_wait(&kv_free[st], ((j / NS) - 1) & 1)) {
          fail(kDevTimeoutEmpty);
          break;
        }
        const int t = j < n1 ? it.t0 + j : it.t2 + (j - n1);
        const int vp0 = 2 * t, vp1 = (2 * t + 1 < hd.n_vpages) ? 2 * t + 1 : 2 * t;
        const int64_t ph[2] = {a.pages[hd.vpage_begin + vp0].phys, a.pages[hd.vpage_begin + vp1].phys};
        uint8_t* k_s = stage_s + st * Sm::kStage;
        uint8_t* v_s = k_s + Sm::kK;
        mbar_arrive_expect_tx(&kv_full[st], Sm::kStage);
#pragma unroll
        for (int pj = 0; pj < 2; ++pj) {
#pragma unroll
          for (int h = 0; h < D / 64; ++h)
            bulk_g2s(k_s + h * 16384 + pj * 8192, kpool + ph[pj] * a.page_bytes + h * 8192, 8192, &kv_full[st]);
          bulk_g2s(v_s + pj * (D * 128), vpool + ph[pj] * a.page_bytes, D * 128, &kv_full[st]);
        }
        issued = j + 1;
      }
      // drain: never leave with bulk copies still writing this CTA's shared memory
      mbar_wait(&bars->q, 0);
      for (int j = (issued > NS ? issued - NS : 0); j < issued; ++j) mbar_wait(&kv_full[j % NS], (j / NS) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------ MMA issuer ------------------------------
    if (lane == 0) {
      constexpr uint32_t idesc_s = tc::idesc_bf16_f32(128, 128);
      constexpr uint32_t idesc_o = tc::idesc_bf16_f32(128, D);
      const uint32_t q_addr = smem_u32(q_s), p_addr = smem_u32(p_s), st_addr = smem_u32(stage_s);
      bool ok = mbar_wait(&bars->q, 0);
      if (!ok) fail(kDevTimeoutFull);
      for (int j = 0; ok && j <= n; ++j) {
        if (*abort_flag) break;
        if (j < n) {
          const int st = j % NS, b = j & 1;
          if (!mbar_wait(&kv_full[st], (j / NS) & 1)) { fail(kDevTimeoutFull); break; }
          if (j >= 2 && !mbar_wait(&bars->s_free[b], ((j >> 1) - 1) & 1)) { fail(kDevTimeoutSoftmax); break; }
          tc::fence_after_sync();
          const uint32_t k_addr = st_addr + st * Sm::kStage;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
            tc::mma_bf16_ss(t_s0 + b * 128, tc::smem_desc_sw128(q_addr + off), tc::smem_desc_sw128(k_addr + off),
                            idesc_s, kk > 0);
          }
          tc::commit(&bars->s_full[b]);
        }
        if (j >= 1) {
          const int jj = j - 1, st = jj % NS;
          if (!mbar_wait(&bars->p_full, jj & 1)) { fail(kDevTimeoutSoftmax); break; }
          tc::fence_after_sync();
          const uint32_t v_addr = st_addr + st * Sm::kStage + Sm::kK;
#pragma unroll
          for (int kk = 0; kk < kTile / 16; ++kk) {
            const uint32_t pa = p_addr + (kk >> 2) * 16384 + (kk & 3) * 32;
            const uint32_t va = v_addr + (kk >> 2) * (D * 128) + (kk & 3) * 32;
            tc::mma_bf16_ss(t_o, tc::smem_desc_sw128(pa), tc::smem_desc_sw128(va), idesc_o, (jj > 0 || kk > 0));
          }
          tc::commit(&bars->o_done);
          tc::commit(&kv_free[st]);
        }
      }
      // all MMAs issued by this thread complete before TMEM is released
      tc::commit(&bars->done);
      mbar_wait(&bars->done, 0);
    }
    __syncwarp();
  } else {
    // ------------------------------ softmax ------------------------------
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t lane_off = uint32_t(quarter * 32) << 16;
    const int p = it.p0 + r;
    const int p_last = it.p0 + it.n_rows - 1;
    const float sl2 = a.scale_log2;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < n; ++j) {
      const int b = j & 1;
      const int t = j < n1 ? it.t0 + j : it.t2 + (j - n1);
      const bool have1 = 2 * t + 1 < hd.n_vpages;
      const PageDesc pg0 = a.pages[hd.vpage_begin + 2 * t];
      const PageDesc pg1 = have1 ? a.pages[hd.vpage_begin + 2 * t + 1] : PageDesc{0, 0, 0, 0};
      const bool full = page_fully_visible(pg0, true, hd, it.p0, p_last) &&
                        page_fully_visible(pg1, have1, hd, it.p0, p_last);
      // tcgen05.ld / st are warp-collective (.sync.aligned): every branch that
      // guards one must be taken by the whole warp, so wait outcomes are voted.
      if (!__all_sync(0xffffffffu, mbar_wait(&bars->s_full[b], (j >> 1) & 1))) {
        fail(kDevTimeoutMma);
        ok = false;
        break;
      }
      tc::fence_after_sync();
      float s[kTile];
#pragma unroll
      for (int c = 0; c < kTile / 32; ++c)
        tc::tmem_ld32(t_s0 + b * 128 + lane_off + c * 32, *reinterpret_cast<float(*)[32]>(s + c * 32));
      tc::tmem_wait_ld();
      tc::fence_before_sync();
      mbar_arrive(&bars->s_free[b]);
      if (!full) {
#pragma unroll
        for (int c = 0; c < kTile; ++c) {
          const PageDesc& pg = c < 64 ? pg0 : pg1;
          const int slot = c & 63;
          const bool vis = slot < pg.nvalid && sees(hd.kind, hd.sink, hd.window, p, pg.abs_start + slot);
          if (!vis) s[c] = -INFINITY;
        }
      }
      float mt = s[0];
#pragma unroll
      for (int c = 1; c < kTile; ++c) mt = fmaxf(mt, s[c]);
      const float mts = mt * sl2;
      float alpha = 1.f;
      bool rescale = false;
      if (mts > m_run + kRescaleLog2) {
        alpha = fast_exp2(m_run - mts);
        rescale = m_run != -INFINITY;
        m_run = mts;
      }
      const float base = m_run == -INFINITY ? 0.f : m_run;
      uint32_t pk[kTile / 2];
      float sum = 0.f;
#pragma unroll
      for (int c = 0; c < kTile / 2; ++c) {
        const float e0 = fast_exp2(fmaf(s[2 * c], sl2, -base));
        const float e1 = fast_exp2(fmaf(s[2 * c + 1], sl2, -base));
        sum += e0 + e1;
        pk[c] = pack_bf16x2(e0, e1);
      }
      l_run = l_run * alpha + sum;
      // P V of the previous tile must be done before P and O are touched
      if (j > 0 && !__all_sync(0xffffffffu, mbar_wait(&bars->o_done, (j - 1) & 1))) {
        fail(kDevTimeoutMma);
        ok = false;
        break;
      }
      tc::fence_after_sync();
      // The rescale decision is per row; the TMEM round trip runs for the whole
      // warp whenever one of its rows needs it (factor 1 for the others).
      const bool need = rescale && j > 0;
      if (__any_sync(0xffffffffu, need)) {
        const float f = need ? alpha : 1.f;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          float o[32];
          tc::tmem_ld32(t_o + lane_off + c * 32, o);
          tc::tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] *= f;
          tc::tmem_st32(t_o + lane_off + c * 32, o);
        }
        tc::tmem_wait_st();
      }
      // P row r -> [2 atoms][128 rows][128 B], 16-byte chunk c at c ^ (r & 7)
#pragma unroll
      for (int cc = 0; cc < kTile / 8; ++cc) {
        const int atom = cc >> 3, c = cc & 7;
        uint8_t* dst = p_s + atom * 16384 + r * 128 + ((c ^ (r & 7)) << 4);
        *reinterpret_cast<uint4*>(dst) = make_uint4(pk[4 * cc], pk[4 * cc + 1], pk[4 * cc + 2], pk[4 * cc + 3]);
      }
      tc::fence_proxy_async_smem();
      tc::fence_before_sync();
      mbar_arrive(&bars->p_full);
    }
    // ------------------------------ epilogue ------------------------------
    bool go = ok && n > 0 && mbar_wait(&bars->o_done, (n - 1) & 1);
    go = __all_sync(0xffffffffu, go && !*abort_flag);
    if (go) {
      tc::fence_after_sync();
      const bool row_ok = r < it.n_rows;
      const float inv_l = 1.f / l_run;
      __nv_bfloat16* orow =
          static_cast<__nv_bfloat16*>(a.out) + (int64_t(it.q_row + r) * a.num_q_heads + it.qh) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        float o[32];
        tc::tmem_ld32(t_o + lane_off + c * 32, o);
        tc::tmem_wait_ld();
        if (row_ok) {
          uint32_t w[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) w[e] = pack_bf16x2(o[2 * e] * inv_l, o[2 * e + 1] * inv_l);
          uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
          for (int e = 0; e < 4; ++e) dst[e] = make_uint4(w[4 * e], w[4 * e + 1], w[4 * e + 2], w[4 * e + 3]);
        }
      }
      if (row_ok && a.lse) a.lse[int64_t(it.q_row + r) * a.num_q_heads + it.qh] = (m_run + log2f(l_run)) * kLn2;
    } else if (ok && n > 0) {
      fail(kDevTimeoutMma);
    }
  }

  tc::fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

template <int D, int NS>
cudaError_t launch_tc(const PrefillLaunch& a, cudaStream_t s) {
  using Sm = TcSmem<D, NS>;
  EncodeTiledFn enc = encode_fn();
  if (!enc) return cudaErrorNotSupported;
  CUtensorMap qmap;
  const cuuint64_t dims[3] = {cuuint64_t(D), cuuint64_t(a.num_q_heads), cuuint64_t(a.total_rows)};
  const cuuint64_t strides[2] = {cuuint64_t(D) * 2, cuuint64_t(a.num_q_heads) * D * 2};
  const cuuint32_t box[3] = {64, 1, kTile};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = enc(&qmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(a.q), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
  auto kern = prefill_tc_kernel<D, NS>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Sm::kBytes);
  if (e != cudaSuccess) return e;
  kern<<<a.n_items, kThreads, Sm::kBytes, s>>>(qmap, a);
  return cudaGetLastError();
}

constexpr int kStages = 2;

}  // namespace

cudaError_t launch_prefill_bf16(const PrefillLaunch& a, cudaStream_t s) {
  if (a.n_items == 0) return cudaSuccess;
  if (a.P != 64) return cudaErrorNotSupported;
  return a.D == 128 ? launch_tc<128, kStages>(a, s) : launch_tc<64, kStages>(a, s);
}

}  // namespace sp
