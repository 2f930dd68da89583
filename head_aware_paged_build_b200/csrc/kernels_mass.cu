// Attention mass per page-size block: the scoring pass behind a retrieval
// head's importance.  The pages leave the scoring rule open ("RedKnot head
// classification", four-kind table: a retrieval head fetches only the pages
// that matter); the reading taken is the head's own attention mass per page.
// For each sequence b and kv-head kv, the query of each q-head h of the GQA
// group at the last position L_b - 1 attends over the whole context [0, L_b):
//   mass[b][kv][i] = (1 / g) * sum_h sum_{j in block i} softmax_j(scale * q_h . k_j)
// with blocks of 64 positions (the bf16 page size).
//
// Pass 1 (block_mass_kernel): one warp per block, in two halves of 32
// positions.  The GQA group's g query rows are the 16 rows of
// mma.sync.m16n8k16 (bf16, fp32 accumulate) and each lane loads its tokens'
// keys straight from the dense cache, 16 bytes at a time: lane tq of a quad
// owns dimensions 32 j + 8 tq .. +7 of its token, and the query fragments use
// the same permutation of the 32 dimensions of each group, so the dot
// products are unchanged.  Per (q-head, block) it writes the block's score
// maximum m and sum 2^(s - m) (log2 units).  (Measured: halves instead of
// whole blocks 3.6 % faster; capping registers for more CTAs per SM slower.)
// Pass 2 (block_mass_combine_kernel): one CTA per (sequence, kv-head): per
// q-head M = max over blocks, Z = sum_blocks s_i 2^(m_i - M); mass_i =
// (1 / g) sum_h s_hi 2^(m_hi - M_h) / Z_h, one warp per q-head for M and Z.
// The pass over the keys has pushed most of the (m, s) pairs out of L2 by
// the time pass 2 reads them, so each lane issues all its loads of a row
// (up to 16 pairs) before it uses one: a single DRAM round trip per 512
// blocks instead of one per few blocks.  Pass 2 is a programmatic dependent
// launch: its CTAs are placed while the pass's last wave runs and wait for
// the pass's results on the device (griddepcontrol), which hides the launch
// gap.  (Measured on the 32K layer: 10.2 us of pass 2 down to 5.1 us.
// Folding pass 2 into the pass, the last CTA of each (sequence, kv-head)
// normalising, was 25 us slower: it changed the pass's register allocation.)
// Every sum runs in a fixed order, so results are bitwise reproducible.
#include <cuda_bf16.h>

#include <algorithm>
#include <cmath>
#include <mutex>
#include <string>

#include "device_common.cuh"
#include "kernels.h"

namespace sp {
namespace {

constexpr uint32_t kFull = 0xffffffffu;
constexpr int kMassThreads = 128;     // pass 1: 4 warps, one block each per step
constexpr int kCombineThreads = 256;  // pass 2

template <int D>
__global__ void __launch_bounds__(kMassThreads) block_mass_kernel(const __grid_constant__ BlockMassLaunch a) {
  // pass 2 may be placed now: it waits on the device for this grid's results
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int bk = blockIdx.y, b = bk / a.Hkv, kv = bk % a.Hkv;
  const int L = a.L[b], nb = (L + kMassBlock - 1) / kMassBlock;
  const int blk0 = blockIdx.x * a.blocks_per_cta, blk1 = min(nb, blk0 + a.blocks_per_cta);
  if (blk0 >= blk1) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, grp = lane >> 2, tq = lane & 3;
  const int G = a.G, r0 = grp, r1 = grp + 8;

  // query fragments: k-steps 2j, 2j+1 cover dimensions 32 j .. 32 j + 31, lane tq
  // holds dimensions 32 j + 8 tq .. +7 (pairs {0,1},{2,3} -> k-step 2j, {4,5},{6,7} -> 2j+1)
  uint32_t qa[D / 16][4];
  const __nv_bfloat16* qrow = static_cast<const __nv_bfloat16*>(a.q) + (int64_t(b) * a.Hq + kv * G) * D;
#pragma unroll
  for (int j = 0; j < D / 32; ++j) {
    const int c0 = 32 * j + 8 * tq;
    const uint4 x0 = r0 < G ? *reinterpret_cast<const uint4*>(qrow + r0 * D + c0) : make_uint4(0, 0, 0, 0);
    const uint4 x1 = r1 < G ? *reinterpret_cast<const uint4*>(qrow + r1 * D + c0) : make_uint4(0, 0, 0, 0);
    qa[2 * j][0] = x0.x, qa[2 * j][2] = x0.y, qa[2 * j + 1][0] = x0.z, qa[2 * j + 1][2] = x0.w;
    qa[2 * j][1] = x1.x, qa[2 * j][3] = x1.y, qa[2 * j + 1][1] = x1.z, qa[2 * j + 1][3] = x1.w;
  }
  const __nv_bfloat16* kb =
      static_cast<const __nv_bfloat16*>(a.k) + int64_t(b) * a.stride_seq + int64_t(kv) * a.stride_head;
  const float sl2 = a.scale_log2;
  const int64_t row0 = (int64_t(b) * a.Hq + kv * G + r0) * a.nb_max;
  const int64_t row1 = (int64_t(b) * a.Hq + kv * G + r1) * a.nb_max;

  for (int blk = blk0 + warp; blk < blk1; blk += kMassThreads / 32) {
    const int t0 = blk * kMassBlock;
    // the block in two halves of 32 tokens (16 score registers at a time); each half's
    // maximum and sum, then the block's: m = max(m_a, m_b), s = s_a 2^(m_a - m) + s_b 2^(m_b - m)
    float bm0 = -INFINITY, bm1 = -INFINITY, bs0 = 0.f, bs1 = 0.f;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      float sc[4][4];
#pragma unroll
      for (int nt = 0; nt < 4; ++nt) {
        sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
        const int tok = t0 + 32 * half + nt * 8 + grp;
        const __nv_bfloat16* kr = kb + int64_t(tok) * a.stride_tok + 8 * tq;
#pragma unroll
        for (int j = 0; j < D / 32; ++j) {
          const uint4 u = tok < L ? __ldg(reinterpret_cast<const uint4*>(kr + 32 * j)) : make_uint4(0, 0, 0, 0);
          mma_bf16_16816(sc[nt], qa[2 * j], u.x, u.y);
          mma_bf16_16816(sc[nt], qa[2 * j + 1], u.z, u.w);
        }
      }
      float m0 = -INFINITY, m1 = -INFINITY;
#pragma unroll
      for (int nt = 0; nt < 4; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int tok = t0 + 32 * half + nt * 8 + 2 * tq + (e & 1);
          const float x = tok < L ? sc[nt][e] * sl2 : -INFINITY;
          sc[nt][e] = x;
          if (e < 2) m0 = fmaxf(m0, x); else m1 = fmaxf(m1, x);
        }
      m0 = fmaxf(m0, __shfl_xor_sync(kFull, m0, 1));
      m0 = fmaxf(m0, __shfl_xor_sync(kFull, m0, 2));
      m1 = fmaxf(m1, __shfl_xor_sync(kFull, m1, 1));
      m1 = fmaxf(m1, __shfl_xor_sync(kFull, m1, 2));
      if (m0 == -INFINITY) continue;  // the second half lies wholly past the context (both rows alike)
      float s0 = 0.f, s1 = 0.f;
#pragma unroll
      for (int nt = 0; nt < 4; ++nt) {
        s0 += fast_exp2(sc[nt][0] - m0) + fast_exp2(sc[nt][1] - m0);
        s1 += fast_exp2(sc[nt][2] - m1) + fast_exp2(sc[nt][3] - m1);
      }
      s0 += __shfl_xor_sync(kFull, s0, 1);
      s0 += __shfl_xor_sync(kFull, s0, 2);
      s1 += __shfl_xor_sync(kFull, s1, 1);
      s1 += __shfl_xor_sync(kFull, s1, 2);
      if (half == 0) {
        bm0 = m0, bm1 = m1, bs0 = s0, bs1 = s1;
      } else {
        const float n0 = fmaxf(bm0, m0), n1 = fmaxf(bm1, m1);
        bs0 = bs0 * fast_exp2(bm0 - n0) + s0 * fast_exp2(m0 - n0);
        bs1 = bs1 * fast_exp2(bm1 - n1) + s1 * fast_exp2(m1 - n1);
        bm0 = n0, bm1 = n1;
      }
    }
    if (tq == 0) {
      if (r0 < G) a.ws_m[row0 + blk] = bm0, a.ws_s[row0 + blk] = bs0;
      if (r1 < G) a.ws_m[row1 + blk] = bm1, a.ws_s[row1 + blk] = bs1;
    }
  }
}

__global__ void __launch_bounds__(kCombineThreads)
    block_mass_combine_kernel(const __grid_constant__ BlockMassLaunch a) {
  // one warp per q-head of the group (two for G > 8): its maximum and sum over the blocks,
  // lane-strided with a fixed butterfly, no block-wide barrier per head
  constexpr int C = 16;  // (m, s) pairs a lane loads before it uses one
  __shared__ float s_max[16], s_inv[16];
  // wait until the pass over the keys has finished and its results are visible
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int bk = blockIdx.x, b = bk / a.Hkv, kv = bk % a.Hkv;
  const int L = a.L[b], nb = (L + kMassBlock - 1) / kMassBlock;
  const int G = a.G, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int h = warp; h < G; h += kCombineThreads / 32) {
    const int64_t row = (int64_t(b) * a.Hq + kv * G + h) * a.nb_max;
    float mv[C], sv[C];
    float m = -INFINITY;
    for (int base = 0; base < nb; base += 32 * C) {
#pragma unroll
      for (int k = 0; k < C; ++k) {
        const int i = base + lane + 32 * k;
        mv[k] = i < nb ? __ldcg(a.ws_m + row + i) : -INFINITY;
        sv[k] = i < nb ? __ldcg(a.ws_s + row + i) : 0.f;
      }
#pragma unroll
      for (int k = 0; k < C; ++k) m = fmaxf(m, mv[k]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(kFull, m, o));
    // Z in block order per lane; a row of at most 32 C blocks is still in registers
    float z = 0.f;
    for (int base = 0; base < nb; base += 32 * C) {
      if (nb > 32 * C) {
#pragma unroll
        for (int k = 0; k < C; ++k) {
          const int i = base + lane + 32 * k;
          mv[k] = i < nb ? __ldcg(a.ws_m + row + i) : -INFINITY;
          sv[k] = i < nb ? __ldcg(a.ws_s + row + i) : 0.f;
        }
      }
#pragma unroll
      for (int k = 0; k < C; ++k)
        if (base + lane + 32 * k < nb) z += sv[k] * exp2f(mv[k] - m);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(kFull, z, o);
    if (lane == 0) s_max[h] = m, s_inv[h] = 1.f / z;
  }
  __syncthreads();
  float* out = a.mass + int64_t(bk) * a.mass_stride;
  const float inv_g = 1.f / float(G);
  for (int i = threadIdx.x; i < nb; i += kCombineThreads) {
    float acc = 0.f;
    for (int h = 0; h < G; ++h) {
      const int64_t idx = (int64_t(b) * a.Hq + kv * G + h) * a.nb_max + i;
      acc += __ldcg(a.ws_s + idx) * exp2f(__ldcg(a.ws_m + idx) - s_max[h]) * s_inv[h];
    }
    out[i] = acc * inv_g;
  }
}

}  // namespace

cudaError_t launch_block_mass(const BlockMassLaunch& a, cudaStream_t s) {
  const dim3 grid((a.nb_max + a.blocks_per_cta - 1) / a.blocks_per_cta, a.B * a.Hkv);
  if (a.D == 128)
    block_mass_kernel<128><<<grid, kMassThreads, 0, s>>>(a);
  else
    block_mass_kernel<64><<<grid, kMassThreads, 0, s>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // pass 2 as a programmatic dependent of the pass (it waits with griddepcontrol.wait)
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.B * a.Hkv);
  cfg.blockDim = dim3(kCombineThreads);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, block_mass_combine_kernel, a);
}

}  // namespace sp

// ---------------------------------------------------------------------------
// C ABI
// ---------------------------------------------------------------------------
namespace sp {
namespace {

sp_status mass_shape(const sp_problem* p, int32_t& G, int32_t& nb_max) {
  if (!p) return fail(SP_ERR_INVALID_ARG, "problem is NULL");
  if (p->batch < 1 || p->num_q_heads < 1 || p->num_kv_heads < 1)
    return fail(SP_ERR_INVALID_ARG, "batch and head counts must be >= 1");
  if (p->batch > kMassMaxBatch) return fail(SP_ERR_UNSUPPORTED, "segpaged_block_mass: at most 2048 sequences");
  if (p->dtype != SP_BF16) return fail(SP_ERR_UNSUPPORTED, "segpaged_block_mass: bf16 keys and queries only");
  if (p->head_dim != 64 && p->head_dim != 128) return fail(SP_ERR_UNSUPPORTED, "head_dim must be 64 or 128");
  if (p->page_size != kMassBlock) return fail(SP_ERR_UNSUPPORTED, "segpaged_block_mass: page_size must be 64");
  if (p->num_q_heads % p->num_kv_heads != 0 || p->num_q_heads / p->num_kv_heads > 16)
    return fail(SP_ERR_UNSUPPORTED, "num_q_heads must be a multiple of num_kv_heads, at most 16 times it");
  if (int64_t(p->batch) * p->num_kv_heads > 65535)  // the pass's grid.y
    return fail(SP_ERR_UNSUPPORTED, "segpaged_block_mass: batch * num_kv_heads above 65535");
  if (!p->ctx_len) return fail(SP_ERR_INVALID_ARG, "ctx_len is NULL");
  int64_t lmax = 0;
  for (int b = 0; b < p->batch; ++b) {
    if (p->ctx_len[b] < 1) return fail(SP_ERR_INVALID_ARG, "ctx_len must be >= 1");
    lmax = std::max<int64_t>(lmax, p->ctx_len[b]);
  }
  G = p->num_q_heads / p->num_kv_heads;
  nb_max = int32_t((lmax + kMassBlock - 1) / kMassBlock);
  return SP_OK;
}

int64_t mass_workspace_bytes(const sp_problem* p, int32_t nb_max) {
  const int64_t raw = 2 * int64_t(p->batch) * p->num_q_heads * nb_max * int64_t(sizeof(float));
  return (raw + 255) / 256 * 256;
}

}  // namespace
}  // namespace sp

extern "C" sp_status segpaged_block_mass_workspace(const sp_problem* problem, size_t* bytes) {
  using namespace sp;
  int32_t G, nb_max;
  const sp_status st = mass_shape(problem, G, nb_max);
  if (st != SP_OK) return st;
  if (!bytes) return fail(SP_ERR_INVALID_ARG, "bytes is NULL");
  *bytes = size_t(mass_workspace_bytes(problem, nb_max));
  return SP_OK;
}

extern "C" sp_status segpaged_block_mass(const sp_problem* problem, const void* k_dense, int64_t stride_seq,
                                         int64_t stride_head, int64_t stride_tok, const void* q, float softmax_scale,
                                         float* mass, int64_t mass_stride, void* workspace, size_t workspace_bytes,
                                         void* stream) {
  using namespace sp;
  int32_t G, nb_max;
  sp_status st = mass_shape(problem, G, nb_max);
  if (st != SP_OK) return st;
  auto al = [](const void* ptr, uintptr_t n) { return (reinterpret_cast<uintptr_t>(ptr) % n) == 0; };
  if (!k_dense || !q || !mass || !workspace)
    return fail(SP_ERR_INVALID_ARG, "k_dense, q, mass and workspace must be non-NULL");
  if (!al(k_dense, 16) || !al(q, 16) || !al(mass, 4) || !al(workspace, 256))
    return fail(SP_ERR_INVALID_ARG, "k_dense and q must be 16-byte aligned, mass 4-byte, workspace 256-byte");
  if (stride_seq < 0 || stride_head < 0 || stride_tok < 0 || stride_seq % 8 || stride_head % 8 || stride_tok % 8)
    return fail(SP_ERR_INVALID_ARG, "strides must be >= 0 and multiples of 8 elements (16-byte rows)");
  if (mass_stride < nb_max) return fail(SP_ERR_INVALID_ARG, "mass_stride below ceil(max ctx_len / page_size)");
  if (int64_t(workspace_bytes) < mass_workspace_bytes(problem, nb_max))
    return fail(SP_ERR_WORKSPACE, "workspace smaller than segpaged_block_mass_workspace");
  if (!std::isfinite(softmax_scale)) return fail(SP_ERR_INVALID_ARG, "softmax_scale must be finite");
  const float scale = softmax_scale > 0.f ? softmax_scale : 1.0f / std::sqrt(float(problem->head_dim));
  static BlockMassLaunch a;  // 8 KB of lengths: kept off the caller's stack
  static std::mutex mu;      // the launch copies it; one call fills it at a time
  std::lock_guard<std::mutex> lock(mu);
  a = BlockMassLaunch{};
  a.k = k_dense, a.q = q;
  a.stride_seq = stride_seq, a.stride_head = stride_head, a.stride_tok = stride_tok;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.B = problem->batch, a.Hq = problem->num_q_heads, a.Hkv = problem->num_kv_heads, a.G = G;
  a.D = problem->head_dim;
  a.nb_max = nb_max;
  a.blocks_per_cta = 16;
  float* ws = static_cast<float*>(workspace);
  a.ws_m = ws;
  a.ws_s = ws + int64_t(a.B) * a.Hq * nb_max;
  a.mass = mass, a.mass_stride = mass_stride;
  for (int b = 0; b < a.B; ++b) a.L[b] = problem->ctx_len[b];
  const cudaError_t e = launch_block_mass(a, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SP_OK
                          : fail(SP_ERR_CUDA, std::string("segpaged_block_mass launch: ") + cudaGetErrorString(e));
}
