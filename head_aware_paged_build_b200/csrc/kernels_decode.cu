// Decode: split-KV attention over each head's own page list, then a combine
// pass for heads split across CTAs ("SegPagedAttention runtime design", §4:
// each head is evaluated at its true KV length, straight from its pages).
//
// bf16: one CTA = 4 consumer warps + 1 producer warp.  The producer streams
// the CTA's pages (a balanced range of the concatenated page lists) into a
// ring of shared-memory stages with 1-D bulk copies (one per K page and one
// per V page: pages are stored in the swizzled layout the consumers read).
// Each consumer warp takes 16 of a page's 64 tokens: S = Q K^T and O += P V
// run on mma.sync m16n8k16 with the GQA group's q-heads as the 16 rows, and
// the online softmax runs on the accumulator fragments with quad shuffles.
// At the end of a head's range the 4 warps' states merge through shared
// memory in a fixed order, so results are bitwise reproducible.  A head split
// across CTAs is finished by whichever of its CTAs publishes its partial last
// (an arrival counter in the workspace): it merges the partials in slot order.
//
// E4M3 pages: the same kernel with 1-byte pages.  Each lane loads the codes
// of its mma.sync B fragments straight from the staged page (one 64-bit load
// per K fragment pair, one 32-bit load per V fragment: the page layout puts
// them side by side) and widens them exactly to f16; Q and P enter the
// tensor cores as f16, so the MMAs run kind f16 with f32 accumulation.  For
// K the head dimension is visited in a permuted order (Q loaded to match),
// which leaves the dot products unchanged.  k_scale is folded into the
// softmax scale and v_scale into the output normalisation.
//
// fp32: a plain SIMT kernel over the same work list (FP32 FMA only), with a
// separate combine pass for split heads.
#include <cmath>

#include "append_common.cuh"
#include "device_common.cuh"
#include "kernels.h"

namespace sp {
namespace {

constexpr int kConsumerWarps = 4;
constexpr int kDecodeThreads = (kConsumerWarps + 1) * 32;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kLazyLog2 = 8.f;  // decode softmax: rescale O only when the max grows by more than 2^8

template <int D, int NST, bool FP8>
struct DecodeSmem {
  static constexpr int kPageBytes = 64 * D * (FP8 ? 1 : 2);
  static constexpr int kMergePitch = D + 8;  // floats per merge row (breaks bank aliasing)
  static constexpr int kStageOff = 0;
  static constexpr int kMergeOff = NST * 2 * kPageBytes;
  static constexpr int kMlOff = kMergeOff + kConsumerWarps * kMaxGroup * kMergePitch * 4;
  static constexpr int kBarOff = kMlOff + kConsumerWarps * kMaxGroup * 2 * 4;
  static constexpr int kDescOff = kBarOff + 2 * NST * 8;  // PageDesc of each stage (16-byte aligned)
  static constexpr int kPatchOff = kDescOff + NST * 16;  // fused step: slot of the stage's new token, or -1
  static constexpr int kBytes = kPatchOff + ((NST * 4 + 15) / 16) * 16;
};

// Final merge of a split head, run by its last CTA over the n_slots partials
// (m, l, acc) at p0 (standard split-KV: O = sum_i 2^(m_i - M) acc_i / L with
// M = max_i m_i, L = sum_i 2^(m_i - M) l_i).  The consumer warps run it.
//   1. one warp per row: (M, L) in one pass over the slots' (m, l) pairs,
//      merged online per lane and then across lanes (a fixed butterfly, so
//      every lane ends with the same bits);
//   2. per 32-slot chunk, the slot weights 2^(m_i - M) go to shared memory
//      (the first chunk's straight from step 1), and each thread adds NE
//      (row, 4-column) entries over the chunk's slots, BATCH slots' loads in
//      flight at a time, slots in increasing order.
// All summation orders are fixed: results are bitwise reproducible.
template <int D, int NE, int BATCH, bool FP8>
__device__ __forceinline__ void merge_split_head(const DecodeLaunch& a, const HeadDesc& hd, int qh0, int G, int ns,
                                                 const float* p0, float* part, float* wts, float* rowml, int warp,
                                                 int lane) {
  constexpr int kT = kConsumerWarps * 32;
  constexpr int kChunk = 32;
  const int64_t stride = partial_slot_floats(G, D);
  float* row_m = rowml;              // [G] merged max (log2 units)
  float* row_l = rowml + kMaxGroup;  // [G] merged sum
  for (int row = warp; row < G; row += kConsumerWarps) {
    float m = -INFINITY, l = 0.f, m_first = -INFINITY;
    for (int i = lane; i < ns; i += 32) {
      const float2 ml = __ldcg(reinterpret_cast<const float2*>(p0 + i * stride + G * D + row * 2));
      if (i == lane) m_first = ml.x;
      const float mn = fmaxf(m, ml.x), b = mn == -INFINITY ? 0.f : mn;
      l = l * fast_exp2(m - b) + ml.y * fast_exp2(ml.x - b);
      m = mn;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float mo = __shfl_xor_sync(0xffffffffu, m, o), lo = __shfl_xor_sync(0xffffffffu, l, o);
      const float mn = fmaxf(m, mo), b = mn == -INFINITY ? 0.f : mn;
      l = l * fast_exp2(m - b) + lo * fast_exp2(mo - b);
      m = mn;
    }
    const float base = m == -INFINITY ? 0.f : m;
    wts[row * kChunk + lane] = lane < ns ? fast_exp2(m_first - base) : 0.f;
    if (lane == 0) row_m[row] = m, row_l[row] = l;
  }
  float4 acc[NE];
#pragma unroll
  for (int t = 0; t < NE; ++t) acc[t] = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int c0 = 0; c0 < ns; c0 += kChunk) {
    if (c0 > 0) {
      asm volatile("bar.sync 1, %0;" ::"n"(kT) : "memory");  // the previous chunk's weights are consumed
      for (int e = threadIdx.x; e < G * kChunk; e += kT) {
        const int row = e / kChunk, i = c0 + e % kChunk;
        const float M = row_m[row], base = M == -INFINITY ? 0.f : M;
        wts[e] = i < ns ? fast_exp2(__ldcg(p0 + i * stride + G * D + row * 2) - base) : 0.f;
      }
    }
    asm volatile("bar.sync 1, %0;" ::"n"(kT) : "memory");
    const int c1 = min(ns, c0 + kChunk);
    for (int i = c0; i < c1; i += BATCH) {
      float4 v[NE][BATCH];
#pragma unroll
      for (int t = 0; t < NE; ++t) {
        const int e4 = threadIdx.x + t * kT, row = e4 / (D / 4), col = (e4 % (D / 4)) * 4;
#pragma unroll
        for (int u = 0; u < BATCH; ++u)
          v[t][u] = e4 < G * D / 4 && i + u < c1
                        ? __ldcg(reinterpret_cast<const float4*>(p0 + (i + u) * stride + row * D + col))
                        : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int t = 0; t < NE; ++t) {
        const int e4 = threadIdx.x + t * kT, row = e4 / (D / 4);
#pragma unroll
        for (int u = 0; u < BATCH; ++u) {
          if (e4 < G * D / 4 && i + u < c1) {
            const float f = wts[row * kChunk + (i + u - c0)];
            acc[t].x += f * v[t][u].x, acc[t].y += f * v[t][u].y;
            acc[t].z += f * v[t][u].z, acc[t].w += f * v[t][u].w;
          }
        }
      }
    }
  }
  if (part) {  // a merge group: the merged partial (acc, M, L) in the same slot layout
#pragma unroll
    for (int t = 0; t < NE; ++t) {
      const int e4 = threadIdx.x + t * kT, row = e4 / (D / 4), col = (e4 % (D / 4)) * 4;
      if (e4 < G * D / 4) *reinterpret_cast<float4*>(part + row * D + col) = acc[t];
    }
    if (threadIdx.x < G)
      part[G * D + threadIdx.x * 2] = row_m[threadIdx.x], part[G * D + threadIdx.x * 2 + 1] = row_l[threadIdx.x];
    return;
  }
#pragma unroll
  for (int t = 0; t < NE; ++t) {
    const int e4 = threadIdx.x + t * kT, row = e4 / (D / 4), col = (e4 % (D / 4)) * 4;
    if (e4 < G * D / 4) {
      const float inv = (FP8 ? a.v_scale : 1.f) / row_l[row];
      __nv_bfloat16* o =
          static_cast<__nv_bfloat16*>(a.out) + (int64_t(hd.q_row0) * a.num_q_heads + qh0 + row) * D + col;
      reinterpret_cast<uint2*>(o)[0] = make_uint2(pack_bf16x2(acc[t].x * inv, acc[t].y * inv),
                                                  pack_bf16x2(acc[t].z * inv, acc[t].w * inv));
    }
  }
  if (threadIdx.x < G && a.lse)
    a.lse[int64_t(hd.q_row0) * a.num_q_heads + qh0 + threadIdx.x] =
        (row_m[threadIdx.x] + log2f(row_l[threadIdx.x])) * kLn2;
}

// Fused decode step: the new token of head `hd` has been written by the CTA
// that owns its target page; the CTA finishing the head (its single item, or
// the final merge of a split head) advances the context, exactly as the
// standalone append does after writing (or reports a ring without room).
template <int P>
__device__ __forceinline__ void finish_append(const DecodeLaunch& a, int head) {
  // re-read from the table (not kept in registers through the page loop); no
  // thread writes this head's descriptor before this point of the launch.
  // Inlined: an out-of-line call here cost ~9 us per launch on the 32K layer.
  const HeadDesc hd = a.heads[head];
  int vp, slot;
  append_target<P>(hd, vp, slot);
  if (vp >= hd.n_vpages) {
    record_error(a.status, kDevAppendFull);
    return;
  }
  const int64_t phys = a.pages[hd.vpage_begin + vp].phys;
  if (phys < 0 || phys >= a.pool_pages) return;  // reported where the page was met
  HeadDesc* w = const_cast<HeadDesc*>(a.heads) + head;
  w->ctx_len = hd.ctx_len + 1;
  w->q_start = hd.ctx_len;
}

// Fused decode step, producer side.  Lane i holds the append of item
// `first + i` of this CTA: the head's target page (index in the table's page
// list, or -1 when the head has no room left) and slot, and the page and slot
// of the token that leaves a LOCAL head's window (-1: none).  The producer
// meets each page of its items once, in order; at the target or eviction page
// it applies the append's record changes to its copy of the record before it
// publishes it, writes the record back, and marks the stage so that the warp
// whose tokens hold the new slot writes the new token into the staged page
// (and the pool page) itself: the page's bulk copy never waits for the append.
struct AppendInfo {
  int vend = 0;  // item's page range end
  int tg = -1, slot = 0, len = 0;
  int eg = -1, eslot = 0, epos = 0;
};

__device__ __forceinline__ AppendInfo append_info(const DecodeLaunch& a, int it, int ie) {
  constexpr int P = 64;
  AppendInfo r;
  if (it >= ie) return r;
  const DecodeItem item = a.items[it];
  const HeadDesc hd = a.heads[item.head];
  r.vend = item.vp_end;
  int vp, slot;
  append_target<P>(hd, vp, slot);
  if (vp >= hd.n_vpages) return r;  // no room: nothing changes (the head's finisher reports it)
  r.tg = hd.vpage_begin + vp, r.slot = slot, r.len = hd.ctx_len;
  int evp, eslot, epos;
  append_eviction<P>(hd, evp, eslot, epos);
  if (evp >= 0) r.eg = hd.vpage_begin + evp, r.eslot = eslot, r.epos = epos;
  return r;
}

template <int D, int NST, bool FP8, bool APPEND>
__device__ __forceinline__ void decode_mma_body(const DecodeLaunch& a) {
  using S = DecodeSmem<D, NST, FP8>;
  constexpr int P = 64;
  constexpr int PB = S::kPageBytes;
  constexpr int KSTEPS = D / 16;
  constexpr int NT = D / 8;  // n-tiles of the output
  extern __shared__ __align__(1024) uint8_t smem[];
  __shared__ int s_last;
  uint8_t* stage = smem + S::kStageOff;
  float* mbuf = reinterpret_cast<float*>(smem + S::kMergeOff);
  float* mlbuf = reinterpret_cast<float*>(smem + S::kMlOff);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S::kBarOff);
  uint64_t* empty = full + NST;
  PageDesc* sdesc = reinterpret_cast<PageDesc*>(smem + S::kDescOff);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ib = a.cta_begin[blockIdx.x], ie = a.cta_begin[blockIdx.x + 1];
  if (ib >= ie) return;
  const int gb = a.items[ib].vp_begin, ge = a.items[ie - 1].vp_end;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kConsumerWarps);
    }
    fence_barrier_init();
  }
  __syncthreads();

  const uint8_t* kpool = static_cast<const uint8_t*>(a.kpool);
  const uint8_t* vpool = static_cast<const uint8_t*>(a.vpool);

  if (warp == kConsumerWarps) {
    // ---------------- producer ----------------
    // The warp's lanes fetch the next 32 page descriptors together, so no global
    // load sits between two stage refills; lane 0 walks them: wait for the stage,
    // publish the descriptor in shared memory (the consumers read it there after
    // the stage's full barrier), start the copies.
    int k = 0;
    bool ok = true;
    int32_t* spatch = reinterpret_cast<int32_t*>(smem + S::kPatchOff);
    // page records this launch may change (fused append) are read through L2
    auto records = [&](int base) {
      const int4* r = reinterpret_cast<const int4*>(a.pages + base + lane);
      return base + lane < ge ? (APPEND ? __ldcg(r) : __ldg(r)) : make_int4(0, 0, 0, 0);
    };
    int4 mine = records(gb);  // issued before the append bookkeeping's loads, so their latencies overlap
    AppendInfo ai;
    int ai_first = ib, cur = ib;  // lane i holds item ai_first + i; cur: the item of the current page
    if constexpr (APPEND) ai = append_info(a, ib + lane, ie);
    for (int base = gb; base < ge && ok; base += 32) {
      if (base != gb) mine = records(base);
      const int n = min(32, ge - base);
      for (int i = 0; i < n; ++i, ++k) {
        PageDesc pgd;
        pgd.phys = __shfl_sync(0xffffffffu, mine.x, i);
        pgd.abs_start = __shfl_sync(0xffffffffu, mine.y, i);
        pgd.span = __shfl_sync(0xffffffffu, mine.z, i);
        pgd.head = __shfl_sync(0xffffffffu, mine.w, i);
        const int s = k % NST;
        int patch = -1;
        if constexpr (APPEND) {
          const int g = base + i;
          while (g >= __shfl_sync(0xffffffffu, ai.vend, cur - ai_first)) {
            if (++cur - ai_first == 32) ai_first = cur, ai = append_info(a, cur + lane, ie);
          }
          const int c = cur - ai_first;
          const int tg = __shfl_sync(0xffffffffu, ai.tg, c), eg = __shfl_sync(0xffffffffu, ai.eg, c);
          if (g == tg || g == eg) {
            PageDesc* rec = const_cast<PageDesc*>(a.pages) + g;
            if (g == tg) {
              if (pgd.phys == kNoPage) {  // a GLOBAL head's reserved record: take a page from the spare pool
                int32_t taken = 0;
                if (lane == 0) {
                  taken = append_take_page(rec, a.free_pool, a.status);
                  __threadfence();  // the record's page before the head's finisher reads it
                }
                pgd.phys = __shfl_sync(0xffffffffu, taken, 0);
              }
              if (pgd.phys >= 0 && pgd.phys < a.pool_pages) {  // else: pool empty (reported) or a corrupted table
                patch = __shfl_sync(0xffffffffu, ai.slot, c);
                append_update_target(&pgd, __shfl_sync(0xffffffffu, ai.len, c), patch);
              }
            }
            if (g == eg)
              append_update_eviction(&pgd, __shfl_sync(0xffffffffu, ai.epos, c),
                                     __shfl_sync(0xffffffffu, ai.eslot, c));
            if (lane == 0) *rec = pgd;
          }
        }
        int good = 1;
        if (lane == 0) {
          if (k >= NST && !mbar_wait(&empty[s], ((k / NST) & 1) ^ 1)) {
            record_error(a.status, kDevTimeoutEmpty);
            good = 0;
          } else {
            if (slot_hi(pgd) > slot_lo(pgd) && (pgd.phys < 0 || pgd.phys >= a.pool_pages)) {
              record_error(a.status, kDevBadPage);  // corrupted table: report, read nothing
              pgd.span = 0;
            }
            sdesc[s] = pgd;
            if constexpr (APPEND) spatch[s] = patch;
            uint8_t* kd = stage + s * 2 * PB;
            if (slot_hi(pgd) > slot_lo(pgd)) {
              mbar_arrive_expect_tx(&full[s], 2 * PB);
              bulk_g2s(kd, kpool + int64_t(pgd.phys) * a.page_bytes, PB, &full[s]);
              bulk_g2s(kd + PB, vpool + int64_t(pgd.phys) * a.page_bytes, PB, &full[s]);
            } else {
              mbar_arrive(&full[s]);  // empty page (ring or reserved): nothing to copy
            }
          }
        }
        if (!__shfl_sync(0xffffffffu, good, 0)) {
          ok = false;
          break;
        }
      }
    }
    // Do not leave while copies into this CTA's shared memory are in flight.
    if (lane == 0)
      for (int j = (k > NST ? k - NST : 0); j < k; ++j)
        if (!mbar_wait(&full[j % NST], (j / NST) & 1)) break;
    return;
  }

  // ---------------- consumers ----------------
  const int grp = lane >> 2, tq = lane & 3;  // fragment row group, thread in quad
  const int r0 = grp, r1 = grp + 8;
  const int G = a.group;
  const __nv_bfloat16* qg = static_cast<const __nv_bfloat16*>(a.q);
  const float scale_log2 = a.scale_log2;
  bool ok = true;
  int k = 0;
  for (int it = ib; it < ie; ++it) {
    const DecodeItem item = a.items[it];
    const HeadDesc hd = a.heads[item.head];
    const int qh0 = hd.kv * G;
    const __nv_bfloat16* qrow = qg + (int64_t(hd.q_row0) * a.num_q_heads + qh0) * D;
    uint32_t qa[KSTEPS][4];
    if constexpr (FP8) {
      // k-steps 2j, 2j+1 cover dims 32j .. 32j+31; lane tq owns dims 32j+8tq .. +7
      // (pairs {0,1},{2,3} -> k-step 2j, {4,5},{6,7} -> k-step 2j+1), matching the K loads.
#pragma unroll
      for (int j = 0; j < D / 32; ++j) {
        const int c0 = j * 32 + tq * 8;
        const uint4 x0 = r0 < G ? *reinterpret_cast<const uint4*>(qrow + r0 * D + c0) : make_uint4(0, 0, 0, 0);
        const uint4 x1 = r1 < G ? *reinterpret_cast<const uint4*>(qrow + r1 * D + c0) : make_uint4(0, 0, 0, 0);
        qa[2 * j][0] = bf16x2_to_f16x2(x0.x), qa[2 * j][2] = bf16x2_to_f16x2(x0.y);
        qa[2 * j + 1][0] = bf16x2_to_f16x2(x0.z), qa[2 * j + 1][2] = bf16x2_to_f16x2(x0.w);
        qa[2 * j][1] = bf16x2_to_f16x2(x1.x), qa[2 * j][3] = bf16x2_to_f16x2(x1.y);
        qa[2 * j + 1][1] = bf16x2_to_f16x2(x1.z), qa[2 * j + 1][3] = bf16x2_to_f16x2(x1.w);
      }
    } else {
#pragma unroll
      for (int kk = 0; kk < KSTEPS; ++kk) {
        const int c0 = kk * 16 + tq * 2;
        qa[kk][0] = r0 < G ? *reinterpret_cast<const uint32_t*>(qrow + r0 * D + c0) : 0u;
        qa[kk][1] = r1 < G ? *reinterpret_cast<const uint32_t*>(qrow + r1 * D + c0) : 0u;
        qa[kk][2] = r0 < G ? *reinterpret_cast<const uint32_t*>(qrow + r0 * D + c0 + 8) : 0u;
        qa[kk][3] = r1 < G ? *reinterpret_cast<const uint32_t*>(qrow + r1 * D + c0 + 8) : 0u;
      }
    }
    float o[NT][4];
#pragma unroll
    for (int j = 0; j < NT; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
    const int qpos = hd.ctx_len - 1;

    for (int g = item.vp_begin; g < item.vp_end; ++g, ++k) {
      const int s = k % NST;
      // ldmatrix / mma.sync are warp-collective: the wait outcome is voted so the
      // whole warp takes the same branch.
      if (ok && !__all_sync(0xffffffffu, mbar_wait(&full[s], (k / NST) & 1))) {
        record_error(a.status, kDevTimeoutFull);
        ok = false;
      }
      const PageDesc pg = sdesc[s];
      const int tok0 = warp * 16;
      const int lo = slot_lo(pg), hi = slot_hi(pg);
      if constexpr (APPEND) {
        const int patch = reinterpret_cast<const int32_t*>(smem + S::kPatchOff)[s];
        if (ok && patch >= tok0 && patch < tok0 + 16) {
          // this warp's tokens hold the new one: write it into the staged page
          // (the bytes the page will hold) and into the pool page
          const __nv_bfloat16* kn = static_cast<const __nv_bfloat16*>(a.k_new) + int64_t(hd.b) * a.new_stride_seq +
                                    int64_t(hd.kv) * a.new_stride_head;
          const __nv_bfloat16* vn = static_cast<const __nv_bfloat16*>(a.v_new) + int64_t(hd.b) * a.new_stride_seq +
                                    int64_t(hd.kv) * a.new_stride_head;
          uint8_t* ks = stage + s * 2 * PB;
          append_write_token<__nv_bfloat16, D, P, FP8>(kn, vn, ks, ks + PB, patch, a.k_inv, a.v_inv, lane, 32);
          append_write_token<__nv_bfloat16, D, P, FP8>(
              kn, vn, static_cast<uint8_t*>(const_cast<void*>(a.kpool)) + int64_t(pg.phys) * a.page_bytes,
              static_cast<uint8_t*>(const_cast<void*>(a.vpool)) + int64_t(pg.phys) * a.page_bytes, patch, a.k_inv,
              a.v_inv, lane, 32);
          // generic writes to the stage before the next bulk copy into it (async proxy)
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
          __syncwarp();
        }
      }
      if (ok && tok0 < hi && tok0 + 16 > lo) {
        const uint32_t kst = smem_u32(stage + s * 2 * PB);
        const uint32_t vst = kst + PB;
        // S = Q K^T over this warp's 16 tokens (two n8 tiles)
        float sc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
        const int mi = lane >> 3, rr = lane & 7;
        if constexpr (FP8) {
          const uint8_t* kp8 = stage + s * 2 * PB;
#pragma unroll
          for (int j = 0; j < D / 32; ++j)
#pragma unroll
            for (int n = 0; n < 2; ++n) {
              const uint2 u =
                  *reinterpret_cast<const uint2*>(kp8 + fp8_kpage_offset(tok0 + n * 8 + grp, j * 32 + tq * 8, D));
              mma_f16_16816(sc[n], qa[2 * j], e4m3x2_to_f16x2(uint16_t(u.x)), e4m3x2_to_f16x2(uint16_t(u.x >> 16)));
              mma_f16_16816(sc[n], qa[2 * j + 1], e4m3x2_to_f16x2(uint16_t(u.y)),
                            e4m3x2_to_f16x2(uint16_t(u.y >> 16)));
            }
        } else {
          const int ktok = tok0 + (mi >> 1) * 8 + rr;
#pragma unroll
          for (int kk = 0; kk < KSTEPS; ++kk) {
            uint32_t b0, b1, b2, b3;
            ldmatrix_x4(b0, b1, b2, b3, kst + uint32_t(kpage_chunk_offset_bf16(ktok, 2 * kk + (mi & 1), P)));
            mma_bf16_16816(sc[0], qa[kk], b0, b1);
            mma_bf16_16816(sc[1], qa[kk], b2, b3);
          }
        }
        // mask and scale (log2 domain); the warp's 16 slots are usually all valid
        if (lo <= tok0 && hi >= tok0 + 16 && !hd.mask_local) {
#pragma unroll
          for (int n = 0; n < 2; ++n)
#pragma unroll
            for (int e = 0; e < 4; ++e) sc[n][e] *= scale_log2;
        } else {
#pragma unroll
          for (int n = 0; n < 2; ++n)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int tok = tok0 + n * 8 + tq * 2 + (e & 1);
              bool vis = tok >= lo && tok < hi;
              if (hd.mask_local) vis = vis && (page_causal(pg) || sees(1, hd.sink, hd.window, qpos, pg.abs_start + tok));
              sc[n][e] = vis ? sc[n][e] * scale_log2 : -INFINITY;
            }
        }
        float mx0 = fmaxf(fmaxf(sc[0][0], sc[0][1]), fmaxf(sc[1][0], sc[1][1]));
        float mx1 = fmaxf(fmaxf(sc[0][2], sc[0][3]), fmaxf(sc[1][2], sc[1][3]));
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
        // Lazy rescaling: a row's reference m moves only when a score exceeds it
        // by more than kLazyLog2; until then the weights 2^(s - m) stay below
        // 2^kLazyLog2 and O and l keep their scale (no multiply of O per page).
        if (__any_sync(0xffffffffu, mx0 > m0 + kLazyLog2 || mx1 > m1 + kLazyLog2)) {
          const float mn0 = mx0 > m0 + kLazyLog2 ? mx0 : m0, mn1 = mx1 > m1 + kLazyLog2 ? mx1 : m1;
          const float al0 = mn0 == m0 ? 1.f : fast_exp2(m0 - mn0), al1 = mn1 == m1 ? 1.f : fast_exp2(m1 - mn1);
          l0 *= al0, l1 *= al1;
#pragma unroll
          for (int j = 0; j < NT; ++j) o[j][0] *= al0, o[j][1] *= al0, o[j][2] *= al1, o[j][3] *= al1;
          m0 = mn0, m1 = mn1;
        }
        const float base0 = m0 == -INFINITY ? 0.f : m0, base1 = m1 == -INFINITY ? 0.f : m1;
        float p[2][4];
#pragma unroll
        for (int n = 0; n < 2; ++n) {
          p[n][0] = fast_exp2(sc[n][0] - base0);
          p[n][1] = fast_exp2(sc[n][1] - base0);
          p[n][2] = fast_exp2(sc[n][2] - base1);
          p[n][3] = fast_exp2(sc[n][3] - base1);
        }
        l0 += (p[0][0] + p[0][1]) + (p[1][0] + p[1][1]);
        l1 += (p[0][2] + p[0][3]) + (p[1][2] + p[1][3]);
        uint32_t pa[4];
        if constexpr (FP8) {
          pa[0] = pack_f16x2(p[0][0], p[0][1]);
          pa[1] = pack_f16x2(p[0][2], p[0][3]);
          pa[2] = pack_f16x2(p[1][0], p[1][1]);
          pa[3] = pack_f16x2(p[1][2], p[1][3]);
          // O = alpha O + P V: lane (grp, tq) needs V rows d = 8 j + grp at this
          // warp's tokens 2tq, 2tq+1, 8+2tq, 9+2tq: positions 4tq .. 4tq+3
          const uint8_t* vp8 = stage + s * 2 * PB + PB;
#pragma unroll
          for (int j = 0; j < NT; ++j) {
            const uint32_t u = *reinterpret_cast<const uint32_t*>(vp8 + fp8_vpage_offset(j * 8 + grp, tok0 + tq * 4));
            mma_f16_16816(o[j], pa, e4m3x2_to_f16x2(uint16_t(u)), e4m3x2_to_f16x2(uint16_t(u >> 16)));
          }
        } else {
        pa[0] = pack_bf16x2(p[0][0], p[0][1]);
        pa[1] = pack_bf16x2(p[0][2], p[0][3]);
        pa[2] = pack_bf16x2(p[1][0], p[1][1]);
        pa[3] = pack_bf16x2(p[1][2], p[1][3]);
        // O = alpha O + P V
        const int vc = 2 * warp + (mi & 1);
#pragma unroll
        for (int j = 0; j < NT / 2; ++j) {
          const int dd = (2 * j + (mi >> 1)) * 8 + rr;
          uint32_t b0, b1, b2, b3;
          ldmatrix_x4(b0, b1, b2, b3, vst + uint32_t(vpage_chunk_offset_bf16(dd, vc)));
          mma_bf16_16816(o[2 * j], pa, b0, b1);
          mma_bf16_16816(o[2 * j + 1], pa, b2, b3);
        }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
    }

    // ---- merge the 4 warps' partial states of this item ----
    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
    float* mw = mbuf + warp * kMaxGroup * S::kMergePitch;
    if (tq == 0) {
      mlbuf[(warp * kMaxGroup + r0) * 2 + 0] = m0;
      mlbuf[(warp * kMaxGroup + r0) * 2 + 1] = l0;
      mlbuf[(warp * kMaxGroup + r1) * 2 + 0] = m1;
      mlbuf[(warp * kMaxGroup + r1) * 2 + 1] = l1;
    }
#pragma unroll
    for (int j = 0; j < NT; ++j) {
      *reinterpret_cast<float2*>(mw + r0 * S::kMergePitch + j * 8 + tq * 2) = make_float2(o[j][0], o[j][1]);
      if (r1 < G)
        *reinterpret_cast<float2*>(mw + r1 * S::kMergePitch + j * 8 + tq * 2) = make_float2(o[j][2], o[j][3]);
    }
    asm volatile("bar.sync 1, %0;" ::"n"(kConsumerWarps * 32) : "memory");
    for (int e = threadIdx.x; e < G * D; e += kConsumerWarps * 32) {
      const int row = e / D, col = e % D;
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, mlbuf[(w * kMaxGroup + row) * 2]);
      const float base = M == -INFINITY ? 0.f : M;
      float acc = 0.f, L = 0.f;
#pragma unroll
      for (int w = 0; w < kConsumerWarps; ++w) {
        const float f = fast_exp2(mlbuf[(w * kMaxGroup + row) * 2] - base);
        acc += f * mbuf[(w * kMaxGroup + row) * S::kMergePitch + col];
        L += f * mlbuf[(w * kMaxGroup + row) * 2 + 1];
      }
      if (item.slot < 0) {
        const int64_t o_idx = (int64_t(hd.q_row0) * a.num_q_heads + qh0 + row) * D + col;
        if constexpr (FP8)
          static_cast<__nv_bfloat16*>(a.out)[o_idx] = __float2bfloat16_rn(acc * a.v_scale / L);
        else
          static_cast<__nv_bfloat16*>(a.out)[o_idx] = __float2bfloat16_rn(acc / L);
        if (col == 0 && a.lse) a.lse[int64_t(hd.q_row0) * a.num_q_heads + qh0 + row] = (M + log2f(L)) * kLn2;
      } else {
        float* slot = a.partial + int64_t(item.slot) * partial_slot_floats(G, D);
        slot[row * D + col] = acc;
        if (col == 0) slot[G * D + row * 2] = M, slot[G * D + row * 2 + 1] = L;
      }
    }
    if constexpr (APPEND) {
      if (item.slot < 0 && threadIdx.x == 0) finish_append<64>(a, item.head);
    }
    if (item.slot >= 0) {
      // Split head: publish this partial, take a ticket; the last CTA to arrive
      // merges in slot order (fixed order: bitwise reproducible) and returns
      // the counter to zero for the next call.  A head with merge groups takes
      // its ticket on its group's counter: the group's last CTA merges the
      // group into the group's slot, then takes a ticket on the head's counter,
      // and the last group's merger merges the group slots.
      int grp = 0, cnt = item.comb, n_arrive = item.n_slots;
      if constexpr (!FP8) {  // E4M3 plans have no merge groups
        if (item.gsz > 0) {
          grp = (item.slot - item.slot0) / item.gsz;
          cnt = item.gcnt0 + grp;
          n_arrive = min(item.gsz, item.n_slots - grp * item.gsz);
        }
      }
      __threadfence();
      asm volatile("bar.sync 1, %0;" ::"n"(kConsumerWarps * 32) : "memory");
      if (threadIdx.x == 0) s_last = atomicAdd(&a.counters[cnt], 1) == n_arrive - 1;
      asm volatile("bar.sync 1, %0;" ::"n"(kConsumerWarps * 32) : "memory");
      if (s_last) {
        __threadfence();
        const int ns = item.n_slots;
        if constexpr (!FP8) {
          const int64_t stride = partial_slot_floats(G, D);
          const float* src = a.partial + int64_t(item.slot0 + grp * item.gsz) * stride;
          int n_src = n_arrive;
          float* part = item.gsz > 0 ? a.partial + int64_t(item.gslot0 + grp) * stride : nullptr;
          for (;;) {
            // 16 float4 loads in flight per thread: 8 slots of two (row, 4-column)
            // entries, or 4 slots of four.
            if (G * D / 4 <= 2 * kConsumerWarps * 32)
              merge_split_head<D, 2, 8, false>(a, hd, qh0, G, n_src, src, part, mbuf, mlbuf, warp, lane);
            else
              merge_split_head<D, 4, 4, false>(a, hd, qh0, G, n_src, src, part, mbuf, mlbuf, warp, lane);
            if (part == nullptr) {
              if (threadIdx.x == 0) {
                a.counters[item.comb] = 0;
                if constexpr (APPEND) finish_append<64>(a, item.head);
              }
              break;
            }
            // group merged: reset its counter, publish the group slot, ticket on the head
            if (threadIdx.x == 0) a.counters[cnt] = 0;
            const int ng = (ns + item.gsz - 1) / item.gsz;
            __threadfence();
            asm volatile("bar.sync 1, %0;" ::"n"(kConsumerWarps * 32) : "memory");
            if (threadIdx.x == 0) s_last = atomicAdd(&a.counters[item.comb], 1) == ng - 1;
            asm volatile("bar.sync 1, %0;" ::"n"(kConsumerWarps * 32) : "memory");
            if (!s_last) break;
            __threadfence();
            src = a.partial + int64_t(item.gslot0) * stride;
            n_src = ng;
            part = nullptr;
          }
        } else {
          // E4M3 pages keep a serial merge (four slots' loads in flight): with the
          // batched one inlined, the kernel's register allocation grew from 153 to
          // 200 and its page loop ran 38% slower (measured on the 32K layer).
          const int64_t stride = partial_slot_floats(G, D);
          const float* p0 = a.partial + int64_t(item.slot0) * stride;
          float* row_m = mlbuf;              // [G] merged max
          float* row_l = mlbuf + kMaxGroup;  // [G] merged sum
          // per row: max and weighted sum over the slots, one warp per row
          for (int row = warp; row < G; row += kConsumerWarps) {
            float m = -INFINITY;
            for (int i = lane; i < ns; i += 32) m = fmaxf(m, __ldcg(p0 + i * stride + G * D + row * 2));
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
            const float base = m == -INFINITY ? 0.f : m;
            float l = 0.f;
            for (int i = lane; i < ns; i += 32) {
              const float* ml = p0 + i * stride + G * D + row * 2;
              l += fast_exp2(__ldcg(ml) - base) * __ldcg(ml + 1);
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
            if (lane == 0) row_m[row] = m, row_l[row] = l;
          }
          asm volatile("bar.sync 1, %0;" ::"n"(kConsumerWarps * 32) : "memory");
          // weighted sum of the slots' accumulators, four columns per thread, slots in order
          for (int e4 = threadIdx.x; e4 < G * D / 4; e4 += kConsumerWarps * 32) {
            const int row = e4 / (D / 4), col = (e4 % (D / 4)) * 4;
            const float M = row_m[row], base = M == -INFINITY ? 0.f : M;
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
            for (int i = 0; i < ns; ++i) {
              const float* sl = p0 + i * stride;
              const float f = fast_exp2(__ldcg(sl + G * D + row * 2) - base);
              const float4 v = __ldcg(reinterpret_cast<const float4*>(sl + row * D + col));
              acc.x += f * v.x, acc.y += f * v.y, acc.z += f * v.z, acc.w += f * v.w;
            }
            const float inv = a.v_scale / row_l[row];
            __nv_bfloat16* o =
                static_cast<__nv_bfloat16*>(a.out) + (int64_t(hd.q_row0) * a.num_q_heads + qh0 + row) * D + col;
            reinterpret_cast<uint2*>(o)[0] = make_uint2(pack_bf16x2(acc.x * inv, acc.y * inv),
                                                        pack_bf16x2(acc.z * inv, acc.w * inv));
          }
          if (threadIdx.x < G && a.lse)
            a.lse[int64_t(hd.q_row0) * a.num_q_heads + qh0 + threadIdx.x] =
                (row_m[threadIdx.x] + log2f(row_l[threadIdx.x])) * kLn2;
          if (threadIdx.x == 0) {
            a.counters[item.comb] = 0;
            if constexpr (APPEND) finish_append<64>(a, item.head);
          }
        }
      }
    }
    asm volatile("bar.sync 1, %0;" ::"n"(kConsumerWarps * 32) : "memory");
  }
}

// The decode kernel, and the fused decode step (append + decode), which must
// keep two CTAs on every SM: its append bookkeeping would otherwise raise the
// register count past the 168 that two 5-warp CTAs leave each thread.
template <int D, int NST, bool FP8>
__global__ void __launch_bounds__(kDecodeThreads) decode_mma_kernel(DecodeLaunch a) {
  decode_mma_body<D, NST, FP8, false>(a);
}
template <int D, int NST, bool FP8>
__global__ void __launch_bounds__(kDecodeThreads, 2) decode_step_kernel(DecodeLaunch a) {
  decode_mma_body<D, NST, FP8, true>(a);
}

// ---------------------------------------------------------------------------
// fp32 SIMT decode (FP32 FMA only, exp2f).
// ---------------------------------------------------------------------------
constexpr int kF32Threads = 128;

template <int D, int P>
__global__ void __launch_bounds__(kF32Threads) decode_f32_kernel(DecodeLaunch a) {
  constexpr int PB = P * D * 4;
  constexpr int ACC = kMaxGroup * D / kF32Threads;
  extern __shared__ __align__(1024) uint8_t smem[];
  float* kp = reinterpret_cast<float*>(smem);        // [P][D]
  float* vp = kp + P * D;                            // [D][P]
  float* qs = vp + P * D;                            // [G][D]
  float* sc = qs + kMaxGroup * D;                    // [G][P]
  float* st = sc + kMaxGroup * P;                    // alpha[G], m[G], l[G]
  const int ib = a.cta_begin[blockIdx.x], ie = a.cta_begin[blockIdx.x + 1];
  const int G = a.group;
  const float* qg = static_cast<const float*>(a.q);
  const uint8_t* kpool = static_cast<const uint8_t*>(a.kpool);
  const uint8_t* vpool = static_cast<const uint8_t*>(a.vpool);
  for (int it = ib; it < ie; ++it) {
    const DecodeItem item = a.items[it];
    const HeadDesc hd = a.heads[item.head];
    const int qh0 = hd.kv * G;
    const int qpos = hd.ctx_len - 1;
    __syncthreads();  // the previous item's output phase still reads st
    for (int e = threadIdx.x; e < G * D; e += kF32Threads)
      qs[e] = qg[(int64_t(hd.q_row0) * a.num_q_heads + qh0) * D + e];
    if (threadIdx.x < G) st[kMaxGroup + threadIdx.x] = -INFINITY, st[2 * kMaxGroup + threadIdx.x] = 0.f;
    float acc[ACC];
#pragma unroll
    for (int j = 0; j < ACC; ++j) acc[j] = 0.f;
    for (int g = item.vp_begin; g < item.vp_end; ++g) {
      const PageDesc pg = a.pages[g];
      if (slot_hi(pg) <= slot_lo(pg)) continue;  // no token (a ring page or a reserved record)
      if (pg.phys < 0 || pg.phys >= a.pool_pages) {  // corrupted table: report, read nothing
        if (threadIdx.x == 0) record_error(a.status, kDevBadPage);
        continue;
      }
      __syncthreads();
      const uint4* ks = reinterpret_cast<const uint4*>(kpool + int64_t(pg.phys) * a.page_bytes);
      const uint4* vs = reinterpret_cast<const uint4*>(vpool + int64_t(pg.phys) * a.page_bytes);
      for (int e = threadIdx.x; e < PB / 16; e += kF32Threads) {
        reinterpret_cast<uint4*>(kp)[e] = ks[e];
        reinterpret_cast<uint4*>(vp)[e] = vs[e];
      }
      __syncthreads();
      for (int e = threadIdx.x; e < G * P; e += kF32Threads) {
        const int h = e / P, t = e % P;
        bool vis = t >= slot_lo(pg) && t < slot_hi(pg);
        if (hd.mask_local) vis = vis && (page_causal(pg) || sees(1, hd.sink, hd.window, qpos, pg.abs_start + t));
        float s = 0.f;
        for (int i = 0; i < D; ++i) s = fmaf(qs[h * D + i], kp[t * D + i], s);
        sc[e] = vis ? s * a.scale_log2 : -INFINITY;
      }
      __syncthreads();
      if (threadIdx.x < G) {
        const int h = threadIdx.x;
        float mx = -INFINITY;
        for (int t = 0; t < P; ++t) mx = fmaxf(mx, sc[h * P + t]);
        const float mo = st[kMaxGroup + h], mn = fmaxf(mo, mx);
        const float base = mn == -INFINITY ? 0.f : mn;
        const float al = exp2f(mo - base);
        float sum = 0.f;
        for (int t = 0; t < P; ++t) {
          const float pv = exp2f(sc[h * P + t] - base);
          sc[h * P + t] = pv;
          sum += pv;
        }
        st[h] = al;
        st[kMaxGroup + h] = mn;
        st[2 * kMaxGroup + h] = st[2 * kMaxGroup + h] * al + sum;
      }
      __syncthreads();
#pragma unroll
      for (int j = 0; j < ACC; ++j) {
        const int e = threadIdx.x + j * kF32Threads;
        const int row = e / D, col = e % D;
        if (row >= G) continue;
        float x = acc[j] * st[row];
        for (int t = 0; t < P; ++t) x = fmaf(sc[row * P + t], vp[col * P + t], x);
        acc[j] = x;
      }
    }
    __syncthreads();
#pragma unroll
    for (int j = 0; j < ACC; ++j) {
      const int e = threadIdx.x + j * kF32Threads;
      const int row = e / D, col = e % D;
      if (row >= G) continue;
      const float M = st[kMaxGroup + row], L = st[2 * kMaxGroup + row];
      if (item.slot < 0) {
        const int64_t o_idx = (int64_t(hd.q_row0) * a.num_q_heads + qh0 + row) * D + col;
        static_cast<float*>(a.out)[o_idx] = acc[j] / L;
        if (col == 0 && a.lse) a.lse[int64_t(hd.q_row0) * a.num_q_heads + qh0 + row] = (M + log2f(L)) * kLn2;
      } else {
        float* slot = a.partial + int64_t(item.slot) * partial_slot_floats(G, D);
        slot[row * D + col] = acc[j];
        if (col == 0) slot[G * D + row * 2] = M, slot[G * D + row * 2 + 1] = L;
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Combine (fp32 path): one warp per (split head, q-head of its group).
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(128) combine_kernel(DecodeLaunch a) {
  const int gw = blockIdx.x * 4 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  const int G = a.group;
  if (gw >= a.n_combine * G) return;
  const CombineItem ci = a.combine[gw / G];
  const int row = gw % G;
  const HeadDesc hd = a.heads[ci.head];
  float M = -INFINITY;
  for (int i = 0; i < ci.n_slots; ++i)
    M = fmaxf(M, a.partial[int64_t(ci.slot_begin + i) * partial_slot_floats(G, D) + G * D + row * 2]);
  const float base = M == -INFINITY ? 0.f : M;
  float acc[D / 32];
#pragma unroll
  for (int j = 0; j < D / 32; ++j) acc[j] = 0.f;
  float L = 0.f;
  for (int i = 0; i < ci.n_slots; ++i) {
    const float* slot = a.partial + int64_t(ci.slot_begin + i) * partial_slot_floats(G, D);
    const float mi = slot[G * D + row * 2];
    const float f = exp2f(mi - base);
    L += f * slot[G * D + row * 2 + 1];
#pragma unroll
    for (int j = 0; j < D / 32; ++j) acc[j] += f * slot[row * D + j * 32 + lane];
  }
  const int qh = hd.kv * G + row;
  const int64_t o_idx = (int64_t(hd.q_row0) * a.num_q_heads + qh) * D;
#pragma unroll
  for (int j = 0; j < D / 32; ++j) static_cast<float*>(a.out)[o_idx + j * 32 + lane] = acc[j] / L;
  if (lane == 0 && a.lse) a.lse[int64_t(hd.q_row0) * a.num_q_heads + qh] = (M + log2f(L)) * kLn2;
}

constexpr int kStagesBf16 = 2;
constexpr int kStagesFp8 = 4;  // half-size pages: twice the stages for the same bytes in flight

template <int D, bool FP8>
cudaError_t launch_mma(const DecodeLaunch& a, cudaStream_t s) {
  constexpr int NST = FP8 ? kStagesFp8 : kStagesBf16;
  using Sm = DecodeSmem<D, NST, FP8>;
  auto kern = a.append ? decode_step_kernel<D, NST, FP8> : decode_mma_kernel<D, NST, FP8>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Sm::kBytes);
  if (e != cudaSuccess) return e;
  kern<<<a.n_ctas, kDecodeThreads, Sm::kBytes, s>>>(a);  // split heads are merged in-kernel
  return cudaGetLastError();
}

template <int D, int P>
cudaError_t launch_f32(const DecodeLaunch& a, cudaStream_t s) {
  const int bytes = (2 * P * D + kMaxGroup * D + kMaxGroup * P + 3 * kMaxGroup) * 4;
  auto kern = decode_f32_kernel<D, P>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return e;
  kern<<<a.n_ctas, kF32Threads, bytes, s>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess || a.n_combine == 0) return e;
  combine_kernel<D><<<(a.n_combine * a.group + 3) / 4, 128, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode(const DecodeLaunch& a, cudaStream_t s) {
  if (a.n_ctas == 0) return cudaSuccess;
  if (a.fp8) return a.D == 128 ? launch_mma<128, true>(a, s) : launch_mma<64, true>(a, s);
  if (a.bf16) return a.D == 128 ? launch_mma<128, false>(a, s) : launch_mma<64, false>(a, s);
  if (a.P == 16) return a.D == 128 ? launch_f32<128, 16>(a, s) : launch_f32<64, 16>(a, s);
  return a.D == 128 ? launch_f32<128, 64>(a, s) : launch_f32<64, 64>(a, s);
}

}  // namespace sp
