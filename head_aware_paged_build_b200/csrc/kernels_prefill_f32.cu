// fp32 prefill: SIMT FP32-FMA kernel over the plan's prefill work list.
//
// One CTA per (q-head, 64-row query tile) (the planner gives fp32 plans
// single-tile items); thread r owns query row r.  KV
// tiles of 64 tokens (the head's pages, in its position order) are staged in
// shared memory; each thread scores the tile's keys for its row, masks them
// (causal, and sink + window for local heads, except on pages flagged to be
// seen causally: a retrieval head's sink and kept blocks), and folds them into an online
// softmax.  Only the tile ranges the planner lists are visited: a local head
// touches its sink tiles and the tiles of its recent window, never the rest of
// the context ("SegPagedAttention runtime design", §4).
#include <cmath>

#include "device_common.cuh"
#include "kernels.h"

namespace sp {
namespace {

constexpr int kRows = kPrefillTileTokensF32;  // query rows per CTA = KV tokens per tile
constexpr float kLn2f = 0.6931471805599453f;
constexpr int kPosCausal = 1 << 30;  // key flag in pos[]: its page is seen causally (positions stay below 2^30)

template <int D, int P>
__global__ void __launch_bounds__(kRows) prefill_f32_kernel(PrefillLaunch a) {
  constexpr int PPT = kRows / P;  // pages per KV tile
  extern __shared__ __align__(1024) uint8_t smem[];
  float* qs = reinterpret_cast<float*>(smem);  // [kRows][D + 1]
  float* ks = qs + kRows * (D + 1);            // [kRows tokens][D]
  float* vs = ks + kRows * D;                  // [D][kRows tokens]
  int* pos = reinterpret_cast<int*>(vs + kRows * D);  // [kRows] absolute position, -1 = empty slot

  const PrefillItem it = a.items[blockIdx.x];
  const HeadDesc hd = a.heads[it.head];
  const int r = threadIdx.x;
  const bool active = r < it.n_rows[0];
  const int p = it.p0[0] + r;
  const float* qg = static_cast<const float*>(a.q);
  for (int e = threadIdx.x; e < kRows * D; e += kRows) {
    const int rr = e / D, i = e % D;
    qs[rr * (D + 1) + i] = rr < it.n_rows[0] ? qg[(int64_t(it.q_row[0] + rr) * a.num_q_heads + it.qh[0]) * D + i] : 0.f;
  }
  float acc[D];
#pragma unroll
  for (int i = 0; i < D; ++i) acc[i] = 0.f;
  float m = -INFINITY, l = 0.f;
  const uint8_t* kpool = static_cast<const uint8_t*>(a.kpool);
  const uint8_t* vpool = static_cast<const uint8_t*>(a.vpool);

  for (int range = 0; range < 2; ++range) {
    const int tb = range ? it.t2 : it.t0, te = range ? it.t3 : it.t1;
    for (int t = tb; t < te; ++t) {
      __syncthreads();
      for (int j = 0; j < PPT; ++j) {
        const int vp = t * PPT + j;
        bool have = vp < hd.n_vpages;
        const PageDesc pg = have ? a.pages[hd.vpage_begin + vp] : PageDesc{0, 0, 0, 0};
        if (have && (pg.phys < 0 || pg.phys >= a.pool_pages)) {  // corrupted table: report, read nothing
          if (threadIdx.x == 0) record_error(a.status, kDevBadPage);
          have = false;
        }
        const float* kp = reinterpret_cast<const float*>(kpool + int64_t(pg.phys) * a.page_bytes);
        const float* vpp = reinterpret_cast<const float*>(vpool + int64_t(pg.phys) * a.page_bytes);
        for (int e = threadIdx.x; e < P * D; e += kRows) {
          const int tt = e / D, i = e % D;
          ks[(j * P + tt) * D + i] = have ? kp[e] : 0.f;
          const int ii = e / P, t2 = e % P;
          vs[ii * kRows + j * P + t2] = have ? vpp[e] : 0.f;
        }
        // key position, with kPosCausal set for a page every row sees causally; -1: no key
        for (int tt = threadIdx.x; tt < P; tt += kRows)
          pos[j * P + tt] = (have && tt >= slot_lo(pg) && tt < slot_hi(pg))
                                ? (pg.abs_start + tt) | (page_causal(pg) ? kPosCausal : 0)
                                : -1;
      }
      __syncthreads();
      if (!active) continue;
      float s[kRows];
      float mx = -INFINITY;
#pragma unroll 4
      for (int c = 0; c < kRows; ++c) {
        const int ap = pos[c] & ~kPosCausal;
        float x = -INFINITY;
        if (pos[c] >= 0 && sees((pos[c] & kPosCausal) ? 0 : hd.kind, hd.sink, hd.window, p, ap)) {
          float d = 0.f;
          for (int i = 0; i < D; ++i) d = fmaf(qs[r * (D + 1) + i], ks[c * D + i], d);
          x = d * a.scale_log2;
        }
        s[c] = x;
        mx = fmaxf(mx, x);
      }
      const float mn = fmaxf(m, mx);
      const float base = mn == -INFINITY ? 0.f : mn;
      const float al = exp2f(m - base);
      m = mn;
      float sum = 0.f;
#pragma unroll
      for (int i = 0; i < D; ++i) acc[i] *= al;
      for (int c = 0; c < kRows; ++c) {
        const float pv = exp2f(s[c] - base);
        sum += pv;
        if (pv != 0.f) {
#pragma unroll
          for (int i = 0; i < D; ++i) acc[i] = fmaf(pv, vs[i * kRows + c], acc[i]);
        }
      }
      l = l * al + sum;
    }
  }
  if (!active) return;
  float* og = static_cast<float*>(a.out) + (int64_t(it.q_row[0] + r) * a.num_q_heads + it.qh[0]) * D;
#pragma unroll
  for (int i = 0; i < D; ++i) og[i] = acc[i] / l;
  if (a.lse) a.lse[int64_t(it.q_row[0] + r) * a.num_q_heads + it.qh[0]] = (m + log2f(l)) * kLn2f;
}

template <int D, int P>
cudaError_t launch_f32(const PrefillLaunch& a, cudaStream_t s) {
  const int bytes = (kRows * (D + 1) + 2 * kRows * D) * 4 + kRows * 4;
  auto kern = prefill_f32_kernel<D, P>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return e;
  kern<<<a.n_items, kRows, bytes, s>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill_f32(const PrefillLaunch& a, cudaStream_t s) {
  if (a.n_items == 0) return cudaSuccess;
  if (a.P == 16) return a.D == 128 ? launch_f32<128, 16>(a, s) : launch_f32<64, 16>(a, s);
  return a.D == 128 ? launch_f32<128, 64>(a, s) : launch_f32<64, 64>(a, s);
}

}  // namespace sp
