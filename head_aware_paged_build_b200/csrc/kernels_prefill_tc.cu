// bf16 prefill on 5th-generation tensor cores (tcgen05, sm_100a).
//
// One CTA per work item: one or two 128-row query tiles of the same
// (sequence, kv-head) — two q-heads of the GQA group at the same positions,
// or neighbouring query tiles.  The CTA visits only the KV tiles of 128
// tokens (two pages) that some row can see, in the head's stored order: the
// sink tiles and the recent-window tiles of a local head, the causal prefix of
// a global head ("SegPagedAttention runtime design", §4: every
// (query-head, kv-head) pair runs over its own true length, with no mask over
// invisible KV).  Only tiles that cross a boundary (causal diagonal, window
// edge, sink page, a segment's partial last page) are masked, per row, by
// visible column intervals.  A retrieval head's sink and kept blocks sit on
// pages flagged to be seen causally; its other pages follow the local rule.
//
// Warp roles (576 threads):
//   warp 0      producer: both Q tiles by TMA (128-byte swizzle); K and V
//               pages by 1-D bulk copies (pool pages are stored in the tensor
//               cores' swizzled K-major operand layout, V transposed), one
//               K/V stage feeding both query tiles
//   warp 1      TMEM owner and MMA issuer (one thread):
//                 S_x = Q_x K^T       tcgen05.mma, A and B from shared memory
//                 O_x += P_x V        tcgen05.mma, A (= P_x) from TMEM
//               in the order S_A, S_B, then per KV tile j:
//                 PV_A(j), S_A(j+1), PV_B(j), S_B(j+1)
//               so that the tensor core alternates between the two tiles while
//               their softmax warpgroups run
//   warps 2-9   softmax of tile A, warps 10-17 softmax of tile B: two threads
//               per row, each owning one of the KV tile's two pages (64
//               columns); S read with tcgen05.ld, online softmax in the log2
//               domain against a running reference kept per row, a lazy
//               rescale of O (only when the row maximum grows by more than
//               2^8), P written back as bf16 over the half's own first 32 S
//               columns; then the epilogue (O / l, LSE).  Usually one pass:
//               each 32-column chunk is exponentiated against the reference as
//               soon as it is read, and the halves only vote; a tile whose
//               scores outgrow some row's reference takes the two-pass step
//               (row maxima exchanged between the halves through shared
//               memory, held-back chunks recomputed from S, stored chunks of
//               rows whose reference moved rescaled in TMEM).
// The commit that signals S_x(j) also covers P_x(j-1) V, so a softmax thread
// holding S_x(j) may rescale O_x and overwrite P_x with no further wait.
// Every wait is bounded; a wait that runs out records a status code, and the
// CTA drains its copies and MMAs, frees its TMEM and returns.
#include <cuda.h>

#include <mutex>

#include "device_common.cuh"
#include "kernels.h"
#include "tc_ptx.cuh"

namespace sp {
namespace {



constexpr int kTile = kPrefillTileTokensBf16;  // 128 query rows, 128 KV tokens
constexpr int kThreads = 576;
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleLog2 = 8.0f;  // rescale O only when the max grows by more than 2^8
constexpr float kLn2 = 0.6931471805599453f;
constexpr uint32_t kFull = 0xffffffffu;
// One exponent pair in every kPolyPeriod is computed on the FMA pipe (0: none).
#ifndef SP_EXP2_POLY_PERIOD
#define SP_EXP2_POLY_PERIOD 16
#endif
constexpr int kPolyPeriod = SP_EXP2_POLY_PERIOD;

template <int D, int NS>
struct TcSmem {
  static constexpr int kQ = D / 64 * 16384;  // one query tile: [D/64][128 rows][128 B]
  static constexpr int kK = D / 64 * 16384;  // [D/64][128 tokens][128 B]
  static constexpr int kV = 2 * D * 128;     // [2 pages][D rows][64 tokens * 2 B]
  static constexpr int kStage = kK + kV;
  static constexpr int kOffQ = 0;
  static constexpr int kOffStage = kOffQ + 2 * kQ;
  static constexpr int kOffBar = kOffStage + NS * kStage;
  static constexpr int kOffX = kOffBar + 256;                // softmax halves' exchange: 2 tiles x 6 x 128 floats
  static constexpr int kBytes = kOffX + 2 * 6 * 128 * 4 + 1024;  // + 1 KB alignment slack
};

struct Bars {
  uint64_t q;
  uint64_t o_done;
  uint64_t done;
  uint64_t pad;
  uint64_t s_full[2];
  uint64_t p_full[2];
};

// Does every row p in [p_first, p_last] see every slot of this page?
__device__ __forceinline__ bool page_fully_visible(const PageDesc& pg, bool exists, const HeadDesc& hd, int p_first,
                                                   int p_last) {
  if (!exists || slot_lo(pg) != 0 || slot_hi(pg) != 64) return false;
  const int a0 = pg.abs_start, a1 = pg.abs_start + 63;
  if (a1 > p_first) return false;
  if (hd.kind == 0 || page_causal(pg)) return true;
  return a1 < hd.sink || a0 > p_last - hd.window;
}

// Slots of a page visible to row p: [0, h1) (sink run) and [l2, h2) (causal
// part / recent window), inside the page's valid range [lo, hi).  A page with
// lo > 0 never holds sink positions (sink pages always start at slot 0; only
// ring pages of decode plans start later), so its sink run is empty.
__device__ __forceinline__ void visible_slots(const PageDesc& pg, bool exists, const HeadDesc& hd, int p, int& h1,
                                              int& l2, int& h2) {
  h1 = l2 = h2 = 0;
  if (!exists) return;
  const int lo = slot_lo(pg);
  const int causal = min(slot_hi(pg), p - pg.abs_start + 1);  // valid slots with position <= p
  if (hd.kind == 0 || page_causal(pg)) {
    l2 = lo, h2 = causal;
  } else {
    h1 = lo > 0 ? 0 : min(causal, hd.sink - pg.abs_start);     // sink run
    l2 = max(lo, p - hd.window + 1 - pg.abs_start);            // recent window
    h2 = causal;
  }
}

template <int D, int NS>
__global__ void __launch_bounds__(kThreads, 1) prefill_tc_kernel(const __grid_constant__ CUtensorMap qmap,
                                                                  PrefillLaunch a) {
  using Sm = TcSmem<D, NS>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* q_s = smem + Sm::kOffQ;
  uint8_t* stage_s = smem + Sm::kOffStage;
  Bars* bars = reinterpret_cast<Bars*>(smem + Sm::kOffBar);
  uint64_t* kv_full = reinterpret_cast<uint64_t*>(bars + 1);
  uint64_t* kv_free = kv_full + NS;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(kv_free + NS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* xbuf = reinterpret_cast<float*>(smem + Sm::kOffX);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const PrefillItem it = a.items[blockIdx.x];
  const HeadDesc hd = a.heads[it.head];
  const int n1 = it.t1 - it.t0;
  const int n = n1 + (it.t3 - it.t2);
  const bool two = it.qh[1] >= 0;

  if (threadIdx.x == 0) {
    mbar_init(&bars->q, 1);
    mbar_init(&bars->o_done, 1);
    mbar_init(&bars->done, 1);
    for (int x = 0; x < 2; ++x) {
      mbar_init(&bars->s_full[x], 1);
      mbar_init(&bars->p_full[x], 256);
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
  // TMEM columns: S/P of tile x at [128 x, 128 x + 128); O of tile x at 256 + x D
  auto t_s = [&](int x) { return tmem + uint32_t(128 * x); };
  auto t_o = [&](int x) { return tmem + uint32_t(256 + x * D); };

  auto fail = [&](int32_t code) {
    record_error(a.status, code);
    *abort_flag = 1;
  };
  auto tile_of = [&](int j) { return j < n1 ? it.t0 + j : it.t2 + (j - n1); };

  if (warp == 0) {
    // ------------------------------ producer ------------------------------
    if (lane == 0) {
      const uint8_t* kpool = static_cast<const uint8_t*>(a.kpool);
      const uint8_t* vpool = static_cast<const uint8_t*>(a.vpool);
      mbar_arrive_expect_tx(&bars->q, (two ? 2 : 1) * Sm::kQ);
#pragma unroll
      for (int x = 0; x < 2; ++x)
        if (x == 0 || two)
#pragma unroll
          for (int h = 0; h < D / 64; ++h)
            tc::tma_load_3d(q_s + x * Sm::kQ + h * 16384, &qmap, h * 64, it.qh[x], it.q_row[x], &bars->q);
      int issued = 0;
      for (int j = 0; j < n && !*abort_flag; ++j) {
        const int st = j % NS;
        if (j >= NS && !mbar_wait(&kv_free[st], ((j / NS) - 1) & 1)) {
          fail(kDevTimeoutEmpty);
          break;
        }
        const int t = tile_of(j);
        const int vp0 = 2 * t, vp1 = (2 * t + 1 < hd.n_vpages) ? 2 * t + 1 : 2 * t;
        const int64_t ph[2] = {a.pages[hd.vpage_begin + vp0].phys, a.pages[hd.vpage_begin + vp1].phys};
        if (ph[0] < 0 || ph[0] >= a.pool_pages || ph[1] < 0 || ph[1] >= a.pool_pages) {
          fail(kDevBadPage);  // corrupted table: read nothing; the other roles' bounded waits end the CTA
          break;
        }
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
      const uint32_t q_addr = smem_u32(q_s), st_addr = smem_u32(stage_s);
      auto issue_s = [&](int x, int st) {
        // a descriptor's start-address field is address >> 4, so each k-step's
        // descriptor is the tile's base descriptor plus a fixed offset
        const uint64_t qd = tc::smem_desc_sw128(q_addr + x * Sm::kQ);
        const uint64_t kd = tc::smem_desc_sw128(st_addr + st * Sm::kStage);
        const uint32_t ts = t_s(x);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = ((kk >> 2) * 16384 + (kk & 3) * 32) >> 4;
          tc::mma_bf16_ss(ts, qd + off, kd + off, idesc_s, kk > 0);
        }
        tc::commit(&bars->s_full[x]);
      };
      auto issue_pv = [&](int x, int st, bool acc) {
        const uint64_t vd = tc::smem_desc_sw128(st_addr + st * Sm::kStage + Sm::kK);
        const uint32_t to = t_o(x), ts = t_s(x);
#pragma unroll
        for (int kk = 0; kk < kTile / 16; ++kk)  // P of page h sits at columns [64 h, 64 h + 32)
          tc::mma_bf16_ts(to, ts + (kk >> 2) * 64 + (kk & 3) * 8, vd + (((kk >> 2) * (D * 128) + (kk & 3) * 32) >> 4),
                          idesc_o, (acc || kk > 0) ? 1u : 0u);
      };
      bool ok = mbar_wait(&bars->q, 0) && mbar_wait(&kv_full[0], 0);
      if (!ok) fail(kDevTimeoutFull);
      if (ok && n > 0) {
        tc::fence_after_sync();
        issue_s(0, 0);
        if (two) issue_s(1, 0);
      }
      for (int j = 0; ok && j < n; ++j) {
        if (*abort_flag) break;
        const int st = j % NS;
        const bool more = j + 1 < n;
        const int st1 = (j + 1) % NS;
        if (!mbar_wait(&bars->p_full[0], j & 1)) { fail(kDevTimeoutSoftmax); break; }
        tc::fence_after_sync();
        issue_pv(0, st, j > 0);
        if (more) {
          if (!mbar_wait(&kv_full[st1], ((j + 1) / NS) & 1)) { fail(kDevTimeoutFull); break; }
          tc::fence_after_sync();
          issue_s(0, st1);
        }
        if (two) {
          if (!mbar_wait(&bars->p_full[1], j & 1)) { fail(kDevTimeoutSoftmax); break; }
          tc::fence_after_sync();
          issue_pv(1, st, j > 0);
        }
        tc::commit(&kv_free[st]);
        if (two && more) issue_s(1, st1);
      }
      tc::commit(&bars->o_done);
      // all MMAs issued by this thread complete before TMEM is released
      tc::commit(&bars->done);
      mbar_wait(&bars->done, 0);
    }
    __syncwarp();
  } else {
    // ------------------------------ softmax ------------------------------
    // Eight warps per query tile, two threads per row: half h takes the tile's
    // page h (columns [64 h, 64 h + 64)).  The halves exchange row maxima
    // through shared memory at a barrier that also votes on every wait, so
    // both halves always take the same path.
    const int x = (warp - 2) >> 3;       // query tile of this warp
    const int h = ((warp - 2) >> 2) & 1;  // page (column half) of the KV tile
    if (x == 0 || two) {
      const int quarter = warp & 3;  // TMEM lane quarter this warp may access
      const int r = quarter * 32 + lane;
      const uint32_t lane_off = uint32_t(quarter * 32) << 16;
      // this tile's fields by select, not by index: the item stays in registers
      const int p0x = x ? it.p0[1] : it.p0[0], rows_x = x ? it.n_rows[1] : it.n_rows[0];
      const int qrow_x = x ? it.q_row[1] : it.q_row[0], qh_x = x ? it.qh[1] : it.qh[0];
      const int p = p0x + r;
      const int p_first = p0x, p_last = p0x + rows_x - 1;
      const float sl2 = a.scale_log2;
      const int bar_id = 1 + x;
      float* xch = xbuf + x * 6 * kTile;  // [parity][half][row] row maxima, then [half][row] row sums
      float m_run = -INFINITY, l_run = 0.f;
      bool ok = true;
      PageDesc nx{};
      auto fetch_desc = [&](int j, PageDesc& d) {
        const int vp = 2 * tile_of(j) + h;
        d = vp < hd.n_vpages ? a.pages[hd.vpage_begin + vp] : PageDesc{0, 0, 0, 0};
      };
      if (n > 0) fetch_desc(0, nx);
      for (int j = 0; j < n; ++j) {
        const bool have = 2 * tile_of(j) + h < hd.n_vpages;
        const PageDesc pg = nx;
        if (j + 1 < n) fetch_desc(j + 1, nx);
        const bool full = page_fully_visible(pg, have, hd, p_first, p_last);
        // tcgen05.ld / st are warp-collective: the wait outcome is voted per warp,
        // then across the tile's eight warps at the exchange barrier below.
        const bool got = __all_sync(kFull, mbar_wait(&bars->s_full[x], j & 1));
        int h1 = 64, l2 = 0, h2 = 0;
        if (!full) visible_slots(pg, have, hd, p, h1, l2, h2);
        auto mask32 = [&](float (&w)[32], int c) {  // chunk c: page slots [32 c, 32 c + 32)
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const int t = 32 * c + e;
            if (!(t < h1 || (t >= l2 && t < h2))) w[e] = -INFINITY;
          }
        };
        auto exp_chunk = [&](const float (&w)[32], uint64_t nbase2, uint32_t (&pk)[16]) -> uint64_t {
          const uint64_t scale2 = f2_pack(sl2, sl2);
          uint64_t s2[2] = {f2_pack(0.f, 0.f), f2_pack(0.f, 0.f)};
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const uint64_t x2 = f2_fma(f2_pack(w[2 * e], w[2 * e + 1]), scale2, nbase2);
            float e0, e1;
            if (kPolyPeriod > 0 && (e % (kPolyPeriod > 0 ? kPolyPeriod : 1)) == kPolyPeriod - 1) {
              exp2_poly_pair(x2, e0, e1);
            } else {
              float x0, x1;
              f2_unpack(x2, x0, x1);
              e0 = fast_exp2(x0), e1 = fast_exp2(x1);
            }
            s2[e & 1] = f2_add(s2[e & 1], f2_pack(e0, e1));
            pk[e] = pack_bf16x2(e0, e1);
          }
          return f2_add(s2[0], s2[1]);
        };
        // One pass: each 32-column chunk's maximum, then P = 2^(s - m_run)
        // against the row's running reference.  A warp stores a chunk's P only
        // when all its rows stay within 2^8 of their reference (the weights the
        // lazy rescale keeps); once a warp holds back a chunk it stores no
        // more, so that chunk's scores stay in TMEM.  If any row of the tile
        // outgrew its reference, the tile takes the two-pass step: maxima
        // exchanged, held-back chunks recomputed from S, stored chunks of rows
        // whose reference moved rescaled in TMEM.
        float mx = -INFINITY;
        uint64_t csum[2] = {f2_pack(0.f, 0.f), f2_pack(0.f, 0.f)};
        int stored = 0;  // chunks of this warp already in TMEM (warp-uniform)
        if (got) {
          tc::fence_after_sync();
          const float base = m_run == -INFINITY ? 0.f : m_run;
          const uint64_t nbase2 = f2_pack(-base, -base);
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            float w[32];
            tc::tmem_ld32(t_s(x) + lane_off + 64 * h + 32 * c, w);
            tc::tmem_wait_ld();
            if (!full) mask32(w, c);
            float m4[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) m4[i] = fmax3(w[i], w[i + 4], mx);
#pragma unroll
            for (int e = 8; e < 32; e += 8)
#pragma unroll
              for (int i = 0; i < 4; ++i) m4[i] = fmax3(m4[i], w[e + i], w[e + 4 + i]);
            mx = fmax3(fmax3(m4[0], m4[1], m4[2]), m4[3], mx);
            const bool fit = m_run != -INFINITY && !(mx * sl2 > m_run + kRescaleLog2);
            if (stored == c && __all_sync(kFull, fit)) {
              uint32_t pk[16];
              csum[c] = exp_chunk(w, nbase2, pk);
              tc::tmem_st16(t_s(x) + lane_off + 64 * h + 16 * c, pk);
              stored = c + 1;
            }
          }
        }
        xch[(j & 1) * 2 * kTile + h * kTile + r] = mx;
        if (bar_red_and(bar_id, 8 * 32, got && stored == 2)) {
          float s0, s1, s2, s3;
          f2_unpack(csum[0], s0, s1);
          f2_unpack(csum[1], s2, s3);
          l_run = l_run + ((s0 + s1) + (s2 + s3));
        } else {
          if (!bar_red_and(bar_id, 8 * 32, got)) {
            fail(kDevTimeoutMma);
            ok = false;
            break;
          }
          tc::tmem_wait_st();  // P chunks stored above are read back below
          const float mt = fmaxf(mx, xch[(j & 1) * 2 * kTile + (1 - h) * kTile + r]);
          const float mts = mt * sl2;
          float alpha = 1.f;
          bool need = false;
          if (mts > m_run + kRescaleLog2) {
            alpha = fast_exp2(m_run - mts);
            need = m_run != -INFINITY;
            m_run = mts;
          }
          const float base = m_run == -INFINITY ? 0.f : m_run;
          const uint64_t nbase2 = f2_pack(-base, -base);
          float lsum = 0.f;
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            if (c < stored) {
              // stored against the old reference: scale by alpha where it moved
              float s0, s1;
              f2_unpack(csum[c], s0, s1);
              lsum += (s0 + s1) * alpha;
              if (__any_sync(kFull, need)) {
                uint32_t pk[16];
                tc::tmem_ld16(t_s(x) + lane_off + 64 * h + 16 * c, pk);
                tc::tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                  const float lo = __uint_as_float(pk[e] << 16), hi = __uint_as_float(pk[e] & 0xffff0000u);
                  pk[e] = pack_bf16x2(lo * alpha, hi * alpha);
                }
                tc::tmem_st16(t_s(x) + lane_off + 64 * h + 16 * c, pk);
              }
            } else {
              float w[32];
              tc::tmem_ld32(t_s(x) + lane_off + 64 * h + 32 * c, w);
              tc::tmem_wait_ld();
              if (!full) mask32(w, c);
              uint32_t pk[16];
              float s0, s1;
              f2_unpack(exp_chunk(w, nbase2, pk), s0, s1);
              lsum += s0 + s1;
              tc::tmem_st16(t_s(x) + lane_off + 64 * h + 16 * c, pk);
            }
          }
          l_run = l_run * alpha + lsum;
          if (__any_sync(kFull, need)) {
            const float f = need ? alpha : 1.f;
#pragma unroll
            for (int c = 0; c < D / 64; ++c) {
              float o[32];
              tc::tmem_ld32(t_o(x) + lane_off + h * (D / 2) + c * 32, o);
              tc::tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 32; ++e) o[e] *= f;
              tc::tmem_st32(t_o(x) + lane_off + h * (D / 2) + c * 32, o);
            }
          }
        }
        tc::tmem_wait_st();
        tc::fence_before_sync();
        mbar_arrive(&bars->p_full[x]);
      }
      // ------------------------------ epilogue ------------------------------
      // The row sum is the two halves' sums; the barrier also votes on the O wait.
      xch[4 * kTile + h * kTile + r] = l_run;
      const bool got = ok && n > 0 && mbar_wait(&bars->o_done, 0);
      const bool go = bar_red_and(bar_id, 8 * 32, got && !*abort_flag);
      if (go) {
        tc::fence_after_sync();
        const float l_tot = xch[4 * kTile + r] + xch[5 * kTile + r];
        const bool row_ok = r < rows_x;
        const float inv_l = 1.f / l_tot;
        __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(a.out) +
                              (int64_t(qrow_x + r) * a.num_q_heads + qh_x) * D + h * (D / 2);
#pragma unroll
        for (int c = 0; c < D / 64; ++c) {
          float o[32];
          tc::tmem_ld32(t_o(x) + lane_off + h * (D / 2) + c * 32, o);
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
        if (h == 0 && row_ok && a.lse)
          a.lse[int64_t(qrow_x + r) * a.num_q_heads + qh_x] = (m_run + log2f(l_tot)) * kLn2;
      } else if (ok && n > 0) {
        fail(kDevTimeoutMma);
      }
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
