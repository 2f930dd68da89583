// Host planner of libsegpaged.so: policy -> segments -> pages -> work lists.
//
// Everything that depends only on the batch's layout is decided here, once,
// when the plan is created ("SegPagedAttention runtime design", §5: page
// tables and layout must be built when KV is written and reused, because
// computing them on every attention call cost a 0.70x slowdown).
#include <algorithm>
#include <cmath>
#include <cstring>
#include <limits>
#include <new>
#include <numeric>
#include <string>
#include <vector>

#include "sp_internal.h"

namespace sp {

thread_local std::string g_last_error;

void set_error(const std::string& msg) { g_last_error = msg; }

sp_status fail(sp_status st, const std::string& msg) {
  g_last_error = msg;
  return st;
}

namespace {

constexpr int kDefaultDecodeCtas = 2 * 148;
constexpr int64_t kItemCostPages100 = 350;  // a head start costs about 3.5 pages (measured)
constexpr int32_t kMergeOneLevel = 16;      // split heads with more items merge in two levels

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

sp_status validate(const sp_problem& p) {
  if (p.batch < 1 || p.num_q_heads < 1 || p.num_kv_heads < 1 || p.head_dim < 1 || p.page_size < 1)
    return fail(SP_ERR_INVALID_ARG, "batch, head counts, head_dim and page_size must be >= 1");
  if (!p.ctx_len || !p.q_start || !p.policy)
    return fail(SP_ERR_INVALID_ARG, "ctx_len, q_start and policy must be non-NULL host arrays");
  if (p.flags & ~uint32_t(SP_FLAG_DENSE_MASKED | SP_FLAG_RING)) return fail(SP_ERR_INVALID_ARG, "unknown flag bits");
  if (p.append_capacity < 0) return fail(SP_ERR_INVALID_ARG, "append_capacity must be >= 0");
  if (p.append_capacity > 0 && !(p.flags & SP_FLAG_RING))
    return fail(SP_ERR_INVALID_ARG, "append_capacity needs SP_FLAG_RING");
  if (p.spare_pages < 0) return fail(SP_ERR_INVALID_ARG, "spare_pages must be >= 0");
  if (p.spare_pages > 0 && !(p.flags & SP_FLAG_RING))
    return fail(SP_ERR_INVALID_ARG, "spare_pages needs SP_FLAG_RING");
  if ((p.flags & SP_FLAG_RING) && (p.flags & SP_FLAG_DENSE_MASKED))
    return fail(SP_ERR_UNSUPPORTED, "ring plans are SegPaged plans (no dense-masked variant)");
  if (p.first_page < 0) return fail(SP_ERR_INVALID_ARG, "first_page must be >= 0");
  if (p.target_ctas < 0) return fail(SP_ERR_INVALID_ARG, "target_ctas must be >= 0");
  if (p.dtype != SP_F32 && p.dtype != SP_BF16) return fail(SP_ERR_UNSUPPORTED, "dtype must be SP_F32 or SP_BF16");
  if (p.head_dim != 64 && p.head_dim != 128) return fail(SP_ERR_UNSUPPORTED, "head_dim must be 64 or 128");
  if (p.dtype == SP_BF16 && p.page_size != 64) return fail(SP_ERR_UNSUPPORTED, "bf16 pools need page_size 64");
  if (p.dtype == SP_F32 && p.page_size != 16 && p.page_size != 64)
    return fail(SP_ERR_UNSUPPORTED, "fp32 pools need page_size 16 or 64");
  if (p.num_q_heads % p.num_kv_heads != 0)
    return fail(SP_ERR_UNSUPPORTED, "num_q_heads must be a multiple of num_kv_heads");
  if (p.num_q_heads / p.num_kv_heads > kMaxGroup)
    return fail(SP_ERR_UNSUPPORTED, "at most 16 q-heads per kv-head");
  if (p.kv_dtype != 0 && p.kv_dtype != p.dtype && p.kv_dtype != SP_E4M3)
    return fail(SP_ERR_UNSUPPORTED, "kv_dtype must be 0, the problem dtype or SP_E4M3");
  if (p.kv_dtype == SP_E4M3) {
    if (p.dtype != SP_BF16) return fail(SP_ERR_UNSUPPORTED, "E4M3 pages need bf16 queries");
    if (!(p.k_scale > 0.f) || !(p.v_scale > 0.f) || p.k_scale > 3.0e38f || p.v_scale > 3.0e38f)
      return fail(SP_ERR_INVALID_ARG, "E4M3 pages need finite k_scale, v_scale > 0");
  }
  int64_t rows = 0;
  for (int b = 0; b < p.batch; ++b) {
    const int64_t L = p.ctx_len[b], q0 = p.q_start[b];
    if (L < 1) return fail(SP_ERR_INVALID_ARG, "ctx_len[" + std::to_string(b) + "] must be >= 1");
    if (L > (int64_t(1) << 30)) return fail(SP_ERR_UNSUPPORTED, "ctx_len above 2^30");
    if (q0 < 0 || q0 >= L)
      return fail(SP_ERR_INVALID_ARG, "q_start[" + std::to_string(b) + "] must lie in [0, ctx_len)");
    rows += L - q0;
  }
  if (rows > std::numeric_limits<int32_t>::max()) return fail(SP_ERR_UNSUPPORTED, "too many query rows");
  for (int64_t i = 0; i < int64_t(p.batch) * p.num_kv_heads; ++i) {
    const sp_head_policy& h = p.policy[i];
    const std::string who = "policy[" + std::to_string(i) + "]";
    if (h.kind != SP_GLOBAL && h.kind != SP_LOCAL && h.kind != SP_DENSE && h.kind != SP_RETRIEVAL)
      return fail(SP_ERR_INVALID_ARG, who + ".kind is not a head kind");
    if ((h.kind == SP_LOCAL || h.kind == SP_RETRIEVAL) && (h.sink < 0 || h.window == 0))
      return fail(SP_ERR_INVALID_ARG, who + ": local and retrieval heads need sink >= 0, window != 0");
    if (h.kind != SP_RETRIEVAL) continue;
    if (!std::isfinite(h.top_p)) return fail(SP_ERR_INVALID_ARG, who + ": top_p must be finite");
    if (p.flags & SP_FLAG_RING) return fail(SP_ERR_UNSUPPORTED, "retrieval heads are not supported in ring plans");
    if (!p.block_mass || !p.block_mass[i])
      return fail(SP_ERR_INVALID_ARG, who + ": a retrieval head needs its block_mass entry");
    const int64_t nb = (int64_t(p.ctx_len[i / p.num_kv_heads]) + p.page_size - 1) / p.page_size;
    for (int64_t j = 0; j < nb; ++j) {
      const float m = p.block_mass[i][j];
      if (!(m >= 0.f) || !std::isfinite(m))
        return fail(SP_ERR_INVALID_ARG, who + ": block_mass values must be finite and >= 0");
    }
  }
  return SP_OK;
}

// Blocks a retrieval head keeps: the candidates (blocks holding a position >=
// sink) in decreasing importance, ties by lower block, and of those the
// shortest prefix whose importance reaches top_p of the candidates' total
// (fp64 sums in that order); top_p >= 1 keeps every candidate, <= 0 none.
std::vector<uint8_t> kept_blocks(int64_t L, int64_t P, int64_t sink, float top_p, const float* mass) {
  const int64_t nb = (L + P - 1) / P;
  std::vector<int64_t> cand;
  for (int64_t i = 0; i < nb; ++i)
    if ((i + 1) * P > sink) cand.push_back(i);
  std::stable_sort(cand.begin(), cand.end(), [&](int64_t a, int64_t b) { return mass[a] > mass[b]; });
  size_t keep = cand.size();
  if (top_p <= 0.f) {
    keep = 0;
  } else if (top_p < 1.f) {
    double total = 0.0;
    for (int64_t i : cand) total += double(mass[i]);
    const double target = double(top_p) * total;
    double run = 0.0;
    keep = 0;
    while (keep < cand.size() && run < target) run += double(mass[cand[keep++]]);
  }
  std::vector<uint8_t> sel(nb, 0);
  for (size_t k = 0; k < keep; ++k) sel[cand[k]] = 1;
  return sel;
}

// Pages of a head (indices into its page list) holding any position of [x, y].
void pages_touching(const sp_plan& pl, int h, int64_t x, int64_t y, int64_t* v0, int64_t* v1) {
  *v0 = std::numeric_limits<int64_t>::max();
  *v1 = std::numeric_limits<int64_t>::min();
  const int P = pl.prob.page_size;
  for (int s = pl.seg_begin[h]; s < pl.seg_begin[h + 1]; ++s) {
    const sp_segment& g = pl.segments[s];
    const int64_t lo = std::max<int64_t>(g.abs_start, x);
    const int64_t hi = std::min<int64_t>(int64_t(g.abs_start) + g.length - 1, y);
    if (lo > hi) continue;
    *v0 = std::min<int64_t>(*v0, g.first_page_index + (lo - g.abs_start) / P);
    *v1 = std::max<int64_t>(*v1, g.first_page_index + (hi - g.abs_start) / P + 1);
  }
  if (*v0 > *v1) *v0 = *v1 = 0;
}

// KV tiles (of `ppt` pages, in the head's page list) that a retrieval head's
// item must visit for rows at positions [p_first, p_last]: every tile holding
// a key some row sees, covered by at most two ranges (split at the widest run
// of tiles no row sees; tiles left inside a range are masked out by the
// kernel).  A page flagged kSpanCausal is seen by a row at p up to p; any
// other page by the local rule (sink, or the window of some row).
void retrieval_tiles(const sp_plan& pl, int h, int64_t p_first, int64_t p_last, int ppt, int64_t* t) {
  const HeadDesc& hd = pl.heads[h];
  std::vector<int64_t> tiles;
  for (int v = 0; v < hd.n_vpages; ++v) {
    const PageDesc& pg = pl.pages[hd.vpage_begin + v];
    const int64_t lo = slot_lo(pg), hi = slot_hi(pg);
    if (hi <= lo) continue;
    const int64_t a0 = pg.abs_start + lo, a1 = pg.abs_start + hi - 1;
    const bool seen = a0 <= p_last && (page_causal(pg) || a0 < hd.sink ||
                                       std::min<int64_t>(a1, p_last) >= p_first - hd.window + 1);
    if (seen && (tiles.empty() || tiles.back() != v / ppt)) tiles.push_back(v / ppt);
  }
  t[0] = t[1] = t[2] = t[3] = 0;
  if (tiles.empty()) return;
  size_t cut = 0;  // the widest gap lies after tiles[cut - 1]
  int64_t gap = 0;
  for (size_t i = 1; i < tiles.size(); ++i)
    if (tiles[i] - tiles[i - 1] - 1 > gap) gap = tiles[i] - tiles[i - 1] - 1, cut = i;
  if (gap == 0) {
    t[0] = tiles.front(), t[1] = tiles.back() + 1;
  } else {
    t[0] = tiles.front(), t[1] = tiles[cut - 1] + 1, t[2] = tiles[cut], t[3] = tiles.back() + 1;
  }
}

void align_to(std::vector<uint8_t>& blob, size_t a) { blob.resize((blob.size() + a - 1) / a * a, 0); }

template <typename T>
int64_t append(std::vector<uint8_t>& blob, const std::vector<T>& v) {
  align_to(blob, 256);
  const int64_t off = int64_t(blob.size());
  blob.resize(blob.size() + v.size() * sizeof(T));
  if (!v.empty()) std::memcpy(blob.data() + off, v.data(), v.size() * sizeof(T));
  return off;
}

sp_status plan_build(sp_plan& pl) {
  const sp_problem& p = pl.prob;
  const int B = p.batch, Hkv = p.num_kv_heads, P = p.page_size, D = p.head_dim;
  const bool dense_masked = (p.flags & SP_FLAG_DENSE_MASKED) != 0;
  pl.group = p.num_q_heads / Hkv;
  pl.elem_bytes = p.dtype == SP_BF16 ? 2 : 4;
  const int nh = B * Hkv;

  // --- segments and pages ---------------------------------------------------
  pl.seg_begin.assign(1, 0);
  pl.heads.resize(nh);
  int64_t n_pages = 0, stored = 0, dense_rows = 0, visible = 0;
  std::vector<int32_t> qrow(B + 1, 0);
  for (int b = 0; b < B; ++b) qrow[b + 1] = qrow[b] + (pl.ctx_len[b] - pl.q_start[b]);
  bool decode = true;
  for (int b = 0; b < B; ++b) decode = decode && (pl.ctx_len[b] - pl.q_start[b] == 1);
  const bool ring = (p.flags & SP_FLAG_RING) != 0;
  if (ring && !decode) return fail(SP_ERR_UNSUPPORTED, "ring plans are decode plans (one query per sequence)");
  pl.fp8 = p.kv_dtype == SP_E4M3;
  if (pl.fp8 && !decode) return fail(SP_ERR_UNSUPPORTED, "E4M3 pages are supported for decode plans");
  pl.k_scale = pl.fp8 ? p.k_scale : 1.f;
  pl.v_scale = pl.fp8 ? p.v_scale : 1.f;
  const int64_t cap = p.append_capacity;
  if (ring) {
    for (int b = 0; b < B; ++b)
      if (int64_t(pl.ctx_len[b]) + cap > (int64_t(1) << 30)) return fail(SP_ERR_UNSUPPORTED, "ctx_len + capacity above 2^30");
  }

  pl.kept_blocks.assign(nh, {});
  int64_t ctx_row = 0;
  for (int b = 0; b < B; ++b, ctx_row += pl.ctx_len[b - 1]) {
    const int64_t L = pl.ctx_len[b], q0 = pl.q_start[b];
    if (ctx_row + L > std::numeric_limits<int32_t>::max())
      return fail(SP_ERR_UNSUPPORTED, "sum of ctx_len above 2^31");
    for (int kv = 0; kv < Hkv; ++kv) {
      const int h = b * Hkv + kv;
      const sp_head_policy& pol = pl.policy[h];
      const bool retrieval = pol.kind == SP_RETRIEVAL;
      const bool local = pol.kind == SP_LOCAL || retrieval;  // the local rule applies (to unflagged pages)
      const int64_t s = local ? pol.sink : 0;
      // adaptive window (window <= -1): max(1, L / -window) for this sequence
      const int64_t w = !local ? 0 : pol.window > 0 ? pol.window : std::max<int64_t>(1, L / (-int64_t(pol.window)));
      // Runs of stored positions (start, length, every query sees them causally).
      struct Run {
        int64_t start, len;
        bool causal;
      };
      std::vector<Run> runs;
      std::vector<uint8_t> sel;
      if (retrieval) {
        sel = kept_blocks(L, P, s, pol.top_p, p.block_mass[h]);
        pl.kept_blocks[h] = sel;
      }
      if (!local || dense_masked) {
        runs.push_back({0, L, false});
      } else if (!retrieval) {
        const int64_t sink_len = std::min<int64_t>(s, L);
        const int64_t rec = std::max<int64_t>(s, q0 - w + 1);
        if (rec <= sink_len) {  // touching: one run [0, L)
          runs.push_back({0, L, false});
        } else {
          if (sink_len > 0) runs.push_back({0, sink_len, false});
          if (rec < L) runs.push_back({rec, L - rec, false});
        }
      } else {
        // Retrieval: per block, its sink part and its kept part are seen causally
        // by every query; an unkept block keeps only its part inside the calls'
        // windows [max(sink, q0 - w + 1), L).  Touching runs merge when they share
        // the flag; in decode plans (one query, which sees every stored position)
        // touching runs always merge.
        const int64_t rec = std::max<int64_t>(s, q0 - w + 1);
        const bool decode_head = q0 == L - 1;
        auto add = [&](int64_t a, int64_t e, bool causal) {
          if (e <= a) return;
          if (!runs.empty() && runs.back().start + runs.back().len == a &&
              (runs.back().causal == causal || decode_head)) {
            runs.back().len += e - a;
            runs.back().causal = runs.back().causal && causal;
          } else {
            runs.push_back({a, e - a, causal});
          }
        };
        for (int64_t i = 0; i * P < L; ++i) {
          const int64_t a = i * P, e = std::min<int64_t>(L, a + P), c = std::max<int64_t>(a, s);
          add(a, std::min<int64_t>(e, s), true);
          if (sel[i])
            add(c, e, true);
          else
            add(std::max<int64_t>(c, rec), e, false);
        }
      }
      if (ring) {
        // Ring plan: pages aligned to absolute multiples of P.  GLOBAL: [0, L)
        // plus pages for `cap` more tokens.  LOCAL: the sink's pages (for all
        // s positions) and a ring of R pages; position a >= s sits in ring slot
        // a mod (R P), so appends never move a token.
        runs.assign(1, Run{0, L, false});
        if (local) {
          const int64_t sink_len = std::min<int64_t>(s, L);
          const int64_t wlo = std::max<int64_t>(s, L - w), whi = L;
          runs.clear();
          if (sink_len > 0) runs.push_back({0, sink_len, false});
          if (whi > wlo) runs.push_back({wlo, whi - wlo, false});
        }
      }
      HeadDesc& hd = pl.heads[h];
      hd = HeadDesc{};
      hd.kind = local ? 1 : 0;
      hd.sink = int32_t(s);
      // windows beyond the 2^30 context cap change nothing; the clamp keeps
      // position arithmetic such as p - window + 1 - a inside int32
      hd.window = int32_t(std::min<int64_t>(w, int64_t(1) << 30));
      hd.ctx_len = int32_t(L);
      hd.q_start = int32_t(q0);
      hd.vpage_begin = int32_t(n_pages);
      hd.mask_local = (local && dense_masked) ? 1 : 0;
      hd.b = b;
      hd.kv = kv;
      hd.q_row0 = qrow[b];
      int32_t vp = 0;
      if (ring) {
        auto add_page = [&](int64_t abs0, int64_t lo, int64_t hi) {
          PageDesc pd{};
          pd.abs_start = int32_t(abs0);
          pd.span = hi > lo ? make_span(int32_t(lo), int32_t(hi)) : 0;
          pd.head = h;
          pl.pages.push_back(pd);
          ++vp;
        };
        if (!local) {
          const int64_t np = ceil_div(L + cap, P);
          for (int64_t k = 0; k < np; ++k) {
            add_page(k * P, 0, std::clamp<int64_t>(L - k * P, 0, P));
            // with a shared spare pool, pages reserved for growth are records only
            if (p.spare_pages > 0 && k * P >= L) pl.pages.back().phys = kNoPage;
          }
          pl.segments.push_back(sp_segment{0, int32_t(L), 0, int32_t(np)});
        } else {
          const int64_t nsink = ceil_div(s, P);
          const int64_t sink_len = std::min<int64_t>(s, L);
          for (int64_t k = 0; k < nsink; ++k) add_page(k * P, 0, std::clamp<int64_t>(sink_len - k * P, 0, P));
          if (sink_len > 0) pl.segments.push_back(sp_segment{0, int32_t(sink_len), 0, int32_t(nsink)});
          const int64_t R = ceil_div(w, P) + 1, RP = R * P;
          const int64_t wlo = std::max<int64_t>(s, L - w), whi = L;
          for (int64_t i = 0; i < R; ++i) {
            // latest run of ring page i (positions q RP + i P ...) that starts before whi
            const int64_t x = whi - 1 - i * P;
            const int64_t q = x >= 0 ? x / RP : -((-x + RP - 1) / RP);
            const int64_t run = q * RP + i * P;
            const int64_t lo = std::max<int64_t>(wlo, run) - run, hi = std::min<int64_t>(whi, run + P) - run;
            add_page(run, std::max<int64_t>(lo, 0), std::max<int64_t>(hi, 0));
          }
          if (whi > wlo)
            pl.segments.push_back(sp_segment{int32_t(wlo), int32_t(whi - wlo), int32_t(nsink), int32_t(R)});
        }
        for (const Run& r : runs) stored += r.len;
      }
      for (size_t i = 0; i < runs.size() && !ring; ++i) {
        const Run& r = runs[i];
        sp_segment g{int32_t(r.start), int32_t(r.len), vp, int32_t(ceil_div(r.len, P))};
        pl.segments.push_back(g);
        for (int k = 0; k < g.num_pages; ++k) {
          PageDesc pd{};
          pd.phys = 0;  // assigned below
          pd.abs_start = g.abs_start + k * P;
          pd.span = make_span(0, int32_t(std::min<int64_t>(P, int64_t(g.abs_start) + g.length - pd.abs_start)));
          // dense-masked retrieval heads: page k is block k, seen causally when kept
          if (r.causal || (retrieval && dense_masked && sel[k])) pd.span |= kSpanCausal;
          pd.head = h;
          pl.pages.push_back(pd);
        }
        vp += g.num_pages;
        stored += r.len;
      }
      hd.n_vpages = vp;
      hd.ctx_row0 = int32_t(ctx_row);
      n_pages += vp;
      if (n_pages > std::numeric_limits<int32_t>::max())
        return fail(SP_ERR_UNSUPPORTED, "more than 2^31 pages");
      pl.seg_begin.push_back(int32_t(pl.segments.size()));
      dense_rows += L;
      // visible (query, key) pairs: global p + 1, local min(p + 1, s + w); retrieval:
      // the sink and kept positions before the window plus the window itself
      if (retrieval) {
        std::vector<int64_t> pc(L + 1, 0);  // pc[j]: positions < j seen causally (sink or kept block)
        for (int64_t j = 0; j < L; ++j) pc[j + 1] = pc[j] + ((j < s || sel[j / P]) ? 1 : 0);
        for (int64_t q = q0; q < L; ++q) {
          const int64_t lo = std::max<int64_t>(0, q - w + 1);
          visible += pc[lo] + (q + 1 - lo);
        }
      } else {
        for (int64_t q = q0; q < L; ++q) visible += local ? std::min<int64_t>(q + 1, s + w) : q + 1;
      }
    }
  }
  visible *= pl.group;

  // --- physical page ids -----------------------------------------------------
  // The plan owns one page per page record with a page, then the spare pool;
  // logical page k (records in order, then the pool) is physical page
  // first_page + (page_ids ? page_ids[k] : k).
  int64_t n_assigned = 0;
  for (const PageDesc& pd : pl.pages) n_assigned += pd.phys != kNoPage;
  const int64_t n_owned = n_assigned + p.spare_pages;
  if (n_owned > std::numeric_limits<int32_t>::max()) return fail(SP_ERR_UNSUPPORTED, "more than 2^31 pages");
  int64_t max_id = n_owned - 1;
  if (p.page_ids) {
    std::vector<int32_t> ids(p.page_ids, p.page_ids + n_owned);
    for (int32_t id : ids)
      if (id < 0) return fail(SP_ERR_INVALID_ARG, "page_ids must be non-negative");
    std::sort(ids.begin(), ids.end());
    if (std::adjacent_find(ids.begin(), ids.end()) != ids.end())
      return fail(SP_ERR_INVALID_ARG, "page_ids must be distinct");
    max_id = n_owned ? ids.back() : -1;
  }
  if (p.first_page + max_id + 1 > std::numeric_limits<int32_t>::max())
    return fail(SP_ERR_UNSUPPORTED, "pool above 2^31 pages");
  auto phys_of = [&](int64_t k) { return int32_t(p.first_page + (p.page_ids ? p.page_ids[k] : k)); };
  int64_t logical = 0;
  for (int64_t i = 0; i < n_pages; ++i)
    if (pl.pages[i].phys != kNoPage) pl.pages[i].phys = phys_of(logical++);
  std::vector<int32_t> free_stack(kFreeIdsOffset + p.spare_pages, 0);
  free_stack[0] = p.spare_pages;
  for (int64_t k = 0; k < p.spare_pages; ++k) free_stack[kFreeIdsOffset + k] = phys_of(n_assigned + k);

  // --- decode: balanced page ranges per CTA, cut at head boundaries ---------
  int n_slots = 0;
  if (decode) {
    const int64_t G = std::min<int64_t>(p.target_ctas ? p.target_ctas : kDefaultDecodeCtas, n_pages);
    // A CTA pays for every head it starts (Q load, warp merge, partial publish) on
    // top of its pages: cut the page list at equal shares of (pages + 3.5 pages
    // per head start), so CTAs that cross a head boundary take fewer pages.
    // Costs are in hundredths of a page.
    std::vector<int64_t> cost(n_pages + 1, 0);  // cost of pages [0, i)
    for (int64_t i = 0; i < n_pages; ++i) {
      const HeadDesc& hd = pl.heads[pl.pages[i].head];
      cost[i + 1] = cost[i] + kItemCostPages100 * (i == hd.vpage_begin ? 1 : 0) + 100;
    }
    std::vector<int64_t> cut(G + 1, n_pages);
    for (int64_t c = 0, i = 0; c <= G; ++c) {
      const int64_t total = cost[n_pages];  // ceil(total * c / G) without overflow
      const int64_t want = total / G * c + ((total % G) * c + G - 1) / G;
      while (i < n_pages && cost[i] < want) ++i;
      cut[c] = c == G ? n_pages : i;
    }
    pl.decode_cta_begin.assign(1, 0);
    for (int64_t c = 0; c < G; ++c) {
      int64_t lo = cut[c], hi = cut[c + 1];
      while (lo < hi) {
        const int h = pl.pages[lo].head;
        const int64_t end = std::min<int64_t>(hi, pl.heads[h].vpage_begin + pl.heads[h].n_vpages);
        pl.decode_items.push_back(DecodeItem{h, int32_t(lo), int32_t(end), -1, -1, 0, 0, 0, 0, 0, {0, 0}});
        lo = end;
      }
      pl.decode_cta_begin.push_back(int32_t(pl.decode_items.size()));
    }
    // items of a head are consecutive; split heads get consecutive slots.  On
    // bf16 pages a head split into more than kMergeOneLevel items merges in two
    // levels (groups of about sqrt(n) slots), so no single CTA reads all of a
    // long head's partials at the end of the call.
    const bool two_level = p.dtype == SP_BF16 && !pl.fp8;
    int32_t n_group_counters = 0;
    size_t i = 0;
    while (i < pl.decode_items.size()) {
      size_t j = i;
      while (j < pl.decode_items.size() && pl.decode_items[j].head == pl.decode_items[i].head) ++j;
      if (j - i > 1) {
        const int32_t ns = int32_t(j - i);
        const int32_t comb = int32_t(pl.combine.size());
        pl.combine.push_back(CombineItem{pl.decode_items[i].head, n_slots, ns, 0});
        const int32_t slot0 = n_slots;
        n_slots += ns;
        int32_t gsz = 0, gslot0 = 0, gcnt0 = 0;
        if (two_level && ns > kMergeOneLevel) {
          gsz = 1;
          while (gsz * gsz < ns) ++gsz;  // ceil(sqrt(ns))
          const int32_t ng = (ns + gsz - 1) / gsz;
          gslot0 = n_slots;
          n_slots += ng;
          gcnt0 = n_group_counters;
          n_group_counters += ng;
        }
        for (size_t k = i; k < j; ++k) {
          DecodeItem& d = pl.decode_items[k];
          d.slot = slot0 + int32_t(k - i);
          d.comb = comb;
          d.n_slots = ns;
          d.slot0 = slot0;
          d.gsz = gsz;
          d.gslot0 = gslot0;
          d.gcnt0 = gcnt0;
        }
      }
      i = j;
    }
    // group counters follow the heads' counters in the workspace
    for (DecodeItem& d : pl.decode_items)
      if (d.gsz > 0) d.gcnt0 += int32_t(pl.combine.size());
    pl.n_counters = int32_t(pl.combine.size()) + n_group_counters;
  } else {
    // --- prefill: query tiles x visited KV tile ranges -----------------------
    // bf16 items pair two query tiles of the same (sequence, kv-head) so that
    // one K/V tile in shared memory feeds two 128-row tiles: two q-heads of the
    // GQA group at the same positions, or (odd group sizes, MHA) neighbouring
    // query tiles, whose visible KV ranges share the sink run and overlap in
    // the window.  fp32 items hold a single 64-row tile.
    const bool pair = p.dtype == SP_BF16;
    const int T = pair ? kPrefillTileTokensBf16 : kPrefillTileTokensF32;
    const int ppt = T / P;
    pl.prefill_tile = T;
    std::vector<std::vector<PrefillItem>> per_head(nh);
    std::vector<int32_t> head_max(nh, 0);
    for (int h = 0; h < nh; ++h) {
      const HeadDesc& hd = pl.heads[h];
      const int64_t C = hd.ctx_len - hd.q_start;
      std::vector<std::pair<int64_t, int>> units;  // (query tile, q-head)
      for (int64_t qt = 0; qt * T < C; ++qt)
        for (int g = 0; g < pl.group; ++g) units.emplace_back(qt, hd.kv * pl.group + g);
      const size_t step = pair ? 2 : 1;
      for (size_t u = 0; u < units.size(); u += step) {
        PrefillItem it{};
        it.head = h;
        it.qh[1] = -1;
        int64_t p_first = std::numeric_limits<int64_t>::max(), p_last = -1;
        for (size_t x = 0; x < step && u + x < units.size(); ++x) {
          const int64_t qt = units[u + x].first;
          it.qh[x] = units[u + x].second;
          it.n_rows[x] = int32_t(std::min<int64_t>(T, C - qt * T));
          it.q_row[x] = int32_t(hd.q_row0 + qt * T);
          it.p0[x] = int32_t(hd.q_start + qt * T);
          p_first = std::min<int64_t>(p_first, it.p0[x]);
          p_last = std::max<int64_t>(p_last, it.p0[x] + it.n_rows[x] - 1);
        }
        int64_t v0, v1, v2, v3;
        if (!pl.kept_blocks[h].empty() && !dense_masked) {
          int64_t t[4];
          retrieval_tiles(pl, h, p_first, p_last, ppt, t);
          it.t0 = int32_t(t[0]), it.t1 = int32_t(t[1]), it.t2 = int32_t(t[2]), it.t3 = int32_t(t[3]);
          it.work = int32_t((t[1] - t[0]) + (t[3] - t[2]));
          head_max[h] = std::max(head_max[h], it.work);
          per_head[h].push_back(it);
          continue;
        }
        if (hd.kind == 0 || dense_masked) {
          pages_touching(pl, h, 0, p_last, &v0, &v1);
          v2 = v3 = 0;
        } else {
          pages_touching(pl, h, 0, std::min<int64_t>(hd.sink, p_last + 1) - 1, &v0, &v1);
          pages_touching(pl, h, std::max<int64_t>(hd.sink, p_first - hd.window + 1), p_last, &v2, &v3);
        }
        int64_t t0 = v0 / ppt, t1 = ceil_div(v1, ppt), t2 = v2 / ppt, t3 = ceil_div(v3, ppt);
        if (v0 == v1) t0 = t1 = 0;
        if (v2 == v3) t2 = t3 = 0;
        if (t0 == t1) std::swap(t0, t2), std::swap(t1, t3);
        if (t2 < t3 && t2 <= t1) t1 = std::max(t1, t3), t2 = t3 = 0;
        it.t0 = int32_t(t0), it.t1 = int32_t(t1), it.t2 = int32_t(t2), it.t3 = int32_t(t3);
        it.work = int32_t((t1 - t0) + (t3 - t2));
        head_max[h] = std::max(head_max[h], it.work);
        per_head[h].push_back(it);
      }
    }
    // Heaviest heads first; within a head the heaviest items first.  Items of
    // one head run back to back so that its KV tiles are reused through L2.
    std::vector<int> order(nh);
    std::iota(order.begin(), order.end(), 0);
    std::stable_sort(order.begin(), order.end(), [&](int a, int c) { return head_max[a] > head_max[c]; });
    for (int h : order) {
      auto& v = per_head[h];
      std::stable_sort(v.begin(), v.end(), [](const PrefillItem& a, const PrefillItem& c) { return a.work > c.work; });
      pl.prefill.insert(pl.prefill.end(), v.begin(), v.end());
    }
  }
  pl.n_partial_slots = n_slots;

  // --- table blob --------------------------------------------------------------
  TableHeader& H = pl.hdr;
  H = TableHeader{};
  H.magic = kTableMagic;
  H.version = SEGPAGED_ABI_VERSION;
  H.n_heads = nh;
  H.n_vpages = int32_t(n_pages);
  H.n_decode_items = int32_t(pl.decode_items.size());
  H.n_decode_ctas = decode ? int32_t(pl.decode_cta_begin.size() - 1) : 0;
  H.n_combine = int32_t(pl.combine.size());
  H.n_prefill_items = int32_t(pl.prefill.size());
  pl.blob.assign(sizeof(TableHeader), 0);
  H.off_heads = append(pl.blob, pl.heads);
  H.off_pages = append(pl.blob, pl.pages);
  H.off_decode_items = append(pl.blob, pl.decode_items);
  H.off_decode_cta = append(pl.blob, pl.decode_cta_begin);
  H.off_combine = append(pl.blob, pl.combine);
  H.off_prefill = append(pl.blob, pl.prefill);
  H.off_free = append(pl.blob, free_stack);
  H.n_spare = p.spare_pages;
  align_to(pl.blob, 256);
  std::memcpy(pl.blob.data(), &H, sizeof(H));

  sp_sizes& z = pl.sizes;
  z = sp_sizes{};
  z.num_pages = n_owned;
  z.pool_pages = p.first_page + max_id + 1;
  z.page_bytes = int64_t(P) * D * (pl.fp8 ? 1 : pl.elem_bytes);
  z.table_bytes = int64_t(pl.blob.size());
  // workspace: status word block | arrival counters (one per split head, then
  // one per merge group) | partial slots (items' slots, then group slots)
  const int64_t partial = int64_t(n_slots) * partial_slot_floats(pl.group, D) * 4;
  pl.partial_offset = kStatusBytes + ceil_div(int64_t(pl.n_counters) * 4, 256) * 256;
  z.workspace_bytes = pl.partial_offset + ceil_div(partial, 256) * 256;
  z.stored_token_heads = stored;
  z.dense_token_heads = dense_rows;
  z.visible_pairs = visible;
  z.num_queries = qrow[B];
  z.is_decode = decode ? 1 : 0;
  z.num_decode_ctas = H.n_decode_ctas;
  z.num_prefill_items = H.n_prefill_items;
  z.num_combine = H.n_combine;
  // bf16 decode merges split heads inside its kernel; fp32 decode adds a combine pass
  z.launches_per_call = decode ? (H.n_decode_ctas > 0) + (p.dtype == SP_F32 && H.n_combine > 0)
                               : (H.n_prefill_items > 0);
  return SP_OK;
}

}  // namespace
}  // namespace sp

extern "C" {

const char* segpaged_last_error(void) { return sp::g_last_error.c_str(); }

int32_t segpaged_abi_version(void) { return SEGPAGED_ABI_VERSION; }

const char* segpaged_status_string(sp_status st) {
  switch (st) {
    case SP_OK: return "SP_OK";
    case SP_ERR_INVALID_ARG: return "SP_ERR_INVALID_ARG";
    case SP_ERR_UNSUPPORTED: return "SP_ERR_UNSUPPORTED";
    case SP_ERR_WORKSPACE: return "SP_ERR_WORKSPACE";
    case SP_ERR_CUDA: return "SP_ERR_CUDA";
    case SP_ERR_DEVICE_CHECK: return "SP_ERR_DEVICE_CHECK";
  }
  return "unknown sp_status";
}

sp_status segpaged_plan_create(const sp_problem* problem, sp_plan** out) {
  if (!problem || !out) return sp::fail(SP_ERR_INVALID_ARG, "problem and out must be non-NULL");
  *out = nullptr;
  try {
    sp_status st = sp::validate(*problem);
    if (st != SP_OK) return st;
    auto* pl = new sp_plan();
    pl->prob = *problem;
    const int B = problem->batch, nh = problem->batch * problem->num_kv_heads;
    pl->ctx_len.assign(problem->ctx_len, problem->ctx_len + B);
    pl->q_start.assign(problem->q_start, problem->q_start + B);
    pl->policy.assign(problem->policy, problem->policy + nh);
    st = sp::plan_build(*pl);
    pl->prob.ctx_len = pl->prob.q_start = nullptr;
    pl->prob.policy = nullptr;
    pl->prob.page_ids = nullptr;
    pl->prob.block_mass = nullptr;
    if (st != SP_OK) {
      delete pl;
      return st;
    }
    *out = pl;
    return SP_OK;
  } catch (const std::bad_alloc&) {
    return sp::fail(SP_ERR_INVALID_ARG, "out of host memory while planning");
  } catch (...) {
    return sp::fail(SP_ERR_INVALID_ARG, "unexpected error while planning");
  }
}

void segpaged_plan_destroy(sp_plan* plan) { delete plan; }

sp_status segpaged_plan_sizes(const sp_plan* plan, sp_sizes* out) {
  if (!plan || !out) return sp::fail(SP_ERR_INVALID_ARG, "plan and out must be non-NULL");
  *out = plan->sizes;
  return SP_OK;
}

sp_status segpaged_plan_head_segments(const sp_plan* plan, int32_t b, int32_t kv, sp_segment* segs,
                                      int32_t max, int32_t* count) {
  if (!plan || !count || (max > 0 && !segs)) return sp::fail(SP_ERR_INVALID_ARG, "NULL argument");
  if (b < 0 || b >= plan->prob.batch || kv < 0 || kv >= plan->prob.num_kv_heads)
    return sp::fail(SP_ERR_INVALID_ARG, "(b, kv) out of range");
  const int h = b * plan->prob.num_kv_heads + kv;
  const int n = plan->seg_begin[h + 1] - plan->seg_begin[h];
  *count = n;
  for (int i = 0; i < n && i < max; ++i) segs[i] = plan->segments[plan->seg_begin[h] + i];
  return SP_OK;
}

sp_status segpaged_plan_head_pages(const sp_plan* plan, int32_t b, int32_t kv, int64_t* page_ids,
                                   int32_t max, int32_t* count) {
  if (!plan || !count || (max > 0 && !page_ids)) return sp::fail(SP_ERR_INVALID_ARG, "NULL argument");
  if (b < 0 || b >= plan->prob.batch || kv < 0 || kv >= plan->prob.num_kv_heads)
    return sp::fail(SP_ERR_INVALID_ARG, "(b, kv) out of range");
  const sp::HeadDesc& hd = plan->heads[b * plan->prob.num_kv_heads + kv];
  *count = hd.n_vpages;
  for (int i = 0; i < hd.n_vpages && i < max; ++i) page_ids[i] = plan->pages[hd.vpage_begin + i].phys;
  return SP_OK;
}

sp_status segpaged_plan_decode_items(const sp_plan* plan, int32_t* records, int32_t max, int32_t* count) {
  if (!plan || !count || (max > 0 && !records)) return sp::fail(SP_ERR_INVALID_ARG, "NULL argument");
  const int32_t n = int32_t(plan->decode_items.size());
  *count = n;
  const int32_t hkv = plan->prob.num_kv_heads;
  int32_t i = 0;
  for (size_t c = 0; c + 1 < plan->decode_cta_begin.size(); ++c) {
    for (int32_t it = plan->decode_cta_begin[c]; it < plan->decode_cta_begin[c + 1]; ++it, ++i) {
      if (i >= max) return SP_OK;
      const sp::DecodeItem& d = plan->decode_items[it];
      const sp::HeadDesc& hd = plan->heads[d.head];
      int32_t* r = records + int64_t(i) * SP_DECODE_ITEM_WORDS;
      r[0] = int32_t(c);
      r[1] = d.head / hkv;
      r[2] = d.head % hkv;
      r[3] = d.vp_begin - hd.vpage_begin;
      r[4] = d.vp_end - hd.vpage_begin;
      r[5] = d.slot;
      r[6] = d.slot >= 0 ? d.n_slots : 1;
      r[7] = d.slot >= 0 ? d.slot0 : -1;
      r[8] = d.gsz;
      r[9] = d.gsz > 0 ? d.gslot0 : -1;
      r[10] = d.slot >= 0 ? d.comb : -1;
      r[11] = d.gsz > 0 ? d.gcnt0 + (d.slot - d.slot0) / d.gsz : -1;
    }
  }
  return SP_OK;
}

sp_status segpaged_plan_prefill_items(const sp_plan* plan, int32_t* records, int32_t max, int32_t* count) {
  if (!plan || !count || (max > 0 && !records)) return sp::fail(SP_ERR_INVALID_ARG, "NULL argument");
  const int32_t n = int32_t(plan->prefill.size());
  *count = n;
  const int32_t hkv = plan->prob.num_kv_heads;
  for (int32_t i = 0; i < n && i < max; ++i) {
    const sp::PrefillItem& it = plan->prefill[i];
    int32_t* r = records + int64_t(i) * SP_PREFILL_ITEM_WORDS;
    r[0] = it.head / hkv;
    r[1] = it.head % hkv;
    r[2] = plan->prefill_tile;
    r[3] = it.qh[0], r[4] = it.qh[1];
    r[5] = it.q_row[0], r[6] = it.qh[1] >= 0 ? it.q_row[1] : 0;
    r[7] = it.n_rows[0], r[8] = it.qh[1] >= 0 ? it.n_rows[1] : 0;
    r[9] = it.p0[0], r[10] = it.qh[1] >= 0 ? it.p0[1] : 0;
    r[11] = it.t0, r[12] = it.t1, r[13] = it.t2, r[14] = it.t3;
    r[15] = it.work;
  }
  return SP_OK;
}

}  // extern "C"
