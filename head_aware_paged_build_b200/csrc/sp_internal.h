// Internal layout of the SegmentPageTable blob and of the plan, shared by the
// host planner and the CUDA kernels of libsegpaged.so.
#pragma once

#include <cstdint>
#include <string>
#include <vector>

#include "segpaged.h"

#if defined(__CUDACC__)
#define SP_HD __host__ __device__
#else
#define SP_HD
#endif

namespace sp {

constexpr int32_t kTableMagic = 0x53504731;  // "SPG1"
constexpr int kStatusBytes = 256;            // workspace prefix holding the status word
constexpr int kPrefillTileTokensBf16 = 128;  // query tile of the tcgen05 prefill kernel
constexpr int kPrefillTileTokensF32 = 64;    // KV / query tile of the fp32 prefill kernel
constexpr int kMaxGroup = 16;                // q-heads per kv-head handled by one decode CTA

// Floats of one decode partial-result slot: acc [G][D], then (m, l) per row in
// a 4G-float block, so that every slot starts 16-byte aligned.
SP_HD constexpr int64_t partial_slot_floats(int G, int D) { return int64_t(G) * (D + 4); }

// Device status codes (workspace word 0); the first error sticks.
enum DeviceCode : int32_t {
  kDevOk = 0,
  kDevTimeoutFull = 1,     // a consumer gave up waiting for a page / tile copy
  kDevTimeoutEmpty = 2,    // the producer gave up waiting for a free stage
  kDevTimeoutMma = 3,      // a wait on a tensor-core commit ran out
  kDevTimeoutSoftmax = 4,  // the MMA issuer gave up waiting for P
  kDevBadPage = 5,         // a table page id outside [0, pool_pages): nothing read or written there
  kDevAppendFull = 6,      // an append found no reserved page left (ring plans)
  kDevPoolEmpty = 7,       // an append found the shared spare pool empty (ring plans with spare pages)
};

// Shared spare pool of a ring plan (table section): word 0 holds how many of
// the page ids at words kFreeIdsOffset ... are still free; appends take the
// last free one with an atomic decrement.  A page record waiting for a page
// from the pool has phys == kNoPage.
constexpr int kFreeIdsOffset = 4;
constexpr int32_t kNoPage = -1;

// One (sequence, kv-head).  Kinds are resolved: 0 reads the whole causal
// context, 1 applies the local rule (sink + window) to every page that is not
// flagged kSpanCausal.  A retrieval head is kind 1 whose sink pages and kept
// blocks' pages carry that flag.
struct alignas(16) HeadDesc {
  int32_t kind;
  int32_t sink;
  int32_t window;
  int32_t ctx_len;
  int32_t q_start;
  int32_t vpage_begin;  // first entry of this head in the page array
  int32_t n_vpages;
  int32_t mask_local;   // 1: kernels apply the local mask per element (dense-masked baseline)
  int32_t b;
  int32_t kv;
  int32_t q_row0;       // first row of sequence b in the varlen query / output arrays
  int32_t ctx_row0;     // L_0 + ... + L_{b-1}: first token row of sequence b when packed
};
static_assert(sizeof(HeadDesc) == 48, "HeadDesc layout");

// One page of a head.  Slot t holds position abs_start + t; only slots
// [lo, hi) hold tokens (lo = span & 0xff, hi = (span >> 16) & 0xff; page sizes
// are at most 64).  Bit 8 of span (kSpanCausal) marks a page every query sees
// causally whatever the head's local rule: the sink and kept blocks of a
// retrieval head.  Pages of a head are in position order except in ring plans,
// where the recent window is a ring of pages (see the planner).
struct alignas(16) PageDesc {
  int32_t phys;       // physical page id in the pools
  int32_t abs_start;  // absolute position of slot 0
  int32_t span;       // lo | hi << 16
  int32_t head;       // owning HeadDesc index
};
static_assert(sizeof(PageDesc) == 16, "PageDesc layout");
constexpr int32_t kSpanCausal = 1 << 8;
SP_HD inline int32_t slot_lo(const PageDesc& p) { return p.span & 0xff; }
SP_HD inline int32_t slot_hi(const PageDesc& p) { return (p.span >> 16) & 0xff; }
SP_HD inline bool page_causal(const PageDesc& p) { return (p.span & kSpanCausal) != 0; }
SP_HD inline int32_t make_span(int32_t lo, int32_t hi) { return lo | (hi << 16); }

// A run of consecutive pages of one head processed by one decode CTA.
struct alignas(16) DecodeItem {
  int32_t head;
  int32_t vp_begin;  // global page-array indices [vp_begin, vp_end)
  int32_t vp_end;
  int32_t slot;      // partial-result slot in the workspace, or -1: the item covers the head
  int32_t comb;      // split head index (arrival counter), -1 if not split
  int32_t n_slots;   // items the split head has
  int32_t slot0;     // first slot of the split head
  // Two-level merge of a head split into many items: its slots form groups of
  // gsz consecutive slots; the last CTA of a group merges the group into a
  // group slot (gslot0 + group) and the last group's merger merges those.
  // gsz = 0: the last of the n_slots CTAs merges all slots.
  int32_t gsz;
  int32_t gslot0;    // first group slot of the head (after its n_slots item slots)
  int32_t gcnt0;     // arrival counter of the head's first group
  int32_t pad[2];
};
static_assert(sizeof(DecodeItem) == 48, "DecodeItem layout");

// A head whose decode result is split across several items.
struct alignas(16) CombineItem {
  int32_t head;
  int32_t slot_begin;
  int32_t n_slots;
  int32_t pad;
};

// One prefill work unit: one or two query tiles of the same (sequence,
// kv-head).  Tile x holds rows [q_row[x], q_row[x] + n_rows[x]) of q-head
// qh[x] at positions p0[x] ...; qh[1] < 0 when there is a single tile.  The
// KV tiles (of the kernel's tile size, counted in the head's page list) that
// any row of either tile can see are visited in [t0, t1) then [t2, t3).
struct alignas(16) PrefillItem {
  int32_t head;
  int32_t qh[2];
  int32_t q_row[2];
  int32_t n_rows[2];
  int32_t p0[2];
  int32_t t0, t1, t2, t3;
  int32_t work;  // visited KV tiles
  int32_t pad[2];
};
static_assert(sizeof(PrefillItem) == 64, "PrefillItem layout");

struct alignas(16) TableHeader {
  int32_t magic;
  int32_t version;
  int32_t n_heads;
  int32_t n_vpages;
  int32_t n_decode_items;
  int32_t n_decode_ctas;
  int32_t n_combine;
  int32_t n_prefill_items;
  int64_t off_heads, off_pages, off_decode_items, off_decode_cta, off_combine, off_prefill;
  int64_t off_free;  // spare pool section (count, then page ids)
  int32_t n_spare;
  int32_t pad;
};

}  // namespace sp

// The plan: a host copy of the problem plus the table blob.
struct sp_plan {
  sp_problem prob{};                      // pointers inside are cleared after copying
  std::vector<int32_t> ctx_len, q_start;
  std::vector<sp_head_policy> policy;
  std::vector<sp_segment> segments;       // per head: its runs of stored positions, flattened
  std::vector<int32_t> seg_begin;         // [n_heads + 1]
  std::vector<std::vector<uint8_t>> kept_blocks;  // per head: kept blocks of a retrieval head, else empty
  std::vector<sp::HeadDesc> heads;
  std::vector<sp::PageDesc> pages;
  std::vector<sp::DecodeItem> decode_items;
  std::vector<int32_t> decode_cta_begin;  // [n_ctas + 1] item ranges per CTA
  std::vector<sp::CombineItem> combine;
  std::vector<sp::PrefillItem> prefill;
  std::vector<uint8_t> blob;              // header + arrays, 256-byte aligned sections
  sp::TableHeader hdr{};
  sp_sizes sizes{};
  int32_t group = 1;
  int32_t elem_bytes = 4;                 // bytes of a Q / K / V / O element (dense inputs)
  bool fp8 = false;                       // pages hold E4M3 codes
  float k_scale = 1.f, v_scale = 1.f;     // E4M3 page scales
  int32_t prefill_tile = 0;
  int32_t n_partial_slots = 0;
  int32_t n_counters = 0;      // arrival counters in the workspace (split heads, then merge groups)
  int64_t partial_offset = 0;  // workspace byte offset of the partial slots (status word, then counters)
};

namespace sp {
void set_error(const std::string& msg);
sp_status fail(sp_status st, const std::string& msg);
}  // namespace sp
