// Tile schedule ("plan") layout and the mask predicates the kernels share.
//
// The mask (page "Attention Sink, Learnable Sink and dsink", section 2: block
// selection, window, causality and sample boundaries restrict the visible
// set) is turned once into explicit tile lists so no kernel visits a fully
// masked tile.  Tiles are square (tile x tile) and sequence-local.
//
// Plan buffer = int32 words:
//   [0, kHdrWords)       header (PlanHdr)
//   tile_base[n_seq+1]   first global tile number of each sequence
//   fwd_items[cap_items] TileItem, forward: one per (query tile, KV-head slot)
//   fwd_order[cap_items] forward items, longest list first
//   fwd_entries[cap_entries]  (key tile << 1) | partial
//   bwd_items / bwd_order / bwd_entries: the reverse lists (per key tile, the
//                        query tiles that see it), entries (query tile << 1) |
//                        partial, each list latest query tile first (the
//                        CTAs of one sequence and KV head then read the
//                        same query tiles at about the same time, so the
//                        second and later reads hit L2)
//   bwd_cursor[cap_items] scratch for the reverse scatter
//   bwd_units[cap_units][4] backward work units: (bwd item, first entry,
//                        entry count, number of units of that item); a
//                        reverse list longer than kBwdChunk entries is split
//                        into near-equal parts, so no single CTA serialises a
//                        very popular key tile and no unit is much longer
//                        than the others
//   bwd_unit_order[cap_units] units in item order: (KV-head slot, sequence,
//                        key tile), so the units of one sequence and KV head
//                        -- which reduce into the same dQ tiles and read the
//                        same Q/dO tiles -- run at about the same time and
//                        find those tiles in L2
//   unit_base[cap_items] first unit of every bwd item
// With no block_indices the lists do not depend on the KV head: one slot
// (kvh = -1) serves every KV head.
#pragma once
#include <stdint.h>

namespace sk {

constexpr int kPlanMagic = 0x534b4150;  // 'SKAP'
constexpr int kHdrWords = 32;
constexpr int kBwdChunk = 16;  // most reverse-list entries per backward work unit

struct PlanHdr {
  int magic;
  int n_fwd_items;    // device-written: valid items in fwd_order
  int n_bwd_items;    // device-written
  int n_tiles;        // device-written: sum over sequences of ceil(len / tile)
  int tile;
  int kh_slots;       // 1 (lists shared by all KV heads) or Hkv
  int T_tot, Hkv, n_seq;
  int cap_tiles, cap_items, cap_entries;
  int n_entries;      // device-written
  int fingerprint;    // hash of the problem scalars (host)
  int off_tile_base, off_fwd_items, off_fwd_order, off_fwd_entries;
  int off_bwd_items, off_bwd_order, off_bwd_entries, off_bwd_cursor;
  int total_words;
  int n_bwd_units;    // device-written
  int cap_units;
  int off_bwd_units, off_bwd_unit_order, off_unit_base;
  int pad[kHdrWords - 28];
};
static_assert(sizeof(PlanHdr) == kHdrWords * 4, "plan header size");

struct TileItem {
  int tile_start;  // sequence-local first token of this tile
  int tile_len;    // valid tokens in this tile (<= tile)
  int seq_start;   // global index of the sequence's first token
  int seq_len;
  int kvh;         // KV head, or -1 = the list serves every KV head
  int entry_off;   // first entry (word index relative to the entries array)
  int entry_len;
  int tile_global; // global tile number
};
static_assert(sizeof(TileItem) == 32, "tile item size");

// Element-level visibility inside a tile (sequence-local positions).
__host__ __device__ __forceinline__ bool visible_elem(int qi, int kj, int seq_len, int causal,
                                                      int n_sink, int window) {
  if (kj >= seq_len) return false;
  if (causal && kj > qi) return false;
  if (window > 0 && !(kj < n_sink || qi - kj < window)) return false;
  return true;
}

// The visible columns c of one query row inside a tile that starts at key
// k0 (sequence-local): c <= hi and (c >= lo or c < ns).  hi is the causal /
// sequence-end bound, lo the window's lower bound (-1 without a window), ns
// the end of the sink prefix (0 without a window).  Same set as visible_elem.
struct RowSpan {
  int lo, hi, ns;
};
__host__ __device__ __forceinline__ RowSpan row_span(int qi, int k0, int seq_len, int causal,
                                                     int n_sink, int window) {
  int last = seq_len - 1;
  if (causal && qi < last) last = qi;
  RowSpan s;
  s.hi = last - k0;
  s.lo = window > 0 ? qi - window + 1 - k0 : -1;
  s.ns = window > 0 ? n_sink - k0 : 0;
  return s;
}
__host__ __device__ __forceinline__ bool span_visible(const RowSpan& s, int c) {
  return c <= s.hi && (c >= s.lo || c < s.ns);
}

// The query tokens t of a tile starting at q0 that see key kj: lo <= t <= hi
// (qi >= kj when causal; past the sink prefix, qi <= kj + window - 1; a key
// past the sequence is seen by none).  Same set as visible_elem.
struct KeySpan {
  int lo, hi;
};
__host__ __device__ __forceinline__ KeySpan key_span(int kj, int q0, int seq_len, int causal,
                                                     int n_sink, int window) {
  constexpr int kFar = 1 << 29;
  KeySpan s;
  s.lo = (causal ? kj : -kFar) - q0;
  s.hi = kj >= seq_len ? -kFar
       : (window > 0 && kj >= n_sink ? kj + window - 1 - q0 : kFar);
  return s;
}

// A StreamingLLM band's first key tile, seen from a query tile whose every
// row's window starts past that tile: only the n_sink <= 16 sink keys of it
// are visible, so a 16-key slice of the tile carries all of its work.
__host__ __device__ __forceinline__ bool sink_only_tile(int key_tile, int q_tile_start, int tile,
                                                        int n_sink, int window) {
  return key_tile == 0 && window > 0 && n_sink > 0 && n_sink <= 16 &&
         q_tile_start - window + 1 >= tile;
}

// Tile classification from the interval bounds (no enumeration):
// 0 = no visible pair, 1 = some, 2 = every (valid row, tile column) pair.
// Rows are [q0, q0 + qlen); columns [k0, k0 + tile), keys past seq_len are
// not visible.  Block selection is applied by the caller (tiles = blocks).
__host__ __device__ __forceinline__ int classify_tile(int q0, int qlen, int k0, int tile,
                                                      int seq_len, int causal, int n_sink,
                                                      int window) {
  if (k0 >= seq_len || qlen <= 0) return 0;
  const int q1 = q0 + qlen;
  const int k1 = (k0 + tile < seq_len) ? k0 + tile : seq_len;
  bool any;
  if (!causal) {
    any = true;
  } else if (window <= 0) {
    any = (k0 <= q1 - 1);
  } else {
    const bool sink_any = (k0 < n_sink) && (k0 <= q1 - 1);
    const bool win_any = ((q1 - 1) - k0 >= 0) && (q0 - (k1 - 1) <= window - 1);
    any = sink_any || win_any;
  }
  if (!any) return 0;
  bool full = (k0 + tile <= seq_len);
  if (causal) full = full && (k1 - 1 <= q0);
  if (window > 0 && k1 > n_sink) {
    const int jlo = k0 > n_sink ? k0 : n_sink;
    full = full && ((q1 - 1) - jlo <= window - 1);
  }
  return full ? 2 : 1;
}

// Host-side sizes of the plan for a problem.
struct PlanSizes {
  int tile, kh_slots, cap_tiles, cap_items, cap_entries, max_list, cap_units;
  int off_tile_base, off_fwd_items, off_fwd_order, off_fwd_entries;
  int off_bwd_items, off_bwd_order, off_bwd_entries, off_bwd_cursor;
  int off_bwd_units, off_bwd_unit_order, off_unit_base, total_words;
};

__host__ __device__ __forceinline__ int bwd_units_of(int entry_len) {
  return entry_len <= kBwdChunk ? 1 : (entry_len + kBwdChunk - 1) / kBwdChunk;
}

inline PlanSizes plan_sizes(int T_tot, int Hkv, int n_seq, int max_seqlen, bool sparse,
                            int block, int max_blocks) {
  PlanSizes s{};
  s.tile = sparse ? block : 128;
  s.kh_slots = sparse ? Hkv : 1;
  const long long cap_tiles = (long long)T_tot / s.tile + n_seq;
  const long long max_kt = ((long long)max_seqlen + s.tile - 1) / s.tile;
  long long per_item = sparse ? (max_blocks < max_kt ? max_blocks : max_kt) : max_kt;
  if (per_item < 1) per_item = 1;
  s.cap_tiles = (int)cap_tiles;
  s.cap_items = (int)(cap_tiles * s.kh_slots);
  long long cap_entries = (long long)s.cap_items * per_item;
  s.cap_entries = (int)cap_entries;
  s.max_list = (int)(max_kt > per_item ? max_kt : per_item);
  long long off = kHdrWords;
  auto take = [&](long long words) {
    long long o = off;
    off += (words + 3) & ~3LL;  // keep 16-byte alignment of every array
    return (int)o;
  };
  s.off_tile_base = take(n_seq + 1);
  s.off_fwd_items = take((long long)s.cap_items * 8);
  s.off_fwd_order = take(s.cap_items);
  s.off_fwd_entries = take(s.cap_entries);
  s.off_bwd_items = take((long long)s.cap_items * 8);
  s.off_bwd_order = take(s.cap_items);
  s.off_bwd_entries = take(s.cap_entries);
  s.off_bwd_cursor = take(s.cap_items);
  s.cap_units = (int)((long long)s.cap_items + cap_entries / kBwdChunk + 1);
  s.off_bwd_units = take((long long)s.cap_units * 4);
  s.off_bwd_unit_order = take(s.cap_units);
  s.off_unit_base = take(s.cap_items);
  s.total_words = (int)off;
  return s;
}

}  // namespace sk
