// Mask -> tile schedule (forward lists and the reverse lists for backward).
//
// For every (query tile, KV-head slot) the list of key tiles with at least
// one visible pair, flagged full or partial; for every key tile the reverse
// list of query tiles (a counting-sort "reverse CSR"; page "Attention Sink,
// Learnable Sink and dsink", section 10, describes a backward split by KV
// block over such reverse lists).  All integer work, deterministic contents.
#include "internal.h"
#include "plan.cuh"

namespace sk {

struct PlanArgs {
  int* plan;
  const int* cu;
  const int* bi;
  int* status;
  int n_seq, T_tot, Hkv, tile, kh_slots, cap_tiles, cap_items, cap_entries;
  int causal, n_sink, window, n_qblk, max_blocks;
  int off_tile_base, off_fwd_items, off_fwd_order, off_fwd_entries;
  int off_bwd_items, off_bwd_order, off_bwd_entries, off_bwd_cursor;
  int cap_units, off_bwd_units, off_bwd_unit_order, off_unit_base;
};

constexpr int kScanThreads = 1024;
constexpr int kLptBins = 4096;

// Block-wide exclusive scan of one int per thread (kScanThreads threads).
__device__ int block_excl_scan(int v, int* warp_tot, int* total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_tot[w] = x;
  __syncthreads();
  if (w == 0) {
    int t = (lane < kScanThreads / 32) ? warp_tot[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += y;
    }
    warp_tot[lane] = t;  // inclusive warp prefix
  }
  __syncthreads();
  const int excl = x - v + (w > 0 ? warp_tot[w - 1] : 0);
  *total = warp_tot[kScanThreads / 32 - 1];
  __syncthreads();
  return excl;
}

__device__ __forceinline__ PlanHdr* hdr(const PlanArgs& a) {
  return reinterpret_cast<PlanHdr*>(a.plan);
}

// Sequence owning global tile tg (binary search over tile_base).
__device__ __forceinline__ int seq_of_tile(const int* tile_base, int n_seq, int tg) {
  int lo = 0, hi = n_seq - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (tile_base[mid] <= tg) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// A: per-sequence tile prefix, validation of cu_seqlens, header counters.
__global__ void __launch_bounds__(kScanThreads) plan_tiles_kernel(PlanArgs a, PlanHdr h0) {
  __shared__ int warp_tot[32];
  __shared__ int carry;
  int* tile_base = a.plan + a.off_tile_base;
  if (threadIdx.x < kHdrWords) a.plan[threadIdx.x] = reinterpret_cast<const int*>(&h0)[threadIdx.x];
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  for (int base = 0; base < a.n_seq; base += kScanThreads) {
    const int s = base + threadIdx.x;
    int nt = 0;
    if (s < a.n_seq) {
      const int st = a.cu[s], en = a.cu[s + 1];
      if (en < st || st < 0 || en > a.T_tot || (s == 0 && st != 0) ||
          (s == a.n_seq - 1 && en != a.T_tot)) {
        set_status(a.status, SINKATTN_ERR_BOUNDS);
      } else {
        nt = (en - st + a.tile - 1) / a.tile;
      }
    }
    int total;
    const int ex = block_excl_scan(nt, warp_tot, &total);
    if (s < a.n_seq) tile_base[s] = carry + ex;
    __syncthreads();
    if (threadIdx.x == 0) carry += total;
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    int n_tiles = carry;
    if (n_tiles > a.cap_tiles) {  // cannot happen for valid cu_seqlens
      set_status(a.status, SINKATTN_ERR_BOUNDS);
      n_tiles = a.cap_tiles;
    }
    if (a.bi && n_tiles != a.n_qblk) set_status(a.status, SINKATTN_ERR_BOUNDS);
    tile_base[a.n_seq] = n_tiles;
    PlanHdr* h = hdr(a);
    h->n_tiles = n_tiles;
    h->n_fwd_items = 0;
    h->n_bwd_items = 0;
    h->n_entries = 0;
  }
}

// The forward list of one item, written in ascending key-tile order to `out`
// (if non-null); returns its length.
__device__ int item_list(const PlanArgs& a, int kh, int tg, int s, int* out) {
  const int* tile_base = a.plan + a.off_tile_base;
  const int st = a.cu[s], len = a.cu[s + 1] - st;
  const int qt = tg - tile_base[s];
  const int q0 = qt * a.tile;
  const int qlen = min(a.tile, len - q0);
  const int n_kt = (len + a.tile - 1) / a.tile;
  int n = 0;
  if (!a.bi) {
    for (int kt = 0; kt < n_kt; ++kt) {
      const int c = classify_tile(q0, qlen, kt * a.tile, a.tile, len, a.causal, a.n_sink, a.window);
      if (c) {
        if (out) out[n] = (kt << 1) | (c == 1 ? 1 : 0);
        ++n;
      }
    }
    return n;
  }
  if (tg >= a.n_qblk) return 0;
  const int* row = a.bi + ((long long)kh * a.n_qblk + tg) * a.max_blocks;
  int kept[32];
  for (int e = 0; e < a.max_blocks; ++e) {
    const int b = row[e];
    if (b == -1) continue;
    if (b < -1 || b >= n_kt) {
      set_status(a.status, SINKATTN_ERR_BOUNDS);
      continue;
    }
    bool dup = false;
    for (int f = 0; f < e; ++f) dup |= (row[f] == b);
    if (dup) continue;
    const int c = classify_tile(q0, qlen, b * a.tile, a.tile, len, a.causal, a.n_sink, a.window);
    if (!c) continue;
    // insertion into the ascending list
    int v = (b << 1) | (c == 1 ? 1 : 0), p = n;
    while (p > 0 && kept[p - 1] > v) { kept[p] = kept[p - 1]; --p; }
    kept[p] = v;
    ++n;
  }
  if (out)
    for (int e = 0; e < n; ++e) out[e] = kept[e];
  return n;
}

// B: count entries of every forward item and fill its fields.
__global__ void plan_fwd_count_kernel(PlanArgs a) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= a.cap_items) return;
  const int* tile_base = a.plan + a.off_tile_base;
  const int n_tiles = tile_base[a.n_seq];
  TileItem* items = reinterpret_cast<TileItem*>(a.plan + a.off_fwd_items);
  const int kh = i / a.cap_tiles, tg = i % a.cap_tiles;
  TileItem it{};
  it.entry_len = -1;  // marks an unused slot
  if (tg < n_tiles) {
    const int s = seq_of_tile(tile_base, a.n_seq, tg);
    const int st = a.cu[s], len = a.cu[s + 1] - st;
    const int qt = tg - tile_base[s];
    it.tile_start = qt * a.tile;
    it.tile_len = min(a.tile, len - it.tile_start);
    it.seq_start = st;
    it.seq_len = len;
    it.kvh = a.bi ? kh : -1;
    it.tile_global = tg;
    it.entry_len = item_list(a, kh, tg, s, nullptr);
  }
  items[i] = it;
}

// C/E: offsets of every list (exclusive scan in item order) and the
// longest-first order of the valid items (counting sort on the length).
__global__ void __launch_bounds__(kScanThreads) plan_offsets_kernel(PlanArgs a, int bwd) {
  __shared__ int warp_tot[32];
  __shared__ int carry, n_valid;
  __shared__ int hist[kLptBins];
  TileItem* items = reinterpret_cast<TileItem*>(a.plan + (bwd ? a.off_bwd_items : a.off_fwd_items));
  int* order = a.plan + (bwd ? a.off_bwd_order : a.off_fwd_order);
  for (int b = threadIdx.x; b < kLptBins; b += kScanThreads) hist[b] = 0;
  if (threadIdx.x == 0) { carry = 0; n_valid = 0; }
  __syncthreads();
  for (int base = 0; base < a.cap_items; base += kScanThreads) {
    const int i = base + threadIdx.x;
    int len = 0, valid = 0;
    if (i < a.cap_items) {
      len = items[i].entry_len;
      valid = len >= 0;
      if (!valid) len = 0;
    }
    int total;
    const int ex = block_excl_scan(len, warp_tot, &total);
    if (i < a.cap_items) {
      items[i].entry_off = carry + ex;
      if (valid) {
        atomicAdd(&hist[kLptBins - 1 - min(len, kLptBins - 1)], 1);
        atomicAdd(&n_valid, 1);
      }
    }
    __syncthreads();
    if (threadIdx.x == 0) carry += total;
    __syncthreads();
  }
  // descending-length bins are stored in reverse, so an ascending exclusive
  // scan of hist gives the first slot of every length
  __shared__ int bin_carry;
  if (threadIdx.x == 0) bin_carry = 0;
  __syncthreads();
  for (int base = 0; base < kLptBins; base += kScanThreads) {
    const int b = base + threadIdx.x;
    const int v = hist[b];
    int total;
    const int ex = block_excl_scan(v, warp_tot, &total);
    hist[b] = bin_carry + ex;
    __syncthreads();
    if (threadIdx.x == 0) bin_carry += total;
    __syncthreads();
  }
  for (int i = threadIdx.x; i < a.cap_items; i += kScanThreads) {
    const int len = items[i].entry_len;
    if (len < 0) continue;
    const int pos = atomicAdd(&hist[kLptBins - 1 - min(len, kLptBins - 1)], 1);
    order[pos] = i;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    PlanHdr* h = hdr(a);
    if (bwd) h->n_bwd_items = n_valid; else h->n_fwd_items = n_valid;
    h->n_entries = carry;
    if (carry > a.cap_entries) set_status(a.status, SINKATTN_ERR_BOUNDS);
  }
}

// D: write forward entries; count the reverse lists.
__global__ void plan_fwd_fill_kernel(PlanArgs a) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= a.cap_items) return;
  const TileItem it = reinterpret_cast<const TileItem*>(a.plan + a.off_fwd_items)[i];
  if (it.entry_len <= 0) return;
  if (it.entry_off + it.entry_len > a.cap_entries) return;
  const int* tile_base = a.plan + a.off_tile_base;
  const int kh = i / a.cap_tiles, tg = i % a.cap_tiles;
  const int s = seq_of_tile(tile_base, a.n_seq, tg);
  int* out = a.plan + a.off_fwd_entries + it.entry_off;
  const int n = item_list(a, kh, tg, s, out);
  TileItem* bitems = reinterpret_cast<TileItem*>(a.plan + a.off_bwd_items);
  for (int e = 0; e < n; ++e) {
    const int kt = out[e] >> 1;
    const int b = kh * a.cap_tiles + tile_base[s] + kt;
    atomicAdd(&bitems[b].entry_len, 1);
  }
}

// Before E: reverse items' fields, entry_len reset to 0 for valid tiles.
__global__ void plan_bwd_init_kernel(PlanArgs a) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= a.cap_items) return;
  const int* tile_base = a.plan + a.off_tile_base;
  const int n_tiles = tile_base[a.n_seq];
  TileItem* items = reinterpret_cast<TileItem*>(a.plan + a.off_bwd_items);
  const int kh = i / a.cap_tiles, tg = i % a.cap_tiles;
  TileItem it{};
  it.entry_len = -1;
  if (tg < n_tiles) {
    const int s = seq_of_tile(tile_base, a.n_seq, tg);
    const int st = a.cu[s], len = a.cu[s + 1] - st;
    const int kt = tg - tile_base[s];
    it.tile_start = kt * a.tile;
    it.tile_len = min(a.tile, len - it.tile_start);
    it.seq_start = st;
    it.seq_len = len;
    it.kvh = a.bi ? kh : -1;
    it.tile_global = tg;
    it.entry_len = 0;
  }
  items[i] = it;
}

// F: scatter forward entries into the reverse lists.
__global__ void plan_bwd_scatter_kernel(PlanArgs a) {
  // one warp per forward item, lanes over its entries
  const int i = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (i >= a.cap_items) return;
  const TileItem it = reinterpret_cast<const TileItem*>(a.plan + a.off_fwd_items)[i];
  if (it.entry_len <= 0 || it.entry_off + it.entry_len > a.cap_entries) return;
  const int* tile_base = a.plan + a.off_tile_base;
  const int kh = i / a.cap_tiles, tg = i % a.cap_tiles;
  const int s = seq_of_tile(tile_base, a.n_seq, tg);
  const int qt = tg - tile_base[s];
  const int* ent = a.plan + a.off_fwd_entries + it.entry_off;
  const TileItem* bitems = reinterpret_cast<const TileItem*>(a.plan + a.off_bwd_items);
  int* cursor = a.plan + a.off_bwd_cursor;
  int* bent = a.plan + a.off_bwd_entries;
  for (int e = lane; e < it.entry_len; e += 32) {
    const int kt = ent[e] >> 1, partial = ent[e] & 1;
    const int b = kh * a.cap_tiles + tile_base[s] + kt;
    const int pos = bitems[b].entry_off + atomicAdd(&cursor[b], 1);
    if (pos < a.cap_entries) bent[pos] = (qt << 1) | partial;
  }
}

__global__ void plan_zero_kernel(int* p, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) p[i] = 0;
}

// H: backward work units.  One CTA scans the per-item unit counts (item
// order), then every item writes its units, then the launch order is set
// (item order).
__global__ void __launch_bounds__(kScanThreads) plan_units_scan_kernel(PlanArgs a) {
  __shared__ int warp_tot[32];
  __shared__ int carry;
  const TileItem* items = reinterpret_cast<const TileItem*>(a.plan + a.off_bwd_items);
  int* base = a.plan + a.off_unit_base;
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  for (int b0 = 0; b0 < a.cap_items; b0 += kScanThreads) {
    const int i = b0 + threadIdx.x;
    int n = 0;
    if (i < a.cap_items) {
      const int len = items[i].entry_len;
      n = len < 0 ? 0 : bwd_units_of(len);
    }
    int total;
    const int ex = block_excl_scan(n, warp_tot, &total);
    if (i < a.cap_items) base[i] = carry + ex;
    __syncthreads();
    if (threadIdx.x == 0) carry += total;
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    hdr(a)->n_bwd_units = carry;
    if (carry > a.cap_units) set_status(a.status, SINKATTN_ERR_BOUNDS);
  }
}

__global__ void plan_units_fill_kernel(PlanArgs a) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= a.cap_items) return;
  const TileItem it = reinterpret_cast<const TileItem*>(a.plan + a.off_bwd_items)[i];
  if (it.entry_len < 0) return;
  const int n = bwd_units_of(it.entry_len);
  const int b = a.plan[a.off_unit_base + i];
  int4* units = reinterpret_cast<int4*>(a.plan + a.off_bwd_units);
  // near-equal parts: unit c takes entries [c len / n, (c + 1) len / n)
  for (int c = 0; c < n && b + c < a.cap_units; ++c) {
    const int first = (int)((long long)c * it.entry_len / n);
    const int last = (int)((long long)(c + 1) * it.entry_len / n);
    units[b + c] = make_int4(i, first, max(last - first, 0), n);
  }
}

__global__ void plan_units_order_kernel(PlanArgs a) {
  // item order: units of one (KV-head slot, sequence) are consecutive
  const int n_units = min(hdr(a)->n_bwd_units, a.cap_units);
  int* order = a.plan + a.off_bwd_unit_order;
  for (int u = blockIdx.x * blockDim.x + threadIdx.x; u < n_units; u += gridDim.x * blockDim.x)
    order[u] = u;
}

// G: sort every reverse list by query tile, latest first.  One warp per
// item: a list of at most kSortShared entries is staged in shared memory and
// every entry goes straight to its rank (the entries it must follow: larger
// values, and equal values earlier in the list); a longer list is sorted in
// place by one lane (insertion sort).
constexpr int kSortShared = 256;
constexpr int kSortWarps = 8;
__global__ void __launch_bounds__(kSortWarps * 32) plan_bwd_sort_kernel(PlanArgs a) {
  __shared__ int buf[kSortWarps][kSortShared];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int i = blockIdx.x * kSortWarps + warp;
  if (i >= a.cap_items) return;  // uniform over the warp
  const TileItem it = reinterpret_cast<const TileItem*>(a.plan + a.off_bwd_items)[i];
  if (it.entry_len <= 1 || it.entry_off + it.entry_len > a.cap_entries) return;
  int* e = a.plan + a.off_bwd_entries + it.entry_off;
  const int n = it.entry_len;
  if (n <= kSortShared) {
    int* w = buf[warp];
    for (int x = lane; x < n; x += 32) w[x] = e[x];
    __syncwarp();
    for (int x = lane; x < n; x += 32) {
      const int v = w[x];
      int rank = 0;
      for (int y = 0; y < n; ++y) {
        const int u = w[y];
        rank += (u > v) || (u == v && y < x);
      }
      e[rank] = v;
    }
    return;
  }
  if (lane == 0) {
    for (int x = 1; x < n; ++x) {
      const int v = e[x];
      int p = x;
      while (p > 0 && e[p - 1] < v) { e[p] = e[p - 1]; --p; }
      e[p] = v;
    }
  }
}

int launch_plan(const PlanLaunch& L, cudaStream_t stream) {
  const PlanSizes& z = L.sizes;
  PlanArgs a{};
  a.plan = static_cast<int*>(L.plan);
  a.cu = L.cu_seqlens;
  a.bi = L.block_indices;
  a.status = L.status;
  a.n_seq = L.n_seq;
  a.T_tot = L.T_tot;
  a.Hkv = L.Hkv;
  a.tile = z.tile;
  a.kh_slots = z.kh_slots;
  a.cap_tiles = z.cap_tiles;
  a.cap_items = z.cap_items;
  a.cap_entries = z.cap_entries;
  a.causal = L.causal;
  a.n_sink = L.n_sink;
  a.window = L.window;
  a.n_qblk = L.n_qblk;
  a.max_blocks = L.max_blocks;
  a.off_tile_base = z.off_tile_base;
  a.off_fwd_items = z.off_fwd_items;
  a.off_fwd_order = z.off_fwd_order;
  a.off_fwd_entries = z.off_fwd_entries;
  a.off_bwd_items = z.off_bwd_items;
  a.off_bwd_order = z.off_bwd_order;
  a.off_bwd_entries = z.off_bwd_entries;
  a.off_bwd_cursor = z.off_bwd_cursor;
  a.cap_units = z.cap_units;
  a.off_bwd_units = z.off_bwd_units;
  a.off_bwd_unit_order = z.off_bwd_unit_order;
  a.off_unit_base = z.off_unit_base;

  // header scalars known on the host (written by the first kernel)
  PlanHdr h{};
  h.magic = kPlanMagic;
  h.tile = z.tile;
  h.kh_slots = z.kh_slots;
  h.T_tot = L.T_tot;
  h.Hkv = L.Hkv;
  h.n_seq = L.n_seq;
  h.cap_tiles = z.cap_tiles;
  h.cap_items = z.cap_items;
  h.cap_entries = z.cap_entries;
  h.fingerprint = L.fingerprint;
  h.off_tile_base = z.off_tile_base;
  h.off_fwd_items = z.off_fwd_items;
  h.off_fwd_order = z.off_fwd_order;
  h.off_fwd_entries = z.off_fwd_entries;
  h.off_bwd_items = z.off_bwd_items;
  h.off_bwd_order = z.off_bwd_order;
  h.off_bwd_entries = z.off_bwd_entries;
  h.off_bwd_cursor = z.off_bwd_cursor;
  h.total_words = z.total_words;
  h.cap_units = z.cap_units;
  h.off_bwd_units = z.off_bwd_units;
  h.off_bwd_unit_order = z.off_bwd_unit_order;
  h.off_unit_base = z.off_unit_base;
  const int nb = (z.cap_items + 255) / 256;
  plan_tiles_kernel<<<1, kScanThreads, 0, stream>>>(a, h);
  plan_fwd_count_kernel<<<nb, 256, 0, stream>>>(a);
  plan_offsets_kernel<<<1, kScanThreads, 0, stream>>>(a, 0);
  plan_bwd_init_kernel<<<nb, 256, 0, stream>>>(a);
  plan_fwd_fill_kernel<<<nb, 256, 0, stream>>>(a);
  plan_offsets_kernel<<<1, kScanThreads, 0, stream>>>(a, 1);
  plan_zero_kernel<<<nb, 256, 0, stream>>>(a.plan + a.off_bwd_cursor, z.cap_items);
  plan_bwd_scatter_kernel<<<(unsigned)(((long long)z.cap_items * 32 + 255) / 256), 256, 0, stream>>>(a);
  plan_bwd_sort_kernel<<<(z.cap_items + kSortWarps - 1) / kSortWarps, kSortWarps * 32, 0, stream>>>(a);
  plan_units_scan_kernel<<<1, kScanThreads, 0, stream>>>(a);
  plan_units_fill_kernel<<<nb, 256, 0, stream>>>(a);
  plan_units_order_kernel<<<(z.cap_units + 255) / 256, 256, 0, stream>>>(a);
  return cudaGetLastError() == cudaSuccess ? SINKATTN_OK : SINKATTN_ERR_CUDA;
}

}  // namespace sk
