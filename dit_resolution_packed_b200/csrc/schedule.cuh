// schedule.cuh -- device-side segment scheduler for the packed attention kernel.
//
// One CTA of 256 threads turns cu_seqlens into the work list of the attention
// kernel, without a host round trip:
//   1. validates cu_seqlens (cu[0] = 0, non-decreasing, cu[B] = T, every
//      segment <= max_seqlen); on failure it records the status and publishes
//      an empty work list;
//   2. (forward, short-segment packing on) packs runs of consecutive short
//      segments (at most 128 tokens each) into shared 128-row tiles, two tiles
//      per unit (see "Short-segment groups" below); every other non-empty
//      segment is a unit of its own;
//   3. orders the units longest-first (stable counting sort on the number of
//      128-key tiles a query tile of the unit meets, i.e. on the per-item cost),
//      so a persistent grid takes the big items first (longest-processing-time
//      order);
//   4. publishes, in that order, the first work-item index of every unit; a
//      segment of L tokens holds heads * ceil(L / 2^rows_log2) items: for the
//      forward (rows_log2 = 8) one per (head, pair of 128-row query tiles), for
//      the backward (rows_log2 = 7) one per (head, 128-key tile); a group of
//      short segments holds one item per head;
//   5. for the forward, writes three tensor maps per unit (q, k, v) whose base
//      is the unit's first token and whose row extent is its token count, so
//      that every TMA tile stops at the unit's end: loads past it read zeros and
//      no tile touches an image outside the unit (maps == nullptr skips this
//      step); the FP8 variant's transposed V map is cut along its key axis;
//   6. records the tile ledger of the call: 128 x 128 score tiles computed and
//      useful (query, key) pairs, over all heads.
//
// Short-segment groups.  A segment of L <= 128 tokens alone would occupy a whole
// 128-row query tile and a whole 128-key tile, most of it masked.  Consecutive
// short segments are instead cut greedily, in packing order, into tiles of at most
// 128 tokens that hold whole segments; two neighbouring tiles form one unit (a
// contiguous token range [beg, beg + len) split at n0: tile 0 = [beg, beg + n0),
// tile 1 = [beg + n0, beg + len)).  Inside a tile the mask is block-diagonal: a
// query row sees only the keys of its own segment, which lie in its own tile, so
// tile t meets only key tile t.  A unit that would hold a single segment leaves that
// segment alone (one tile of its own: nothing to share).  To walk the runs in parallel, a run is also cut
// where a segment starts in a later 1024-token block of the stream than the one
// before it (at most one part-filled tile per 1024 tokens); each warp walks its
// own parts.
//
// The mask of the method (Mage-Flow page, "Packing + Flash Attention varlen":
// images attend only to themselves, no padding) is thereby carried entirely by
// the tensor-map bounds plus the key mask of each segment's last tile (of each
// row's own segment inside a group tile).
#pragma once
#include <cuda.h>

#include <cstdint>

#include "sm100_ptx.cuh"

namespace pa {

constexpr int kSchedThreads = 256;
constexpr int kSortBuckets = 1024;     // tile counts >= 1023 share the first bucket
constexpr int kCuInSmem = 4096 + 1;    // cu_seqlens staged in shared memory up to this many entries
constexpr int kGroupRows = 128;        // tokens of one tile of a short-segment group
constexpr int kGroupBlockLog2 = 10;    // runs of short segments are also cut at 1024-token blocks

// Unit descriptor of segment i (SchedParams::info): a group head stores its tile
// split n0 and token count len as n0 | len << 9 (both <= 256); kUnitAlone marks a
// segment that is a unit by itself, kUnitNone one that is empty or inside a group.
constexpr int32_t kUnitAlone = -1;
constexpr int32_t kUnitNone = -2;
__host__ __device__ constexpr int32_t group_info(int32_t n0, int32_t len) { return n0 | (len << 9); }
__host__ __device__ constexpr int32_t group_n0(int32_t info) { return info & 0x1ff; }
__host__ __device__ constexpr int32_t group_len(int32_t info) { return (info >> 9) & 0x1ff; }

struct SchedParams {
  CUtensorMap tmpl[3];     // q, k, v over the whole [T, H*d] matrix (host-encoded)
  const void* base[3];     // q, k, v base pointers
  const int32_t* cu;       // [B+1]
  int32_t* status;         // status word
  int32_t* counts;         // [0] = work items, [1] = units, [2] = work counter (zeroed)
  int32_t* order;          // [B] unit ids (a unit's first segment), longest first
  int32_t* item_start;     // [B+1] first item of each ordered unit
  uint8_t* maps;           // [B][3] tensor maps, 128 bytes each (nullptr: none); unit i uses slot i
  int32_t* info;           // [B] unit descriptor per segment (nullptr: every non-empty segment is a unit)
  int64_t* stats;          // [4] tile ledger: score tiles, useful pairs, groups, grouped segments
  uint64_t row_bytes;      // H * d * 2
  int32_t batch, total, heads, max_seqlen;
  int32_t rows_log2;        // rows of a work item: 2^rows_log2 (8 forward, 7 backward)
  // nonzero: the third map (v) is over a [channels][keys] matrix whose segment s
  // starts at key 16*ceil(cu[s]/16) + 16*s (the FP8 variant's transposed V); its
  // per-segment map moves the base to that key and sets the key extent to L
  int32_t v_keys_inner;
  int32_t err_cu, err_max;  // status codes to record
  int32_t group_short;      // nonzero (and info set): pack consecutive short segments into shared tiles
};

__device__ __forceinline__ int seg_key(int32_t len) {
  int t = (len + 127) >> 7;
  return t < kSortBuckets - 1 ? t : kSortBuckets - 1;
}

// Exclusive prefix sum over the threads of the block; also returns the block total.
__device__ __forceinline__ int64_t block_exclusive_scan(int64_t v, int64_t* s_warp, int64_t* s_total) {
  constexpr int kWarps = kSchedThreads / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int64_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int64_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) s_warp[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int64_t w = lane < kWarps ? s_warp[lane] : 0, wx = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int64_t y = __shfl_up_sync(0xffffffffu, wx, o);
      if (lane >= o) wx += y;
    }
    if (lane < kWarps) s_warp[lane] = wx - w;
    if (lane == 31) *s_total = wx;
  }
  __syncthreads();
  int64_t r = x - v + s_warp[warp];
  __syncthreads();
  return r;
}

// ---- short-segment groups (the walk runs on validated cu_seqlens, 0 <= L_i) ----

__device__ __forceinline__ bool seg_short(const int32_t* cu, int i) { return cu[i + 1] - cu[i] <= kGroupRows; }

// Segment i > 0 starts in a later 1024-token block of the stream than segment i - 1.
__device__ __forceinline__ bool new_block(const int32_t* cu, int i) {
  return (cu[i - 1] >> kGroupBlockLog2) != (cu[i] >> kGroupBlockLog2);
}

// A walk starts at every short segment that does not continue the walk of the
// segment before it.
__device__ __forceinline__ bool walk_start(const int32_t* cu, int i) {
  return seg_short(cu, i) && (i == 0 || !seg_short(cu, i - 1) || new_block(cu, i));
}

// First segment index e in (i, B] that does not join the tile starting at segment i:
// the end of the pack, a segment that is not short or starts a new walk, or one that
// would take the tile past kGroupRows tokens.  Called by a whole warp.
__device__ __forceinline__ int tile_end(const int32_t* cu, int B, int i) {
  const int lane = threadIdx.x & 31;
  const int32_t base = cu[i];
  for (int e0 = i + 1;; e0 += 32) {
    const int j = e0 + lane;
    const bool stop = j >= B || !seg_short(cu, j) || new_block(cu, j) || cu[j + 1] - base > kGroupRows;
    const uint32_t m = __ballot_sync(0xffffffffu, stop);
    if (m) return e0 + __ffs(m) - 1;
  }
}

// Cuts the walk that starts at segment s into pairs of tiles; writes the unit
// descriptor of every segment it covers.  Called by a whole warp.
__device__ __forceinline__ void walk_groups(const int32_t* cu, int B, int s, int32_t* __restrict__ info) {
  const int lane = threadIdx.x & 31;
  for (int i = s;;) {
    const int e1 = tile_end(cu, B, i);
    int e2 = e1;
    if (e1 < B && seg_short(cu, e1) && !new_block(cu, e1)) e2 = tile_end(cu, B, e1);
    const int32_t n0 = cu[e1] - cu[i], len = cu[e2] - cu[i];
    // a group of one segment gains nothing from sharing: that segment stays a unit alone
    if (lane == 0) info[i] = len <= 0 ? kUnitNone : e2 == i + 1 ? kUnitAlone : group_info(n0, len);
    for (int j = i + 1 + lane; j < e2; j += 32) info[j] = kUnitNone;
    if (e2 >= B || !seg_short(cu, e2) || new_block(cu, e2)) break;
    i = e2;
  }
}

// Token count a unit's tensor maps cover (0: segment i is not a unit).
__device__ __forceinline__ int32_t unit_span(int32_t len, int32_t inf) {
  return inf == kUnitAlone ? len : inf == kUnitNone ? 0 : group_len(inf);
}

__global__ void __launch_bounds__(kSchedThreads, 1) schedule_kernel(const __grid_constant__ SchedParams p) {
  __shared__ int s_bad;
  __shared__ int32_t s_cu_buf[kCuInSmem];
  __shared__ int32_t s_hist[kSortBuckets];
  __shared__ int32_t s_start[kSortBuckets];
  __shared__ int32_t s_keys[kSchedThreads];
  __shared__ int32_t s_info_buf[kCuInSmem - 1];
  __shared__ int64_t s_warp[32];
  __shared__ int64_t s_total;
  __shared__ unsigned long long s_ledger[4];
  const int tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  const int B = p.batch;
  // the attention kernel may start its prologue now; it waits for this grid
  // to complete before it reads anything written here
  pdl_launch_dependents();

  // cu_seqlens in shared memory (one pass over global memory) when it fits
  const bool staged = B + 1 <= kCuInSmem;
  for (int i = tid; staged && i <= B; i += kSchedThreads) s_cu_buf[i] = p.cu[i];
  const int32_t* cu = staged ? s_cu_buf : p.cu;
  if (tid == 0) s_bad = 0;
  if (tid < 4) s_ledger[tid] = 0;
  for (int b = tid; b < kSortBuckets; b += kSchedThreads) s_hist[b] = 0;
  __syncthreads();

  // 1. validation
  if (tid == 0 && (cu[0] != 0 || cu[B] != p.total)) atomicMax(&s_bad, 2);
  for (int i = tid; i < B; i += kSchedThreads) {
    const int32_t a = cu[i], b = cu[i + 1];
    if (b < a) {
      atomicMax(&s_bad, 2);
    } else if (b - a > p.max_seqlen) {
      atomicMax(&s_bad, 1);
    }
  }
  __syncthreads();
  if (s_bad) {
    if (tid == 0) {
      atomicCAS(p.status, 0, s_bad == 2 ? p.err_cu : p.err_max);
      p.counts[0] = 0;
      p.counts[1] = 0;
      p.counts[2] = 0;
      if (p.stats)
        for (int i = 0; i < 4; ++i) p.stats[i] = 0;
    }
    return;
  }

  // 2. units: short-segment groups (each warp walks the runs that start in its
  // 32-segment chunks), every other non-empty segment alone.  The descriptors are
  // built in shared memory when the pack is staged there (copied out at the end)
  const bool grouping = p.info != nullptr && p.group_short;
  int32_t* info = staged ? s_info_buf : p.info;  // working copy (nullptr: computed on the fly)
  if (grouping) {
    for (int c0 = warp * 32; c0 < B; c0 += kSchedThreads) {
      const int i = c0 + lane;
      uint32_t m = __ballot_sync(0xffffffffu, i < B && walk_start(cu, i));
      while (m) {
        const int s = c0 + __ffs(m) - 1;
        m &= m - 1;
        walk_groups(cu, B, s, info);
      }
      if (i < B && !seg_short(cu, i)) info[i] = kUnitAlone;
    }
  } else if (info != nullptr) {
    for (int i = tid; i < B; i += kSchedThreads) info[i] = cu[i + 1] > cu[i] ? kUnitAlone : kUnitNone;
  }
  __syncthreads();
  auto unit_of = [&](int i) -> int32_t {
    if (info != nullptr) return info[i];
    return cu[i + 1] > cu[i] ? kUnitAlone : kUnitNone;
  };

  // 3. histogram of the units' sort keys, and the tile ledger
  {
    unsigned long long tiles = 0, pairs = 0, groups = 0, grouped = 0;
    for (int i = tid; i < B; i += kSchedThreads) {
      const int32_t len = cu[i + 1] - cu[i];
      const int32_t inf = unit_of(i);
      pairs += static_cast<unsigned long long>(len) * static_cast<unsigned long long>(len);
      if (len > 0 && inf != kUnitAlone) ++grouped;  // a non-empty segment inside a group
      if (inf == kUnitNone) continue;
      if (inf == kUnitAlone) {
        const unsigned long long t = static_cast<unsigned long long>((len + 127) >> 7);
        tiles += t * t;
        atomicAdd(&s_hist[seg_key(len)], 1);
      } else {
        tiles += group_len(inf) > group_n0(inf) ? 2 : 1;
        ++groups;
        atomicAdd(&s_hist[1], 1);  // a group's query tile meets one key tile
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      tiles += __shfl_xor_sync(0xffffffffu, tiles, o);
      pairs += __shfl_xor_sync(0xffffffffu, pairs, o);
      groups += __shfl_xor_sync(0xffffffffu, groups, o);
      grouped += __shfl_xor_sync(0xffffffffu, grouped, o);
    }
    if (lane == 0) {
      atomicAdd(&s_ledger[0], tiles * static_cast<unsigned long long>(p.heads));
      atomicAdd(&s_ledger[1], pairs * static_cast<unsigned long long>(p.heads));
      atomicAdd(&s_ledger[2], groups);
      atomicAdd(&s_ledger[3], grouped);
    }
  }
  __syncthreads();

  // 4. per-unit tensor maps: copy the template, then move its base and row extent
  for (int idx = tid; p.maps != nullptr && idx < 3 * B; idx += kSchedThreads) {
    const int s = idx / 3, which = idx - 3 * s;
    const int32_t beg = cu[s], len = cu[s + 1] - beg;
    const int32_t span = unit_span(len, unit_of(s));
    if (span <= 0) continue;
    uint8_t* dst = p.maps + static_cast<size_t>(idx) * 128;
    const uint4* src = reinterpret_cast<const uint4*>(&p.tmpl[which]);
#pragma unroll
    for (int w = 0; w < 8; ++w) reinterpret_cast<uint4*>(dst)[w] = src[w];
    if (which == 2 && p.v_keys_inner) {
      const uint64_t key0 = 16ull * ((static_cast<uint64_t>(beg) + 15) / 16) + 16ull * static_cast<uint64_t>(s);
      tmap_replace_address(dst, static_cast<const uint8_t*>(p.base[2]) + key0);
      tmap_replace_dim0(dst, static_cast<uint32_t>(span));
      continue;
    }
    const uint8_t* seg_base = static_cast<const uint8_t*>(p.base[which]) + static_cast<uint64_t>(beg) * p.row_bytes;
    tmap_replace_address(dst, seg_base);
    tmap_replace_dim1(dst, static_cast<uint32_t>(span));
  }

  // 5. bucket offsets in descending key order (each thread owns 4 buckets)
  {
    constexpr int per = kSortBuckets / kSchedThreads;
    int64_t local = 0;
#pragma unroll
    for (int j = 0; j < per; ++j) local += s_hist[kSortBuckets - 1 - (tid * per + j)];
    int64_t off = block_exclusive_scan(local, s_warp, &s_total);
#pragma unroll
    for (int j = 0; j < per; ++j) {
      const int b = kSortBuckets - 1 - (tid * per + j);
      s_start[b] = static_cast<int32_t>(off);
      off += s_hist[b];
      s_hist[b] = 0;  // reused below as the running count of placed units
    }
  }
  const int32_t n_sorted = static_cast<int32_t>(s_total);
  __syncthreads();

  // 6. stable placement (within a bucket units keep their packing order) and,
  // in the same pass, the first work item of every ordered unit
  for (int c0 = 0; c0 < B; c0 += kSchedThreads) {
    const int i = c0 + tid;
    int key = -1;
    if (i < B) {
      const int32_t len = cu[i + 1] - cu[i];
      const int32_t inf = unit_of(i);
      if (inf == kUnitAlone) key = seg_key(len);
      else if (inf != kUnitNone) key = 1;
    }
    s_keys[tid] = key;
    __syncthreads();
    if (key >= 0) {
      int rank = 0;
      for (int j = 0; j < tid; ++j) rank += (s_keys[j] == key);
      p.order[s_start[key] + s_hist[key] + rank] = i;
    }
    __syncthreads();
    if (key >= 0) atomicAdd(&s_hist[key], 1);
    __syncthreads();
  }
  __threadfence_block();
  __syncthreads();

  int64_t carry = 0;
  for (int c0 = 0; c0 < n_sorted; c0 += kSchedThreads) {
    const int k = c0 + tid;
    int64_t items = 0;
    if (k < n_sorted) {
      const int s = p.order[k];
      const int32_t len = cu[s + 1] - cu[s];
      const int32_t inf = unit_of(s);
      items = inf == kUnitAlone
                  ? static_cast<int64_t>(p.heads) * ((static_cast<int64_t>(len) + (1 << p.rows_log2) - 1) >> p.rows_log2)
                  : static_cast<int64_t>(p.heads);
    }
    const int64_t ex = block_exclusive_scan(items, s_warp, &s_total);
    if (k < n_sorted) p.item_start[k] = static_cast<int32_t>(carry + ex);
    carry += s_total;
    __syncthreads();
  }
  // the attention kernel reads the descriptors from global memory
  for (int i = tid; staged && p.info != nullptr && i < B; i += kSchedThreads) p.info[i] = s_info_buf[i];
  if (tid == 0) {
    p.item_start[n_sorted] = static_cast<int32_t>(carry);
    p.counts[0] = static_cast<int32_t>(carry);
    p.counts[1] = n_sorted;
    p.counts[2] = 0;
    if (p.stats)
      for (int i = 0; i < 4; ++i) p.stats[i] = static_cast<int64_t>(s_ledger[i]);
  }
  fence_tmap_release();
}

}  // namespace pa
