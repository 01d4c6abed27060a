// schedule.cuh -- device-side segment scheduler for the packed attention kernel.
//
// One CTA of 256 threads turns cu_seqlens into the work list of the attention
// kernel, without a host round trip:
//   1. validates cu_seqlens (cu[0] = 0, non-decreasing, cu[B] = T, every
//      segment <= max_seqlen); on failure it records the status and publishes
//      an empty work list;
//   2. orders the non-empty segments longest-first (stable counting sort on the
//      number of 128-key tiles, i.e. on the per-item cost), so a persistent grid
//      takes the big items first (longest-processing-time order);
//   3. publishes, in that order, the first work-item index of every segment;
//      a segment of L tokens holds heads * ceil(L / 2^rows_log2) items: for the
//      forward (rows_log2 = 8) one per (head, pair of 128-row query tiles), for
//      the backward (rows_log2 = 7) one per (head, 128-key tile);
//   4. for the forward, writes three tensor maps per segment (q, k, v) whose
//      base is the segment's first token and whose row extent is L, so that
//      every TMA tile stops at the segment boundary: loads past it read zeros
//      and no tile touches another image (maps == nullptr skips this step);
//      the FP8 variant's transposed V map is cut along its key axis instead.
//
// The mask of the method (Mage-Flow page, "Packing + Flash Attention varlen":
// images attend only to themselves, no padding) is thereby carried entirely by
// the tensor-map bounds plus the key mask of each segment's last tile.
#pragma once
#include <cuda.h>

#include <cstdint>

#include "sm100_ptx.cuh"

namespace pa {

constexpr int kSchedThreads = 256;
constexpr int kSortBuckets = 1024;     // tile counts >= 1023 share the first bucket
constexpr int kCuInSmem = 4096 + 1;    // cu_seqlens staged in shared memory up to this many entries

struct SchedParams {
  CUtensorMap tmpl[3];     // q, k, v over the whole [T, H*d] matrix (host-encoded)
  const void* base[3];     // q, k, v base pointers
  const int32_t* cu;       // [B+1]
  int32_t* status;         // status word
  int32_t* counts;         // [0] = work items, [1] = non-empty segments, [2] = work counter (zeroed)
  int32_t* order;          // [B] segment ids, longest first
  int32_t* item_start;     // [B+1] first item of each ordered segment
  uint8_t* maps;           // [B][3] tensor maps, 128 bytes each (nullptr: none)
  uint64_t row_bytes;      // H * d * 2
  int32_t batch, total, heads, max_seqlen;
  int32_t rows_log2;        // rows of a work item: 2^rows_log2 (8 forward, 7 backward)
  // nonzero: the third map (v) is over a [channels][keys] matrix whose segment s
  // starts at key 16*ceil(cu[s]/16) + 16*s (the FP8 variant's transposed V); its
  // per-segment map moves the base to that key and sets the key extent to L
  int32_t v_keys_inner;
  int32_t err_cu, err_max;  // status codes to record
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

__global__ void __launch_bounds__(kSchedThreads, 1) schedule_kernel(const __grid_constant__ SchedParams p) {
  __shared__ int s_bad;
  __shared__ int32_t s_cu_buf[kCuInSmem];
  __shared__ int32_t s_hist[kSortBuckets];
  __shared__ int32_t s_start[kSortBuckets];
  __shared__ int32_t s_keys[kSchedThreads];
  __shared__ int64_t s_warp[32];
  __shared__ int64_t s_total;
  const int tid = threadIdx.x;
  const int B = p.batch;
  // the attention kernel may start its prologue now; it waits for this grid
  // to complete before it reads anything written here
  pdl_launch_dependents();

  // cu_seqlens in shared memory (one pass over global memory) when it fits
  const bool staged = B + 1 <= kCuInSmem;
  for (int i = tid; staged && i <= B; i += kSchedThreads) s_cu_buf[i] = p.cu[i];
  const int32_t* cu = staged ? s_cu_buf : p.cu;
  if (tid == 0) s_bad = 0;
  for (int b = tid; b < kSortBuckets; b += kSchedThreads) s_hist[b] = 0;
  __syncthreads();

  // 1. validation and histogram of tile counts
  if (tid == 0 && (cu[0] != 0 || cu[B] != p.total)) atomicMax(&s_bad, 2);
  for (int i = tid; i < B; i += kSchedThreads) {
    const int32_t a = cu[i], b = cu[i + 1];
    if (b < a) {
      atomicMax(&s_bad, 2);
    } else if (b - a > p.max_seqlen) {
      atomicMax(&s_bad, 1);
    } else if (b > a) {
      atomicAdd(&s_hist[seg_key(b - a)], 1);
    }
  }
  __syncthreads();
  if (s_bad) {
    if (tid == 0) {
      atomicCAS(p.status, 0, s_bad == 2 ? p.err_cu : p.err_max);
      p.counts[0] = 0;
      p.counts[1] = 0;
      p.counts[2] = 0;
    }
    return;
  }

  // 2. per-segment tensor maps: copy the template, then move its base and row extent
  for (int idx = tid; p.maps != nullptr && idx < 3 * B; idx += kSchedThreads) {
    const int s = idx / 3, which = idx - 3 * s;
    const int32_t beg = cu[s], len = cu[s + 1] - beg;
    if (len <= 0) continue;
    uint8_t* dst = p.maps + static_cast<size_t>(idx) * 128;
    const uint4* src = reinterpret_cast<const uint4*>(&p.tmpl[which]);
#pragma unroll
    for (int w = 0; w < 8; ++w) reinterpret_cast<uint4*>(dst)[w] = src[w];
    if (which == 2 && p.v_keys_inner) {
      const uint64_t key0 = 16ull * ((static_cast<uint64_t>(beg) + 15) / 16) + 16ull * static_cast<uint64_t>(s);
      tmap_replace_address(dst, static_cast<const uint8_t*>(p.base[2]) + key0);
      tmap_replace_dim0(dst, static_cast<uint32_t>(len));
      continue;
    }
    const uint8_t* seg_base = static_cast<const uint8_t*>(p.base[which]) + static_cast<uint64_t>(beg) * p.row_bytes;
    tmap_replace_address(dst, seg_base);
    tmap_replace_dim1(dst, static_cast<uint32_t>(len));
  }

  // 3. bucket offsets in descending tile-count order (each thread owns 4 buckets)
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
      s_hist[b] = 0;  // reused below as the running count of placed segments
    }
  }
  const int32_t n_sorted = static_cast<int32_t>(s_total);
  __syncthreads();

  // 4. stable placement (within a bucket segments keep their packing order) and,
  // in the same pass, the first work item of every ordered segment
  for (int c0 = 0; c0 < B; c0 += kSchedThreads) {
    const int i = c0 + tid;
    int key = -1;
    if (i < B) {
      const int32_t len = cu[i + 1] - cu[i];
      if (len > 0) key = seg_key(len);
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
      items = static_cast<int64_t>(p.heads) * ((static_cast<int64_t>(len) + (1 << p.rows_log2) - 1) >> p.rows_log2);
    }
    const int64_t ex = block_exclusive_scan(items, s_warp, &s_total);
    if (k < n_sorted) p.item_start[k] = static_cast<int32_t>(carry + ex);
    carry += s_total;
    __syncthreads();
  }
  if (tid == 0) {
    p.item_start[n_sorted] = static_cast<int32_t>(carry);
    p.counts[0] = static_cast<int32_t>(carry);
    p.counts[1] = n_sorted;
    p.counts[2] = 0;
  }
  fence_tmap_release();
}

}  // namespace pa
