// attn_fwd_sm100.cuh -- packed variable-length bidirectional attention forward
// for B200 (sm_100a): TMA tile loads, tcgen05 MMAs accumulating in tensor
// memory, online softmax in registers, 16-byte row stores of the output.
//
// Math (SparseAttn page, section 3.1; GigaPath-Flash page, sections 3.2/4.2 for
// the blockwise online softmax): per query row, with x = scale*log2(e)*q.k,
//     m  = running max used for the exponentials,
//     P  = exp2(x - m),  l = l*exp2(m_old - m) + rowsum(P),
//     O  = O*exp2(m_old - m) + P V,
//     out = O / l,   lse = (m + log2 l) * ln 2.
// The exponent shift m is only moved when a new tile's max exceeds it by more
// than kRescaleLog2 (then O and l are rescaled); otherwise P <= 2^kRescaleLog2
// and the result is unchanged, because out and lse do not depend on m.
//
// Work item = (unit, head, pair of 128-row query tiles), a unit being a segment
// alone or a group of consecutive short segments that share tiles (the scheduler
// forms them; each row then sees only its own segment's keys).  Items are taken
// longest first from a global counter by the producer warp (dynamic
// longest-processing-time scheduling) and handed to the other warps through a
// two-slot shared-memory ring.  CTA layout, 12 warps:
//   warps 0-3  softmax + epilogue of query tile 0 (one thread per row)
//   warps 4-7  softmax + epilogue of query tile 1
//   warp 8     TMA producer: Q tiles, then K_j, V_j into a ring of smem slots
//   warp 9     tensor-memory owner and MMA issuer (the whole warp runs the issue
//              loop so its operand arithmetic stays warp-uniform; one elected
//              lane issues the MMAs and commits)
//   warps 10-11 idle (they complete the third warpgroup for the register split)
// Tensor memory (512 columns x 128 lanes, fp32): S0 | S1 | O0 | O1.  P (bf16)
// overwrites the first half of its S columns and feeds the P.V MMA from tensor
// memory.  Ping-pong: while warps 0-3 turn S0 into P0, the tensor core runs
// S1 = Q1 K^T, and the other way round.
#pragma once
#include <cuda.h>

#include <cstdint>

#include "sm100_ptx.cuh"

namespace pa {

// P <= 2^12 between moves of the shift: exact in bf16's exponent range, and O, l
// stay far from fp32 overflow.  Measured on B200: 12 instead of 8 saves ~2 % on a
// single 16384-token segment (fewer O rescales), nothing elsewhere.
constexpr float kRescaleLog2 = 12.0f;
// In every group of four key pairs of a full score tile, this many are
// exponentiated on the FMA pipe (polynomial, max relative error below 1e-4, far
// under the bf16 rounding of P) instead of the MUFU unit, per head_dim.  Measured
// on B200 with the warp-wide MMA issuer: 1 of 4 gains ~2 % at d = 128.
#ifndef PA_POLY_PAIRS_D128
#define PA_POLY_PAIRS_D128 1
#endif
#ifndef PA_POLY_PAIRS_D64
#define PA_POLY_PAIRS_D64 0
#endif
template <int D>
constexpr int kPolyPairsPer4 = D == 128 ? PA_POLY_PAIRS_D128 : PA_POLY_PAIRS_D64;
// Normaliser of the output at head_dim 128: 1 = the sum of the bf16-rounded weights
// that P.V uses (each output row an exact convex combination of value rows; three
// more instructions per key pair), 0 = the fp32 sum of the unrounded weights.
#ifndef PA_NORM_ROUNDED_D128
#define PA_NORM_ROUNDED_D128 1
#endif
static_assert(PA_POLY_PAIRS_D128 >= 0 && PA_POLY_PAIRS_D128 <= 4 && PA_POLY_PAIRS_D64 >= 0 && PA_POLY_PAIRS_D64 <= 4,
              "polynomial share out of range");
constexpr int kFwdThreads = 384;
// Register split of the 384-thread block launched at 168 registers per thread
// (384 x 168 = 64512): the two softmax warpgroups rise to 216, the producer /
// MMA warpgroup drops to 72.  2*128*216 + 128*72 = 64512.  The build checks
// that the kernels are compiled at exactly kLaunchRegs.
constexpr int kLaunchRegs = 168;
constexpr int kSoftmaxRegs = 216;
constexpr int kControlRegs = 72;
static_assert(2 * 128 * kSoftmaxRegs + 128 * kControlRegs <= kFwdThreads * kLaunchRegs, "register split");

template <int D>
struct FwdCfg {
  static_assert(D == 64 || D == 128, "head_dim 64 or 128");
  static constexpr int kRows = 128;                      // rows of a Q/K/V/O tile
  static constexpr int kTileBytes = kRows * D * 2;       // bf16 tile
  static constexpr int kColBlocks = D / 64;              // 128-byte swizzle atoms across d
  static constexpr int kBlockBytes = kRows * 128;        // one 64-column block of a tile
  static constexpr int kSlots = (D == 128) ? 5 : 10;     // K/V ring depth (tiles)
  static constexpr int kOffQ = 0;
  static constexpr int kOffKV = kOffQ + 2 * kTileBytes;
  // d = 64: V is extended by a tile of bf16 ones (one 64-column swizzle atom, shared
  // by all slots), so the P.V product also yields sum_k bf16(P) in O's column d:
  // the exact normaliser of the output, computed by the tensor core.
  static constexpr bool kSumColumn = (D == 64);
  static constexpr int kOCols = kSumColumn ? D + 16 : D;  // O columns written by P.V
  static constexpr int kOffOnes = kOffKV + kSlots * kTileBytes;
  static constexpr int kOffBar = kOffOnes + (kSumColumn ? kRows * 128 : 0);
  static constexpr int kSmemBytes = kOffBar + 512 + 1024;  // + 1024 for base alignment
  static constexpr uint32_t kTmemCols = 512;
  // tensor memory: d = 128: S0 [0,128) S1 [128,256) O0 [256,384) O1 [384,512);
  //                d = 64:  S0 [0,128) O0 [128,208) S1 [256,384) O1 [384,464)
  __host__ __device__ static constexpr uint32_t col_s(int tile) { return kSumColumn ? (tile ? 256u : 0u) : (tile ? 128u : 0u); }
  __host__ __device__ static constexpr uint32_t col_o(int tile) {
    return kSumColumn ? (tile ? 384u : 128u) : (tile ? 256u + D : 256u);
  }
};

struct FwdParams {
  const int32_t* cu;
  void* out;                  // bf16 [T, H, d]
  float* lse;
  const int32_t* counts;      // [0] items, [1] ordered segments
  int32_t* next_item;         // work counter, zeroed by the scheduler kernel
  const int32_t* order;
  const int32_t* item_start;
  const uint8_t* maps;        // [B][3] tensor maps: q, k, v
  const int32_t* info;        // [B] unit descriptors (short-segment groups); nullptr: one unit per segment
  int32_t* status;
  int32_t heads;
  int32_t batch;
  float scale_log2;           // scale * log2(e)
  uint64_t wait_limit_ns;
  int32_t err_timeout;
};

struct Bars {
  uint64_t q_full, q_empty;
  uint64_t kv_full[12], kv_empty[12];
  uint64_t s_full[2], o_full[2], o_empty[2];
  uint64_t p_full[2][2];  // [tile][half]: P columns of keys 0-63 / 64-127 are in tensor memory
  uint64_t sched_full[2], sched_empty[2];  // work-item hand-off from the producer
  uint64_t drain;
  int32_t sched_item[2][10];  // decoded items (WorkItem fields in order); seg < 0 = done
  uint32_t tmem_base;
  int abort_flag;
};

// A work item: query tiles 0 and 1 of one unit and head.  For a segment alone,
// tile t holds rows [q0 + 128 t, q0 + 128 t + 128) of the segment and meets all
// nkv key tiles.  For a group of short segments (n0 > 0), tile 0 holds the unit's
// tokens [0, n0) and tile 1 the tokens [n0, len); tile t meets only key tile t,
// which starts at the same token as its query tile.
struct WorkItem {
  int32_t seg, beg, len, head, q0, nkv;
  bool two;    // second query tile has rows
  int32_t id;  // index in the longest-first order
  int32_t n0;  // group split (tokens of tile 0); 0: a segment alone
  int32_t kt;  // score tiles per query tile: nkv alone, 1 in a group
};

__device__ __forceinline__ WorkItem decode_item(int32_t item, const FwdParams& p, int32_t n_sorted) {
  int32_t lo = 0, hi = n_sorted;
  while (hi - lo > 1) {
    const int32_t mid = (lo + hi) >> 1;
    if (__ldg(p.item_start + mid) <= item) lo = mid; else hi = mid;
  }
  WorkItem w;
  w.seg = __ldg(p.order + lo);
  const int32_t local = item - __ldg(p.item_start + lo);
  w.beg = __ldg(p.cu + w.seg);
  w.id = item;
  const int32_t inf = p.info != nullptr ? __ldg(p.info + w.seg) : -1;
  if (inf >= 0) {  // a group of short segments: one item per head
    w.n0 = inf & 0x1ff;
    w.len = (inf >> 9) & 0x1ff;
    w.head = local;
    w.q0 = 0;
    w.two = w.len > w.n0;
    w.nkv = w.two ? 2 : 1;
    w.kt = 1;
    return w;
  }
  w.len = __ldg(p.cu + w.seg + 1) - w.beg;
  const int32_t npairs = (w.len + 255) >> 8;
  w.head = local / npairs;
  w.q0 = (local - w.head * npairs) * 256;
  w.nkv = (w.len + 127) >> 7;
  w.two = w.q0 + 128 < w.len;
  w.n0 = 0;
  w.kt = w.nkv;
  return w;
}

// Work items travel decoded through the shared-memory ring: one global-memory
// lookup per item by the producer instead of one per warp.
__device__ __forceinline__ void store_item(volatile int32_t* d, const WorkItem& w) {
  d[0] = w.seg;
  d[1] = w.beg;
  d[2] = w.len;
  d[3] = w.head;
  d[4] = w.q0;
  d[5] = w.nkv;
  d[6] = w.two ? 1 : 0;
  d[7] = w.id;
  d[8] = w.n0;
  d[9] = w.kt;
}
__device__ __forceinline__ WorkItem load_item(const volatile int32_t* d) {
  WorkItem w;
  w.seg = d[0];
  w.beg = d[1];
  w.len = d[2];
  w.head = d[3];
  w.q0 = d[4];
  w.nkv = d[5];
  w.two = d[6] != 0;
  w.id = d[7];
  w.n0 = d[8];
  w.kt = d[9];
  return w;
}

__device__ __forceinline__ const void* seg_map(const FwdParams& p, int32_t seg, int which) {
  return p.maps + (static_cast<size_t>(seg) * 3 + which) * 128;
}

// A wait used while draining after an abort: ignores the abort flag, bounded by its own limit.
__device__ __forceinline__ bool drain_wait(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
  const uint32_t a = smem_u32(bar);
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(a, parity)) {
    if (global_timer_ns() - t0 > limit_ns) return false;
  }
  return true;
}

// ------------------------------------------------------------------ producer
template <int D>
__device__ __forceinline__ void run_producer(const FwdParams& p, uint8_t* smem, Bars* bars, const WaitCtl& wc,
                                             int32_t n_items, int32_t n_sorted) {
  using C = FwdCfg<D>;
  int slot = 0;
  uint32_t phase = 0;
  uint32_t q_round = 0, sk = 0;
  // last armed phase of every slot, for the drain after an abort
  uint32_t armed = 0, armed_phase = 0;
  bool q_armed = false;
  uint32_t q_armed_phase = 0;
  bool ok = true;
  for (;;) {
    // hand the next item (or -1 = done) to the other warps
    const int ss = sk & 1;
    const uint32_t sph = (sk >> 1) & 1u;
    ++sk;
    if (!(ok = mbar_wait(&bars->sched_empty[ss], sph ^ 1u, wc))) break;
    const int32_t item = atomicAdd(p.next_item, 1);
    WorkItem w;
    if (item < n_items) {
      w = decode_item(item, p, n_sorted);
    } else {
      w.seg = -1;
    }
    store_item(bars->sched_item[ss], w);
    mbar_arrive(&bars->sched_full[ss]);
    if (w.seg < 0) break;

    const void* mq = seg_map(p, w.seg, 0);
    const void* mk = seg_map(p, w.seg, 1);
    const void* mv = seg_map(p, w.seg, 2);
    fence_tmap_acquire(mq);
    fence_tmap_acquire(mk);
    fence_tmap_acquire(mv);
    const int32_t xcol = w.head * D;
    if (w.n0) {
      // A group of short segments streams its query tiles through the ring too, in the
      // order Q_0, K_0, V_0 [, Q_1, K_1, V_1] (tile t at the unit's token t * n0), so the
      // loads of neighbouring items overlap: the only buffer such an item waits for is a
      // ring slot.
      const int ntile = w.two ? 2 : 1;
      for (int t = 0; ok && t < ntile; ++t) {
        for (int which = 0; which < 3; ++which) {
          if (!(ok = mbar_wait(&bars->kv_empty[slot], phase ^ 1u, wc))) break;
          mbar_arrive_expect_tx(&bars->kv_full[slot], C::kTileBytes);
          armed |= 1u << slot;
          armed_phase = (armed_phase & ~(1u << slot)) | (phase << slot);
          uint8_t* dst = smem + C::kOffKV + slot * C::kTileBytes;
          const void* m = which == 0 ? mq : which == 1 ? mk : mv;
#pragma unroll
          for (int cb = 0; cb < C::kColBlocks; ++cb)
            tma_load_2d(dst + cb * C::kBlockBytes, m, xcol + cb * 64, t * w.n0, &bars->kv_full[slot]);
          if (++slot == C::kSlots) {
            slot = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) break;
      continue;
    }
    if (!(ok = mbar_wait(&bars->q_empty, (q_round & 1u) ^ 1u, wc))) break;
    mbar_arrive_expect_tx(&bars->q_full, (w.two ? 2u : 1u) * C::kTileBytes);
    q_armed = true;
    q_armed_phase = q_round & 1u;
#pragma unroll
    for (int cb = 0; cb < C::kColBlocks; ++cb) {
      tma_load_2d(smem + C::kOffQ + cb * C::kBlockBytes, mq, xcol + cb * 64, w.q0, &bars->q_full);
      if (w.two)
        tma_load_2d(smem + C::kOffQ + C::kTileBytes + cb * C::kBlockBytes, mq, xcol + cb * 64, w.q0 + 128,
                    &bars->q_full);
    }
    ++q_round;
    for (int32_t j = 0; ok && j < w.nkv; ++j) {
#pragma unroll
      for (int which = 0; which < 2; ++which) {
        if (!(ok = mbar_wait(&bars->kv_empty[slot], phase ^ 1u, wc))) break;
        mbar_arrive_expect_tx(&bars->kv_full[slot], C::kTileBytes);
        armed |= 1u << slot;
        armed_phase = (armed_phase & ~(1u << slot)) | (phase << slot);
        uint8_t* dst = smem + C::kOffKV + slot * C::kTileBytes;
        const void* m = which ? mv : mk;
#pragma unroll
        for (int cb = 0; cb < C::kColBlocks; ++cb)
          tma_load_2d(dst + cb * C::kBlockBytes, m, xcol + cb * 64, j * 128, &bars->kv_full[slot]);
        if (++slot == C::kSlots) {
          slot = 0;
          phase ^= 1u;
        }
      }
    }
    if (!ok) break;
  }
  if (!ok) {
    // Let every copy this thread started land before the CTA can exit.
    const uint64_t lim = wc.limit_ns;
    for (int s = 0; s < C::kSlots; ++s)
      if (armed & (1u << s)) drain_wait(&bars->kv_full[s], (armed_phase >> s) & 1u, lim);
    if (q_armed) drain_wait(&bars->q_full, q_armed_phase, lim);
  }
}

// Takes the next decoded item from the producer's hand-off ring.  Returns 1 with
// `w` filled, 0 when the work is done, -2 when the wait gave up.  `arrive`
// releases the slot (one arrival per caller).
__device__ __forceinline__ int next_item_from_ring(Bars* bars, uint32_t& sk, const WaitCtl& wc, bool arrive,
                                                   WorkItem& w) {
  const int ss = sk & 1;
  const uint32_t sph = (sk >> 1) & 1u;
  ++sk;
  if (!mbar_wait(&bars->sched_full[ss], sph, wc)) return -2;
  w = load_item(bars->sched_item[ss]);
  if (arrive) mbar_arrive(&bars->sched_empty[ss]);
  return w.seg < 0 ? 0 : 1;
}

// ------------------------------------------------------------------ MMA issuer
// Unrolled issue loops over split descriptors: per MMA only the 32-bit start
// addresses change (no carry leaves the 14-bit field: shared-memory addresses
// are below 256 KB), the high word is one constant.
template <int D>
__device__ __forceinline__ void issue_s(uint32_t issue, uint32_t d_tmem, uint32_t q_addr, uint32_t k_addr) {
  constexpr uint32_t idesc = idesc_bf16_f32(128, 128, false);
  constexpr uint32_t hi = sdesc_sw128_hi(1024);
  const uint32_t a0 = sdesc_sw128_lo(q_addr, 16), b0 = sdesc_sw128_lo(k_addr, 16);
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint32_t off = ((kk >> 2) * FwdCfg<D>::kBlockBytes + (kk & 3) * 32) >> 4;
    mma_bf16_ss_lo_if(issue, d_tmem, a0 + off, b0 + off, hi, idesc, kk > 0 ? 1u : 0u);
  }
}

// O (+)= P V over the keys [64*half, 64*half + 64) of the tile.  With a sum
// column, V's second 64-column swizzle atom is the shared tile of ones: the
// descriptor's leading byte offset points from the V slot to it.
template <int D>
__device__ __forceinline__ void issue_pv_half(uint32_t issue, uint32_t d_tmem, uint32_t p_tmem, uint32_t v_addr,
                                              uint32_t ones_addr, int half, bool accumulate) {
  using C = FwdCfg<D>;
  constexpr uint32_t idesc = idesc_bf16_f32(128, C::kOCols, true);
  constexpr uint32_t hi = sdesc_sw128_hi(1024);
  const uint32_t lbo = C::kSumColumn ? ones_addr - v_addr : C::kBlockBytes;
  const uint32_t b0 = sdesc_sw128_lo(v_addr, lbo);
#pragma unroll
  for (int kq = 0; kq < 4; ++kq) {
    const int kk = half * 4 + kq;
    mma_bf16_ts_lo_if(issue, d_tmem, p_tmem + kk * 8, b0 + ((kk * 16 * 128) >> 4), hi, idesc,
                   (accumulate || kk > 0) ? 1u : 0u);
  }
}

template <int D>
__device__ __forceinline__ void run_mma(const FwdParams& p, uint8_t* smem, Bars* bars, const WaitCtl& wc,
                                        uint32_t tmem, int32_t n_sorted) {
  using C = FwdCfg<D>;
  const uint32_t q_addr0 = smem_u32(smem + C::kOffQ);
  const uint32_t kv_addr0 = smem_u32(smem + C::kOffKV);
  const uint32_t ones_addr = smem_u32(smem + C::kOffOnes);
  int slot = 0;
  uint32_t phase = 0, q_round = 0;
  uint32_t p_ph = 0, oe_ph = 0;  // bit t: phase of tile t
  uint32_t sk = 0;
  bool ok = true;
  const uint32_t leader = elect_one_sync();
  for (;;) {
    WorkItem w;
    const int got = next_item_from_ring(bars, sk, wc, false, w);
    if (got != -2 && leader) mbar_arrive(&bars->sched_empty[(sk - 1) & 1]);
    if (got == -2) ok = false;
    if (got <= 0) break;
    if (w.n0) {
      // A group of short segments: S_t = Q_t K_t^T and O_t = P_t V_t, tile t meeting only
      // key tile t.  The ring holds Q_0, K_0, V_0 [, Q_1, K_1, V_1] in this order.
      const int ntile = w.two ? 2 : 1;
      int rs[6];
      uint32_t rp[6];
#pragma unroll
      for (int o = 0; o < 6; ++o) {
        int s2 = slot + o;
        uint32_t ph2 = phase;
        if (s2 >= C::kSlots) {
          s2 -= C::kSlots;
          ph2 ^= 1u;
        }
        rs[o] = s2;
        rp[o] = ph2;
      }
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        if (t == ntile) break;
        const int qs = rs[3 * t], ks = rs[3 * t + 1];
        if (!(ok = mbar_wait(&bars->kv_full[qs], rp[3 * t], wc))) break;
        if (!(ok = mbar_wait(&bars->kv_full[ks], rp[3 * t + 1], wc))) break;
        tc_fence_after();
        issue_s<D>(leader, tmem + C::col_s(t), kv_addr0 + qs * C::kTileBytes, kv_addr0 + ks * C::kTileBytes);
        mma_commit_if(leader, &bars->s_full[t]);
        mma_commit_if(leader, &bars->kv_empty[qs]);
        mma_commit_if(leader, &bars->kv_empty[ks]);
      }
      if (!ok) break;
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        if (t == ntile) break;
        if (!(ok = mbar_wait(&bars->o_empty[t], ((oe_ph >> t) & 1u) ^ 1u, wc))) break;
        oe_ph ^= 1u << t;
        const int vs = rs[3 * t + 2];
        if (!(ok = mbar_wait(&bars->kv_full[vs], rp[3 * t + 2], wc))) break;
        if (!(ok = mbar_wait(&bars->p_full[t][0], (p_ph >> t) & 1u, wc))) break;
        tc_fence_after();
        issue_pv_half<D>(leader, tmem + C::col_o(t), tmem + C::col_s(t), kv_addr0 + vs * C::kTileBytes, ones_addr, 0, false);
        if (!(ok = mbar_wait(&bars->p_full[t][1], (p_ph >> t) & 1u, wc))) break;
        p_ph ^= 1u << t;
        tc_fence_after();
        issue_pv_half<D>(leader, tmem + C::col_o(t), tmem + C::col_s(t), kv_addr0 + vs * C::kTileBytes, ones_addr, 1, true);
        mma_commit_if(leader, &bars->o_full[t]);
        mma_commit_if(leader, &bars->kv_empty[vs]);
      }
      if (!ok) break;
      slot = w.two ? rs[5] + 1 : rs[2] + 1;
      phase = w.two ? rp[5] : rp[2];
      if (slot == C::kSlots) {
        slot = 0;
        phase ^= 1u;
      }
      continue;
    }
    if (!(ok = mbar_wait(&bars->q_full, q_round & 1u, wc))) break;
    ++q_round;
    int ks = slot;
    if (!(ok = mbar_wait(&bars->kv_full[slot], phase, wc))) break;
    if (++slot == C::kSlots) { slot = 0; phase ^= 1u; }
    tc_fence_after();
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      if (t == 1 && !w.two) break;
      issue_s<D>(leader, tmem + C::col_s(t), q_addr0 + t * C::kTileBytes, kv_addr0 + ks * C::kTileBytes);
      mma_commit_if(leader, &bars->s_full[t]);
    }
    mma_commit_if(leader, &bars->kv_empty[ks]);
    if (w.nkv == 1) mma_commit_if(leader, &bars->q_empty);
    for (int32_t j = 0; ok && j < w.nkv; ++j) {
      const bool has_next = j + 1 < w.nkv;
      const int vs = slot;
      if (!(ok = mbar_wait(&bars->kv_full[slot], phase, wc))) break;
      if (++slot == C::kSlots) { slot = 0; phase ^= 1u; }
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        if (t == 1 && !w.two) break;
        if (j == 0) {
          if (!(ok = mbar_wait(&bars->o_empty[t], ((oe_ph >> t) & 1u) ^ 1u, wc))) break;
          oe_ph ^= 1u << t;
        }
        if (!(ok = mbar_wait(&bars->p_full[t][0], (p_ph >> t) & 1u, wc))) break;
        tc_fence_after();
        issue_pv_half<D>(leader, tmem + C::col_o(t), tmem + C::col_s(t), kv_addr0 + vs * C::kTileBytes, ones_addr, 0, j > 0);
        if (!(ok = mbar_wait(&bars->p_full[t][1], (p_ph >> t) & 1u, wc))) break;
        p_ph ^= 1u << t;
        tc_fence_after();
        issue_pv_half<D>(leader, tmem + C::col_o(t), tmem + C::col_s(t), kv_addr0 + vs * C::kTileBytes, ones_addr, 1, true);
        if (has_next) {
          if (t == 0) {  // K_{j+1} is needed only now, after P.V of tile 0 is queued
            ks = slot;
            if (!(ok = mbar_wait(&bars->kv_full[slot], phase, wc))) break;
            if (++slot == C::kSlots) { slot = 0; phase ^= 1u; }
            tc_fence_after();
          }
          issue_s<D>(leader, tmem + C::col_s(t), q_addr0 + t * C::kTileBytes, kv_addr0 + ks * C::kTileBytes);
          mma_commit_if(leader, &bars->s_full[t]);
        } else {
          mma_commit_if(leader, &bars->o_full[t]);
        }
      }
      if (!ok) break;
      mma_commit_if(leader, &bars->kv_empty[vs]);
      if (has_next) {
        mma_commit_if(leader, &bars->kv_empty[ks]);
        if (j + 2 == w.nkv) mma_commit_if(leader, &bars->q_empty);
      }
    }
    if (!ok) break;
  }
  // Every MMA issued so far completes before tensor memory is released.
  mma_commit_if(leader, &bars->drain);
  drain_wait(&bars->drain, 0, wc.limit_ns);
}

// ------------------------------------------------------------------ softmax + epilogue
// Row extreme of the 128 scores (64 register pairs): max (kNeg = false) or min
// (kNeg = true, for a negative scale), only keys in [kv_lo, kv_hi) when kPartial.
// Eight independent chains of three-input max/min keep the dependency depth
// near 10.
template <bool kPartial, bool kNeg>
__device__ __forceinline__ float row_extreme(const uint64_t (&v)[64], int kv_lo, int kv_hi) {
  const float fill = kNeg ? INFINITY : -INFINITY;
  float a[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) a[i] = fill;
#pragma unroll
  for (int k = 0; k < 64; k += 8) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      float x0 = f2_lo(v[k + i]), x1 = f2_hi(v[k + i]);
      if (kPartial) {
        x0 = (2 * (k + i) >= kv_lo && 2 * (k + i) < kv_hi) ? x0 : fill;
        x1 = (2 * (k + i) + 1 >= kv_lo && 2 * (k + i) + 1 < kv_hi) ? x1 : fill;
      }
      a[i] = kNeg ? min3f(a[i], x0, x1) : max3f(a[i], x0, x1);
    }
  }
  if (kNeg) return min3f(min3f(a[0], a[1], a[2]), min3f(a[3], a[4], a[5]), fminf(a[6], a[7]));
  return max3f(max3f(a[0], a[1], a[2]), max3f(a[3], a[4], a[5]), fmaxf(a[6], a[7]));
}

// One 128 x 128 score tile of one row (thread): row extreme, exponent-shift
// update (rescaling O first when it moves), then P = exp2(s*c - m) -> bf16 into
// tensor memory in two halves of 64 keys; each half is handed to the MMA warp
// as soon as it is stored, so P.V of keys 0-63 overlaps the exponentials of
// keys 64-127.  Scores stay in register pairs and use packed fp32 arithmetic.
// With kPartial, keys outside [kv_lo, kv_hi) get weight 0: the ragged last tile
// of a segment (kv_lo = 0), or a row's own segment inside a group tile.
template <bool kPartial, bool kNeg, int D>
__device__ __forceinline__ void softmax_tile(const uint64_t (&v)[64], int kv_lo, int kv_hi, bool first, float c,
                                             uint32_t tS, uint32_t tO, float& m, float& l, float& lr,
                                             uint64_t* p_full_half, int lane) {
  const float xmax = row_extreme<kPartial, kNeg>(v, kv_lo, kv_hi) * c;  // log2 units
  bool rescale = false;  // warp-uniform
  float alpha = 1.f;
  if (first) {
    m = xmax;
  } else if (__any_sync(0xffffffffu, xmax > m + kRescaleLog2)) {
    const float m_new = fmaxf(m, xmax);
    alpha = ex2_approx(m - m_new);
    l *= alpha;
    lr *= alpha;
    m = m_new;
    rescale = true;
  }
  const uint64_t c2 = f2_pack(c, c);
  const uint64_t negm2 = f2_pack(-m, -m);
  const float magic = 12582912.0f;  // 1.5 * 2^23
  const Exp2PolyConsts ek{f2_pack(magic, magic), f2_pack(-magic, -magic), f2_pack(kExp2C0, kExp2C0),
                          f2_pack(kExp2C1, kExp2C1), f2_pack(kExp2C2, kExp2C2), f2_pack(kExp2C3, kExp2C3)};
  uint64_t su[2] = {0, 0}, sr[2] = {0, 0};  // packed partial sums (0.0f bit patterns)
#pragma unroll
  for (int half = 0; half < 2; ++half) {
#pragma unroll
    for (int cc = 2 * half; cc < 2 * half + 2; ++cc) {
      uint32_t pk[16];
#pragma unroll
      for (int k = 0; k < 16; ++k) {
        const int i = cc * 16 + k;  // pair index: keys 2i, 2i+1
        uint64_t x = f2_fma(v[i], c2, negm2);
        if (kPartial) {
          x = f2_pack(2 * i >= kv_lo && 2 * i < kv_hi ? f2_lo(x) : -INFINITY,
                      2 * i + 1 >= kv_lo && 2 * i + 1 < kv_hi ? f2_hi(x) : -INFINITY);
        }
        const uint64_t pp =
            (!kPartial && (k & 3) >= 4 - kPolyPairsPer4<D>) ? ex2x2_poly(x, ek) : ex2x2(x);
        const uint32_t pr = pack_bf16x2_pair(pp);
        su[k & 1] = f2_add(su[k & 1], pp);
        if (!FwdCfg<D>::kSumColumn && PA_NORM_ROUNDED_D128) sr[k & 1] = add_bf16x2_as_f32x2(sr[k & 1], pr);
        pk[k] = pr;
      }
      PA_TMEM_ST16(tS + cc * 16, pk);
    }
    if (half == 1 && rescale) {
      // O *= alpha, done after the exponentials, when the score registers are dead (with
      // all 128 live, this block forced a spill whose reloads sat in the hot loop).  P.V
      // of this tile has not started (half 0 is handed over only below, in rescale
      // tiles) and that of the previous tile has completed (S of this tile was issued
      // after it).  With a sum column, the rescale covers it too.
#pragma unroll
      for (int cc = 0; cc < FwdCfg<D>::kOCols / 16; ++cc) {
        uint32_t o[16];
        PA_TMEM_LD16(tO + cc * 16, o);
        tmem_wait_ld();
#pragma unroll
        for (int k = 0; k < 16; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha);
        PA_TMEM_ST16(tO + cc * 16, o);
      }
    }
    tmem_wait_st();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) {
      if (half == 1 && rescale) mbar_arrive(&p_full_half[0]);
      if (half == 1 || !rescale) mbar_arrive(&p_full_half[half]);
    }
  }
  const uint64_t su2 = f2_add(su[0], su[1]), sr2 = f2_add(sr[0], sr[1]);
  l += f2_lo(su2) + f2_hi(su2);
  if (!FwdCfg<D>::kSumColumn) lr += PA_NORM_ROUNDED_D128 ? f2_lo(sr2) + f2_hi(sr2) : f2_lo(su2) + f2_hi(su2);
}

template <int D>
__device__ __forceinline__ void run_softmax(const FwdParams& p, uint8_t* smem, Bars* bars, const WaitCtl& wc,
                                            uint32_t tmem, int32_t n_sorted, int tile) {
  using C = FwdCfg<D>;
  const int t = threadIdx.x & 127;  // row of the query tile
  const int lane = threadIdx.x & 31;
  const uint32_t lane_base = static_cast<uint32_t>(t & ~31) << 16;
  const uint32_t tS = tmem + lane_base + C::col_s(tile);
  const uint32_t tO = tmem + lane_base + C::col_o(tile);
  const float c = p.scale_log2;
  uint32_t s_ph = 0, of_ph = 0, sk = 0;
  bool ok = true;

  for (;;) {
    WorkItem w;
    int got = next_item_from_ring(bars, sk, wc, false, w);
    if (__any_sync(0xffffffffu, got == -2)) got = -2;
    __syncwarp();
    if (lane == 0 && got != -2) mbar_arrive(&bars->sched_empty[(sk - 1) & 1]);
    if (got == -2) ok = false;
    if (got <= 0) break;
    if (tile == 1 && !w.two) continue;
    // l: sum of the fp32 exponentials (gives lse); lr: sum of the same values rounded to
    // bf16, i.e. of the weights the P.V product actually used (normalises the output,
    // so each output row is an exact convex combination of value rows).
    float m = 0.f, l = 0.f, lr = 0.f;
    uint64_t* ph = bars->p_full[tile];
    if (w.n0) {
      // A tile of a group of short segments: one score tile; this row's keys are those of
      // its own segment, [glo, ghi) relative to the tile (the key tile starts at the query
      // tile's first token).  Rows past the tile's tokens see [0, nrows) and are not written.
      const int32_t row0 = w.beg + tile * w.n0;
      const int32_t nrows = tile ? w.len - w.n0 : w.n0;
      int32_t glo = 0, ghi = nrows;
      if (t < nrows) {
        const int32_t tok = row0 + t;
        int32_t a = w.seg, b = p.batch;  // cu[a] <= tok < cu[b]
        while (b - a > 1) {
          const int32_t mid = (a + b) >> 1;
          if (__ldg(p.cu + mid) <= tok) a = mid; else b = mid;
        }
        glo = __ldg(p.cu + a) - row0;
        ghi = __ldg(p.cu + a + 1) - row0;
      }
      ok = mbar_wait(&bars->s_full[tile], s_ph, wc);
      if (__any_sync(0xffffffffu, !ok)) {
        ok = false;
        break;
      }
      s_ph ^= 1u;
      tc_fence_after();
      uint64_t r[64];
      tmem_ld128_pairs(tS, r);
      if (c >= 0.f) softmax_tile<true, false, D>(r, glo, ghi, true, c, tS, tO, m, l, lr, ph, lane);
      else softmax_tile<true, true, D>(r, glo, ghi, true, c, tS, tO, m, l, lr, ph, lane);
    } else {
      for (int32_t j = 0; j < w.nkv; ++j) {
        ok = mbar_wait(&bars->s_full[tile], s_ph, wc);
        if (__any_sync(0xffffffffu, !ok)) { ok = false; break; }
        s_ph ^= 1u;
        tc_fence_after();
        uint64_t r[64];
        tmem_ld128_pairs(tS, r);
        const int kv_valid = w.len - j * 128;  // keys of this tile inside the segment
        if (kv_valid >= 128) {
          if (c >= 0.f) softmax_tile<false, false, D>(r, 0, 128, j == 0, c, tS, tO, m, l, lr, ph, lane);
          else softmax_tile<false, true, D>(r, 0, 128, j == 0, c, tS, tO, m, l, lr, ph, lane);
        } else {
          if (c >= 0.f) softmax_tile<true, false, D>(r, 0, kv_valid, j == 0, c, tS, tO, m, l, lr, ph, lane);
          else softmax_tile<true, true, D>(r, 0, kv_valid, j == 0, c, tS, tO, m, l, lr, ph, lane);
        }
      }
    }
    if (!ok) break;

    // ---- epilogue: O / l -> bf16 -> 16-byte stores of this thread's row (rows past the
    // tile's tokens are not written); lse from the unrounded sum.
    ok = mbar_wait(&bars->o_full[tile], of_ph, wc);
    if (__any_sync(0xffffffffu, !ok)) { ok = false; break; }
    of_ph ^= 1u;
    tc_fence_after();
    // rows of this query tile: tokens [row0, row0 + nrows) of the pack
    const int32_t row0 = w.beg + (w.n0 ? tile * w.n0 : w.q0 + tile * 128);
    const int32_t nrows = w.n0 ? (tile ? w.len - w.n0 : w.n0) : w.len - w.q0 - tile * 128;
    const bool row_ok = t < nrows;
    const int32_t token = row0 + (row_ok ? t : 0);
    uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.out) +
                                          (static_cast<size_t>(token) * p.heads + w.head) * D);
    if (C::kSumColumn) {
      // sum of the bf16 weights, accumulated by the tensor core in O's column d
      uint32_t sc[16];
      PA_TMEM_LD16(tO + D, sc);
      tmem_wait_ld();
      lr = __uint_as_float(sc[0]);
    }
    const float inv_l = 1.0f / lr;
#pragma unroll
    for (int cc = 0; cc < D / 32; ++cc) {
      uint32_t o[32];
      PA_TMEM_LD32(tO + cc * 32, o);
      tmem_wait_ld();
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        uint4 v;
        v.x = pack_bf16x2(__uint_as_float(o[q4 * 8 + 0]) * inv_l, __uint_as_float(o[q4 * 8 + 1]) * inv_l);
        v.y = pack_bf16x2(__uint_as_float(o[q4 * 8 + 2]) * inv_l, __uint_as_float(o[q4 * 8 + 3]) * inv_l);
        v.z = pack_bf16x2(__uint_as_float(o[q4 * 8 + 4]) * inv_l, __uint_as_float(o[q4 * 8 + 5]) * inv_l);
        v.w = pack_bf16x2(__uint_as_float(o[q4 * 8 + 6]) * inv_l, __uint_as_float(o[q4 * 8 + 7]) * inv_l);
        if (row_ok) dst[cc * 4 + q4] = v;
      }
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&bars->o_empty[tile]);  // O columns may be overwritten now
    if (row_ok) {
      const float lse2 = m + __log2f(l);
      p.lse[static_cast<size_t>(token) * p.heads + w.head] = lse2 * 0.69314718055994531f;
    }
  }
}

template <int D>
__global__ void __launch_bounds__(kFwdThreads, 1) attn_fwd_kernel(const __grid_constant__ FwdParams p) {
  using C = FwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned base, derived by an offset from the shared array (not through an
  // integer round trip), so the compiler keeps every address below in the shared window.
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  Bars* bars = reinterpret_cast<Bars*>(smem + C::kOffBar);
  const int warp = threadIdx.x >> 5;

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    mbar_init(&bars->q_empty, 1);
    for (int s = 0; s < C::kSlots; ++s) {
      mbar_init(&bars->kv_full[s], 1);
      mbar_init(&bars->kv_empty[s], 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&bars->s_full[t], 1);
      mbar_init(&bars->p_full[t][0], 4);
      mbar_init(&bars->p_full[t][1], 4);
      mbar_init(&bars->o_full[t], 1);
      mbar_init(&bars->o_empty[t], 4);
      mbar_init(&bars->sched_full[t], 1);
      mbar_init(&bars->sched_empty[t], 9);  // the MMA thread + one lane of each softmax warp
    }
    mbar_init(&bars->drain, 1);
    bars->abort_flag = 0;
    fence_mbar_init();
  }
  if (C::kSumColumn) {
    // the tile of ones read by P.V as V's extra columns (bf16 1.0 = 0x3F80)
    uint4* ones = reinterpret_cast<uint4*>(smem + C::kOffOnes);
    for (int i = threadIdx.x; i < C::kRows * 128 / 16; i += kFwdThreads)
      ones[i] = make_uint4(0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u);
    fence_proxy_async_smem();  // visible to the tensor core (async proxy)
  }
  if (warp == 9) {
    tmem_alloc(&bars->tmem_base, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  const WaitCtl wc{&bars->abort_flag, p.status, p.wait_limit_ns, p.err_timeout};
  // Everything above overlaps the schedule kernel (programmatic dependent
  // launch); the work list, the tensor maps and the counters are read only
  // after it has completed.
  pdl_wait_primary();
  const int32_t n_items = p.counts[0];
  const int32_t n_sorted = p.counts[1];

  // The two register regions never merge again: each branch ends with its own
  // barrier over the whole block, and only the tensor-memory owner continues.
  if (warp < 8) {
    regs_increase<kSoftmaxRegs>();
    run_softmax<D>(p, smem, bars, wc, tmem, n_sorted, warp >> 2);
    tc_fence_before();
    named_bar_sync(1, kFwdThreads);
  } else {
    regs_decrease<kControlRegs>();
    if (warp == 8) {
      if ((threadIdx.x & 31) == 0) run_producer<D>(p, smem, bars, wc, n_items, n_sorted);
    } else if (warp == 9) {
      run_mma<D>(p, smem, bars, wc, tmem, n_sorted);  // the whole warp; one elected lane issues
    }
    __syncwarp();
    tc_fence_before();
    named_bar_sync(1, kFwdThreads);
    if (warp == 9) {
      tc_fence_after();
      tmem_dealloc(tmem, C::kTmemCols);
    }
  }
}

// A one-warp kernel that waits on a barrier nothing completes, through the same
// bounded wait as the attention kernel; it must record a timeout and return.
__global__ void wait_timeout_selftest_kernel(int32_t* status, uint64_t limit_ns, int32_t err_timeout) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  const WaitCtl wc{&abort_flag, status, limit_ns, err_timeout};
  mbar_wait(&bar, 0, wc);
  __syncthreads();
}

}  // namespace pa
