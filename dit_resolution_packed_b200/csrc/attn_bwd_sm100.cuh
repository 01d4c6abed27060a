// attn_bwd_sm100.cuh -- gradients of the packed variable-length bidirectional
// attention for B200 (sm_100a): dq, dk, dv from q, k, v, out, lse and dout.
//
// Math (chain rule through the row softmax of the forward definition; SparseAttn
// page, section 3.1; GigaPath-Flash page, sections 3.2 / 4.2 for the blockwise
// recomputation of P from the saved log-sum-exp): per segment, head, query row r
// and key j of the segment,
//     P_rj  = exp2(s_rj * scale * log2 e - lse_r * log2 e)     (recomputed)
//     D_r   = dout_r . out_r                                    (prep kernel)
//     dS_rj = scale * P_rj * (dout_r . v_j - D_r)
//     dv_j += P_rj dout_r,   dk_j += dS_rj q_r,   dq_r += dS_rj k_j.
//
// Work item = (segment, head, 128-key tile): a persistent grid takes items
// longest segment first (the scheduler kernel with 128-row items).  The CTA
// keeps its K and V tiles in shared memory and dK, dV in tensor memory, and
// walks the segment's 128-row query tiles; per query tile, five MMAs:
//     S^T  = K Q^T        (A = K, B = Q, both K-major)        -> TMEM A
//     dP^T = V dO^T       (A = V, B = dO, both K-major)       -> TMEM B
//     dV  += P^T dO       (A = P^T bf16 in TMEM A, B = dO MN-major)
//     dK  += dS^T Q       (A = dS^T bf16 in TMEM B, B = Q MN-major)
//     dQ   = dS K         (A = dS^T in shared memory, read MN-major; B = K MN-major) -> TMEM B
// and then the next tile's S^T (so the read-out of dQ overlaps it).  The dQ partial of every
// (key tile, query tile) is added into an fp32 accumulator laid out [H][d/4][T]
// (float4 per element group, token fastest), so that the 32 reductions of a warp
// cover 512 contiguous bytes; a last kernel converts it to bf16 [T, H, d].
//
// Rows past the segment end are loaded (one tensor map per tensor over the whole
// [T, H*d] matrix; past T the load reads zeros) and masked: a query past the
// end has lse = +inf (so P = 0) and D = 0; a key past the end gets P = dS = 0.
//
// CTA layout, 16 warps (128 registers each; no register split):
//   warps 0-3, 4-7  two elementwise warpgroups, one per half of the query tile: P^T
//              and dS^T of its 64 queries (one thread per key row)
//   warp 8     TMA producer (K, V once per item; Q, dO through a two-slot ring)
//   warp 9     tensor-memory owner and MMA issuer (whole warp, one elected lane issues)
//   warps 10-11 idle
//   warps 12-15 dQ partial -> fp32 reductions (one thread per query row); dK, dV
//              epilogue at the end of the item (one thread per key row)
#pragma once
#include <cuda.h>

#include <cstdint>

#include "exp2_poly.cuh"
#include "sm100_ptx.cuh"

// Key-column pairs of every 4 whose P is exponentiated on the FMA pipe (polynomial,
// max relative error below 1e-4, far under P's bf16 rounding) instead of the MUFU, in
// query tiles with no row past the segment end (there every x is finite).
#ifndef PA_BWD_POLY_PAIRS
#define PA_BWD_POLY_PAIRS 0
#endif
static_assert(PA_BWD_POLY_PAIRS >= 0 && PA_BWD_POLY_PAIRS <= 4, "polynomial share out of range");

namespace pa {

// 16 warps at 128 registers each (the whole register file): every role fits, so there is
// no register split between the warpgroups.
constexpr int kBwdThreads = 512;

template <int D>
struct BwdCfg {
  static_assert(D == 64 || D == 128, "head_dim 64 or 128");
  static constexpr int kRows = 128;
  static constexpr int kTileBytes = kRows * D * 2;      // bf16 tile of 128 rows
  static constexpr int kColBlocks = D / 64;             // 128-byte swizzle blocks across d
  static constexpr int kBlockBytes = kRows * 128;       // one 64-column block of a tile
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kOffK + kTileBytes;
  static constexpr int kOffQ = kOffV + kTileBytes;      // two ring slots
  static constexpr int kOffDO = kOffQ + 2 * kTileBytes;  // two ring slots
  static constexpr int kOffDS = kOffDO + 2 * kTileBytes;  // dS^T: 128 keys x 128 queries bf16, 2 blocks
  static constexpr int kOffStage = kOffDS + 2 * kBlockBytes;  // -lse2 and -D*scale of the 128 queries
  static constexpr int kOffBar = kOffStage + 2 * 128 * 4;
  static constexpr int kSmemBytes = kOffBar + 512 + 1024;  // + 1024 for base alignment
  static constexpr uint32_t kTmemCols = 512;
  // tensor memory: A [0,128) S^T then P^T; B [128,256) dP^T, dS^T (and dQ at d = 128);
  // dV [256, 256+d); dK [256+d, 256+2d); at d = 64 dQ has its own columns [384, 448),
  // so the next dP^T does not wait for the read-out of the last dQ.
  static constexpr bool kOwnDq = 256 + 3 * D <= 512;
  static constexpr uint32_t kColA = 0, kColB = 128, kColDV = 256, kColDK = 256 + D;
  static constexpr uint32_t kColDQ = kOwnDq ? 256 + 2 * D : kColB;
};

struct BwdParams {
  CUtensorMap tm_q, tm_k, tm_v, tm_do;  // [T, H*d] bf16, box {64, 128}, 128-byte swizzle
  const int32_t* cu;
  const int32_t* counts;     // [0] items, [1] ordered segments
  int32_t* next_item;        // work counter, zeroed by the scheduler kernel
  const int32_t* order;
  const int32_t* item_start;
  const float* lse2;         // [H][T] lse * log2(e)
  const float* delta;        // [H][T] D = dout . out
  float* dq_acc;             // [H][d/4][T] x 4 fp32
  void* dk;                  // bf16 [T, H, d]
  void* dv;                  // bf16 [T, H, d]
  int32_t* status;
  int32_t heads, total;
  float scale, scale_log2;
  uint64_t wait_limit_ns;
  int32_t err_timeout;
};

struct BwdBars {
  uint64_t kv_full, kv_empty;
  uint64_t qd_full[2], qd_empty[2];
  uint64_t s_full[2];    // S^T and dP^T of query half h of the current tile are in tensor memory
  uint64_t pds_full[2];  // P^T, dS^T of query half h stored (tensor memory and shared memory)
  uint64_t dq_full, dq_empty[2];  // dQ in tensor memory; its column halves read out
  uint64_t dkv_full, dkv_empty;
  uint64_t stage_full[2], stage_empty[2];  // per warpgroup: its queries' -lse2, -D*scale staging
  uint64_t sched_full[2], sched_empty[2];
  uint64_t drain;
  int32_t sched_item[2][8];  // seg, beg, len, head, k0, n query tiles, -, id; seg < 0 = done
  uint32_t tmem_base;
  int abort_flag;
};
static_assert(sizeof(BwdBars) <= 512, "backward barrier block");

struct BwdItem {
  int32_t seg, beg, len, head, k0, nq, id;
};

__device__ __forceinline__ BwdItem bwd_decode_item(int32_t item, const BwdParams& p, int32_t n_sorted) {
  int32_t lo = 0, hi = n_sorted;
  while (hi - lo > 1) {
    const int32_t mid = (lo + hi) >> 1;
    if (__ldg(p.item_start + mid) <= item) lo = mid; else hi = mid;
  }
  BwdItem w;
  w.seg = __ldg(p.order + lo);
  const int32_t local = item - __ldg(p.item_start + lo);
  w.beg = __ldg(p.cu + w.seg);
  w.len = __ldg(p.cu + w.seg + 1) - w.beg;
  w.nq = (w.len + 127) >> 7;
  w.head = local / w.nq;
  w.k0 = (local - w.head * w.nq) * 128;
  w.id = item;
  return w;
}

__device__ __forceinline__ void bwd_store_item(volatile int32_t* d, const BwdItem& w) {
  d[0] = w.seg; d[1] = w.beg; d[2] = w.len; d[3] = w.head; d[4] = w.k0; d[5] = w.nq; d[7] = w.id;
}
__device__ __forceinline__ BwdItem bwd_load_item(const volatile int32_t* d) {
  BwdItem w;
  w.seg = d[0]; w.beg = d[1]; w.len = d[2]; w.head = d[3]; w.k0 = d[4]; w.nq = d[5]; w.id = d[7];
  return w;
}

// Next decoded item from the producer's ring: 1 with `w`, 0 when done, -2 when the wait gave up.
__device__ __forceinline__ int bwd_next_item(BwdBars* bars, uint32_t& sk, const WaitCtl& wc, BwdItem& w) {
  const int ss = sk & 1;
  const uint32_t sph = (sk >> 1) & 1u;
  ++sk;
  if (!mbar_wait(&bars->sched_full[ss], sph, wc)) return -2;
  w = bwd_load_item(bars->sched_item[ss]);
  return w.seg < 0 ? 0 : 1;
}

__device__ __forceinline__ bool bwd_drain_wait(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
  const uint32_t a = smem_u32(bar);
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(a, parity)) {
    if (global_timer_ns() - t0 > limit_ns) return false;
  }
  return true;
}

// ------------------------------------------------------------------ producer
template <int D>
__device__ __forceinline__ void bwd_producer(const BwdParams& p, uint8_t* smem, BwdBars* bars, const WaitCtl& wc,
                                             int32_t n_items, int32_t n_sorted) {
  using C = BwdCfg<D>;
  uint32_t sk = 0, kv_round = 0;
  int qslot = 0;
  uint32_t qphase = 0;
  bool kv_armed = false;
  uint32_t kv_armed_ph = 0, q_armed = 0, q_armed_ph = 0;
  bool ok = true;
  for (;;) {
    const int ss = sk & 1;
    const uint32_t sph = (sk >> 1) & 1u;
    ++sk;
    if (!(ok = mbar_wait(&bars->sched_empty[ss], sph ^ 1u, wc))) break;
    const int32_t item = atomicAdd(p.next_item, 1);
    BwdItem w;
    if (item < n_items) {
      w = bwd_decode_item(item, p, n_sorted);
    } else {
      w.seg = -1;
    }
    bwd_store_item(bars->sched_item[ss], w);
    mbar_arrive(&bars->sched_full[ss]);
    if (w.seg < 0) break;

    const int32_t xcol = w.head * D;
    if (!(ok = mbar_wait(&bars->kv_empty, (kv_round & 1u) ^ 1u, wc))) break;
    mbar_arrive_expect_tx(&bars->kv_full, 2u * C::kTileBytes);
    kv_armed = true;
    kv_armed_ph = kv_round & 1u;
    ++kv_round;
#pragma unroll
    for (int cb = 0; cb < C::kColBlocks; ++cb) {
      tma_load_2d(smem + C::kOffK + cb * C::kBlockBytes, &p.tm_k, xcol + cb * 64, w.beg + w.k0, &bars->kv_full);
      tma_load_2d(smem + C::kOffV + cb * C::kBlockBytes, &p.tm_v, xcol + cb * 64, w.beg + w.k0, &bars->kv_full);
    }
    for (int32_t i = 0; ok && i < w.nq; ++i) {
      if (!(ok = mbar_wait(&bars->qd_empty[qslot], qphase ^ 1u, wc))) break;
      mbar_arrive_expect_tx(&bars->qd_full[qslot], 2u * C::kTileBytes);
      q_armed |= 1u << qslot;
      q_armed_ph = (q_armed_ph & ~(1u << qslot)) | (qphase << qslot);
#pragma unroll
      for (int cb = 0; cb < C::kColBlocks; ++cb) {
        tma_load_2d(smem + C::kOffQ + qslot * C::kTileBytes + cb * C::kBlockBytes, &p.tm_q, xcol + cb * 64,
                    w.beg + i * 128, &bars->qd_full[qslot]);
        tma_load_2d(smem + C::kOffDO + qslot * C::kTileBytes + cb * C::kBlockBytes, &p.tm_do, xcol + cb * 64,
                    w.beg + i * 128, &bars->qd_full[qslot]);
      }
      if (++qslot == 2) {
        qslot = 0;
        qphase ^= 1u;
      }
    }
    if (!ok) break;
  }
  if (!ok) {
    // Let every copy this thread started land before the CTA can exit.
    const uint64_t lim = wc.limit_ns;
    if (kv_armed) bwd_drain_wait(&bars->kv_full, kv_armed_ph, lim);
    for (int s = 0; s < 2; ++s)
      if (q_armed & (1u << s)) bwd_drain_wait(&bars->qd_full[s], (q_armed_ph >> s) & 1u, lim);
  }
}

// ------------------------------------------------------------------ MMA issuer
// A (M x K) from shared memory K-major, B (N x K) K-major: a score-like product
// over d (S^T = K Q^T with N = 128; dP^T = V dO^T one half of the queries at a time,
// N = 64, B starting at the half's first row: 64 rows of 128 bytes into each block).
template <int D, int N = 128>
__device__ __forceinline__ void bwd_issue_kmajor(uint32_t issue, uint32_t d_tmem, uint32_t a_addr, uint32_t b_addr) {
  constexpr uint32_t idesc = idesc_bf16_f32(128, N, false);
  constexpr uint32_t hi = sdesc_sw128_hi(1024);
  const uint32_t a0 = sdesc_sw128_lo(a_addr, 16), b0 = sdesc_sw128_lo(b_addr, 16);
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint32_t off = ((kk >> 2) * BwdCfg<D>::kBlockBytes + (kk & 3) * 32) >> 4;
    mma_bf16_ss_lo_if(issue, d_tmem, a0 + off, b0 + off, hi, idesc, kk > 0 ? 1u : 0u);
  }
}

// D (+)= A B with A (128 rows x 128 along K) bf16 in tensor memory and B (K = 128
// token rows x N = d) MN-major in shared memory: dV += P^T dO, dK += dS^T Q.  Only the
// K steps [K0, K1) of 16 query rows each: half h of the queries is steps [4h, 4h + 4).
template <int D, int K0, int K1>
__device__ __forceinline__ void bwd_issue_tmem_a(uint32_t issue, uint32_t d_tmem, uint32_t a_tmem, uint32_t b_addr,
                                                 bool accumulate) {
  constexpr uint32_t idesc = idesc_bf16_f32(128, D, true);
  constexpr uint32_t hi = sdesc_sw128_hi(1024);
  const uint32_t b0 = sdesc_sw128_lo(b_addr, BwdCfg<D>::kBlockBytes);
#pragma unroll
  for (int kk = K0; kk < K1; ++kk)
    mma_bf16_ts_lo_if(issue, d_tmem, a_tmem + kk * 8, b0 + ((kk * 16 * 128) >> 4), hi, idesc,
                      (accumulate || kk > 0) ? 1u : 0u);
}

// dQ = dS K: A = dS (M = 128 queries x K = 128 keys) read MN-major from the dS^T
// buffer (rows = keys, queries contiguous), B = K (K = 128 keys x N = d) MN-major.
template <int D>
__device__ __forceinline__ void bwd_issue_dq(uint32_t issue, uint32_t d_tmem, uint32_t ds_addr, uint32_t k_addr) {
  constexpr uint32_t idesc = idesc_bf16_f32_ab(128, D, true, true);
  constexpr uint32_t hi = sdesc_sw128_hi(1024);
  const uint32_t a0 = sdesc_sw128_lo(ds_addr, BwdCfg<D>::kBlockBytes);
  const uint32_t b0 = sdesc_sw128_lo(k_addr, BwdCfg<D>::kBlockBytes);
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) {
    const uint32_t off = (kk * 16 * 128) >> 4;
    mma_bf16_ss_lo_if(issue, d_tmem, a0 + off, b0 + off, hi, idesc, kk > 0 ? 1u : 0u);
  }
}

template <int D>
__device__ __forceinline__ void bwd_mma(const BwdParams& p, uint8_t* smem, BwdBars* bars, const WaitCtl& wc,
                                        uint32_t tmem) {
  using C = BwdCfg<D>;
  const uint32_t k_addr = smem_u32(smem + C::kOffK);
  const uint32_t v_addr = smem_u32(smem + C::kOffV);
  const uint32_t q_addr0 = smem_u32(smem + C::kOffQ);
  const uint32_t do_addr0 = smem_u32(smem + C::kOffDO);
  const uint32_t ds_addr = smem_u32(smem + C::kOffDS);
  uint32_t sk = 0, kv_round = 0, qphase = 0, pds_ph = 0, dqe_ph = 0, dkve_ph = 0;
  int qslot = 0;
  bool dq_pending = false, dkv_pending = false, ok = true;
  const uint32_t leader = elect_one_sync();
  for (;;) {
    BwdItem w;
    const int got = bwd_next_item(bars, sk, wc, w);
    if (got != -2 && leader) mbar_arrive(&bars->sched_empty[(sk - 1) & 1]);
    if (got == -2) ok = false;
    if (got <= 0) break;
    if (!(ok = mbar_wait(&bars->kv_full, kv_round & 1u, wc))) break;
    ++kv_round;
    if (!(ok = mbar_wait(&bars->qd_full[qslot], qphase, wc))) break;
    tc_fence_after();
    bwd_issue_kmajor<D>(leader, tmem + C::kColA, k_addr, q_addr0 + qslot * C::kTileBytes);
    for (int32_t i = 0; i < w.nq; ++i) {
      const int cur = qslot;
      // dP^T in two halves of 64 queries, one per elementwise warpgroup; at d = 128 each
      // half reuses the tensor-memory columns of one half of the previous dQ partial
      if (!C::kOwnDq && dq_pending) {
        if (!(ok = mbar_wait(&bars->dq_empty[0], dqe_ph, wc))) break;
        tc_fence_after();
      }
      bwd_issue_kmajor<D, 64>(leader, tmem + C::kColB, v_addr, do_addr0 + cur * C::kTileBytes);
      mma_commit_if(leader, &bars->s_full[0]);
      if (!C::kOwnDq && dq_pending) {
        if (!(ok = mbar_wait(&bars->dq_empty[1], dqe_ph, wc))) break;
        dqe_ph ^= 1u;
        tc_fence_after();
      }
      bwd_issue_kmajor<D, 64>(leader, tmem + C::kColB + 64, v_addr, do_addr0 + cur * C::kTileBytes + 64 * 128);
      mma_commit_if(leader, &bars->s_full[1]);
      if (!(ok = mbar_wait(&bars->pds_full[0], pds_ph, wc))) break;
      tc_fence_after();
      if (i == 0 && dkv_pending) {  // the previous item's dK, dV have been read
        if (!(ok = mbar_wait(&bars->dkv_empty, dkve_ph, wc))) break;
        dkve_ph ^= 1u;
        tc_fence_after();
      }
      // the first half's dV, dK run while the second warpgroup finishes its half
      bwd_issue_tmem_a<D, 0, 4>(leader, tmem + C::kColDV, tmem + C::kColA, do_addr0 + cur * C::kTileBytes, i > 0);
      bwd_issue_tmem_a<D, 0, 4>(leader, tmem + C::kColDK, tmem + C::kColB, q_addr0 + cur * C::kTileBytes, i > 0);
      if (!(ok = mbar_wait(&bars->pds_full[1], pds_ph, wc))) break;
      pds_ph ^= 1u;
      tc_fence_after();
      // dK's second half reads dS^T from tensor memory B before dQ (d = 128) overwrites it
      bwd_issue_tmem_a<D, 4, 8>(leader, tmem + C::kColDK, tmem + C::kColB + 32, q_addr0 + cur * C::kTileBytes, true);
      if (C::kOwnDq && dq_pending) {  // dQ's own columns: the previous partial has been read
        if (!(ok = mbar_wait(&bars->dq_empty[0], dqe_ph, wc))) break;
        if (!(ok = mbar_wait(&bars->dq_empty[1], dqe_ph, wc))) break;
        dqe_ph ^= 1u;
        tc_fence_after();
      }
      // dQ before dV's second half and the next S^T, so that its read-out overlaps both
      bwd_issue_dq<D>(leader, tmem + C::kColDQ, ds_addr, k_addr);
      mma_commit_if(leader, &bars->dq_full);
      dq_pending = true;
      bwd_issue_tmem_a<D, 4, 8>(leader, tmem + C::kColDV, tmem + C::kColA + 32, do_addr0 + cur * C::kTileBytes, true);
      mma_commit_if(leader, &bars->qd_empty[cur]);
      if (++qslot == 2) {
        qslot = 0;
        qphase ^= 1u;
      }
      if (i + 1 < w.nq) {
        if (!(ok = mbar_wait(&bars->qd_full[qslot], qphase, wc))) break;
        tc_fence_after();
        bwd_issue_kmajor<D>(leader, tmem + C::kColA, k_addr, q_addr0 + qslot * C::kTileBytes);
      }
    }
    if (!ok) break;
    mma_commit_if(leader, &bars->dkv_full);
    dkv_pending = true;
    mma_commit_if(leader, &bars->kv_empty);
  }
  // Every MMA issued so far completes before tensor memory is released.
  mma_commit_if(leader, &bars->drain);
  bwd_drain_wait(&bars->drain, 0, wc.limit_ns);
}

// P^T and dS^T of one query half: units u = 0..3 of 16 query columns; after units 1
// and 3 the 32 packed queries of the pair are stored (to columns 16(u>>1) ..: the loads
// in flight then read 32..).  kPoly of every 4 pairs take the polynomial exponential.
template <int D, int kPoly>
__device__ __forceinline__ void bwd_ew_units(uint32_t tA, uint32_t tB, const float* stage, uint8_t* ds_blk, int h,
                                             int t, bool key_ok, uint64_t c2, uint64_t sc2,
                                             const Exp2PolyConsts& ek) {
  const uint64_t zero2 = 0;
  uint32_t sb[2][16], db[2][16], pk[16], dk[16];
  PA_TMEM_LD16(tA, sb[0]);
  PA_TMEM_LD16(tB, db[0]);
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    tmem_wait_ld();
    if (u < 3) {
      PA_TMEM_LD16(tA + 16 * (u + 1), sb[(u + 1) & 1]);
      PA_TMEM_LD16(tB + 16 * (u + 1), db[(u + 1) & 1]);
    }
    const uint32_t (&sv)[16] = sb[u & 1];
    const uint32_t (&dpv)[16] = db[u & 1];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int q = 64 * h + 16 * u + 2 * k;
      const uint64_t nl2 = *reinterpret_cast<const uint64_t*>(stage + q);
      const uint64_t nd2 = *reinterpret_cast<const uint64_t*>(stage + 128 + q);
      const uint64_t x = f2_fma(f2_pack(__uint_as_float(sv[2 * k]), __uint_as_float(sv[2 * k + 1])), c2, nl2);
      const uint64_t pp = (k & 3) >= 4 - kPoly ? ex2x2_poly(x, ek) : ex2x2(x);
      const uint64_t tt = f2_fma(f2_pack(__uint_as_float(dpv[2 * k]), __uint_as_float(dpv[2 * k + 1])), sc2, nd2);
      const uint64_t ds = f2_fma(pp, tt, zero2);
      pk[8 * (u & 1) + k] = key_ok ? pack_bf16x2_pair(pp) : 0u;
      dk[8 * (u & 1) + k] = key_ok ? pack_bf16x2_pair(ds) : 0u;
    }
    if (u & 1) {
      const int ch = u >> 1;
      PA_TMEM_ST16(tA + 16 * ch, pk);
      PA_TMEM_ST16(tB + 16 * ch, dk);
      // dS^T row t, queries 64h + 32ch .. +31, into the 128-byte-swizzled MN-major layout
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        const int c = ch * 4 + v;
        *reinterpret_cast<uint4*>(ds_blk + ((c ^ (t & 7)) << 4)) =
            make_uint4(dk[4 * v], dk[4 * v + 1], dk[4 * v + 2], dk[4 * v + 3]);
      }
    }
  }
}

// ------------------------------------------------------------------ elementwise: P^T, dS^T
// Warpgroup h (warps 4h .. 4h+3) computes P^T and dS^T of queries [64h, 64h + 64) of
// every tile, one thread per key row, in units of 16 query columns (the loads of unit
// u + 1 in flight while unit u is computed).  They go to tensor-memory columns
// [64h, 64h + 32) of A and B: each warpgroup reads and writes only its own 64 columns.
template <int D>
__device__ __forceinline__ void bwd_elementwise(const BwdParams& p, uint8_t* smem, BwdBars* bars, const WaitCtl& wc,
                                                uint32_t tmem, int h) {
  using C = BwdCfg<D>;
  const int t = threadIdx.x & 127;  // key row of the tile (tensor-memory lane)
  const int lane = threadIdx.x & 31;
  const uint32_t lane_base = static_cast<uint32_t>(t & ~31) << 16;
  const uint32_t tA = tmem + lane_base + C::kColA + 64 * h;
  const uint32_t tB = tmem + lane_base + C::kColB + 64 * h;
  float* stage = reinterpret_cast<float*>(smem + C::kOffStage);  // [0,128): -lse2, [128,256): -D*scale
  uint8_t* ds_blk = smem + C::kOffDS + h * C::kBlockBytes + t * 128;
  const uint64_t c2 = f2_pack(p.scale_log2, p.scale_log2);
  const uint64_t sc2 = f2_pack(p.scale, p.scale);
  const float magic = 12582912.0f;  // 1.5 * 2^23
  const Exp2PolyConsts ek{f2_pack(magic, magic), f2_pack(-magic, -magic), f2_pack(kExp2C0, kExp2C0),
                          f2_pack(kExp2C1, kExp2C1), f2_pack(kExp2C2, kExp2C2), f2_pack(kExp2C3, kExp2C3)};
  uint32_t sk = 0, s_ph = 0, st_ph = 0;
  for (;;) {
    BwdItem w;
    int got = bwd_next_item(bars, sk, wc, w);
    if (__any_sync(0xffffffffu, got == -2)) got = -2;
    __syncwarp();
    if (lane == 0 && got != -2) mbar_arrive(&bars->sched_empty[(sk - 1) & 1]);
    if (got <= 0) break;
    const bool key_ok = t < w.len - w.k0;
    bool ok = true;
    for (int32_t i = 0; i < w.nq; ++i) {
      // this half's 64 queries' -lse2 and -D*scale (+inf lse past the segment end: P = 0)
      const int32_t qh = i * 128 + 64 * h + (t & 63);
      float nl = -INFINITY, nd = 0.f;
      if (t < 64 && qh < w.len) {
        const size_t hi = static_cast<size_t>(w.head) * p.total + w.beg + qh;
        nl = -__ldg(p.lse2 + hi);
        nd = -__ldg(p.delta + hi) * p.scale;
      }
      // (bounded mbarrier waits, not named barriers: a warp that gives up must not
      // leave the others blocked)
      ok = mbar_wait(&bars->stage_empty[h], st_ph ^ 1u, wc);  // all warps are done with the last stage
      if (__any_sync(0xffffffffu, !ok)) { ok = false; break; }
      if (t < 64) {
        stage[64 * h + t] = nl;
        stage[128 + 64 * h + t] = nd;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->stage_full[h]);
      ok = mbar_wait(&bars->stage_full[h], st_ph, wc);
      if (__any_sync(0xffffffffu, !ok)) { ok = false; break; }
      st_ph ^= 1u;
      ok = mbar_wait(&bars->s_full[h], s_ph, wc);
      if (__any_sync(0xffffffffu, !ok)) { ok = false; break; }
      s_ph ^= 1u;
      tc_fence_after();
      if (PA_BWD_POLY_PAIRS > 0 && (i + 1) * 128 <= w.len)
        bwd_ew_units<D, PA_BWD_POLY_PAIRS>(tA, tB, stage, ds_blk, h, t, key_ok, c2, sc2, ek);
      else
        bwd_ew_units<D, 0>(tA, tB, stage, ds_blk, h, t, key_ok, c2, sc2, ek);
      tmem_wait_st();
      fence_proxy_async_smem();  // the dS^T stores are read by the tensor core
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&bars->pds_full[h]);
        mbar_arrive(&bars->stage_empty[h]);
      }
    }
    if (!ok) break;
  }
}

// ------------------------------------------------------------------ dQ reductions and dK, dV epilogue
// Warps 12-15: per tile the dQ partial of query row i*128 + t, one column half at a time
// (each half's columns are released as soon as they are in registers, for the next
// dP^T half), into the fp32 reductions; at the end of the item dV and dK of key row t.
template <int D>
__device__ __forceinline__ void bwd_reduce_store(const BwdParams& p, BwdBars* bars, const WaitCtl& wc, uint32_t tmem) {
  using C = BwdCfg<D>;
  const int t = threadIdx.x & 127;
  const int lane = threadIdx.x & 31;
  const uint32_t lane_base = static_cast<uint32_t>(t & ~31) << 16;
  const uint32_t tQ = tmem + lane_base + C::kColDQ;  // the dQ partial
  const uint32_t tDV = tmem + lane_base + C::kColDV;
  const uint32_t tDK = tmem + lane_base + C::kColDK;
  uint32_t sk = 0, dqf_ph = 0, dkvf_ph = 0;
  for (;;) {
    BwdItem w;
    int got = bwd_next_item(bars, sk, wc, w);
    if (__any_sync(0xffffffffu, got == -2)) got = -2;
    __syncwarp();
    if (lane == 0 && got != -2) mbar_arrive(&bars->sched_empty[(sk - 1) & 1]);
    if (got <= 0) break;
    bool ok = true;
    for (int32_t i = 0; i < w.nq; ++i) {
      ok = mbar_wait(&bars->dq_full, dqf_ph, wc);
      if (__any_sync(0xffffffffu, !ok)) { ok = false; break; }
      dqf_ph ^= 1u;
      tc_fence_after();
      const int32_t qrow = i * 128 + t;
      const bool row_ok = qrow < w.len;
      const size_t tok = static_cast<size_t>(w.beg) + qrow;
      float* base = p.dq_acc + (static_cast<size_t>(w.head) * (D / 4) * p.total + tok) * 4;
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        uint32_t o[D / 2];
#pragma unroll
        for (int cc = 0; cc < D / 64; ++cc) PA_TMEM_LD32(tQ + hh * (D / 2) + 32 * cc, (o + 32 * cc));
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->dq_empty[hh]);
        if (row_ok) {
#pragma unroll
          for (int u = 0; u < D / 8; ++u)
            red_add_v4_f32(base + static_cast<size_t>(hh * (D / 8) + u) * p.total * 4, __uint_as_float(o[4 * u]),
                           __uint_as_float(o[4 * u + 1]), __uint_as_float(o[4 * u + 2]),
                           __uint_as_float(o[4 * u + 3]));
        }
      }
    }
    if (!ok) break;
    ok = mbar_wait(&bars->dkv_full, dkvf_ph, wc);
    if (__any_sync(0xffffffffu, !ok)) break;
    dkvf_ph ^= 1u;
    tc_fence_after();
    const bool key_ok = t < w.len - w.k0;
    const size_t row = (static_cast<size_t>(w.beg + w.k0 + (key_ok ? t : 0)) * p.heads + w.head) * D;
    uint4* dvp = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.dv) + row);
    uint4* dkp = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.dk) + row);
#pragma unroll
    for (int cc = 0; cc < 2 * (D / 32); ++cc) {
      const bool is_k = cc >= D / 32;
      const int c = is_k ? cc - D / 32 : cc;
      uint32_t a[32];
      PA_TMEM_LD32((is_k ? tDK : tDV) + 32 * c, a);
      tmem_wait_ld();
      uint4* dst = is_k ? dkp : dvp;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        uint4 va;
        va.x = pack_bf16x2(__uint_as_float(a[8 * u + 0]), __uint_as_float(a[8 * u + 1]));
        va.y = pack_bf16x2(__uint_as_float(a[8 * u + 2]), __uint_as_float(a[8 * u + 3]));
        va.z = pack_bf16x2(__uint_as_float(a[8 * u + 4]), __uint_as_float(a[8 * u + 5]));
        va.w = pack_bf16x2(__uint_as_float(a[8 * u + 6]), __uint_as_float(a[8 * u + 7]));
        if (key_ok) dst[c * 4 + u] = va;
      }
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&bars->dkv_empty);
  }
}

// ------------------------------------------------------------------ kernels
template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1) attn_bwd_kernel(const __grid_constant__ BwdParams p) {
  using C = BwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  BwdBars* bars = reinterpret_cast<BwdBars*>(smem + C::kOffBar);
  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    mbar_init(&bars->kv_full, 1);
    mbar_init(&bars->kv_empty, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars->qd_full[s], 1);
      mbar_init(&bars->qd_empty[s], 1);
      mbar_init(&bars->sched_full[s], 1);
      mbar_init(&bars->sched_empty[s], 13);  // the MMA warp + one lane of each of 12 math warps
    }
    for (int h = 0; h < 2; ++h) {
      mbar_init(&bars->s_full[h], 1);
      mbar_init(&bars->pds_full[h], 4);
    }
    mbar_init(&bars->dq_full, 1);
    mbar_init(&bars->dkv_full, 1);
    mbar_init(&bars->dkv_empty, 4);
    for (int h = 0; h < 2; ++h) {
      mbar_init(&bars->dq_empty[h], 4);
      mbar_init(&bars->stage_full[h], 4);
      mbar_init(&bars->stage_empty[h], 4);
    }
    mbar_init(&bars->drain, 1);
    bars->abort_flag = 0;
    fence_mbar_init();
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
  const int32_t n_items = p.counts[0];
  const int32_t n_sorted = p.counts[1];
  if (warp < 8) {
    bwd_elementwise<D>(p, smem, bars, wc, tmem, warp >> 2);
  } else if (warp >= 12) {
    bwd_reduce_store<D>(p, bars, wc, tmem);
  } else if (warp == 8) {
    if ((threadIdx.x & 31) == 0) bwd_producer<D>(p, smem, bars, wc, n_items, n_sorted);
  } else if (warp == 9) {
    bwd_mma<D>(p, smem, bars, wc, tmem);  // the whole warp; one elected lane issues
  }
  __syncwarp();
  tc_fence_before();
  named_bar_sync(1, kBwdThreads);
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// D = dout . out per (token, head) and lse * log2(e), both written head-major [H][T];
// the same launch zeroes the fp32 dq accumulator (acc_n4 float4).  A group of d/8
// lanes takes one (token, head) row with 16-byte loads; each warp takes 8 rows.
constexpr int kPrepRowsPerWarp = 8;
template <int D>
__global__ void bwd_prep_kernel(const uint16_t* __restrict__ out, const uint16_t* __restrict__ dout,
                                const float* __restrict__ lse, float* __restrict__ delta, float* __restrict__ lse2,
                                float4* __restrict__ acc, int64_t acc_n4, int32_t total, int32_t heads) {
  constexpr int kLanes = D / 8;                          // lanes per row
  constexpr int kIter = kPrepRowsPerWarp * kLanes / 32;  // loads per lane and tensor
  const int64_t gtid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t nthreads = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = gtid; i < acc_n4; i += nthreads) acc[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  const int lane = threadIdx.x & 31;
  const int sub = lane / kLanes, col = lane % kLanes;
  const int64_t nrows = static_cast<int64_t>(total) * heads;
  const int64_t row0 = (gtid >> 5) * kPrepRowsPerWarp;
  uint4 a[kIter], g[kIter];
#pragma unroll
  for (int it = 0; it < kIter; ++it) {
    const int64_t row = row0 + it * (32 / kLanes) + sub;
    a[it] = g[it] = make_uint4(0u, 0u, 0u, 0u);
    if (row < nrows) {
      a[it] = __ldg(reinterpret_cast<const uint4*>(out + row * D) + col);
      g[it] = __ldg(reinterpret_cast<const uint4*>(dout + row * D) + col);
    }
  }
#pragma unroll
  for (int it = 0; it < kIter; ++it) {
    const uint32_t av[4] = {a[it].x, a[it].y, a[it].z, a[it].w};
    const uint32_t gv[4] = {g[it].x, g[it].y, g[it].z, g[it].w};
    float acc_d = 0.f;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      acc_d += __uint_as_float(av[e] << 16) * __uint_as_float(gv[e] << 16);
      acc_d += __uint_as_float(av[e] & 0xffff0000u) * __uint_as_float(gv[e] & 0xffff0000u);
    }
#pragma unroll
    for (int s = kLanes / 2; s > 0; s >>= 1) acc_d += __shfl_xor_sync(0xffffffffu, acc_d, s);
    const int64_t row = row0 + it * (32 / kLanes) + sub;
    if (col == 0 && row < nrows) {
      const int32_t tok = static_cast<int32_t>(row / heads), h = static_cast<int32_t>(row - static_cast<int64_t>(tok) * heads);
      const size_t hi = static_cast<size_t>(h) * total + tok;
      delta[hi] = acc_d;
      lse2[hi] = lse[row] * 1.4426950408889634f;
    }
  }
}

// dq [T, H, d] bf16 from the fp32 accumulator [H][d/4][T] x 4.  One block per (32
// tokens, head): the 32 x d/4 float4 are read token-fastest (512 contiguous bytes per
// warp), packed to bf16 in shared memory and written as whole rows, 16 bytes per thread.
template <int D>
__global__ void __launch_bounds__(256) bwd_dq_convert_kernel(const float4* __restrict__ acc, uint16_t* __restrict__ dq,
                                                             int32_t total, int32_t heads) {
  constexpr int kC4 = D / 4;
  constexpr int kStride = kC4 * 8 + 16;  // bytes per token row in shared memory (16-byte aligned)
  constexpr int kChunks = D / 8;         // 16-byte chunks per bf16 row
  __shared__ __align__(16) uint8_t tile[32 * kStride];
  const int32_t h = static_cast<int32_t>(blockIdx.x % static_cast<uint32_t>(heads));
  const int32_t t0 = static_cast<int32_t>(blockIdx.x / static_cast<uint32_t>(heads)) * 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int32_t tok = t0 + lane;
  for (int c4 = warp; c4 < kC4; c4 += 8) {
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (tok < total) v = __ldcs(acc + (static_cast<size_t>(h) * kC4 + c4) * total + tok);
    *reinterpret_cast<uint2*>(tile + lane * kStride + c4 * 8) = make_uint2(pack_bf16x2(v.x, v.y), pack_bf16x2(v.z, v.w));
  }
  __syncthreads();
  for (int j = threadIdx.x; j < 32 * kChunks; j += 256) {
    const int r = j / kChunks, c = j % kChunks;
    if (t0 + r < total)
      *reinterpret_cast<uint4*>(dq + (static_cast<size_t>(t0 + r) * heads + h) * D + c * 8) =
          *reinterpret_cast<const uint4*>(tile + r * kStride + c * 16);
  }
}

}  // namespace pa
