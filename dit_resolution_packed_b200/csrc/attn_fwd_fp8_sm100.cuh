// attn_fwd_fp8_sm100.cuh -- FP8 (E4M3) variant of the packed varlen attention
// forward for B200 (sm_100a), head_dim 128.
//
// Quantisation granularity (FPS Attention slides of the Mage-Flow talk: Q and K
// per tensor, V per channel, P per tensor):
//   q = s_q * q8,  k = s_k * k8            one fp32 scale per tensor
//   v[:, h, c] = s_v[h, c] * v8[:, h, c]   one fp32 scale per (head, channel)
//   P8 = E4M3(2^(x - m + kFp8PShift))       one static power-of-two scale for P
// with x = scale * log2(e) * s_q * s_k * (q8 . k8).  The tensor core computes
// S = q8 k8^T and O = P8 v8 with kind::f8f6f4 MMAs (fp32 accumulators in tensor
// memory, K = 32 per instruction: twice the bf16 rate), and the epilogue applies
//   out[c] = s_v[c] * O[c] / sum(P8),   lse = (m - kFp8PShift + log2 sum(P)) * ln 2,
// where sum(P8) adds the E4M3 weights the MMA used (so each output row is a convex
// combination of the dequantised value rows) and sum(P) the unrounded ones.
//
// Differences from the bf16 kernel (attn_fwd_sm100.cuh), whose work items,
// scheduler hand-off, barriers and warp roles this kernel shares:
//   * Q / K tiles are 128 rows x 128 bytes (one 128-byte swizzle atom), V arrives
//     transposed ([channels][keys], K-major for the P.V MMA) from the quantiser;
//   * P goes to shared memory (E4M3, 128-byte swizzled, K-major) and both MMAs
//     read shared memory; tensor memory holds S0 | S1 | O0 | O1 as before;
//   * the K/V ring holds 10 tiles of 16 KB.
#pragma once
#include <cuda.h>

#include <cstdint>

#include "attn_fwd_sm100.cuh"
#include "sm100_ptx.cuh"

namespace pa {

// Between moves of the shift, x - m <= kFp8Rescale, so the stored weights stay
// <= 2^(kFp8Rescale + kFp8PShift) = 256, inside E4M3's finite range (448), and the
// row maximum lands at >= 2^kFp8PShift = 16, far above the subnormals (< 2^-6).
constexpr float kFp8Rescale = 4.0f;
constexpr float kFp8PShift = 4.0f;
// Key pairs of every group of four exponentiated on the FMA pipe (polynomial).
constexpr int kFp8PolyPairsPer4 = 1;

struct Fp8Cfg {
  static constexpr int D = 128;
  static constexpr int kRows = 128;
  static constexpr int kTileBytes = 128 * 128;  // 128 rows of 128 one-byte values
  static constexpr int kSlots = 10;             // K/V ring depth (tiles)
  static constexpr int kOffQ = 0;
  static constexpr int kOffP = kOffQ + 2 * kTileBytes;
  static constexpr int kOffKV = kOffP + 2 * kTileBytes;
  static constexpr int kOffBar = kOffKV + kSlots * kTileBytes;
  static constexpr int kSmemBytes = kOffBar + 512 + 1024;  // + 1024 for base alignment
  static constexpr uint32_t kTmemCols = 512;
  // tensor memory: S0 [0,128) S1 [128,256) O0 [256,384) O1 [384,512)
  __host__ __device__ static constexpr uint32_t col_s(int tile) { return tile ? 128u : 0u; }
  __host__ __device__ static constexpr uint32_t col_o(int tile) { return tile ? 384u : 256u; }
};
static_assert(Fp8Cfg::kSlots <= 12, "barrier arrays");
static_assert(sizeof(Bars) <= 512, "barrier block");

struct Fp8Params {
  FwdParams f;           // maps: q8, k8 per segment and the transposed v8 per segment
  const float* scales;   // [0] s_q, [1] s_k, [4 + h * 128 + c] s_v
};

// ---------------------------------------------------------------- FP8 PTX
// Instruction descriptor, kind::f8f6f4: E4M3 A and B (format 0), fp32 D, both
// K-major; N/8 at bit 17, M/16 at bit 24 as for kind::f16.
__host__ __device__ constexpr uint32_t idesc_e4m3_f32(uint32_t M, uint32_t N) {
  return (1u << 4) | ((N >> 3) << 17) | ((M >> 4) << 24);
}
__device__ __forceinline__ void mma_f8_ss_lo_if(uint32_t issue, uint32_t d_tmem, uint32_t a_lo, uint32_t b_lo,
                                                uint32_t hi, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t.reg .b64 da, db;\n\t"
      "setp.ne.b32 p, %5, 0;\n\t"
      "setp.ne.b32 q, %6, 0;\n\t"
      "mov.b64 da, {%1, %3};\n\t"
      "mov.b64 db, {%2, %3};\n\t"
      "@q tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], da, db, %4, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_lo), "r"(b_lo), "r"(hi), "r"(idesc), "r"(accumulate), "r"(issue)
      : "memory");
}
// E4M3 pair of an fp32 pair (low lane -> low byte), round to nearest even, saturating.
__device__ __forceinline__ uint32_t pack_e4m3x2_pair(uint64_t x) {
  uint16_t r;
  asm("{\n\t.reg .f32 a, b;\n\t"
      "mov.b64 {a, b}, %1;\n\t"
      "cvt.rn.satfinite.e4m3x2.f32 %0, b, a;\n\t}"
      : "=h"(r)
      : "l"(x));
  return r;
}
// Exact f16 pair of an E4M3 pair (low byte -> low half).
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t x) {
  uint32_t r;
  const uint16_t h = static_cast<uint16_t>(x);
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"(h));
  return r;
}
__device__ __forceinline__ uint32_t add_f16x2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("add.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}
// fp32 sum of the two halves of an f16 pair.
__device__ __forceinline__ float f16x2_sum_f32(uint32_t a) {
  float r;
  asm("{\n\t.reg .b16 lo, hi;\n\t.reg .f32 x, y;\n\t"
      "mov.b32 {lo, hi}, %1;\n\t"
      "cvt.f32.f16 x, lo;\n\t"
      "cvt.f32.f16 y, hi;\n\t"
      "add.rn.f32 %0, x, y;\n\t}"
      : "=f"(r)
      : "r"(a));
  return r;
}
__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d)
               : "memory");
}

// ------------------------------------------------------------------ producer
__device__ __forceinline__ void run_producer_fp8(const Fp8Params& pp, uint8_t* smem, Bars* bars, const WaitCtl& wc,
                                                 int32_t n_items, int32_t n_sorted) {
  using C = Fp8Cfg;
  const FwdParams& p = pp.f;
  int slot = 0;
  uint32_t phase = 0;
  uint32_t q_round = 0, sk = 0;
  uint32_t armed = 0, armed_phase = 0;
  bool q_armed = false;
  uint32_t q_armed_phase = 0;
  bool ok = true;
  for (;;) {
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
    const int32_t xcol = w.head * C::D;  // byte column of the head in a q8 / k8 row; row of v8^T
    if (!(ok = mbar_wait(&bars->q_empty, (q_round & 1u) ^ 1u, wc))) break;
    mbar_arrive_expect_tx(&bars->q_full, (w.two ? 2u : 1u) * C::kTileBytes);
    q_armed = true;
    q_armed_phase = q_round & 1u;
    tma_load_2d(smem + C::kOffQ, mq, xcol, w.q0, &bars->q_full);
    if (w.two) tma_load_2d(smem + C::kOffQ + C::kTileBytes, mq, xcol, w.q0 + 128, &bars->q_full);
    ++q_round;
    for (int32_t j = 0; ok && j < w.nkv; ++j) {
#pragma unroll
      for (int which = 0; which < 2; ++which) {
        if (!(ok = mbar_wait(&bars->kv_empty[slot], phase ^ 1u, wc))) break;
        mbar_arrive_expect_tx(&bars->kv_full[slot], C::kTileBytes);
        armed |= 1u << slot;
        armed_phase = (armed_phase & ~(1u << slot)) | (phase << slot);
        uint8_t* dst = smem + C::kOffKV + slot * C::kTileBytes;
        if (which == 0)
          tma_load_2d(dst, mk, xcol, j * 128, &bars->kv_full[slot]);  // K_j: keys x channels
        else
          tma_load_2d(dst, mv, j * 128, xcol, &bars->kv_full[slot]);  // V_j^T: channels x keys
        if (++slot == C::kSlots) {
          slot = 0;
          phase ^= 1u;
        }
      }
    }
    if (!ok) break;
  }
  if (!ok) {
    const uint64_t lim = wc.limit_ns;
    for (int s = 0; s < C::kSlots; ++s)
      if (armed & (1u << s)) drain_wait(&bars->kv_full[s], (armed_phase >> s) & 1u, lim);
    if (q_armed) drain_wait(&bars->q_full, q_armed_phase, lim);
  }
}

// ------------------------------------------------------------------ MMA issuer
// S = Q8 K8^T: four K = 32 steps across the 128-byte rows.
__device__ __forceinline__ void issue_s_fp8(uint32_t issue, uint32_t d_tmem, uint32_t q_addr, uint32_t k_addr) {
  constexpr uint32_t idesc = idesc_e4m3_f32(128, 128);
  constexpr uint32_t hi = sdesc_sw128_hi(1024);
  const uint32_t a0 = sdesc_sw128_lo(q_addr, 16), b0 = sdesc_sw128_lo(k_addr, 16);
#pragma unroll
  for (int kk = 0; kk < 4; ++kk) mma_f8_ss_lo_if(issue, d_tmem, a0 + kk * 2, b0 + kk * 2, hi, idesc, kk > 0 ? 1u : 0u);
}
// O (+)= P8 V8 over the keys [64*half, 64*half + 64): A = P (rows x keys), B = V^T
// (channels x keys), both K-major in shared memory.
__device__ __forceinline__ void issue_pv_half_fp8(uint32_t issue, uint32_t d_tmem, uint32_t p_addr, uint32_t v_addr,
                                                  int half, bool accumulate) {
  constexpr uint32_t idesc = idesc_e4m3_f32(128, 128);
  constexpr uint32_t hi = sdesc_sw128_hi(1024);
  const uint32_t a0 = sdesc_sw128_lo(p_addr, 16), b0 = sdesc_sw128_lo(v_addr, 16);
#pragma unroll
  for (int kq = 0; kq < 2; ++kq) {
    const int kk = half * 2 + kq;
    mma_f8_ss_lo_if(issue, d_tmem, a0 + kk * 2, b0 + kk * 2, hi, idesc, (accumulate || kk > 0) ? 1u : 0u);
  }
}

__device__ __forceinline__ void run_mma_fp8(uint8_t* smem, Bars* bars, const WaitCtl& wc, uint32_t tmem) {
  using C = Fp8Cfg;
  const uint32_t q_addr0 = smem_u32(smem + C::kOffQ);
  const uint32_t p_addr0 = smem_u32(smem + C::kOffP);
  const uint32_t kv_addr0 = smem_u32(smem + C::kOffKV);
  int slot = 0;
  uint32_t phase = 0, q_round = 0;
  uint32_t p_ph = 0, oe_ph = 0;
  uint32_t sk = 0;
  bool ok = true;
  const uint32_t leader = elect_one_sync();
  for (;;) {
    WorkItem w;
    const int got = next_item_from_ring(bars, sk, wc, false, w);
    if (got != -2 && leader) mbar_arrive(&bars->sched_empty[(sk - 1) & 1]);
    if (got == -2) ok = false;
    if (got <= 0) break;
    if (!(ok = mbar_wait(&bars->q_full, q_round & 1u, wc))) break;
    ++q_round;
    int ks = slot;
    if (!(ok = mbar_wait(&bars->kv_full[slot], phase, wc))) break;
    if (++slot == C::kSlots) { slot = 0; phase ^= 1u; }
    tc_fence_after();
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      if (t == 1 && !w.two) break;
      issue_s_fp8(leader, tmem + C::col_s(t), q_addr0 + t * C::kTileBytes, kv_addr0 + ks * C::kTileBytes);
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
        const uint32_t pt = p_addr0 + t * C::kTileBytes;
        if (!(ok = mbar_wait(&bars->p_full[t][0], (p_ph >> t) & 1u, wc))) break;
        tc_fence_after();
        issue_pv_half_fp8(leader, tmem + C::col_o(t), pt, kv_addr0 + vs * C::kTileBytes, 0, j > 0);
        if (!(ok = mbar_wait(&bars->p_full[t][1], (p_ph >> t) & 1u, wc))) break;
        p_ph ^= 1u << t;
        tc_fence_after();
        issue_pv_half_fp8(leader, tmem + C::col_o(t), pt, kv_addr0 + vs * C::kTileBytes, 1, true);
        if (has_next) {
          if (t == 0) {
            ks = slot;
            if (!(ok = mbar_wait(&bars->kv_full[slot], phase, wc))) break;
            if (++slot == C::kSlots) { slot = 0; phase ^= 1u; }
            tc_fence_after();
          }
          // S_{j+1} of this tile is issued after P_j . V_j, so by the time the softmax
          // warps see it complete, P_j in shared memory has been consumed.
          issue_s_fp8(leader, tmem + C::col_s(t), q_addr0 + t * C::kTileBytes, kv_addr0 + ks * C::kTileBytes);
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
  mma_commit_if(leader, &bars->drain);
  drain_wait(&bars->drain, 0, wc.limit_ns);
}

// ------------------------------------------------------------------ softmax + epilogue
// One 128 x 128 score tile of one row: shift update (rescaling O when it moves),
// P8 = E4M3(2^(x - m + kFp8PShift)) into this row of the swizzled P tile, 16 keys
// (one 16-byte chunk) at a time, in two halves handed to the MMA warp as in the
// bf16 kernel.  l sums the fp32 weights, lr the E4M3 ones (f16 partial sums per
// chunk are exact up to 2^-11 relative).
template <bool kPartial, bool kNeg>
__device__ __forceinline__ void softmax_tile_fp8(const uint64_t (&v)[64], int kv_valid, bool first, float c,
                                                 uint32_t tO, uint32_t p_row, uint32_t sw, float& m, float& l,
                                                 float& lr, uint64_t* p_full_half, int lane) {
  const float xmax = row_extreme<kPartial, kNeg>(v, 0, kv_valid) * c;
  bool rescale = false;
  float alpha = 1.f;
  if (first) {
    m = xmax;
  } else if (__any_sync(0xffffffffu, xmax > m + kFp8Rescale)) {
    const float m_new = fmaxf(m, xmax);
    alpha = ex2_approx(m - m_new);
    l *= alpha;
    lr *= alpha;
    m = m_new;
    rescale = true;
  }
  const uint64_t c2 = f2_pack(c, c);
  const float off = kFp8PShift - m;
  const uint64_t off2 = f2_pack(off, off);
  const float magic = 12582912.0f;  // 1.5 * 2^23
  const Exp2PolyConsts ek{f2_pack(magic, magic), f2_pack(-magic, -magic), f2_pack(kExp2C0, kExp2C0),
                          f2_pack(kExp2C1, kExp2C1), f2_pack(kExp2C2, kExp2C2), f2_pack(kExp2C3, kExp2C3)};
  uint64_t su[2] = {0, 0};
  float lr_t = 0.f;
#pragma unroll
  for (int half = 0; half < 2; ++half) {
#pragma unroll
    for (int ch = 4 * half; ch < 4 * half + 4; ++ch) {
      uint32_t e[8];
      uint32_t hs[2] = {0u, 0u};
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int i = ch * 8 + k;  // pair index: keys 2i, 2i+1
        uint64_t x = f2_fma(v[i], c2, off2);
        if (kPartial) {
          x = f2_pack(2 * i < kv_valid ? f2_lo(x) : -INFINITY, 2 * i + 1 < kv_valid ? f2_hi(x) : -INFINITY);
        }
        const uint64_t pp = (!kPartial && (k & 3) >= 4 - kFp8PolyPairsPer4) ? ex2x2_poly(x, ek) : ex2x2(x);
        su[k & 1] = f2_add(su[k & 1], pp);
        e[k] = pack_e4m3x2_pair(pp);
        hs[k & 1] = add_f16x2(hs[k & 1], e4m3x2_to_f16x2(e[k]));
      }
      lr_t += f16x2_sum_f32(add_f16x2(hs[0], hs[1]));
      st_shared_v4(p_row + ((static_cast<uint32_t>(ch) ^ sw) << 4), e[0] | (e[1] << 16), e[2] | (e[3] << 16),
                   e[4] | (e[5] << 16), e[6] | (e[7] << 16));
    }
    if (half == 1 && rescale) {
      // O *= alpha, as in the bf16 kernel: P.V of this tile has not started (half 0
      // is handed over only below in rescale tiles) and that of the previous tile
      // has completed.
#pragma unroll
      for (int cc = 0; cc < Fp8Cfg::D / 16; ++cc) {
        uint32_t o[16];
        PA_TMEM_LD16(tO + cc * 16, o);
        tmem_wait_ld();
#pragma unroll
        for (int k = 0; k < 16; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha);
        PA_TMEM_ST16(tO + cc * 16, o);
      }
      tmem_wait_st();
    }
    fence_proxy_async_smem();  // P chunks visible to the tensor core
    tc_fence_before();
    __syncwarp();
    if (lane == 0) {
      if (half == 1 && rescale) mbar_arrive(&p_full_half[0]);
      if (half == 1 || !rescale) mbar_arrive(&p_full_half[half]);
    }
  }
  const uint64_t su2 = f2_add(su[0], su[1]);
  l += f2_lo(su2) + f2_hi(su2);
  lr += lr_t;
}

__device__ __forceinline__ void run_softmax_fp8(const Fp8Params& pp, uint8_t* smem, Bars* bars, const WaitCtl& wc,
                                                uint32_t tmem, int tile) {
  using C = Fp8Cfg;
  const FwdParams& p = pp.f;
  const int t = threadIdx.x & 127;
  const int lane = threadIdx.x & 31;
  const uint32_t lane_base = static_cast<uint32_t>(t & ~31) << 16;
  const uint32_t tS = tmem + lane_base + C::col_s(tile);
  const uint32_t tO = tmem + lane_base + C::col_o(tile);
  // this thread's row of the P tile: 8-row groups of 1024 bytes, rows of 128 bytes,
  // 16-byte chunk j of row r stored at chunk position j ^ (r % 8)
  const uint32_t p_row = smem_u32(smem + C::kOffP + tile * C::kTileBytes) + (t >> 3) * 1024 + (t & 7) * 128;
  const uint32_t sw = static_cast<uint32_t>(t & 7);
  const float c = p.scale_log2 * __ldg(pp.scales) * __ldg(pp.scales + 1);
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
    float m = 0.f, l = 0.f, lr = 0.f;
    for (int32_t j = 0; j < w.nkv; ++j) {
      ok = mbar_wait(&bars->s_full[tile], s_ph, wc);
      if (__any_sync(0xffffffffu, !ok)) { ok = false; break; }
      s_ph ^= 1u;
      tc_fence_after();
      uint64_t r[64];
      tmem_ld128_pairs(tS, r);
      const int kv_valid = w.len - j * 128;
      uint64_t* ph = bars->p_full[tile];
      if (kv_valid >= 128) {
        if (c >= 0.f) softmax_tile_fp8<false, false>(r, kv_valid, j == 0, c, tO, p_row, sw, m, l, lr, ph, lane);
        else softmax_tile_fp8<false, true>(r, kv_valid, j == 0, c, tO, p_row, sw, m, l, lr, ph, lane);
      } else {
        if (c >= 0.f) softmax_tile_fp8<true, false>(r, kv_valid, j == 0, c, tO, p_row, sw, m, l, lr, ph, lane);
        else softmax_tile_fp8<true, true>(r, kv_valid, j == 0, c, tO, p_row, sw, m, l, lr, ph, lane);
      }
    }
    if (!ok) break;

    ok = mbar_wait(&bars->o_full[tile], of_ph, wc);
    if (__any_sync(0xffffffffu, !ok)) { ok = false; break; }
    of_ph ^= 1u;
    tc_fence_after();
    const int32_t row = w.q0 + tile * 128 + t;
    const bool row_ok = row < w.len;
    uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.out) +
                                          (static_cast<size_t>(w.beg + (row_ok ? row : 0)) * p.heads + w.head) * C::D);
    const float4* sv = reinterpret_cast<const float4*>(pp.scales + 4 + static_cast<size_t>(w.head) * C::D);
    const float inv_l = 1.0f / lr;
#pragma unroll
    for (int cc = 0; cc < C::D / 32; ++cc) {
      uint32_t o[32];
      PA_TMEM_LD32(tO + cc * 32, o);
      tmem_wait_ld();
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        const float4 a = __ldg(sv + cc * 8 + q4 * 2), b = __ldg(sv + cc * 8 + q4 * 2 + 1);
        const uint32_t* ob = o + q4 * 8;
        uint4 vv;
        vv.x = pack_bf16x2(__uint_as_float(ob[0]) * a.x * inv_l, __uint_as_float(ob[1]) * a.y * inv_l);
        vv.y = pack_bf16x2(__uint_as_float(ob[2]) * a.z * inv_l, __uint_as_float(ob[3]) * a.w * inv_l);
        vv.z = pack_bf16x2(__uint_as_float(ob[4]) * b.x * inv_l, __uint_as_float(ob[5]) * b.y * inv_l);
        vv.w = pack_bf16x2(__uint_as_float(ob[6]) * b.z * inv_l, __uint_as_float(ob[7]) * b.w * inv_l);
        if (row_ok) dst[cc * 4 + q4] = vv;
      }
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&bars->o_empty[tile]);
    if (row_ok) {
      const float lse2 = m - kFp8PShift + __log2f(l);
      p.lse[static_cast<size_t>(w.beg + row) * p.heads + w.head] = lse2 * 0.69314718055994531f;
    }
  }
}

__global__ void __launch_bounds__(kFwdThreads, 1) attn_fwd_fp8_kernel(const __grid_constant__ Fp8Params p) {
  using C = Fp8Cfg;
  extern __shared__ uint8_t smem_raw[];
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
      mbar_init(&bars->sched_empty[t], 9);
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
  const WaitCtl wc{&bars->abort_flag, p.f.status, p.f.wait_limit_ns, p.f.err_timeout};
  pdl_wait_primary();
  const int32_t n_items = p.f.counts[0];
  const int32_t n_sorted = p.f.counts[1];

  if (warp < 8) {
    regs_increase<kSoftmaxRegs>();
    run_softmax_fp8(p, smem, bars, wc, tmem, warp >> 2);
    tc_fence_before();
    named_bar_sync(1, kFwdThreads);
  } else {
    regs_decrease<kControlRegs>();
    if (warp == 8) {
      if ((threadIdx.x & 31) == 0) run_producer_fp8(p, smem, bars, wc, n_items, n_sorted);
    } else if (warp == 9) {
      run_mma_fp8(smem, bars, wc, tmem);
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

// ------------------------------------------------------------------ quantiser
// Absolute maxima of q, k (whole tensors) and v (per (head, channel) column), as
// the bit patterns of non-negative floats (which order like the floats).  Block:
// 32 lanes over 8-channel chunks x 8 token lanes; the grid's y dimension splits
// the tokens.  amax: [0] q, [1] k, [4 + channel] v; zeroed by the caller.
constexpr int kQuantThreads = 256;
__global__ void __launch_bounds__(kQuantThreads) fp8_amax_kernel(const uint4* q, const uint4* k, const uint4* v,
                                                                 int32_t total, int32_t nch8, uint32_t* amax) {
  __shared__ uint32_t s_v[8][32][8];
  __shared__ uint32_t s_qk[8][2];
  const int cl = threadIdx.x & 31, tl = threadIdx.x >> 5;
  const int ch8 = blockIdx.x * 32 + cl;
  uint32_t mq = 0, mk = 0;
  uint32_t mv[4] = {0, 0, 0, 0};  // pairs of bf16 magnitudes
  if (ch8 < nch8) {
    for (int64_t t = static_cast<int64_t>(blockIdx.y) * 8 + tl; t < total; t += static_cast<int64_t>(gridDim.y) * 8) {
      const int64_t idx = t * nch8 + ch8;
      const uint4 a = __ldg(q + idx), b = __ldg(k + idx), c = __ldg(v + idx);
      mq = __vmaxu2(mq, __vmaxu2(__vmaxu2(a.x & 0x7FFF7FFFu, a.y & 0x7FFF7FFFu),
                                  __vmaxu2(a.z & 0x7FFF7FFFu, a.w & 0x7FFF7FFFu)));
      mk = __vmaxu2(mk, __vmaxu2(__vmaxu2(b.x & 0x7FFF7FFFu, b.y & 0x7FFF7FFFu),
                                  __vmaxu2(b.z & 0x7FFF7FFFu, b.w & 0x7FFF7FFFu)));
      mv[0] = __vmaxu2(mv[0], c.x & 0x7FFF7FFFu);
      mv[1] = __vmaxu2(mv[1], c.y & 0x7FFF7FFFu);
      mv[2] = __vmaxu2(mv[2], c.z & 0x7FFF7FFFu);
      mv[3] = __vmaxu2(mv[3], c.w & 0x7FFF7FFFu);
    }
  }
  // bf16 magnitude bits -> fp32 bits (shift by 16)
  uint32_t fq = max(mq & 0xFFFFu, mq >> 16) << 16, fk = max(mk & 0xFFFFu, mk >> 16) << 16;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    fq = max(fq, __shfl_xor_sync(0xffffffffu, fq, o));
    fk = max(fk, __shfl_xor_sync(0xffffffffu, fk, o));
  }
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    s_v[tl][cl][2 * e] = (mv[e] & 0xFFFFu) << 16;
    s_v[tl][cl][2 * e + 1] = (mv[e] >> 16) << 16;
  }
  if (cl == 0) {
    s_qk[tl][0] = fq;
    s_qk[tl][1] = fk;
  }
  __syncthreads();
  // 256 threads: one (chunk lane, element) column each, reduced over the 8 token lanes
  {
    const int col = threadIdx.x;  // 32 chunks x 8 elements
    const int c = col >> 3, e = col & 7;
    uint32_t r = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) r = max(r, s_v[i][c][e]);
    const int chunk = blockIdx.x * 32 + c;
    if (chunk < nch8 && r != 0) atomicMax(amax + 4 + chunk * 8 + e, r);
  }
  if (threadIdx.x < 2) {
    uint32_t r = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) r = max(r, s_qk[i][threadIdx.x]);
    if (r != 0) atomicMax(amax + threadIdx.x, r);
  }
}

// fp32 quantisation multiplier 448 / amax and dequantisation scale amax / 448
// (both 1 for an all-zero group), each one correctly rounded division.
__device__ __forceinline__ float fp8_mult(uint32_t amax_bits) {
  const float a = __uint_as_float(amax_bits);
  return a == 0.f ? 1.f : __fdiv_rn(448.0f, a);
}
__device__ __forceinline__ float fp8_scale(uint32_t amax_bits) {
  const float a = __uint_as_float(amax_bits);
  return a == 0.f ? 1.f : __fdiv_rn(a, 448.0f);
}
// Eight bf16 (one 16-byte chunk) times m, rounded once to fp32 each, then to E4M3.
__device__ __forceinline__ uint2 quant8(uint4 x, float m) {
  const uint32_t w[4] = {x.x, x.y, x.z, x.w};
  uint32_t o[2] = {0, 0};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float lo = __fmul_rn(__uint_as_float(w[i] << 16), m);
    const float hi = __fmul_rn(__uint_as_float(w[i] & 0xFFFF0000u), m);
    o[i >> 1] |= pack_e4m3x2_pair(f2_pack(lo, hi)) << ((i & 1) * 16);
  }
  return make_uint2(o[0], o[1]);
}

// Block (32-token tile, head h): q8, k8 in q's layout, and v8 transposed to
// [h * 128 + c][key] with segment s's keys starting at 16*ceil(cu[s]/16) + 16*s
// (for token t of segment s: key t + 16*ceil(cu[s]/16) + 16*s - cu[s]).
// Also writes the scales: [0] s_q, [1] s_k, [4 + h * 128 + c] s_v.
// kTrack: the maxima of this call's q, k, v are also accumulated into amax_out (same
// layout as amax, zeroed by the caller), for the next call's scales (delayed scaling).
// Small tiles keep the grid many blocks deep, so its last partial wave is short.
constexpr int kQuantTile = 32;       // tokens per block
constexpr int kQuantizeThreads = 128;
template <bool kTrack>
__global__ void __launch_bounds__(kQuantizeThreads) fp8_quantize_kernel(
    const uint4* q, const uint4* k, const uint4* v, const int32_t* cu, int32_t batch, int32_t total, int32_t heads,
    const uint32_t* amax, uint2* q8, uint2* k8, uint8_t* v8t, int64_t vt_keys, float* scales, uint32_t* amax_out) {
  constexpr int D = 128, kT = kQuantTile, NT = kQuantizeThreads;
  constexpr int kChunks = kT / 16;  // 16-token chunks of the tile
  static_assert(kT % 16 == 0 && (kT / 4) * (D / 8) == NT, "one 4-token x 8-channel unit per thread");
  __shared__ __align__(16) uint8_t s_t[D][kT + 4];  // [channel][token] of this tile (word-aligned rows)
  __shared__ float s_mv[D];
  __shared__ int64_t s_off[kT];
  __shared__ int s_vec[kChunks];  // 16-token chunk goes out as one 16-byte store
  __shared__ uint32_t s_am[kTrack ? D + 2 : 1];  // this tile's maxima: v per channel, then q, k
  const int h = blockIdx.y;
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * kT;
  const float mq = fp8_mult(__ldg(amax)), mk = fp8_mult(__ldg(amax + 1));
  if (kTrack)
    for (int i = threadIdx.x; i < D + 2; i += NT) s_am[i] = 0u;
  for (int c = threadIdx.x; c < D; c += NT) {
    const uint32_t a = __ldg(amax + 4 + h * D + c);
    s_mv[c] = fp8_mult(a);
    if (blockIdx.x == 0) scales[4 + h * D + c] = fp8_scale(a);
  }
  if (threadIdx.x < kT) {
    // key offset of each token of the tile in the transposed layout
    const int i = threadIdx.x;
    const int64_t t = t0 + i;
    int64_t off = 0;
    if (t < total) {
      int lo = 0, hi = batch;  // last segment s with cu[s] <= t
      while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (__ldg(cu + mid) <= t) lo = mid; else hi = mid;
      }
      const int64_t beg = __ldg(cu + lo);
      off = 16 * ((beg + 15) / 16) + 16 * static_cast<int64_t>(lo) - beg;
    }
    s_off[i] = off;
  }
  if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) {
    scales[0] = fp8_scale(__ldg(amax));
    scales[1] = fp8_scale(__ldg(amax + 1));
    scales[2] = 0.f;
    scales[3] = 0.f;
  }
  __syncthreads();
  // q, k: 8 codes per 16-byte load; v: four tokens of one 8-channel chunk per thread, so
  // that each channel's four codes go to the transposed tile as one 32-bit word
  uint32_t tq = 0u, tk = 0u;  // pairs of bf16 magnitudes (kTrack)
  {
    const int tg = threadIdx.x >> 4, c8 = threadIdx.x & 15;
    uint32_t pk[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};  // [channel of the chunk]: 4 token bytes
    uint32_t tv[4] = {0u, 0u, 0u, 0u};                   // pairs of bf16 magnitudes of v (kTrack)
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int64_t t = t0 + tg * 4 + u;
      if (t >= total) break;
      const int64_t idx = (t * heads + h) * (D / 8) + c8;
      const uint4 a = __ldg(q + idx), b = __ldg(k + idx);
      q8[idx] = quant8(a, mq);
      k8[idx] = quant8(b, mk);
      const uint4 x = __ldg(v + idx);
      const uint32_t w[4] = {x.x, x.y, x.z, x.w};
      if (kTrack) {
        tq = __vmaxu2(tq, __vmaxu2(__vmaxu2(a.x & 0x7FFF7FFFu, a.y & 0x7FFF7FFFu),
                                   __vmaxu2(a.z & 0x7FFF7FFFu, a.w & 0x7FFF7FFFu)));
        tk = __vmaxu2(tk, __vmaxu2(__vmaxu2(b.x & 0x7FFF7FFFu, b.y & 0x7FFF7FFFu),
                                   __vmaxu2(b.z & 0x7FFF7FFFu, b.w & 0x7FFF7FFFu)));
#pragma unroll
        for (int e = 0; e < 4; ++e) tv[e] = __vmaxu2(tv[e], w[e] & 0x7FFF7FFFu);
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int c = c8 * 8 + 2 * e;
        const float lo = __fmul_rn(__uint_as_float(w[e] << 16), s_mv[c]);
        const float hi = __fmul_rn(__uint_as_float(w[e] & 0xFFFF0000u), s_mv[c + 1]);
        const uint32_t pr = pack_e4m3x2_pair(f2_pack(lo, hi));
        pk[2 * e] |= (pr & 0xFFu) << (8 * u);
        pk[2 * e + 1] |= ((pr >> 8) & 0xFFu) << (8 * u);
      }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) *reinterpret_cast<uint32_t*>(&s_t[c8 * 8 + e][tg * 4]) = pk[e];
    if (kTrack) {  // bf16 magnitude bits << 16 are the fp32 bits of the same value
#pragma unroll
      for (int e = 0; e < 4; ++e) {  // lanes l and l + 16 hold the same channels (two token groups)
        tv[e] = __vmaxu2(tv[e], __shfl_xor_sync(0xffffffffu, tv[e], 16));
        if ((threadIdx.x & 16) == 0) {
          if (tv[e] & 0xFFFFu) atomicMax(&s_am[c8 * 8 + 2 * e], (tv[e] & 0xFFFFu) << 16);
          if (tv[e] >> 16) atomicMax(&s_am[c8 * 8 + 2 * e + 1], (tv[e] >> 16) << 16);
        }
      }
    }
  }
  if (kTrack) {
    uint32_t fq = max(tq & 0xFFFFu, tq >> 16) << 16, fk = max(tk & 0xFFFFu, tk >> 16) << 16;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      fq = max(fq, __shfl_xor_sync(0xffffffffu, fq, o));
      fk = max(fk, __shfl_xor_sync(0xffffffffu, fk, o));
    }
    if ((threadIdx.x & 31) == 0) {
      if (fq) atomicMax(&s_am[D], fq);
      if (fk) atomicMax(&s_am[D + 1], fk);
    }
  }
  // v8^T rows: a 16-token chunk goes out as one 16-byte store when its tokens lie in one
  // segment (equal key offsets: the offset grows at every segment start) and its first key
  // is 16-byte aligned (decided once per block, the same for every row); the other tokens
  // as bytes. Keys are in range for every valid cu_seqlens; the checks keep a malformed one
  // (not validated here) from writing outside the buffer.
  if (threadIdx.x < kChunks) {
    const int tt0 = threadIdx.x * 16;
    const int64_t t_first = t0 + tt0, key0 = t_first + s_off[tt0];
    s_vec[threadIdx.x] = t_first + 15 < total && s_off[tt0] == s_off[tt0 + 15] && (key0 & 15) == 0 &&
                         key0 >= 0 && key0 + 16 <= vt_keys;
  }
  __syncthreads();
  if (kTrack) {
    // maxima only grow: a tile whose maximum is not above the value already in amax_out
    // (read from L2) skips its atomic, so the two whole-tensor words are not hit by every block
    for (int i = threadIdx.x; i < D + 2; i += NT) {
      uint32_t* dst = i < D ? amax_out + 4 + h * D + i : amax_out + i - D;
      if (s_am[i] > __ldcg(dst)) atomicMax(dst, s_am[i]);
    }
  }
  // (channel row, chunk) pairs, chunk fastest: 16-byte stores
  for (int j = threadIdx.x; j < D * kChunks; j += NT) {
    const int c = j / kChunks, ch = j % kChunks;
    if (!s_vec[ch]) continue;
    const uint32_t* src = reinterpret_cast<const uint32_t*>(&s_t[c][ch * 16]);
    uint8_t* row = v8t + static_cast<int64_t>(h * D + c) * vt_keys;
    *reinterpret_cast<uint4*>(row + t0 + ch * 16 + s_off[ch * 16]) = make_uint4(src[0], src[1], src[2], src[3]);
  }
  // (channel row, 4-token group) pairs of the other chunks: bytes
  for (int j = threadIdx.x; j < D * (kT / 4); j += NT) {
    const int c = j / (kT / 4), g = j % (kT / 4);
    if (s_vec[g >> 2]) continue;
    uint8_t* row = v8t + static_cast<int64_t>(h * D + c) * vt_keys;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int tt = g * 4 + e;
      const int64_t t = t0 + tt;
      const int64_t key = t + s_off[tt];
      if (t < total && key >= 0 && key < vt_keys) row[key] = s_t[c][tt];
    }
  }
}

}  // namespace pa
