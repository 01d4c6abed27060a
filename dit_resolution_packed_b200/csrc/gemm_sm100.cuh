// gemm_sm100.cuh -- the projections around the attention, y = x W^T on tcgen05
// (sm_100a), with two epilogues:
//   * plain: y [M, N] bf16 (the output projection, o W_o^T);
//   * QKV + RoPE: the fused QKV projection (Mage-Flow page, "DiT Block" data flow
//     and "fusion strategy one": one GEMM with the stacked weight W_qkv, its output
//     split into q, k, v), written straight into three [M, H, d] tensors, with q and
//     k rotated by the rotary embedding at each token's position inside its image.
//
// Tiles of 128 x 256 outputs; K in blocks of 64 (one 128-byte swizzle row) through a
// four-stage TMA ring (48 KB per stage); tcgen05 M = 128, N = 256, K = 16 MMAs into
// one of two 256-column tensor-memory accumulators, so that the epilogue of a tile
// overlaps the MMAs of the next.  Persistent grid, tiles taken in bands of row tiles
// (kGemmGroupM), so that the CTAs running at once share x rows and W panels in L2.
//
// CTA: warps 0-3 epilogue (one thread per output row), warp 4 TMA producer, warp 5
// tensor-memory owner and MMA issuer (whole warp, one elected lane issues).
#pragma once
#include <cuda.h>

#include <cstdint>

#include "sm100_ptx.cuh"

namespace pa {

constexpr int kGemmThreads = 192;
constexpr int kGemmBM = 128, kGemmBN = 256, kGemmBK = 64;
constexpr int kGemmStages = 4;
constexpr int kGemmABytes = kGemmBM * kGemmBK * 2;  // 16 KB
constexpr int kGemmBBytes = kGemmBN * kGemmBK * 2;  // 32 KB
constexpr int kGemmStageBytes = kGemmABytes + kGemmBBytes;
constexpr int kGemmOffBar = kGemmStages * kGemmStageBytes;
constexpr int kGemmSmemBytes = kGemmOffBar + 256 + 1024;  // + 1024 for base alignment

enum GemmEpilogue : int { kEpiPlain = 0, kEpiQkvRope = 1 };

// Tile order: bands of kGemmGroupM row tiles, each band walked N tile by N tile, so the
// tiles running at once share a few x rows and about half of W's panels.  Measured on
// B200 at the mixed and training shapes against plain row-major order (1): 8 gains
// 5-6 % on the QKV GEMM and up to 2 % on the output projection; 16 is close; column-
// major loses 15-25 % once x outgrows L2.
constexpr int kGemmGroupM = 8;

// Row and column tile of the t-th tile in that order.
__device__ __forceinline__ void gemm_tile(int t, int tiles_m, int tiles_n, int& mt, int& nt) {
  const int per = kGemmGroupM * tiles_n;
  const int g = t / per;
  const int first = g * kGemmGroupM;
  const int size = min(kGemmGroupM, tiles_m - first);
  const int local = t - g * per;
  mt = first + local % size;
  nt = local / size;
}

struct GemmParams {
  CUtensorMap tm_a;      // x [M, K] bf16, box {64, 128}, 128-byte swizzle
  CUtensorMap tm_b;      // W [N, K] bf16, box {64, 256}, 128-byte swizzle
  int32_t M, N, K;
  void* y;               // plain: bf16 [M, N]
  void* q;               // QKV: bf16 [M, H, d] each
  void* k;
  void* v;
  int32_t heads, head_dim;
  const int32_t* pos;    // QKV: position of every token inside its segment
  const float2* rope;    // QKV: (cos, sin) [rope_rows][d/2], nullptr = no rotation
  int32_t* status;
  uint64_t wait_limit_ns;
  int32_t err_timeout;
};

struct GemmBars {
  uint64_t full[kGemmStages], empty[kGemmStages];
  uint64_t acc_full[2], acc_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};
static_assert(sizeof(GemmBars) <= 256, "gemm barrier block");

__device__ __forceinline__ bool gemm_drain_wait(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
  const uint32_t a = smem_u32(bar);
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(a, parity)) {
    if (global_timer_ns() - t0 > limit_ns) return false;
  }
  return true;
}

__device__ __forceinline__ void gemm_producer(const GemmParams& p, uint8_t* smem, GemmBars* bars, const WaitCtl& wc) {
  const int tiles_n = (p.N + kGemmBN - 1) / kGemmBN;
  const int tiles_m = (p.M + kGemmBM - 1) / kGemmBM;
  const int tiles = tiles_m * tiles_n;
  const int kblocks = (p.K + kGemmBK - 1) / kGemmBK;
  int stage = 0;
  uint32_t phase = 0, armed = 0, armed_ph = 0;
  bool ok = true;
  for (int t = blockIdx.x; ok && t < tiles; t += gridDim.x) {
    int mt, nt;
    gemm_tile(t, tiles_m, tiles_n, mt, nt);
    const int m0 = mt * kGemmBM, n0 = nt * kGemmBN;
    for (int kb = 0; kb < kblocks; ++kb) {
      if (!(ok = mbar_wait(&bars->empty[stage], phase ^ 1u, wc))) break;
      mbar_arrive_expect_tx(&bars->full[stage], kGemmStageBytes);
      armed |= 1u << stage;
      armed_ph = (armed_ph & ~(1u << stage)) | (phase << stage);
      uint8_t* dst = smem + stage * kGemmStageBytes;
      tma_load_2d(dst, &p.tm_a, kb * kGemmBK, m0, &bars->full[stage]);
      tma_load_2d(dst + kGemmABytes, &p.tm_b, kb * kGemmBK, n0, &bars->full[stage]);
      if (++stage == kGemmStages) {
        stage = 0;
        phase ^= 1u;
      }
    }
  }
  if (!ok) {
    for (int s = 0; s < kGemmStages; ++s)
      if (armed & (1u << s)) gemm_drain_wait(&bars->full[s], (armed_ph >> s) & 1u, wc.limit_ns);
  }
}

__device__ __forceinline__ void gemm_mma(const GemmParams& p, uint8_t* smem, GemmBars* bars, const WaitCtl& wc,
                                         uint32_t tmem) {
  const int tiles_n = (p.N + kGemmBN - 1) / kGemmBN;
  const int tiles = ((p.M + kGemmBM - 1) / kGemmBM) * tiles_n;
  const int kblocks = (p.K + kGemmBK - 1) / kGemmBK;
  constexpr uint32_t idesc = idesc_bf16_f32(kGemmBM, kGemmBN, false);
  constexpr uint32_t hi = sdesc_sw128_hi(1024);
  const uint32_t base = smem_u32(smem);
  const uint32_t leader = elect_one_sync();
  int stage = 0;
  uint32_t phase = 0, ae_ph = 0;
  int local = 0;
  bool ok = true;
  for (int t = blockIdx.x; ok && t < tiles; t += gridDim.x, ++local) {
    const int buf = local & 1;
    if (!(ok = mbar_wait(&bars->acc_empty[buf], ((ae_ph >> buf) & 1u) ^ 1u, wc))) break;
    ae_ph ^= 1u << buf;
    tc_fence_after();
    const uint32_t d_tmem = tmem + buf * kGemmBN;
    for (int kb = 0; kb < kblocks; ++kb) {
      if (!(ok = mbar_wait(&bars->full[stage], phase, wc))) break;
      tc_fence_after();
      const uint32_t a0 = sdesc_sw128_lo(base + stage * kGemmStageBytes, 16);
      const uint32_t b0 = sdesc_sw128_lo(base + stage * kGemmStageBytes + kGemmABytes, 16);
#pragma unroll
      for (int kk = 0; kk < kGemmBK / 16; ++kk)
        mma_bf16_ss_lo_if(leader, d_tmem, a0 + ((kk * 32) >> 4), b0 + ((kk * 32) >> 4), hi, idesc,
                          (kb > 0 || kk > 0) ? 1u : 0u);
      mma_commit_if(leader, &bars->empty[stage]);
      if (++stage == kGemmStages) {
        stage = 0;
        phase ^= 1u;
      }
    }
    if (!ok) break;
    mma_commit_if(leader, &bars->acc_full[buf]);
  }
  mma_commit_if(leader, &bars->drain);
  gemm_drain_wait(&bars->drain, 0, wc.limit_ns);
}

// Rotate-half RoPE of 32 consecutive pairs (x_c, x_{c+d/2}), c = c0 .. c0+31, in place.
__device__ __forceinline__ void rope32(uint32_t (&lo)[32], uint32_t (&hi)[32], const float2* cs) {
#pragma unroll
  for (int i = 0; i < 32; i += 2) {
    const float4 t = *reinterpret_cast<const float4*>(cs + i);  // (cos, sin) of c0+i and c0+i+1
    const float a0 = __uint_as_float(lo[i]), b0 = __uint_as_float(hi[i]);
    const float a1 = __uint_as_float(lo[i + 1]), b1 = __uint_as_float(hi[i + 1]);
    lo[i] = __float_as_uint(a0 * t.x - b0 * t.y);
    hi[i] = __float_as_uint(a0 * t.y + b0 * t.x);
    lo[i + 1] = __float_as_uint(a1 * t.z - b1 * t.w);
    hi[i + 1] = __float_as_uint(a1 * t.w + b1 * t.z);
  }
}

// 32 fp32 values -> bf16 -> four 16-byte stores at dst.
__device__ __forceinline__ void store32_bf16(uint16_t* dst, const uint32_t (&v)[32]) {
  uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    uint4 w;
    w.x = pack_bf16x2(__uint_as_float(v[8 * u + 0]), __uint_as_float(v[8 * u + 1]));
    w.y = pack_bf16x2(__uint_as_float(v[8 * u + 2]), __uint_as_float(v[8 * u + 3]));
    w.z = pack_bf16x2(__uint_as_float(v[8 * u + 4]), __uint_as_float(v[8 * u + 5]));
    w.w = pack_bf16x2(__uint_as_float(v[8 * u + 6]), __uint_as_float(v[8 * u + 7]));
    d4[u] = w;
  }
}

template <int kEpi>
__device__ __forceinline__ void gemm_epilogue(const GemmParams& p, GemmBars* bars, const WaitCtl& wc, uint32_t tmem) {
  const int tiles_n = (p.N + kGemmBN - 1) / kGemmBN;
  const int tiles_m = (p.M + kGemmBM - 1) / kGemmBM;
  const int tiles = tiles_m * tiles_n;
  const int r = threadIdx.x & 127;
  const int lane = threadIdx.x & 31;
  const uint32_t lane_base = static_cast<uint32_t>(r & ~31) << 16;
  uint32_t af_ph = 0;
  int local = 0;
  for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++local) {
    const int buf = local & 1;
    const bool ok = mbar_wait(&bars->acc_full[buf], (af_ph >> buf) & 1u, wc);
    if (__any_sync(0xffffffffu, !ok)) break;
    af_ph ^= 1u << buf;
    tc_fence_after();
    int mt, nt;
    gemm_tile(t, tiles_m, tiles_n, mt, nt);
    const int m0 = mt * kGemmBM, n0 = nt * kGemmBN;
    const int row = m0 + r;
    const bool row_ok = row < p.M;
    const uint32_t tacc = tmem + lane_base + buf * kGemmBN;
    if (kEpi == kEpiPlain) {
#pragma unroll 1
      for (int cc = 0; cc < kGemmBN / 32; ++cc) {
        uint32_t v[32];
        PA_TMEM_LD32(tacc + 32 * cc, v);
        tmem_wait_ld();
        const int col = n0 + 32 * cc;
        if (row_ok && col < p.N)
          store32_bf16(static_cast<uint16_t*>(p.y) + static_cast<size_t>(row) * p.N + col, v);
      }
    } else {
      const int d = p.head_dim, hd = p.heads * p.head_dim;
      const int half = d >> 1;
      const int prow = (row_ok && p.rope != nullptr) ? __ldg(p.pos + row) : 0;  // no positions without RoPE
      // the tile holds 256 / d whole heads (d in {64, 128}, n0 a multiple of 256, and the
      // q / k / v boundaries are multiples of d)
      const int heads_in_tile = kGemmBN / d;
#pragma unroll 1
      for (int hb = 0; hb < heads_in_tile; ++hb) {
        const int c_head0 = hb * d;  // first column of this head inside the tile
        const int col = n0 + c_head0;
        if (col >= p.N) break;
        const int which = col / hd, head = (col % hd) / d;
        uint16_t* dst = static_cast<uint16_t*>(which == 0 ? p.q : which == 1 ? p.k : p.v) +
                        (static_cast<size_t>(row) * p.heads + head) * d;
        const bool rotate = p.rope != nullptr && which < 2;
#pragma unroll 1
        for (int c0 = 0; c0 < half; c0 += 32) {
          uint32_t lo[32], hi[32];
          PA_TMEM_LD32(tacc + c_head0 + c0, lo);
          PA_TMEM_LD32(tacc + c_head0 + half + c0, hi);
          tmem_wait_ld();
          if (row_ok) {
            if (rotate) rope32(lo, hi, p.rope + static_cast<size_t>(prow) * half + c0);
            store32_bf16(dst + c0, lo);
            store32_bf16(dst + half + c0, hi);
          }
        }
      }
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&bars->acc_empty[buf]);
  }
}

template <int kEpi>
__global__ void __launch_bounds__(kGemmThreads, 1) gemm_kernel(const __grid_constant__ GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  GemmBars* bars = reinterpret_cast<GemmBars*>(smem + kGemmOffBar);
  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kGemmStages; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars->acc_full[b], 1);
      mbar_init(&bars->acc_empty[b], 4);
    }
    mbar_init(&bars->drain, 1);
    bars->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(&bars->tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  const WaitCtl wc{&bars->abort_flag, p.status, p.wait_limit_ns, p.err_timeout};
  if (warp < 4) {
    gemm_epilogue<kEpi>(p, bars, wc, tmem);
  } else if (warp == 4) {
    if ((threadIdx.x & 31) == 0) gemm_producer(p, smem, bars, wc);
  } else {
    gemm_mma(p, smem, bars, wc, tmem);
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// Position of every token inside its segment; a token of no valid segment gets 0 and
// the status word records the problem, as does a position at or past max_seqlen.
// Positions are clamped below rope_rows (the table's rows, >= max_seqlen).
__global__ void rope_positions_kernel(const int32_t* __restrict__ cu, int32_t batch, int32_t total,
                                      int32_t max_seqlen, int32_t rope_rows, int32_t* __restrict__ pos,
                                      int32_t* status, int32_t err_cu, int32_t err_max) {
  const int32_t t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= total) return;
  if (t == 0 && (__ldg(cu) != 0 || __ldg(cu + batch) != total)) atomicCAS(status, 0, err_cu);
  int32_t lo = 0, hi = batch;  // segment lo with cu[lo] <= t < cu[lo + 1]
  while (hi - lo > 1) {
    const int32_t mid = (lo + hi) >> 1;
    if (__ldg(cu + mid) <= t) lo = mid; else hi = mid;
  }
  int32_t pp = t - __ldg(cu + lo);
  if (pp < 0) {
    atomicCAS(status, 0, err_cu);
    pp = 0;
  }
  if (pp >= max_seqlen) atomicCAS(status, 0, err_max);
  if (pp >= rope_rows) pp = rope_rows - 1;
  pos[t] = pp;
}

// (cos, sin) of p * theta^(-2i/d) for p < rows, i < d/2, computed in fp64.
__global__ void rope_table_kernel(float2* __restrict__ table, int32_t rows, int32_t d, double theta) {
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int half = d >> 1;
  if (idx >= static_cast<int64_t>(rows) * half) return;
  const int32_t p = static_cast<int32_t>(idx / half), i = static_cast<int32_t>(idx % half);
  const double ang = static_cast<double>(p) * pow(theta, -2.0 * i / d);
  double s, c;
  sincos(ang, &s, &c);
  table[idx] = make_float2(static_cast<float>(c), static_cast<float>(s));
}

}  // namespace pa
