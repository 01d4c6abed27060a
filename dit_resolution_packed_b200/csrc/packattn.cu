// packattn.cu -- host side of the C ABI declared in include/packattn.h.
//
// A call validates its arguments on the host, finds (or grows) the workspace of
// its (device, stream) pair, encodes three template tensor maps over the whole
// q / k / v matrices, and enqueues two kernels on the caller's stream:
// the segment scheduler (one CTA) and the persistent attention kernel (one CTA
// per SM).  Nothing synchronises on this path.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <vector>

#include "attn_bwd_sm100.cuh"
#include "attn_fwd_fp8_sm100.cuh"
#include "attn_fwd_sm100.cuh"
#include "gemm_sm100.cuh"
#include "packattn.h"
#include "schedule.cuh"

namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

struct DeviceInfo {
  bool ready = false;
  int sms = 0;
};

struct StreamState {
  int device = -1;
  cudaStream_t stream = nullptr;
  int32_t* status = nullptr;  // never moves once allocated
  uint8_t* ws = nullptr;
  size_t ws_bytes = 0;
  // rotary-embedding table of the last QKV projection: (cos, sin) [rope_rows][rope_d/2]
  float2* rope = nullptr;
  int32_t rope_rows = 0, rope_d = 0;
  double rope_theta = 0.0;
};

std::mutex g_mu;
std::vector<StreamState*> g_states;
DeviceInfo g_dev[64];
int g_wait_limit_ms = 4000;
bool g_short_packing = true;  // pack consecutive short segments into shared tiles (bf16 forward)

// profiling
bool g_prof_on = false;
std::vector<std::pair<cudaEvent_t, cudaEvent_t>> g_prof_events;
size_t g_prof_used = 0;

constexpr size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Forward workspace: counts (4 int32) and the tile ledger (4 int64, from byte 16) in
// the first 128 bytes, then order [B], item_start [B+1], the unit descriptors [B]
// and 3 tensor maps per segment.
struct WsLayout {
  size_t counts, order, item_start, info, maps, total;
};

constexpr size_t kStatsOffset = 16;

WsLayout ws_layout(int32_t batch) {
  WsLayout L;
  L.counts = 0;
  L.order = 128;
  L.item_start = align_up(L.order + 4 * static_cast<size_t>(batch), 128);
  L.info = align_up(L.item_start + 4 * (static_cast<size_t>(batch) + 1), 128);
  L.maps = align_up(L.info + 4 * static_cast<size_t>(batch), 128);
  L.total = L.maps + 384 * static_cast<size_t>(batch);
  return L;
}

int device_of(const void* ptr, int* dev) {
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, ptr) != cudaSuccess) {
    cudaGetLastError();
    return PA_ERR_NOT_DEVICE;
  }
  if (a.type != cudaMemoryTypeDevice && a.type != cudaMemoryTypeManaged) return PA_ERR_NOT_DEVICE;
  *dev = a.device;
  return PA_OK;
}

// Finds or creates the state of (device, stream); the device must be current.  g_mu held.
StreamState* state_for(int device, cudaStream_t stream) {
  for (StreamState* s : g_states)
    if (s->device == device && s->stream == stream) return s;
  StreamState* s = new StreamState();
  s->device = device;
  s->stream = stream;
  g_states.push_back(s);
  return s;
}

int ensure_status(StreamState* s) {
  if (s->status) return PA_OK;
  if (cudaMallocAsync(reinterpret_cast<void**>(&s->status), 128, s->stream) != cudaSuccess) return PA_ERR_CUDA;
  if (cudaMemsetAsync(s->status, 0, 128, s->stream) != cudaSuccess) return PA_ERR_CUDA;
  return PA_OK;
}

int ensure_workspace(StreamState* s, size_t bytes) {
  if (s->ws_bytes >= bytes) return PA_OK;
  if (s->ws) cudaFreeAsync(s->ws, s->stream);
  s->ws = nullptr;
  s->ws_bytes = 0;
  const size_t want = std::max<size_t>(bytes + bytes / 2, 64 * 1024);
  if (cudaMallocAsync(reinterpret_cast<void**>(&s->ws), want, s->stream) != cudaSuccess) return PA_ERR_CUDA;
  s->ws_bytes = want;
  return PA_OK;
}

int ensure_device(int device) {
  if (device < 0 || device >= 64) return PA_ERR_CUDA;
  DeviceInfo& d = g_dev[device];
  if (d.ready) return PA_OK;
  if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, device) != cudaSuccess) return PA_ERR_CUDA;
  if (cudaFuncSetAttribute(pa::attn_fwd_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           pa::FwdCfg<64>::kSmemBytes) != cudaSuccess)
    return PA_ERR_CUDA;
  if (cudaFuncSetAttribute(pa::attn_fwd_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           pa::FwdCfg<128>::kSmemBytes) != cudaSuccess)
    return PA_ERR_CUDA;
  if (cudaFuncSetAttribute(pa::attn_fwd_fp8_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           pa::Fp8Cfg::kSmemBytes) != cudaSuccess)
    return PA_ERR_CUDA;
  if (cudaFuncSetAttribute(pa::gemm_kernel<pa::kEpiPlain>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           pa::kGemmSmemBytes) != cudaSuccess)
    return PA_ERR_CUDA;
  if (cudaFuncSetAttribute(pa::gemm_kernel<pa::kEpiQkvRope>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           pa::kGemmSmemBytes) != cudaSuccess)
    return PA_ERR_CUDA;
  if (cudaFuncSetAttribute(pa::attn_bwd_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           pa::BwdCfg<64>::kSmemBytes) != cudaSuccess)
    return PA_ERR_CUDA;
  if (cudaFuncSetAttribute(pa::attn_bwd_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           pa::BwdCfg<128>::kSmemBytes) != cudaSuccess)
    return PA_ERR_CUDA;
  d.ready = true;
  return PA_OK;
}

bool encode_map(CUtensorMap* m, const void* base, int32_t rows, int32_t heads, int32_t head_dim) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(heads) * head_dim, static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(heads) * head_dim * 2};
  const cuuint32_t box[2] = {64, 128};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// A bf16 row-major [outer, inner] matrix, box {64, box_outer}, 128-byte swizzle.
bool encode_2d(CUtensorMap* m, const void* base, int64_t inner, int64_t outer, uint32_t box_outer) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(outer)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(inner) * 2};
  const cuuint32_t box[2] = {64, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// A byte matrix [outer, inner] with a row stride of `stride` bytes, box 128 x 128,
// 128-byte swizzle (the FP8 operands).
bool encode_u8(CUtensorMap* m, const void* base, int64_t inner, int64_t outer, int64_t stride) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(outer)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(stride)};
  const cuuint32_t box[2] = {128, 128};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int64_t fp8_vt_keys(int32_t batch, int32_t total) {
  return 16 * ((static_cast<int64_t>(total) + 15) / 16) + 16 * static_cast<int64_t>(batch);
}

// Events around the main kernel of a call when profiling is on (ev0 recorded here).
int prof_begin(cudaStream_t stream, cudaEvent_t* ev1) {
  *ev1 = nullptr;
  if (!g_prof_on) return PA_OK;
  if (g_prof_used == g_prof_events.size()) {
    cudaEvent_t a, b;
    if (cudaEventCreate(&a) != cudaSuccess || cudaEventCreate(&b) != cudaSuccess) return PA_ERR_CUDA;
    g_prof_events.emplace_back(a, b);
  }
  cudaEventRecord(g_prof_events[g_prof_used].first, stream);
  *ev1 = g_prof_events[g_prof_used].second;
  ++g_prof_used;
  return PA_OK;
}

// Schedule parameters of a forward call (the template maps are filled by the caller):
// workspace slices, the pack, pair items (2^8 query rows), the status codes.  With
// `units`, the scheduler writes unit descriptors (and packs short segments into shared
// tiles when short-segment packing is on); the FP8 kernel takes one unit per segment.
pa::SchedParams forward_sched(const int32_t* cu, int32_t* status, uint8_t* ws, const WsLayout& L, int32_t batch,
                              int32_t total, int32_t heads, int32_t max_seqlen, uint64_t row_bytes, bool units) {
  pa::SchedParams sp;
  std::memset(&sp, 0, sizeof(sp));
  sp.cu = cu;
  sp.status = status;
  sp.counts = reinterpret_cast<int32_t*>(ws + L.counts);
  sp.order = reinterpret_cast<int32_t*>(ws + L.order);
  sp.item_start = reinterpret_cast<int32_t*>(ws + L.item_start);
  sp.maps = ws + L.maps;
  sp.info = units ? reinterpret_cast<int32_t*>(ws + L.info) : nullptr;
  sp.stats = reinterpret_cast<int64_t*>(ws + L.counts + kStatsOffset);
  sp.group_short = units && g_short_packing ? 1 : 0;
  sp.row_bytes = row_bytes;
  sp.batch = batch;
  sp.total = total;
  sp.heads = heads;
  sp.max_seqlen = max_seqlen;
  sp.rows_log2 = 8;
  sp.err_cu = PA_ERR_CU_SEQLENS;
  sp.err_max = PA_ERR_MAX_SEQLEN;
  return sp;
}

// Attention-kernel parameters of a forward call, reading the schedule that `sp` describes.
pa::FwdParams forward_params(const pa::SchedParams& sp, void* out, float* lse, float scale) {
  pa::FwdParams fp;
  std::memset(&fp, 0, sizeof(fp));
  fp.cu = sp.cu;
  fp.out = out;
  fp.lse = lse;
  fp.counts = sp.counts;
  fp.next_item = sp.counts + 2;
  fp.order = sp.order;
  fp.item_start = sp.item_start;
  fp.maps = sp.maps;
  fp.info = sp.info;
  fp.status = sp.status;
  fp.heads = sp.heads;
  fp.batch = sp.batch;
  fp.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
  fp.wait_limit_ns = static_cast<uint64_t>(g_wait_limit_ms) * 1000000ull;
  fp.err_timeout = PA_ERR_TIMEOUT;
  return fp;
}

// Launches an attention kernel right behind the schedule kernel.  With `pdl`, as a
// programmatic dependent launch: its prologue (barrier set-up, tensor-memory
// allocation) overlaps the schedule kernel, whose results it reads only after
// griddepcontrol.wait.
template <class P>
int launch_after_schedule(void (*kernel)(P), const P& params, int grid, size_t smem, cudaStream_t stream, bool pdl) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(pa::kFwdThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kernel, params) != cudaSuccess || cudaGetLastError() != cudaSuccess) return PA_ERR_CUDA;
  return PA_OK;
}

// Launches the projection GEMM (epilogue kEpi) on the persistent grid.
template <int kEpi>
int launch_gemm(const pa::GemmParams& gp, int dev, cudaStream_t stream) {
  const int64_t tiles = ((static_cast<int64_t>(gp.M) + pa::kGemmBM - 1) / pa::kGemmBM) *
                        ((static_cast<int64_t>(gp.N) + pa::kGemmBN - 1) / pa::kGemmBN);
  const int grid = static_cast<int>(std::min<int64_t>(g_dev[dev].sms, tiles));
  pa::gemm_kernel<kEpi><<<grid, pa::kGemmThreads, pa::kGemmSmemBytes, stream>>>(gp);
  return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

// Backward workspace: the schedule, then lse * log2(e) and D head-major [H][T],
// then the fp32 dq accumulator [H][d/4][T] x 4.
struct BwdWsLayout {
  size_t counts, order, item_start, lse2, delta, dq_acc, total;
};

BwdWsLayout bwd_ws_layout(int32_t batch, int32_t total, int32_t heads, int32_t head_dim) {
  BwdWsLayout L;
  const size_t rows = static_cast<size_t>(total) * heads;
  L.counts = 0;
  L.order = 128;
  L.item_start = align_up(L.order + 4 * static_cast<size_t>(batch), 128);
  L.lse2 = align_up(L.item_start + 4 * (static_cast<size_t>(batch) + 1), 256);
  L.delta = align_up(L.lse2 + 4 * rows, 256);
  L.dq_acc = align_up(L.delta + 4 * rows, 256);
  L.total = L.dq_acc + 4 * rows * static_cast<size_t>(head_dim);
  return L;
}

}  // namespace

// ---- scratch of pa_varlen_attn_fwd_noalloc ----------------------------------
// One fixed array in the library's device image: the status word (bytes
// [0, 256)) and, from byte 256, the schedule + per-segment tensor maps laid out
// as in the allocating path.  Every GPU that loads the library holds it until
// the process exits; every call on that GPU shares it.
constexpr int32_t kNoAllocMaxBatch = 1024;
constexpr size_t kNoAllocStatusBytes = 256;
constexpr size_t kNoAllocScratchBytes = 400 * 1024;
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

namespace {

// Device address of g_noalloc_scratch per device (the host-side name is only a
// stand-in for the symbol); filled by the first call on each device.
uint8_t* g_noalloc_ptr[64] = {};

// The device must be current; g_mu held.
int noalloc_setup(int device) {
  if (g_noalloc_ptr[device]) return PA_OK;
  if (kNoAllocStatusBytes + ws_layout(kNoAllocMaxBatch).total > kNoAllocScratchBytes) return PA_ERR_CUDA;
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) {
    cudaGetLastError();
    return PA_ERR_CUDA;
  }
  if (!p || !aligned(p, 256)) return PA_ERR_CUDA;
  g_noalloc_ptr[device] = static_cast<uint8_t*>(p);
  return PA_OK;
}

}  // namespace

extern "C" {

int pa_varlen_attn_fwd(const void* q, const void* k, const void* v, const int32_t* cu_seqlens, int32_t batch,
                       int32_t total_tokens, int32_t heads, int32_t head_dim, int32_t max_seqlen, float scale,
                       void* out, float* lse, void* stream_handle) {
  // ---- host-visible argument checks: nothing is enqueued on failure
  if (head_dim != 64 && head_dim != 128) return PA_ERR_HEAD_DIM;
  if (heads < 1 || batch < 0 || total_tokens < 0) return PA_ERR_SHAPE;
  if (!std::isfinite(scale)) return PA_ERR_SCALE;
  if (batch == 0 && total_tokens > 0) return PA_ERR_SHAPE;
  if (batch == 0 || total_tokens == 0) return PA_OK;
  if (max_seqlen < 1) return PA_ERR_MAX_SEQLEN;
  if (!q || !k || !v || !cu_seqlens || !out || !lse) return PA_ERR_NULL;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) || !aligned(lse, 4) ||
      !aligned(cu_seqlens, 4))
    return PA_ERR_ALIGN;
  // work items: heads * sum ceil(L_i / 256) <= heads * (ceil(T / 256) + batch) must fit int32
  const int64_t item_bound = static_cast<int64_t>(heads) * ((static_cast<int64_t>(total_tokens) + 255) / 256 + batch);
  if (item_bound >= (int64_t(1) << 31) || static_cast<int64_t>(heads) * head_dim >= (int64_t(1) << 24))
    return PA_ERR_SHAPE;

  int dev = -1, d2 = -1;
  int rc;
  if ((rc = device_of(q, &dev)) != PA_OK) return rc;
  const void* others[5] = {k, v, out, lse, cu_seqlens};
  for (const void* p : others) {
    if ((rc = device_of(p, &d2)) != PA_OK) return rc;
    if (d2 != dev) return PA_ERR_NOT_DEVICE;
  }
  cudaStream_t stream = static_cast<cudaStream_t>(stream_handle);

  std::lock_guard<std::mutex> lock(g_mu);
  if (cudaSetDevice(dev) != cudaSuccess) return PA_ERR_CUDA;
  if ((rc = ensure_device(dev)) != PA_OK) return rc;
  StreamState* st = state_for(dev, stream);
  if ((rc = ensure_status(st)) != PA_OK) return rc;
  const WsLayout L = ws_layout(batch);
  if ((rc = ensure_workspace(st, L.total)) != PA_OK) return rc;

  pa::SchedParams sp = forward_sched(cu_seqlens, st->status, st->ws, L, batch, total_tokens, heads, max_seqlen,
                                     static_cast<uint64_t>(heads) * head_dim * 2, true);
  const void* bases[3] = {q, k, v};
  for (int i = 0; i < 3; ++i) {
    if (!encode_map(&sp.tmpl[i], bases[i], total_tokens, heads, head_dim)) return PA_ERR_CUDA;
    sp.base[i] = bases[i];
  }
  pa::schedule_kernel<<<1, pa::kSchedThreads, 0, stream>>>(sp);
  if (cudaGetLastError() != cudaSuccess) return PA_ERR_CUDA;

  const pa::FwdParams fp = forward_params(sp, out, lse, scale);
  const int grid = static_cast<int>(std::min<int64_t>(g_dev[dev].sms, item_bound));
  cudaEvent_t ev1 = nullptr;
  if ((rc = prof_begin(stream, &ev1)) != PA_OK) return rc;
  // (no programmatic overlap while profiling: the events then bracket the attention kernel alone)
  rc = head_dim == 128 ? launch_after_schedule(pa::attn_fwd_kernel<128>, fp, grid, pa::FwdCfg<128>::kSmemBytes,
                                               stream, !g_prof_on)
                       : launch_after_schedule(pa::attn_fwd_kernel<64>, fp, grid, pa::FwdCfg<64>::kSmemBytes,
                                               stream, !g_prof_on);
  if (rc != PA_OK) return rc;
  if (ev1) cudaEventRecord(ev1, stream);
  return PA_OK;
}

int pa_varlen_attn_bwd(const void* q, const void* k, const void* v, const void* out, const float* lse,
                       const void* dout, const int32_t* cu_seqlens, int32_t batch, int32_t total_tokens,
                       int32_t heads, int32_t head_dim, int32_t max_seqlen, float scale, void* dq, void* dk,
                       void* dv, void* stream_handle) {
  // ---- host-visible argument checks: nothing is enqueued on failure
  if (head_dim != 64 && head_dim != 128) return PA_ERR_HEAD_DIM;
  if (heads < 1 || batch < 0 || total_tokens < 0) return PA_ERR_SHAPE;
  if (!std::isfinite(scale)) return PA_ERR_SCALE;
  if (batch == 0 && total_tokens > 0) return PA_ERR_SHAPE;
  if (batch == 0 || total_tokens == 0) return PA_OK;
  if (max_seqlen < 1) return PA_ERR_MAX_SEQLEN;
  if (!q || !k || !v || !out || !lse || !dout || !cu_seqlens || !dq || !dk || !dv) return PA_ERR_NULL;
  const void* a16[8] = {q, k, v, out, dout, dq, dk, dv};
  for (const void* ptr : a16)
    if (!aligned(ptr, 16)) return PA_ERR_ALIGN;
  if (!aligned(lse, 4) || !aligned(cu_seqlens, 4)) return PA_ERR_ALIGN;
  const int64_t item_bound = static_cast<int64_t>(heads) * ((static_cast<int64_t>(total_tokens) + 127) / 128 + batch);
  if (item_bound >= (int64_t(1) << 31) || static_cast<int64_t>(heads) * head_dim >= (int64_t(1) << 24) ||
      static_cast<int64_t>(total_tokens) * heads * head_dim >= (int64_t(1) << 40))
    return PA_ERR_SHAPE;

  int dev = -1, d2 = -1;
  int rc;
  if ((rc = device_of(q, &dev)) != PA_OK) return rc;
  const void* others[10] = {k, v, out, lse, dout, cu_seqlens, dq, dk, dv, q};
  for (const void* ptr : others) {
    if ((rc = device_of(ptr, &d2)) != PA_OK) return rc;
    if (d2 != dev) return PA_ERR_NOT_DEVICE;
  }
  cudaStream_t stream = static_cast<cudaStream_t>(stream_handle);

  std::lock_guard<std::mutex> lock(g_mu);
  if (cudaSetDevice(dev) != cudaSuccess) return PA_ERR_CUDA;
  if ((rc = ensure_device(dev)) != PA_OK) return rc;
  StreamState* st = state_for(dev, stream);
  if ((rc = ensure_status(st)) != PA_OK) return rc;
  const BwdWsLayout L = bwd_ws_layout(batch, total_tokens, heads, head_dim);
  if ((rc = ensure_workspace(st, L.total)) != PA_OK) return rc;

  pa::BwdParams bp;
  std::memset(&bp, 0, sizeof(bp));
  if (!encode_map(&bp.tm_q, q, total_tokens, heads, head_dim) || !encode_map(&bp.tm_k, k, total_tokens, heads, head_dim) ||
      !encode_map(&bp.tm_v, v, total_tokens, heads, head_dim) ||
      !encode_map(&bp.tm_do, dout, total_tokens, heads, head_dim))
    return PA_ERR_CUDA;
  float* lse2 = reinterpret_cast<float*>(st->ws + L.lse2);
  float* delta = reinterpret_cast<float*>(st->ws + L.delta);
  float* dq_acc = reinterpret_cast<float*>(st->ws + L.dq_acc);
  const size_t rows = static_cast<size_t>(total_tokens) * heads;

  // one launch: D and lse * log2(e), and the zeroed dq accumulator
  const int64_t acc_n4 = static_cast<int64_t>(rows) * (head_dim / 4);
  const size_t prep_warps = (rows + pa::kPrepRowsPerWarp - 1) / pa::kPrepRowsPerWarp;
  const unsigned prep_blocks = static_cast<unsigned>((prep_warps * 32 + 255) / 256);
  if (head_dim == 128)
    pa::bwd_prep_kernel<128><<<prep_blocks, 256, 0, stream>>>(static_cast<const uint16_t*>(out),
                                                            static_cast<const uint16_t*>(dout), lse, delta, lse2,
                                                            reinterpret_cast<float4*>(dq_acc), acc_n4, total_tokens,
                                                            heads);
  else
    pa::bwd_prep_kernel<64><<<prep_blocks, 256, 0, stream>>>(static_cast<const uint16_t*>(out),
                                                           static_cast<const uint16_t*>(dout), lse, delta, lse2,
                                                           reinterpret_cast<float4*>(dq_acc), acc_n4, total_tokens,
                                                           heads);
  if (cudaGetLastError() != cudaSuccess) return PA_ERR_CUDA;

  pa::SchedParams sp;
  std::memset(&sp, 0, sizeof(sp));
  sp.cu = cu_seqlens;
  sp.status = st->status;
  sp.counts = reinterpret_cast<int32_t*>(st->ws + L.counts);
  sp.order = reinterpret_cast<int32_t*>(st->ws + L.order);
  sp.item_start = reinterpret_cast<int32_t*>(st->ws + L.item_start);
  sp.maps = nullptr;
  sp.stats = reinterpret_cast<int64_t*>(st->ws + L.counts + kStatsOffset);
  sp.batch = batch;
  sp.total = total_tokens;
  sp.heads = heads;
  sp.max_seqlen = max_seqlen;
  sp.rows_log2 = 7;
  sp.err_cu = PA_ERR_CU_SEQLENS;
  sp.err_max = PA_ERR_MAX_SEQLEN;
  pa::schedule_kernel<<<1, pa::kSchedThreads, 0, stream>>>(sp);
  if (cudaGetLastError() != cudaSuccess) return PA_ERR_CUDA;

  bp.cu = cu_seqlens;
  bp.counts = sp.counts;
  bp.next_item = sp.counts + 2;
  bp.order = sp.order;
  bp.item_start = sp.item_start;
  bp.lse2 = lse2;
  bp.delta = delta;
  bp.dq_acc = dq_acc;
  bp.dk = dk;
  bp.dv = dv;
  bp.status = st->status;
  bp.heads = heads;
  bp.total = total_tokens;
  bp.scale = scale;
  bp.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
  bp.wait_limit_ns = static_cast<uint64_t>(g_wait_limit_ms) * 1000000ull;
  bp.err_timeout = PA_ERR_TIMEOUT;
  const int grid = static_cast<int>(std::min<int64_t>(g_dev[dev].sms, item_bound));
  cudaEvent_t ev1 = nullptr;
  if (g_prof_on) {  // events around the backward main kernel, as for the forward
    if (g_prof_used == g_prof_events.size()) {
      cudaEvent_t a, b;
      if (cudaEventCreate(&a) != cudaSuccess || cudaEventCreate(&b) != cudaSuccess) return PA_ERR_CUDA;
      g_prof_events.emplace_back(a, b);
    }
    cudaEventRecord(g_prof_events[g_prof_used].first, stream);
    ev1 = g_prof_events[g_prof_used].second;
    ++g_prof_used;
  }
  if (head_dim == 128)
    pa::attn_bwd_kernel<128><<<grid, pa::kBwdThreads, pa::BwdCfg<128>::kSmemBytes, stream>>>(bp);
  else
    pa::attn_bwd_kernel<64><<<grid, pa::kBwdThreads, pa::BwdCfg<64>::kSmemBytes, stream>>>(bp);
  if (cudaGetLastError() != cudaSuccess) return PA_ERR_CUDA;
  if (ev1) cudaEventRecord(ev1, stream);

  const unsigned conv_blocks = static_cast<unsigned>(((static_cast<size_t>(total_tokens) + 31) / 32) * heads);
  if (head_dim == 128)
    pa::bwd_dq_convert_kernel<128><<<conv_blocks, 256, 0, stream>>>(reinterpret_cast<const float4*>(dq_acc),
                                                                  static_cast<uint16_t*>(dq), total_tokens, heads);
  else
    pa::bwd_dq_convert_kernel<64><<<conv_blocks, 256, 0, stream>>>(reinterpret_cast<const float4*>(dq_acc),
                                                                 static_cast<uint16_t*>(dq), total_tokens, heads);
  return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

int pa_linear_fwd(const void* x, const void* w, int32_t rows, int32_t in_features, int32_t out_features, void* y,
                  void* stream_handle) {
  if (rows < 0 || in_features < 1 || out_features < 1) return PA_ERR_SHAPE;
  if (in_features % 8 != 0 || out_features % 32 != 0) return PA_ERR_SHAPE;
  if (rows == 0) return PA_OK;
  if (!x || !w || !y) return PA_ERR_NULL;
  if (!aligned(x, 16) || !aligned(w, 16) || !aligned(y, 16)) return PA_ERR_ALIGN;
  int dev = -1, d2 = -1, rc;
  if ((rc = device_of(x, &dev)) != PA_OK) return rc;
  for (const void* ptr : {w, static_cast<const void*>(y)}) {
    if ((rc = device_of(ptr, &d2)) != PA_OK) return rc;
    if (d2 != dev) return PA_ERR_NOT_DEVICE;
  }
  cudaStream_t stream = static_cast<cudaStream_t>(stream_handle);
  std::lock_guard<std::mutex> lock(g_mu);
  if (cudaSetDevice(dev) != cudaSuccess) return PA_ERR_CUDA;
  if ((rc = ensure_device(dev)) != PA_OK) return rc;
  StreamState* st = state_for(dev, stream);
  if ((rc = ensure_status(st)) != PA_OK) return rc;
  pa::GemmParams gp;
  std::memset(&gp, 0, sizeof(gp));
  if (!encode_2d(&gp.tm_a, x, in_features, rows, 128) || !encode_2d(&gp.tm_b, w, in_features, out_features, 256))
    return PA_ERR_CUDA;
  gp.M = rows;
  gp.N = out_features;
  gp.K = in_features;
  gp.y = y;
  gp.status = st->status;
  gp.wait_limit_ns = static_cast<uint64_t>(g_wait_limit_ms) * 1000000ull;
  gp.err_timeout = PA_ERR_TIMEOUT;
  return launch_gemm<pa::kEpiPlain>(gp, dev, stream);
}

int pa_qkv_rope_fwd(const void* x, const void* w_qkv, const int32_t* cu_seqlens, int32_t batch,
                    int32_t total_tokens, int32_t hidden, int32_t heads, int32_t head_dim, int32_t max_seqlen,
                    float rope_theta, void* q, void* k, void* v, void* stream_handle) {
  if (head_dim != 64 && head_dim != 128) return PA_ERR_HEAD_DIM;
  if (heads < 1 || batch < 0 || total_tokens < 0 || hidden < 1 || hidden % 8 != 0) return PA_ERR_SHAPE;
  if (!std::isfinite(rope_theta)) return PA_ERR_SCALE;
  if (batch == 0 && total_tokens > 0) return PA_ERR_SHAPE;
  if (batch == 0 || total_tokens == 0) return PA_OK;
  const bool rotate = rope_theta > 0.f;
  if (rotate && max_seqlen < 1) return PA_ERR_MAX_SEQLEN;
  if (static_cast<int64_t>(heads) * head_dim * 3 >= (int64_t(1) << 30)) return PA_ERR_SHAPE;
  if (!x || !w_qkv || !q || !k || !v || (rotate && !cu_seqlens)) return PA_ERR_NULL;
  const void* a16[5] = {x, w_qkv, q, k, v};
  for (const void* ptr : a16)
    if (!aligned(ptr, 16)) return PA_ERR_ALIGN;
  if (rotate && !aligned(cu_seqlens, 4)) return PA_ERR_ALIGN;
  int dev = -1, d2 = -1, rc;
  if ((rc = device_of(x, &dev)) != PA_OK) return rc;
  for (const void* ptr : {w_qkv, static_cast<const void*>(q), static_cast<const void*>(k),
                          static_cast<const void*>(v), static_cast<const void*>(cu_seqlens)}) {
    if (ptr == nullptr) continue;
    if ((rc = device_of(ptr, &d2)) != PA_OK) return rc;
    if (d2 != dev) return PA_ERR_NOT_DEVICE;
  }
  cudaStream_t stream = static_cast<cudaStream_t>(stream_handle);
  std::lock_guard<std::mutex> lock(g_mu);
  if (cudaSetDevice(dev) != cudaSuccess) return PA_ERR_CUDA;
  if ((rc = ensure_device(dev)) != PA_OK) return rc;
  StreamState* st = state_for(dev, stream);
  if ((rc = ensure_status(st)) != PA_OK) return rc;
  const int32_t N = 3 * heads * head_dim;
  pa::GemmParams gp;
  std::memset(&gp, 0, sizeof(gp));
  if (!encode_2d(&gp.tm_a, x, hidden, total_tokens, 128) || !encode_2d(&gp.tm_b, w_qkv, hidden, N, 256))
    return PA_ERR_CUDA;
  if (rotate) {
    // positions in the workspace; the (cos, sin) table cached per (device, stream)
    if ((rc = ensure_workspace(st, 4 * static_cast<size_t>(total_tokens))) != PA_OK) return rc;
    if (st->rope == nullptr || st->rope_rows < max_seqlen || st->rope_d != head_dim ||
        st->rope_theta != static_cast<double>(rope_theta)) {
      if (st->rope) cudaFreeAsync(st->rope, stream);
      st->rope = nullptr;
      const size_t n = static_cast<size_t>(max_seqlen) * (head_dim / 2);
      if (cudaMallocAsync(reinterpret_cast<void**>(&st->rope), n * sizeof(float2), stream) != cudaSuccess)
        return PA_ERR_CUDA;
      pa::rope_table_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, stream>>>(
          st->rope, max_seqlen, head_dim, static_cast<double>(rope_theta));
      if (cudaGetLastError() != cudaSuccess) return PA_ERR_CUDA;
      st->rope_rows = max_seqlen;
      st->rope_d = head_dim;
      st->rope_theta = static_cast<double>(rope_theta);
    }
    int32_t* pos = reinterpret_cast<int32_t*>(st->ws);
    pa::rope_positions_kernel<<<static_cast<unsigned>((total_tokens + 255) / 256), 256, 0, stream>>>(
        cu_seqlens, batch, total_tokens, max_seqlen, st->rope_rows, pos, st->status, PA_ERR_CU_SEQLENS,
        PA_ERR_MAX_SEQLEN);
    if (cudaGetLastError() != cudaSuccess) return PA_ERR_CUDA;
    gp.pos = pos;
    gp.rope = st->rope;
  }
  gp.M = total_tokens;
  gp.N = N;
  gp.K = hidden;
  gp.q = q;
  gp.k = k;
  gp.v = v;
  gp.heads = heads;
  gp.head_dim = head_dim;
  gp.status = st->status;
  gp.wait_limit_ns = static_cast<uint64_t>(g_wait_limit_ms) * 1000000ull;
  gp.err_timeout = PA_ERR_TIMEOUT;
  return launch_gemm<pa::kEpiQkvRope>(gp, dev, stream);
}

int pa_get_error(void* stream_handle) {
  cudaStream_t stream = static_cast<cudaStream_t>(stream_handle);
  std::lock_guard<std::mutex> lock(g_mu);
  int dev = 0;
  if (stream != nullptr) {
    if (cudaStreamGetDevice(stream, &dev) != cudaSuccess) return PA_ERR_CUDA;
  } else if (cudaGetDevice(&dev) != cudaSuccess) {
    return PA_ERR_CUDA;
  }
  if (cudaSetDevice(dev) != cudaSuccess) return PA_ERR_CUDA;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return PA_ERR_CUDA;
  StreamState* st = nullptr;
  for (StreamState* s : g_states)
    if (s->device == dev && s->stream == stream) st = s;
  if (!st || !st->status) return PA_OK;
  int32_t h = 0;
  if (cudaMemcpy(&h, st->status, 4, cudaMemcpyDeviceToHost) != cudaSuccess) return PA_ERR_CUDA;
  if (h != 0 && cudaMemset(st->status, 0, 4) != cudaSuccess) return PA_ERR_CUDA;
  return h;
}

const char* pa_status_string(int code) {
  switch (code) {
    case PA_OK: return "ok";
    case PA_ERR_NULL: return "a required pointer is NULL";
    case PA_ERR_ALIGN: return "pointer misaligned (q/k/v/out need 16 bytes, lse/cu_seqlens 4 bytes)";
    case PA_ERR_HEAD_DIM: return "head_dim must be 64 or 128";
    case PA_ERR_SHAPE: return "invalid sizes (heads, batch, total_tokens)";
    case PA_ERR_CU_SEQLENS: return "invalid cu_seqlens (must start at 0, not decrease, end at total_tokens)";
    case PA_ERR_MAX_SEQLEN: return "max_seqlen below 1 or below a segment length";
    case PA_ERR_TIMEOUT: return "a device pipeline wait exceeded its limit";
    case PA_ERR_CUDA: return "CUDA runtime error";
    case PA_ERR_SCALE: return "scale is not finite";
    case PA_ERR_NOT_DEVICE: return "a buffer is not device memory of one GPU";
    case PA_ERR_NOALLOC_LIMIT: return "batch exceeds the 1024 segments of pa_varlen_attn_fwd_noalloc's fixed scratch";
    default: return "unknown status";
  }
}

int pa_version(void) { return 100; }

void pa_release_workspace(void) {
  std::lock_guard<std::mutex> lock(g_mu);
  for (StreamState* s : g_states) {
    if (cudaSetDevice(s->device) == cudaSuccess) {
      cudaDeviceSynchronize();
      if (s->ws) cudaFree(s->ws);
      if (s->rope) cudaFree(s->rope);
      if (s->status) cudaFree(s->status);
    }
    delete s;
  }
  g_states.clear();
}

void pa_set_short_packing(int on) {
  std::lock_guard<std::mutex> lock(g_mu);
  g_short_packing = on != 0;
}

int pa_schedule_stats(void* stream_handle, int64_t* out) {
  if (!out) return PA_ERR_NULL;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_handle);
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return PA_ERR_CUDA;
  uint8_t* ws = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    for (StreamState* s : g_states)
      if (s->device == dev && s->stream == stream) ws = s->ws;
  }
  if (!ws) return PA_ERR_NOT_DEVICE;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return PA_ERR_CUDA;
  int32_t counts[2];
  int64_t stats[4];
  if (cudaMemcpy(counts, ws, sizeof(counts), cudaMemcpyDeviceToHost) != cudaSuccess ||
      cudaMemcpy(stats, ws + kStatsOffset, sizeof(stats), cudaMemcpyDeviceToHost) != cudaSuccess)
    return PA_ERR_CUDA;
  out[0] = counts[0];
  out[1] = counts[1];
  for (int i = 0; i < 4; ++i) out[2 + i] = stats[i];
  return PA_OK;
}

void pa_set_wait_limit_ms(int ms) {
  std::lock_guard<std::mutex> lock(g_mu);
  g_wait_limit_ms = ms < 1 ? 1 : ms;
}

int pa_selftest_wait_timeout(uint32_t limit_us, void* stream_handle) {
  cudaStream_t stream = static_cast<cudaStream_t>(stream_handle);
  std::lock_guard<std::mutex> lock(g_mu);
  int dev = 0;
  if (stream != nullptr) {
    if (cudaStreamGetDevice(stream, &dev) != cudaSuccess) return PA_ERR_CUDA;
  } else if (cudaGetDevice(&dev) != cudaSuccess) {
    return PA_ERR_CUDA;
  }
  if (cudaSetDevice(dev) != cudaSuccess) return PA_ERR_CUDA;
  StreamState* st = state_for(dev, stream);
  if (ensure_status(st) != PA_OK) return PA_ERR_CUDA;
  pa::wait_timeout_selftest_kernel<<<1, 32, 0, stream>>>(st->status, static_cast<uint64_t>(limit_us) * 1000ull,
                                                         PA_ERR_TIMEOUT);
  return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

void pa_profile_enable(int on) {
  std::lock_guard<std::mutex> lock(g_mu);
  g_prof_on = on != 0;
}

int pa_profile_read(double* total_ms, int32_t* launches) {
  std::lock_guard<std::mutex> lock(g_mu);
  double sum = 0.0;
  for (size_t i = 0; i < g_prof_used; ++i) {
    if (cudaEventSynchronize(g_prof_events[i].second) != cudaSuccess) return PA_ERR_CUDA;
    float ms = 0.f;
    if (cudaEventElapsedTime(&ms, g_prof_events[i].first, g_prof_events[i].second) != cudaSuccess) return PA_ERR_CUDA;
    sum += ms;
  }
  if (total_ms) *total_ms = sum;
  if (launches) *launches = static_cast<int32_t>(g_prof_used);
  g_prof_used = 0;
  return PA_OK;
}

int pa_varlen_attn_fwd_noalloc(const void* q, const void* k, const void* v, const int32_t* cu_seqlens,
                               int32_t batch, int32_t total_tokens, int32_t heads, int32_t head_dim,
                               int32_t max_seqlen, float scale, void* out, float* lse, int32_t* status,
                               void* stream_handle) {
  // ---- host-visible argument checks: nothing is enqueued on failure
  if (head_dim != 64 && head_dim != 128) return PA_ERR_HEAD_DIM;
  if (heads < 1 || batch < 0 || total_tokens < 0) return PA_ERR_SHAPE;
  if (batch > kNoAllocMaxBatch) return PA_ERR_NOALLOC_LIMIT;
  if (!std::isfinite(scale)) return PA_ERR_SCALE;
  if (batch == 0 && total_tokens > 0) return PA_ERR_SHAPE;
  if (batch == 0 || total_tokens == 0) return PA_OK;
  if (max_seqlen < 1) return PA_ERR_MAX_SEQLEN;
  if (!q || !k || !v || !cu_seqlens || !out || !lse) return PA_ERR_NULL;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) || !aligned(lse, 4) ||
      !aligned(cu_seqlens, 4) || (status && !aligned(status, 4)))
    return PA_ERR_ALIGN;
  const int64_t item_bound = static_cast<int64_t>(heads) * ((static_cast<int64_t>(total_tokens) + 255) / 256 + batch);
  if (item_bound >= (int64_t(1) << 31) || static_cast<int64_t>(heads) * head_dim >= (int64_t(1) << 24))
    return PA_ERR_SHAPE;

  int dev = -1, d2 = -1;
  int rc;
  if ((rc = device_of(q, &dev)) != PA_OK) return rc;
  const void* others[6] = {k, v, out, lse, cu_seqlens, status};
  for (const void* p : others) {
    if (!p) continue;  // only status may be NULL here
    if ((rc = device_of(p, &d2)) != PA_OK) return rc;
    if (d2 != dev) return PA_ERR_NOT_DEVICE;
  }
  cudaStream_t stream = static_cast<cudaStream_t>(stream_handle);

  std::lock_guard<std::mutex> lock(g_mu);
  if (cudaSetDevice(dev) != cudaSuccess) return PA_ERR_CUDA;
  if ((rc = ensure_device(dev)) != PA_OK) return rc;
  if ((rc = noalloc_setup(dev)) != PA_OK) return rc;
  uint8_t* scratch = g_noalloc_ptr[dev];
  uint8_t* ws = scratch + kNoAllocStatusBytes;
  int32_t* st = status ? status : reinterpret_cast<int32_t*>(scratch);
  const WsLayout L = ws_layout(batch);

  // The status word must start at zero; the schedule kernel rewrites the rest
  // (counts, work counter, order, item starts, unit descriptors, tensor maps)
  // before it is read.
  if (cudaMemsetAsync(st, 0, sizeof(int32_t), stream) != cudaSuccess) return PA_ERR_CUDA;

  pa::SchedParams sp = forward_sched(cu_seqlens, st, ws, L, batch, total_tokens, heads, max_seqlen,
                                     static_cast<uint64_t>(heads) * head_dim * 2, true);
  const void* bases[3] = {q, k, v};
  for (int i = 0; i < 3; ++i) {
    if (!encode_map(&sp.tmpl[i], bases[i], total_tokens, heads, head_dim)) return PA_ERR_CUDA;
    sp.base[i] = bases[i];
  }
  pa::schedule_kernel<<<1, pa::kSchedThreads, 0, stream>>>(sp);
  if (cudaGetLastError() != cudaSuccess) return PA_ERR_CUDA;

  const pa::FwdParams fp = forward_params(sp, out, lse, scale);
  const int grid = static_cast<int>(std::min<int64_t>(g_dev[dev].sms, item_bound));
  return head_dim == 128 ? launch_after_schedule(pa::attn_fwd_kernel<128>, fp, grid, pa::FwdCfg<128>::kSmemBytes,
                                                 stream, true)
                         : launch_after_schedule(pa::attn_fwd_kernel<64>, fp, grid, pa::FwdCfg<64>::kSmemBytes,
                                                 stream, true);
}

int64_t pa_fp8_vt_keys(int32_t batch, int32_t total_tokens) {
  if (batch < 0 || total_tokens < 0) return -1;
  return fp8_vt_keys(batch, total_tokens);
}

namespace {
// The FP8 quantiser. amax_in null: the maxima of this call's q, k, v (a first pass)
// give the scales. Otherwise amax_in's maxima do (delayed scaling: one pass), and this
// call's maxima go to amax_out.
int fp8_quantize(const void* q, const void* k, const void* v, const int32_t* cu_seqlens, int32_t batch,
                 int32_t total_tokens, int32_t heads, int32_t head_dim, const float* amax_in, float* amax_out,
                 void* q8, void* k8, void* v8t, float* scales, void* stream_handle) {
  if (head_dim != 128) return PA_ERR_HEAD_DIM;
  if (heads < 1 || batch < 0 || total_tokens < 0) return PA_ERR_SHAPE;
  if (batch == 0 && total_tokens > 0) return PA_ERR_SHAPE;
  const bool delayed = amax_in != nullptr || amax_out != nullptr;
  if (delayed && (!amax_in || !amax_out)) return PA_ERR_NULL;
  const size_t amax_bytes = 4 * (4 + static_cast<size_t>(heads) * head_dim);
  if (delayed) {
    if (!aligned(amax_in, 4) || !aligned(amax_out, 4)) return PA_ERR_ALIGN;
    const uintptr_t ai = reinterpret_cast<uintptr_t>(amax_in), ao = reinterpret_cast<uintptr_t>(amax_out);
    if (ai < ao + amax_bytes && ao < ai + amax_bytes) return PA_ERR_SHAPE;  // the two must not overlap
  }
  if (batch == 0 || total_tokens == 0) {
    if (!delayed) return PA_OK;
    // no tokens: this call's maxima are all zero
    int dev0 = -1, rc0;
    if ((rc0 = device_of(amax_out, &dev0)) != PA_OK) return rc0;
    std::lock_guard<std::mutex> lock(g_mu);
    if (cudaSetDevice(dev0) != cudaSuccess) return PA_ERR_CUDA;
    return cudaMemsetAsync(amax_out, 0, amax_bytes, static_cast<cudaStream_t>(stream_handle)) == cudaSuccess
               ? PA_OK
               : PA_ERR_CUDA;
  }
  if (!q || !k || !v || !cu_seqlens || !q8 || !k8 || !v8t || !scales) return PA_ERR_NULL;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(q8, 16) || !aligned(k8, 16) ||
      !aligned(v8t, 16) || !aligned(scales, 16) || !aligned(cu_seqlens, 4))
    return PA_ERR_ALIGN;
  const int64_t tiles = (static_cast<int64_t>(total_tokens) + pa::kQuantTile - 1) / pa::kQuantTile;
  if (heads > 65535 || static_cast<int64_t>(heads) * head_dim >= (int64_t(1) << 24) ||
      fp8_vt_keys(batch, total_tokens) >= (int64_t(1) << 32))
    return PA_ERR_SHAPE;
  int dev = -1, d2 = -1;
  int rc;
  if ((rc = device_of(q, &dev)) != PA_OK) return rc;
  const void* others[9] = {k, v, cu_seqlens, q8, k8, v8t, scales, delayed ? amax_in : q, delayed ? amax_out : q};
  for (const void* p : others) {
    if ((rc = device_of(p, &d2)) != PA_OK) return rc;
    if (d2 != dev) return PA_ERR_NOT_DEVICE;
  }
  cudaStream_t stream = static_cast<cudaStream_t>(stream_handle);
  std::lock_guard<std::mutex> lock(g_mu);
  if (cudaSetDevice(dev) != cudaSuccess) return PA_ERR_CUDA;
  if ((rc = ensure_device(dev)) != PA_OK) return rc;
  const dim3 qgrid(static_cast<unsigned>(tiles), heads);
  const int64_t vt_keys = fp8_vt_keys(batch, total_tokens);
  if (delayed) {
    if (cudaMemsetAsync(amax_out, 0, amax_bytes, stream) != cudaSuccess) return PA_ERR_CUDA;
    pa::fp8_quantize_kernel<true><<<qgrid, pa::kQuantizeThreads, 0, stream>>>(
        static_cast<const uint4*>(q), static_cast<const uint4*>(k), static_cast<const uint4*>(v), cu_seqlens, batch,
        total_tokens, heads, reinterpret_cast<const uint32_t*>(amax_in), static_cast<uint2*>(q8),
        static_cast<uint2*>(k8), static_cast<uint8_t*>(v8t), vt_keys, scales, reinterpret_cast<uint32_t*>(amax_out));
    return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
  }
  StreamState* st = state_for(dev, stream);
  if ((rc = ensure_status(st)) != PA_OK) return rc;
  if ((rc = ensure_workspace(st, amax_bytes)) != PA_OK) return rc;
  uint32_t* amax = reinterpret_cast<uint32_t*>(st->ws);
  if (cudaMemsetAsync(amax, 0, amax_bytes, stream) != cudaSuccess) return PA_ERR_CUDA;
  const int32_t nch8 = heads * head_dim / 8;
  const int gx = (nch8 + 31) / 32;
  const int64_t gy_want = std::max<int64_t>(1, (4 * static_cast<int64_t>(g_dev[dev].sms)) / gx);
  const int gy = static_cast<int>(std::min<int64_t>({gy_want, (static_cast<int64_t>(total_tokens) + 7) / 8, 65535}));
  pa::fp8_amax_kernel<<<dim3(gx, gy), pa::kQuantThreads, 0, stream>>>(
      static_cast<const uint4*>(q), static_cast<const uint4*>(k), static_cast<const uint4*>(v), total_tokens, nch8,
      amax);
  if (cudaGetLastError() != cudaSuccess) return PA_ERR_CUDA;
  pa::fp8_quantize_kernel<false><<<qgrid, pa::kQuantizeThreads, 0, stream>>>(
      static_cast<const uint4*>(q), static_cast<const uint4*>(k), static_cast<const uint4*>(v), cu_seqlens, batch,
      total_tokens, heads, amax, static_cast<uint2*>(q8), static_cast<uint2*>(k8), static_cast<uint8_t*>(v8t),
      vt_keys, scales, nullptr);
  return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}
}  // namespace

int pa_fp8_quantize_qkv(const void* q, const void* k, const void* v, const int32_t* cu_seqlens, int32_t batch,
                        int32_t total_tokens, int32_t heads, int32_t head_dim, void* q8, void* k8, void* v8t,
                        float* scales, void* stream_handle) {
  return fp8_quantize(q, k, v, cu_seqlens, batch, total_tokens, heads, head_dim, nullptr, nullptr, q8, k8, v8t,
                      scales, stream_handle);
}

int pa_fp8_quantize_qkv_delayed(const void* q, const void* k, const void* v, const int32_t* cu_seqlens,
                                int32_t batch, int32_t total_tokens, int32_t heads, int32_t head_dim,
                                const float* amax_in, float* amax_out, void* q8, void* k8, void* v8t, float* scales,
                                void* stream_handle) {
  if (!amax_in || !amax_out) return PA_ERR_NULL;
  return fp8_quantize(q, k, v, cu_seqlens, batch, total_tokens, heads, head_dim, amax_in, amax_out, q8, k8, v8t,
                      scales, stream_handle);
}

int pa_varlen_attn_fwd_fp8(const void* q8, const void* k8, const void* v8t, const float* scales,
                           const int32_t* cu_seqlens, int32_t batch, int32_t total_tokens, int32_t heads,
                           int32_t head_dim, int32_t max_seqlen, float scale, void* out, float* lse,
                           void* stream_handle) {
  if (head_dim != 128) return PA_ERR_HEAD_DIM;
  if (heads < 1 || batch < 0 || total_tokens < 0) return PA_ERR_SHAPE;
  if (!std::isfinite(scale)) return PA_ERR_SCALE;
  if (batch == 0 && total_tokens > 0) return PA_ERR_SHAPE;
  if (batch == 0 || total_tokens == 0) return PA_OK;
  if (max_seqlen < 1) return PA_ERR_MAX_SEQLEN;
  if (!q8 || !k8 || !v8t || !scales || !cu_seqlens || !out || !lse) return PA_ERR_NULL;
  if (!aligned(q8, 16) || !aligned(k8, 16) || !aligned(v8t, 16) || !aligned(scales, 16) || !aligned(out, 16) ||
      !aligned(lse, 4) || !aligned(cu_seqlens, 4))
    return PA_ERR_ALIGN;
  const int64_t item_bound = static_cast<int64_t>(heads) * ((static_cast<int64_t>(total_tokens) + 255) / 256 + batch);
  const int64_t vt_keys = fp8_vt_keys(batch, total_tokens);
  if (item_bound >= (int64_t(1) << 31) || static_cast<int64_t>(heads) * head_dim >= (int64_t(1) << 24) ||
      vt_keys >= (int64_t(1) << 32))
    return PA_ERR_SHAPE;
  int dev = -1, d2 = -1;
  int rc;
  if ((rc = device_of(q8, &dev)) != PA_OK) return rc;
  const void* others[6] = {k8, v8t, scales, out, lse, cu_seqlens};
  for (const void* p : others) {
    if ((rc = device_of(p, &d2)) != PA_OK) return rc;
    if (d2 != dev) return PA_ERR_NOT_DEVICE;
  }
  cudaStream_t stream = static_cast<cudaStream_t>(stream_handle);
  std::lock_guard<std::mutex> lock(g_mu);
  if (cudaSetDevice(dev) != cudaSuccess) return PA_ERR_CUDA;
  if ((rc = ensure_device(dev)) != PA_OK) return rc;
  StreamState* st = state_for(dev, stream);
  if ((rc = ensure_status(st)) != PA_OK) return rc;
  const WsLayout L = ws_layout(batch);
  if ((rc = ensure_workspace(st, L.total)) != PA_OK) return rc;

  const int64_t hd = static_cast<int64_t>(heads) * head_dim;
  pa::SchedParams sp = forward_sched(cu_seqlens, st->status, st->ws, L, batch, total_tokens, heads, max_seqlen,
                                     static_cast<uint64_t>(hd), false);
  if (!encode_u8(&sp.tmpl[0], q8, hd, total_tokens, hd) || !encode_u8(&sp.tmpl[1], k8, hd, total_tokens, hd) ||
      !encode_u8(&sp.tmpl[2], v8t, vt_keys, hd, vt_keys))
    return PA_ERR_CUDA;
  sp.base[0] = q8;
  sp.base[1] = k8;
  sp.base[2] = v8t;
  sp.v_keys_inner = 1;
  pa::schedule_kernel<<<1, pa::kSchedThreads, 0, stream>>>(sp);
  if (cudaGetLastError() != cudaSuccess) return PA_ERR_CUDA;

  pa::Fp8Params fp;
  std::memset(&fp, 0, sizeof(fp));
  fp.f = forward_params(sp, out, lse, scale);
  fp.scales = scales;
  const int grid = static_cast<int>(std::min<int64_t>(g_dev[dev].sms, item_bound));
  cudaEvent_t ev1 = nullptr;
  if ((rc = prof_begin(stream, &ev1)) != PA_OK) return rc;
  if ((rc = launch_after_schedule(pa::attn_fwd_fp8_kernel, fp, grid, pa::Fp8Cfg::kSmemBytes, stream, !g_prof_on)) !=
      PA_OK)
    return rc;
  if (ev1) cudaEventRecord(ev1, stream);
  return PA_OK;
}

}  // extern "C"
