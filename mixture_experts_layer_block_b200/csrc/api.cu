// api.cu -- the C ABI declared in include/moe_b200.h: argument checks, the workspace,
// tensor-map encoding (cached per weight pointer), kernel launches and status readback.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <new>
#include <vector>

#include "launch.h"
#include "moe_b200.h"
#include "mx.cuh"

namespace moe {
cudaError_t configure_router_kernel();
cudaError_t configure_gemm_kernel();
cudaError_t configure_gemm_pair_kernel(int* max_pairs);
int small_fused_blocks_per_sm();
}  // namespace moe

using namespace moe;

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

struct MapKey {
  const void* ptr;
  uint64_t inner, outer, stride;
  uint32_t box0, box1;
  int dtype;
  bool operator==(const MapKey& o) const {
    return ptr == o.ptr && inner == o.inner && outer == o.outer && stride == o.stride &&
           box0 == o.box0 && box1 == o.box1 && dtype == o.dtype;
  }
};

struct MapEntry {
  MapKey key;
  CUtensorMap map;
};

constexpr int64_t kDefaultTimeoutNs = 2000000000LL;
constexpr size_t kMapCacheMax = 64;
constexpr int kTimingRing = 256;  // forwards whose kernel durations moe_stage_times averages
constexpr int kNumStages = 6;     // router, gating, align scatter, row gather, expert GEMMs, combine

}  // namespace

struct moe_handle {
  moe_config cfg{};
  int device = 0;
  int num_sms = 0;
  char* ws_mem = nullptr;
  size_t ws_bytes = 0;
  Workspace ws{};
  int max_tiles = 0, max_lag = 0, max_units = 0;
  int64_t sorted_len_max = 0, blocks_len_max = 0;
  size_t gate_smem = 0;
  EncodeTiledFn encode = nullptr;
  std::vector<MapEntry> cache;
  CUtensorMap h_routed{}, h_shared{}, xs_map{}, y_map{};
  CUtensorMap h_routed16{}, h_shared16{}, xs_map16{};  // 16-row boxes for batches of <= 16 tokens
  CUtensorMap h_routed32{}, h_shared32{}, xs_map32{}, y_map32{};  // 32-row boxes (SM-pair tiles)
  int max_routed_tiles = 0;
  int64_t routed_rows = 0, tile_rows = 0;  // rows of xs, and of h and y, for either tile height
  int max_pairs = 0;                       // 2-CTA clusters of the pair kernel that fit at once
  int last_workers = 0, last_tile_m = kBM;
  int last_shape = 0;  // expert-GEMM shape of the last forward: 0 general, 1 small, 2 tail, 3 pair
  int last_kernels = 0;  // kernels launched by the last forward
  bool fused_ok = false;  // batches of <= 16 tokens may run as one fused launch on this device
  bool mx_fused_ok = false;  // the same for moe_forward_mxfp8
  int32_t epoch = 0;      // fused forwards launched (the arrival counter's target / grid size)
  int parts_rows = 0;  // rows of the K-split partial logits buffer
  std::vector<cudaEvent_t> ev;  // kTimingRing x (kNumStages + 1) events around the kernels
  int timed = 0;                // forwards recorded since the last moe_stage_times
  bool timing = false;
  cudaStream_t last_stream = nullptr;
  bool have_forward = false;
  int last_T = 0, last_k = 0, last_lag = 0;
  void* x_stage = nullptr;   // [2 slots][max_tokens][H] bf16 (slot 0 for moe_forward_host)
  float* out_stage = nullptr;  // [2 slots][max_tokens][H] fp32 or bf16
  size_t x_slot_bytes = 0, out_slot_bytes = 0;
  // moe_forward_host_async: copy streams and, per staging slot, the events that order the
  // copy in, the forward and the copy back
  cudaStream_t copy_in = nullptr, copy_out = nullptr;
  cudaEvent_t ev_in[2] = {nullptr, nullptr}, ev_done[2] = {nullptr, nullptr}, ev_out[2] = {nullptr, nullptr};
  bool slot_used[2] = {false, false};
  int async_slot = 0;
  bool async_pending = false;
  int dep_extra_next = 0;
  int64_t timeout_ns = kDefaultTimeoutNs;
  // MXFP8 workspace (MOE_FLAG_MXFP8): x in token order and in tile order, h, with their scales
  MxBuffers mx{};
  CUtensorMap mx_xs_map{}, mx_h_map{}, mx_xs_map32{}, mx_h_map32{};
};

namespace {

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int encode_map(moe_handle* h, CUtensorMap* out, const void* ptr, uint64_t inner, uint64_t outer,
               uint64_t stride_bytes, uint32_t box0, uint32_t box1,
               CUtensorMapDataType dtype = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16) {
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {stride_bytes};
  cuuint32_t box[2] = {box0, box1};
  cuuint32_t es[2] = {1, 1};
  CUresult r = h->encode(out, dtype, 2, const_cast<void*>(ptr), dims,
                         strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? MOE_OK : MOE_ERR_CUDA;
}

// Weight maps are cached by (pointer, shape, box): encoding is cheap, but caching keeps the
// per-call host work to a lookup.
int cached_map(moe_handle* h, CUtensorMap* out, const void* ptr, uint64_t inner, uint64_t outer,
               uint64_t stride_bytes, uint32_t box0, uint32_t box1,
               CUtensorMapDataType dtype = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16) {
  const MapKey key{ptr, inner, outer, stride_bytes, box0, box1, (int)dtype};
  for (const MapEntry& e : h->cache)
    if (e.key == key) {
      *out = e.map;
      return MOE_OK;
    }
  MapEntry e{key, {}};
  const int rc = encode_map(h, &e.map, ptr, inner, outer, stride_bytes, box0, box1, dtype);
  if (rc != MOE_OK) return rc;
  if (h->cache.size() >= kMapCacheMax) h->cache.erase(h->cache.begin());
  h->cache.push_back(e);
  *out = e.map;
  return MOE_OK;
}

int capacity_of(const moe_config& c, int T, int k) {
  if (!(c.capacity_factor > 0.f)) return 0;
  const double v = std::ceil((double)c.capacity_factor * (double)T * (double)k / (double)c.num_experts);
  return (int)std::min<double>(v, (double)T * k);
}

Shape make_shape(const moe_handle* h, int T, int k, int tile_m = kBM, int workers = 0) {
  const moe_config& c = h->cfg;
  Shape sh{};
  sh.T = T;
  sh.H = c.hidden;
  sh.D = c.inter;
  sh.Ds = c.inter_shared;
  sh.E = c.num_experts;
  sh.k = k;
  sh.block_m = c.block_m;
  sh.capacity = capacity_of(c, T, k);
  // a chunk holds a whole number of gating CTAs (kGateTokensPerCta tokens each)
  sh.chunk_tokens = ceil_div(std::max(kMinChunkTokens, ceil_div(std::max(T, 1), kMaxChunks)),
                             kGateTokensPerCta) * kGateTokensPerCta;
  sh.num_chunks = std::max(1, ceil_div(T, sh.chunk_tokens));
  sh.sorted_len = T * k + c.num_experts * (c.block_m - 1);
  sh.blocks_len = ceil_div(sh.sorted_len, c.block_m);
  // A group's down tasks are numbered `lag` units after its up tasks: at least four waves of
  // tasks and three waves of up tasks in between, so that a claimed down task rarely finds its
  // tile's up tasks still running (measured: half this lag was 1% slower on the prefill layer,
  // a quarter of it up to 16% slower on the decode layer).
  const int n1 = ceil_div(c.inter, kBN1), n2 = ceil_div(c.hidden, kBN2);
  const int W = workers > 0 ? workers : h->num_sms;  // SMs, or SM pairs
  const int lag = std::max(ceil_div(4 * W, n1 + n2), ceil_div(3 * W, n1));
  sh.lag = std::max(1, std::min(h->max_lag, lag));
  sh.dep_extra = 0;
  sh.tile_m = tile_m;
  sh.claim_batch = std::max(1, c.claim_batch);
  sh.timeout_ns = h->timeout_ns;
  return sh;
}

int check_cuda(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

// Router N tile: the narrowest power of two >= E (at most kRouterMaxN, so that x is read once
// per K split), narrowed while the m-tiles x N tiles x the deepest K split give less than half
// a wave of CTAs (a few tokens then still spread the router weights over many SMs).
int router_bn(int E, int T, int num_sms) {
  int bn = 16;
  while (bn < E && bn < kRouterMaxN) bn *= 2;
  const int mt = ceil_div(std::max(T, 1), kBM);
  while (bn > 16 && (int64_t)mt * ceil_div(E, bn) * kMaxRouterSplits < num_sms / 2) bn /= 2;
  return bn;
}

int select_device(moe_handle* h) { return check_cuda(cudaSetDevice(h->device)); }

}  // namespace

extern "C" {

const char* moe_status_string(int code) {
  switch (code) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED: return "unsupported shape";
    case MOE_ERR_CUDA: return "CUDA error";
    case MOE_ERR_OUT_OF_MEMORY: return "out of device memory";
    case MOE_ERR_MISALIGNED: return "device pointer not 16-byte aligned";
    case MOE_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
    case MOE_ERR_NOT_READY: return "not ready";
    default: return "unknown status";
  }
}

int moe_init(const moe_config* cfg, moe_handle** out) {
  if (!cfg || !out) return MOE_ERR_INVALID_ARG;
  *out = nullptr;
  const moe_config c = *cfg;
  // ---- argument checks (no CUDA call before these pass) ----
  if (c.hidden < 8 || c.hidden % 8 != 0) return MOE_ERR_INVALID_ARG;
  if (c.inter < 8 || c.inter % 8 != 0) return MOE_ERR_INVALID_ARG;
  if (c.inter_shared < 0 || c.inter_shared % 8 != 0) return MOE_ERR_INVALID_ARG;
  if (c.num_experts < 1 || c.num_experts > kMaxExperts) return MOE_ERR_INVALID_ARG;
  if (c.top_k < 1 || c.top_k > std::min(c.num_experts, 32)) return MOE_ERR_INVALID_ARG;
  if (c.block_m < 1 || c.block_m > 4096) return MOE_ERR_INVALID_ARG;
  if (!(c.capacity_factor >= 0.f) || std::isinf(c.capacity_factor)) return MOE_ERR_INVALID_ARG;
  if (c.max_tokens < 1) return MOE_ERR_INVALID_ARG;
  if (c.claim_batch < 0 || c.claim_batch > kMaxClaimBatch) return MOE_ERR_INVALID_ARG;
  const int64_t S_max = (int64_t)c.max_tokens * c.top_k;
  const int64_t sorted_len_max = S_max + (int64_t)c.num_experts * (c.block_m - 1);
  if (sorted_len_max > (int64_t)INT32_MAX / 2) return MOE_ERR_UNSUPPORTED;
  if ((int64_t)c.num_experts * std::max(c.inter, c.hidden) > (int64_t)INT32_MAX / 2) return MOE_ERR_UNSUPPORTED;
  if ((int64_t)c.max_tokens * c.hidden > ((int64_t)1 << 40)) return MOE_ERR_UNSUPPORTED;
  const bool mxfp8 = (c.flags & MOE_FLAG_MXFP8) != 0;
  if (mxfp8 && (c.hidden % kMxBK != 0 || c.inter % kMxBK != 0 || c.inter_shared % kMxBK != 0))
    return MOE_ERR_UNSUPPORTED;

  moe_handle* h = new (std::nothrow) moe_handle();
  if (!h) return MOE_ERR_OUT_OF_MEMORY;
  h->cfg = c;
  h->timeout_ns = c.timeout_ns > 0 ? c.timeout_ns : kDefaultTimeoutNs;
  h->timing = (c.flags & MOE_FLAG_STAGE_TIMING) != 0;
  int rc = MOE_OK;
  auto fail = [&](int code) {
    moe_destroy(h);
    return code;
  };

  if (c.device >= 0) {
    if (cudaSetDevice(c.device) != cudaSuccess) return fail(MOE_ERR_CUDA);
  }
  if (cudaGetDevice(&h->device) != cudaSuccess) return fail(MOE_ERR_CUDA);
  int major = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, h->device) != cudaSuccess)
    return fail(MOE_ERR_CUDA);
  if (major != 10) return fail(MOE_ERR_UNSUPPORTED);
  if (cudaDeviceGetAttribute(&h->num_sms, cudaDevAttrMultiProcessorCount, h->device) != cudaSuccess)
    return fail(MOE_ERR_CUDA);

  // driver entry point for tensor-map encoding (no link-time dependency on libcuda)
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q{};
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess || !fn)
    return fail(MOE_ERR_CUDA);
  h->encode = reinterpret_cast<EncodeTiledFn>(fn);

  // ---- sizes ----
  const int E = c.num_experts;
  h->sorted_len_max = sorted_len_max;
  h->blocks_len_max = ceil_div((int)sorted_len_max, c.block_m);
  h->max_routed_tiles = ceil_div((int)S_max, kBM) + E;  // tile count (128-row tiles: the most)
  // rows: 256-row tiles pad the most (at most 255 rows per expert and per batch)
  h->routed_rows = (int64_t)(ceil_div((int)S_max, 2 * kBM) + E) * 2 * kBM;
  h->tile_rows = h->routed_rows + (c.inter_shared > 0 ? (int64_t)ceil_div(c.max_tokens, 2 * kBM) * 2 * kBM : 0);
  // splits * T <= #SMs * 128 (see router_splits) and splits <= 4
  h->parts_rows = std::min(kMaxRouterSplits * c.max_tokens, (h->num_sms + 1) * kBM);
  h->max_tiles = h->max_routed_tiles + (c.inter_shared > 0 ? ceil_div(c.max_tokens, kBM) : 0);
  h->max_lag = 2 * h->num_sms;
  h->max_units = h->max_tiles + h->max_lag;
  const int ldh = std::max(c.inter, c.inter_shared);
  const int n_task_max = ceil_div(ldh, kBN1) + ceil_div(c.hidden, kBN2);
  const int trace_cap = (c.flags & MOE_FLAG_TRACE) ? h->max_tiles * n_task_max : 0;

  struct Piece {
    void** dst;
    size_t bytes;
  };
  Workspace& w = h->ws;
  const size_t T_ = (size_t)c.max_tokens, K_ = (size_t)c.top_k, E_ = (size_t)E;
  const size_t T_pad = (size_t)ceil_div(c.max_tokens, kBM) * kBM;
  std::vector<Piece> pieces = {
      {(void**)&w.meta, sizeof(DeviceMeta)},
      {(void**)&w.logits, T_ * E_ * 4},
      {(void**)&w.logit_parts, (size_t)h->parts_rows * E_ * 4},
      {(void**)&w.topk_ids, T_ * K_ * 4},
      {(void**)&w.topk_w, T_ * K_ * 4},
      {(void**)&w.chunk_hist, (size_t)kMaxChunks * E_ * 4},
      {(void**)&w.chunk_base, (size_t)kMaxChunks * E_ * 4},
      {(void**)&w.expert_off, (E_ + 1) * 4},
      {(void**)&w.expert_kept, E_ * 4},
      {(void**)&w.sorted_ids, (size_t)sorted_len_max * 4},
      {(void**)&w.expert_ids, (size_t)h->blocks_len_max * 4},
      {(void**)&w.tile_expert, (size_t)h->max_tiles * 4},
      {(void**)&w.tile_row0, (size_t)h->max_tiles * 4},
      {(void**)&w.tile_nrows, (size_t)h->max_tiles * 4},
      {(void**)&w.group_tile0, (size_t)h->max_tiles * 4},
      {(void**)&w.group_ntiles, (size_t)h->max_tiles * 4},
      {(void**)&w.group_tasks, (size_t)h->max_tiles * 4},
      {(void**)&w.expert_group0, (E_ + 2) * 4},
      {(void**)&w.unit_start, (size_t)(h->max_units + 1) * 4},
      {(void**)&w.done1, (size_t)h->max_tiles * 4},
      {(void**)&w.h, (size_t)h->tile_rows * ldh * 2},
      {(void**)&w.expert_tile0, E_ * 4},
      {(void**)&w.row_of_slot, (size_t)S_max * 4},
      {(void**)&w.xs, (size_t)h->routed_rows * c.hidden * 2},
      {(void**)&w.y, (size_t)h->tile_rows * c.hidden * 2},
      {(void**)&w.trace, (size_t)trace_cap * 4 * 8},
      {(void**)&w.waits, (c.flags & MOE_FLAG_TRACE) ? (size_t)h->num_sms * kNumWaits * 8 : 0},
      {(void**)&w.task_tab, (size_t)h->max_tiles * n_task_max * sizeof(int4)},
      {(void**)&w.front, sizeof(FrontSync)},
      {(void**)&w.tok_done, (size_t)kSmallRows * ceil_div(c.hidden, kBN2) * 4},
      {(void**)&w.gather_done, (size_t)h->max_tiles * 4},
      {(void**)&h->x_stage, (c.flags & MOE_FLAG_HOST_STAGING) ? 2 * T_ * c.hidden * 2 : 0},
      {(void**)&h->out_stage, (c.flags & MOE_FLAG_HOST_STAGING) ? 2 * T_ * c.hidden * 4 : 0},
      // MXFP8: codes plus scales (1 byte per 32 elements); token rows padded to whole atoms
      {(void**)&h->mx.xq, mxfp8 && c.inter_shared > 0 ? T_pad * c.hidden : 0},
      {(void**)&h->mx.sf_xq, mxfp8 && c.inter_shared > 0 ? T_pad * c.hidden / kMxBlock : 0},
      {(void**)&h->mx.xs, mxfp8 ? (size_t)h->routed_rows * c.hidden : 0},
      {(void**)&h->mx.sf_xs, mxfp8 ? (size_t)h->routed_rows * c.hidden / kMxBlock : 0},
      {(void**)&h->mx.h, mxfp8 ? (size_t)h->tile_rows * ldh : 0},
      {(void**)&h->mx.sf_h, mxfp8 ? (size_t)h->tile_rows * ldh / kMxBlock : 0},
  };
  size_t total = 0;
  for (const Piece& p : pieces) total += (p.bytes + 255) & ~size_t(255);
  if (cudaMalloc(&h->ws_mem, total) != cudaSuccess) {
    cudaGetLastError();
    return fail(MOE_ERR_OUT_OF_MEMORY);
  }
  h->ws_bytes = total;
  size_t off = 0;
  for (const Piece& p : pieces) {
    *p.dst = p.bytes ? h->ws_mem + off : nullptr;
    off += (p.bytes + 255) & ~size_t(255);
  }
  w.trace_cap = trace_cap;
  w.task_cap = h->max_tiles * n_task_max;
  w.ldh = ldh;
  h->x_slot_bytes = T_ * c.hidden * 2;
  h->out_slot_bytes = T_ * c.hidden * 4;
  if (c.flags & MOE_FLAG_HOST_STAGING) {
    if (cudaStreamCreateWithFlags(&h->copy_in, cudaStreamNonBlocking) != cudaSuccess ||
        cudaStreamCreateWithFlags(&h->copy_out, cudaStreamNonBlocking) != cudaSuccess)
      return fail(MOE_ERR_CUDA);
    for (int i = 0; i < 2; ++i)
      if (cudaEventCreateWithFlags(&h->ev_in[i], cudaEventDisableTiming) != cudaSuccess ||
          cudaEventCreateWithFlags(&h->ev_done[i], cudaEventDisableTiming) != cudaSuccess ||
          cudaEventCreateWithFlags(&h->ev_out[i], cudaEventDisableTiming) != cudaSuccess)
        return fail(MOE_ERR_CUDA);
  }
  if (cudaMemset(h->ws_mem, 0, total) != cudaSuccess) return fail(MOE_ERR_CUDA);

  // h tensor maps (fixed for the handle's lifetime)
  const uint64_t h_rows = (uint64_t)h->tile_rows;
  const uint64_t xs_rows = (uint64_t)h->routed_rows;
  if ((rc = encode_map(h, &h->h_routed, w.h, c.inter, h_rows, (uint64_t)ldh * 2, kBK, kBM))) return fail(rc);
  if (c.inter_shared > 0) {
    if ((rc = encode_map(h, &h->h_shared, w.h, c.inter_shared, h_rows, (uint64_t)ldh * 2, kBK, kBM)))
      return fail(rc);
  } else {
    h->h_shared = h->h_routed;
  }
  if ((rc = encode_map(h, &h->xs_map, w.xs, c.hidden, xs_rows, (uint64_t)c.hidden * 2, kBK, kBM)))
    return fail(rc);
  if ((rc = encode_map(h, &h->xs_map16, w.xs, c.hidden, xs_rows, (uint64_t)c.hidden * 2, kBK, kSmallRows)))
    return fail(rc);
  if ((rc = encode_map(h, &h->xs_map32, w.xs, c.hidden, xs_rows, (uint64_t)c.hidden * 2, kBK, kPairBoxRows)))
    return fail(rc);
  if ((rc = encode_map(h, &h->h_routed32, w.h, c.inter, h_rows, (uint64_t)ldh * 2, kBK, kPairBoxRows)))
    return fail(rc);
  if (c.inter_shared > 0) {
    if ((rc = encode_map(h, &h->h_shared32, w.h, c.inter_shared, h_rows, (uint64_t)ldh * 2, kBK, kPairBoxRows)))
      return fail(rc);
  } else {
    h->h_shared32 = h->h_routed32;
  }
  if ((rc = encode_map(h, &h->y_map32, w.y, c.hidden, h_rows, (uint64_t)c.hidden * 2, kBK, kPairBoxRows)))
    return fail(rc);
  if ((rc = encode_map(h, &h->h_routed16, w.h, c.inter, h_rows, (uint64_t)ldh * 2, kBK, kSmallRows)))
    return fail(rc);
  if (c.inter_shared > 0) {
    if ((rc = encode_map(h, &h->h_shared16, w.h, c.inter_shared, h_rows, (uint64_t)ldh * 2, kBK, kSmallRows)))
      return fail(rc);
  } else {
    h->h_shared16 = h->h_routed16;
  }
  if ((rc = encode_map(h, &h->y_map, w.y, c.hidden, h_rows, (uint64_t)c.hidden * 2, kBK, kBM))) return fail(rc);
  if (mxfp8) {
    if ((rc = encode_map(h, &h->mx_xs_map, h->mx.xs, c.hidden, xs_rows, (uint64_t)c.hidden, kMxBK, kBM,
                         CU_TENSOR_MAP_DATA_TYPE_UINT8)))
      return fail(rc);
    if ((rc = encode_map(h, &h->mx_h_map, h->mx.h, ldh, h_rows, (uint64_t)ldh, kMxBK, kBM,
                         CU_TENSOR_MAP_DATA_TYPE_UINT8)))
      return fail(rc);
    if ((rc = encode_map(h, &h->mx_xs_map32, h->mx.xs, c.hidden, xs_rows, (uint64_t)c.hidden, kMxBK, kPairBoxRows,
                         CU_TENSOR_MAP_DATA_TYPE_UINT8)))
      return fail(rc);
    if ((rc = encode_map(h, &h->mx_h_map32, h->mx.h, ldh, h_rows, (uint64_t)ldh, kMxBK, kPairBoxRows,
                         CU_TENSOR_MAP_DATA_TYPE_UINT8)))
      return fail(rc);
    if (check_cuda(configure_gemm_mx_kernel())) return fail(MOE_ERR_CUDA);
  }

  // kernel attributes
  Shape sh = make_shape(h, c.max_tokens, c.top_k);
  h->gate_smem = gate_smem_bytes(sh, h->max_units);
  const size_t scatter_smem = scatter_smem_bytes(E, sh.chunk_tokens * c.top_k);
  // on the handle's device (current here); raise-only, so no other handle or call loses out
  if (check_cuda(raise_align_smem(h->gate_smem, h->gate_smem, scatter_smem))) return fail(MOE_ERR_CUDA);
  if (check_cuda(configure_router_kernel()) || check_cuda(configure_gemm_kernel())) return fail(MOE_ERR_CUDA);
  if (check_cuda(configure_gemm_pair_kernel(&h->max_pairs))) return fail(MOE_ERR_CUDA);
  // the fused small-batch forward needs one resident CTA per SM at once (cooperative launch)
  int coop = 0;
  if (cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, h->device) != cudaSuccess) return fail(MOE_ERR_CUDA);
  h->fused_ok = coop != 0 && E <= kFusedMaxExperts && small_fused_blocks_per_sm() >= 1 &&
                !(c.flags & MOE_FLAG_UNFUSED_SMALL) && !(c.flags & MOE_FLAG_STATIC_QUOTA);
  h->mx_fused_ok = coop != 0 && E <= kFusedMaxExperts && (c.flags & MOE_FLAG_MXFP8) &&
                   mx_small_fused_blocks_per_sm() >= 1 && !(c.flags & MOE_FLAG_UNFUSED_SMALL);
  h->max_pairs = std::min(h->max_pairs, h->num_sms / 2);
  h->last_workers = h->num_sms;
  if (h->timing) {
    h->ev.assign((size_t)kTimingRing * (kNumStages + 1), nullptr);
    for (auto& e : h->ev)
      if (cudaEventCreate(&e) != cudaSuccess) return fail(MOE_ERR_CUDA);
  }
  *out = h;
  return MOE_OK;
}

void moe_destroy(moe_handle* h) {
  if (!h) return;
  if (h->ws_mem || !h->ev.empty()) {
    cudaSetDevice(h->device);
    cudaDeviceSynchronize();
  }
  for (auto& e : h->ev)
    if (e) cudaEventDestroy(e);
  for (int i = 0; i < 2; ++i) {
    if (h->ev_in[i]) cudaEventDestroy(h->ev_in[i]);
    if (h->ev_done[i]) cudaEventDestroy(h->ev_done[i]);
    if (h->ev_out[i]) cudaEventDestroy(h->ev_out[i]);
  }
  if (h->copy_in) cudaStreamDestroy(h->copy_in);
  if (h->copy_out) cudaStreamDestroy(h->copy_out);
  if (h->ws_mem) cudaFree(h->ws_mem);
  delete h;
}

int64_t moe_sorted_len(const moe_handle* h, int32_t T, int32_t top_k) {
  if (!h || T < 0 || top_k < 0) return -1;
  return (int64_t)T * top_k + (int64_t)h->cfg.num_experts * (h->cfg.block_m - 1);
}

int64_t moe_blocks_len(const moe_handle* h, int32_t T, int32_t top_k) {
  const int64_t n = moe_sorted_len(h, T, top_k);
  if (n < 0) return -1;
  return (n + h->cfg.block_m - 1) / h->cfg.block_m;
}

static int check_tokens(const moe_handle* h, int32_t T, int32_t top_k) {
  if (T < 0 || T > h->cfg.max_tokens) return MOE_ERR_INVALID_ARG;
  if (top_k < 1 || top_k > h->cfg.top_k) return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}

static int forward_impl(moe_handle* h, const void* x, int32_t T, const void* w_router,
                        const float* router_bias, const void* w_up, const void* w_gate,
                        const void* w_down, const moe_shared_w* w_shared, int32_t top_k,
                        void* out, cudaStream_t st) {
  const moe_config& c = h->cfg;
  int rc;
  if ((rc = check_tokens(h, T, top_k))) return rc;
  if (!w_router || !w_up || !w_gate || !w_down) return MOE_ERR_INVALID_ARG;
  if (T > 0 && (!x || !out)) return MOE_ERR_INVALID_ARG;  // an empty batch may pass null x / out
  const bool has_shared = c.inter_shared > 0;
  if (has_shared && (!w_shared || !w_shared->up || !w_shared->gate || !w_shared->down))
    return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(w_router) || !aligned16(w_up) || !aligned16(w_gate) ||
      !aligned16(w_down) || !aligned16(out) || (router_bias && !aligned16(router_bias)))
    return MOE_ERR_MISALIGNED;
  if (has_shared && (!aligned16(w_shared->up) || !aligned16(w_shared->gate) || !aligned16(w_shared->down)))
    return MOE_ERR_MISALIGNED;
  if ((rc = select_device(h))) return rc;
  h->last_stream = st;
  h->last_T = T;
  h->last_k = top_k;
  h->have_forward = true;
  if (T == 0) return MOE_OK;

  const int E = c.num_experts, H = c.hidden, D = c.inter, Ds = c.inter_shared;
  // With at most 16 tokens every m-tile has at most 16 rows (an expert appears once per token):
  // the expert GEMMs use their small-tile shape with 16-row A boxes, and the whole forward runs
  // as one fused launch where the device allows it.
  const bool small = T <= kSmallRows;
  const bool fused = small && h->fused_ok;
  bool pair = false;
  // The pair shape is chosen only on request: on the measured workloads (skewed routing, and
  // 256 experts x top-8 with a shared expert) it was slower than single SMs, whose operand rings
  // already keep the tensor pipe as busy as the memory system allows.
  if (!small && h->max_pairs > 0 && (c.flags & MOE_FLAG_PAIR_TILES) && !(c.flags & MOE_FLAG_SINGLE_TILES))
    pair = true;
  const int workers = pair ? h->max_pairs : h->num_sms;
  Shape sh = make_shape(h, T, top_k, pair ? 2 * kBM : kBM, workers);
  // Merging tails of at most 32 rows into the previous tile's tasks pays when experts get a few
  // 128-row tiles each (many of them then end in a short tail), and costs the general shape's
  // second staging buffer: by default it is used when the mean load per expert is 96..384
  // slots and the capacity allows more than one tile per expert.
  int gemm_shape = small ? kShapeSmall : kShapeGeneral;
  if (!small && !pair) {
    if (c.flags & MOE_FLAG_TWO_TILES) {
      gemm_shape = kShapeTwo;
    } else if (c.flags & MOE_FLAG_TAIL_TILES) {
      gemm_shape = kShapeTail;
    } else if (!(c.flags & MOE_FLAG_NO_TAIL_TILES)) {
      // two-tile task sets once the mean load per expert is above 96 slots and the capacity
      // lets an expert fill more than one tile (measured: 21% faster on the skewed layer, 2% on
      // the DSV3-style layer; 7% slower where every expert has one tile, from the shallower ring)
      const int64_t load = (int64_t)T * top_k;  // slots over E experts
      const int cap = capacity_of(c, T, top_k);
      if (load > (int64_t)96 * E && (cap == 0 || cap > kBM)) gemm_shape = kShapeTwo;
    }
  }
  h->last_shape = pair ? 3 : (gemm_shape == kShapeTwo ? 5 : gemm_shape);
  sh.merge_tail = (gemm_shape == kShapeTail) ? 1 : (gemm_shape == kShapeTwo ? 2 : 0);
  sh.static_quota = (!pair && (c.flags & MOE_FLAG_STATIC_QUOTA)) ? 1 : 0;
  h->last_workers = workers;
  h->last_tile_m = sh.tile_m;
  sh.dep_extra = h->dep_extra_next;
  h->dep_extra_next = 0;
  h->last_lag = sh.lag;
  const Workspace& w = h->ws;

  // tensor maps
  CUtensorMap wr_map;
  GemmMaps maps;
  const int bn = router_bn(E, T, h->num_sms);
  CUtensorMap x_router;
  if ((rc = encode_map(h, &x_router, x, H, T, (uint64_t)H * 2, kBK, kBM))) return rc;
  if (small || pair) {
    if ((rc = encode_map(h, &maps.x_tile, x, H, T, (uint64_t)H * 2, kBK, small ? kSmallRows : kPairBoxRows)))
      return rc;
  } else {
    maps.x_tile = x_router;
  }
  maps.xs = small ? h->xs_map16 : (pair ? h->xs_map32 : h->xs_map);
  maps.y = pair ? h->y_map32 : h->y_map;
  // the pair shape stages half of B (128 rows) per CTA
  const uint32_t bn2 = pair ? (uint32_t)kBN2 / 2 : (uint32_t)kBN2;
  if ((rc = cached_map(h, &wr_map, w_router, H, E, (uint64_t)H * 2, kBK, bn))) return rc;
  if ((rc = cached_map(h, &maps.w_up, w_up, H, (uint64_t)E * D, (uint64_t)H * 2, kBK, kBN1))) return rc;
  if ((rc = cached_map(h, &maps.w_gate, w_gate, H, (uint64_t)E * D, (uint64_t)H * 2, kBK, kBN1))) return rc;
  if ((rc = cached_map(h, &maps.w_down, w_down, D, (uint64_t)E * H, (uint64_t)D * 2, kBK, bn2))) return rc;
  maps.h_routed = small ? h->h_routed16 : (pair ? h->h_routed32 : h->h_routed);
  maps.xs32 = h->xs_map32;
  maps.h_routed32 = h->h_routed32;
  maps.h_shared32 = h->h_shared32;
  if (small || pair) {
    maps.x_tile32 = maps.x_tile;  // unused by these shapes (the pair shape's x_tile has 32-row boxes)
  } else if ((rc = encode_map(h, &maps.x_tile32, x, H, T, (uint64_t)H * 2, kBK, kPairBoxRows))) {
    return rc;
  }
  if (has_shared) {
    if ((rc = cached_map(h, &maps.ws_up, w_shared->up, H, Ds, (uint64_t)H * 2, kBK, kBN1))) return rc;
    if ((rc = cached_map(h, &maps.ws_gate, w_shared->gate, H, Ds, (uint64_t)H * 2, kBK, kBN1))) return rc;
    if ((rc = cached_map(h, &maps.ws_down, w_shared->down, Ds, H, (uint64_t)Ds * 2, kBK, bn2))) return rc;
    maps.h_shared = small ? h->h_shared16 : (pair ? h->h_shared32 : h->h_shared);
  } else {
    maps.ws_up = maps.w_up;
    maps.ws_gate = maps.w_gate;
    maps.ws_down = maps.w_down;
    maps.h_shared = maps.h_routed;
  }

  cudaEvent_t* ev = nullptr;
  if (h->timing && h->timed < kTimingRing) ev = &h->ev[(size_t)h->timed++ * (kNumStages + 1)];
  auto mark = [&](int i) { return (ev && cudaEventRecord(ev[i], st) != cudaSuccess) ? MOE_ERR_CUDA : MOE_OK; };
  const uint16_t* x16 = static_cast<const uint16_t*>(x);
  // tracing: the per-CTA wait accounting of this forward starts from zero
  if (w.waits && cudaMemsetAsync(w.waits, 0, (size_t)h->num_sms * kNumWaits * 8, st) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (fused) {
    // one launch: the stage events before it time nothing, the expert-GEMM slot times the launch
    for (int i = 0; i <= 4; ++i)
      if ((rc = mark(i))) return rc;
    FrontArgs fa{};
    fa.x = x16;
    fa.w_router = static_cast<const uint16_t*>(w_router);
    fa.bias = router_bias;
    fa.out = out;
    fa.out_bf16 = (c.flags & MOE_FLAG_OUT_BF16) ? 1 : 0;
    fa.epoch = h->epoch + 1;
    const cudaError_t le = launch_moe_small_fused(maps, w, sh, fa, h->num_sms, st);
    if (le == cudaSuccess) {
      h->epoch = fa.epoch;
      h->last_kernels = 1;
      if ((rc = mark(5))) return rc;
      return mark(6);
    }
    // the device refused the cooperative launch (nothing ran): the separate kernels from now on
    cudaGetLastError();
    h->fused_ok = false;
    if (ev) --h->timed;
    h->dep_extra_next = sh.dep_extra;
    return forward_impl(h, x, T, w_router, router_bias, w_up, w_gate, w_down, w_shared, top_k, out, st);
  }
  h->last_kernels = 6;
  if ((rc = mark(0))) return rc;
  int splits = router_splits(T, E, H, bn, h->num_sms);
  while (splits > 1 && (int64_t)splits * T > h->parts_rows) splits /= 2;
  float* parts = splits > 1 ? w.logit_parts : w.logits;
  if ((rc = check_cuda(launch_router(x_router, wr_map, router_bias, parts, T, E, H, bn, splits, w.meta,
                                     h->timeout_ns, st))))
    return rc;
  if ((rc = mark(1))) return rc;
  if ((rc = check_cuda(launch_gate(parts, splits, splits > 1 ? w.logits : nullptr, w.topk_ids, w.topk_w, w,
                                   sh, true, true, h->gate_smem, st))))
    return rc;
  if ((rc = mark(2))) return rc;
  if ((rc = check_cuda(launch_scatter(w.topk_ids, w.sorted_ids, w.expert_ids, nullptr, w.row_of_slot, w,
                                      sh, 2 * h->num_sms, st))))
    return rc;
  if ((rc = mark(3))) return rc;
  if ((rc = check_cuda(launch_gather_rows(x16, w, sh, 4 * h->num_sms, st)))) return rc;
  if ((rc = mark(4))) return rc;
  if (pair) {
    if ((rc = check_cuda(launch_moe_gemm_pair(maps, w, sh, h->max_pairs, st)))) return rc;
  } else {
    if ((rc = check_cuda(launch_moe_gemm(maps, w, sh, h->num_sms, gemm_shape, st)))) return rc;
  }
  if ((rc = mark(5))) return rc;
  if ((rc = check_cuda(launch_combine(out, (c.flags & MOE_FLAG_OUT_BF16) != 0, w, sh, st)))) return rc;
  if ((rc = mark(6))) return rc;
  return MOE_OK;
}

int64_t moe_mxfp8_scale_bytes(int64_t rows, int64_t cols) {
  if (rows <= 0 || cols <= 0 || rows % kMxBK != 0 || cols % kMxBK != 0) return -1;
  return rows * cols / kMxBlock;
}

int moe_quantize_mxfp8(moe_handle* h, const void* src, int64_t rows, int64_t cols, void* q, void* scales,
                       void* stream) {
  if (!h || !src || !q || !scales) return MOE_ERR_INVALID_ARG;
  if (moe_mxfp8_scale_bytes(rows, cols) < 0 || cols > INT32_MAX) return MOE_ERR_UNSUPPORTED;
  if (!aligned16(src) || !aligned16(q) || !aligned16(scales)) return MOE_ERR_MISALIGNED;
  int rc;
  if ((rc = select_device(h))) return rc;
  // one warp per row, 8 rows per CTA, grid-stride beyond 16 CTAs per SM
  const int grid = (int)std::min<int64_t>((rows + 7) / 8, (int64_t)16 * h->num_sms);
  return check_cuda(launch_mx_quantize(static_cast<const uint16_t*>(src), rows, (int)cols, static_cast<uint8_t*>(q),
                                       static_cast<uint8_t*>(scales), grid,
                                       static_cast<cudaStream_t>(stream)));
}

int moe_forward_mxfp8(moe_handle* h, const void* x, int32_t T, const void* w_router, const float* router_bias,
                      const moe_mxfp8_experts* wq, int32_t top_k, void* out, void* stream) {
  if (!h) return MOE_ERR_INVALID_ARG;
  const moe_config& c = h->cfg;
  if (!(c.flags & MOE_FLAG_MXFP8)) return MOE_ERR_NOT_READY;
  int rc;
  if ((rc = check_tokens(h, T, top_k))) return rc;
  if (!w_router || !wq || !wq->up.q || !wq->up.scales || !wq->gate.q || !wq->gate.scales || !wq->down.q ||
      !wq->down.scales)
    return MOE_ERR_INVALID_ARG;
  if (T > 0 && (!x || !out)) return MOE_ERR_INVALID_ARG;
  const bool has_shared = c.inter_shared > 0;
  if (has_shared && (!wq->shared_up.q || !wq->shared_up.scales || !wq->shared_gate.q || !wq->shared_gate.scales ||
                     !wq->shared_down.q || !wq->shared_down.scales))
    return MOE_ERR_INVALID_ARG;
  const moe_mxfp8_mat* mats[6] = {&wq->up, &wq->gate, &wq->down, &wq->shared_up, &wq->shared_gate, &wq->shared_down};
  for (int i = 0; i < (has_shared ? 6 : 3); ++i)
    if (!aligned16(mats[i]->q) || !aligned16(mats[i]->scales)) return MOE_ERR_MISALIGNED;
  if (!aligned16(x) || !aligned16(w_router) || !aligned16(out) || (router_bias && !aligned16(router_bias)))
    return MOE_ERR_MISALIGNED;
  if ((rc = select_device(h))) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  h->last_stream = st;
  h->last_T = T;
  h->last_k = top_k;
  h->have_forward = true;
  if (T == 0) return MOE_OK;

  const int E = c.num_experts, H = c.hidden, D = c.inter, Ds = c.inter_shared;
  Shape sh = make_shape(h, T, top_k);
  sh.dep_extra = h->dep_extra_next;
  h->dep_extra_next = 0;
  h->last_shape = 4;
  h->last_kernels = 6;
  h->last_workers = h->num_sms;
  h->last_tile_m = kBM;
  h->last_lag = sh.lag;
  const Workspace& w = h->ws;
  constexpr CUtensorMapDataType kU8 = CU_TENSOR_MAP_DATA_TYPE_UINT8;

  CUtensorMap x_router, wr_map;
  MxMaps maps;
  const int bn = router_bn(E, T, h->num_sms);
  if ((rc = encode_map(h, &x_router, x, H, T, (uint64_t)H * 2, kBK, kBM))) return rc;
  if ((rc = cached_map(h, &wr_map, w_router, H, E, (uint64_t)H * 2, kBK, bn))) return rc;
  maps.xs = h->mx_xs_map;
  maps.h = h->mx_h_map;
  maps.xs32 = h->mx_xs_map32;
  maps.h32 = h->mx_h_map32;
  maps.y = h->y_map;
  if ((rc = cached_map(h, &maps.w_up, wq->up.q, H, (uint64_t)E * D, H, kMxBK, kBN1, kU8))) return rc;
  if ((rc = cached_map(h, &maps.w_gate, wq->gate.q, H, (uint64_t)E * D, H, kMxBK, kBN1, kU8))) return rc;
  if ((rc = cached_map(h, &maps.w_down, wq->down.q, D, (uint64_t)E * H, D, kMxBK, kBN2, kU8))) return rc;
  MxBuffers mx = h->mx;
  mx.sf_up = static_cast<const uint8_t*>(wq->up.scales);
  mx.sf_gate = static_cast<const uint8_t*>(wq->gate.scales);
  mx.sf_down = static_cast<const uint8_t*>(wq->down.scales);
  if (has_shared) {
    if ((rc = encode_map(h, &maps.x_tile, mx.xq, H, T, H, kMxBK, kBM, kU8))) return rc;
    if ((rc = encode_map(h, &maps.x_tile32, mx.xq, H, T, H, kMxBK, kPairBoxRows, kU8))) return rc;
    if ((rc = cached_map(h, &maps.ws_up, wq->shared_up.q, H, Ds, H, kMxBK, kBN1, kU8))) return rc;
    if ((rc = cached_map(h, &maps.ws_gate, wq->shared_gate.q, H, Ds, H, kMxBK, kBN1, kU8))) return rc;
    if ((rc = cached_map(h, &maps.ws_down, wq->shared_down.q, Ds, H, Ds, kMxBK, kBN2, kU8))) return rc;
    mx.sfs_up = static_cast<const uint8_t*>(wq->shared_up.scales);
    mx.sfs_gate = static_cast<const uint8_t*>(wq->shared_gate.scales);
    mx.sfs_down = static_cast<const uint8_t*>(wq->shared_down.scales);
  } else {
    maps.x_tile = maps.xs;
    maps.x_tile32 = maps.xs32;
    maps.ws_up = maps.w_up;
    maps.ws_gate = maps.w_gate;
    maps.ws_down = maps.w_down;
    mx.sfs_up = mx.sf_up;
    mx.sfs_gate = mx.sf_gate;
    mx.sfs_down = mx.sf_down;
  }

  cudaEvent_t* ev = nullptr;
  if (h->timing && h->timed < kTimingRing) ev = &h->ev[(size_t)h->timed++ * (kNumStages + 1)];
  auto mark = [&](int i) { return (ev && cudaEventRecord(ev[i], st) != cudaSuccess) ? MOE_ERR_CUDA : MOE_OK; };
  // tracing: the per-CTA wait accounting of this forward starts from zero
  if (w.waits && cudaMemsetAsync(w.waits, 0, (size_t)h->num_sms * kNumWaits * 8, st) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (T <= kSmallRows && h->mx_fused_ok) {
    // one launch, as for bf16 experts: router slices, schedule, quantising gather, GEMMs, combine
    for (int i = 0; i <= 4; ++i)
      if ((rc = mark(i))) return rc;
    FrontArgs fa{};
    fa.x = static_cast<const uint16_t*>(x);
    fa.w_router = static_cast<const uint16_t*>(w_router);
    fa.bias = router_bias;
    fa.out = out;
    fa.out_bf16 = (c.flags & MOE_FLAG_OUT_BF16) ? 1 : 0;
    fa.epoch = h->epoch + 1;
    const cudaError_t le = launch_moe_mx_small_fused(maps, w, mx, sh, fa, h->num_sms, st);
    if (le == cudaSuccess) {
      h->epoch = fa.epoch;
      h->last_kernels = 1;
      if ((rc = mark(5))) return rc;
      return mark(6);
    }
    // the device refused the cooperative launch (nothing ran): the separate kernels from now on
    cudaGetLastError();
    h->mx_fused_ok = false;
    if (ev) --h->timed;
    h->dep_extra_next = sh.dep_extra;
    return moe_forward_mxfp8(h, x, T, w_router, router_bias, wq, top_k, out, stream);
  }
  if ((rc = mark(0))) return rc;
  int splits = router_splits(T, E, H, bn, h->num_sms);
  while (splits > 1 && (int64_t)splits * T > h->parts_rows) splits /= 2;
  float* parts = splits > 1 ? w.logit_parts : w.logits;
  if ((rc = check_cuda(launch_router(x_router, wr_map, router_bias, parts, T, E, H, bn, splits, w.meta,
                                     h->timeout_ns, st))))
    return rc;
  if ((rc = mark(1))) return rc;
  if ((rc = check_cuda(launch_gate(parts, splits, splits > 1 ? w.logits : nullptr, w.topk_ids, w.topk_w, w,
                                   sh, true, true, h->gate_smem, st))))
    return rc;
  if ((rc = mark(2))) return rc;
  if ((rc = check_cuda(launch_scatter(w.topk_ids, w.sorted_ids, w.expert_ids, nullptr, w.row_of_slot, w,
                                      sh, 2 * h->num_sms, st))))
    return rc;
  if ((rc = mark(3))) return rc;
  if ((rc = check_cuda(launch_mx_gather(static_cast<const uint16_t*>(x), w, mx, sh, has_shared,
                                        4 * h->num_sms, st))))
    return rc;
  if ((rc = mark(4))) return rc;
  if ((rc = check_cuda(launch_moe_gemm_mx(maps, w, mx, sh, h->num_sms, st)))) return rc;
  if ((rc = mark(5))) return rc;
  if ((rc = check_cuda(launch_combine(out, (c.flags & MOE_FLAG_OUT_BF16) != 0, w, sh, st)))) return rc;
  if ((rc = mark(6))) return rc;
  return MOE_OK;
}

int moe_forward(moe_handle* h, const void* x, int32_t T, const void* w_router,
                const float* router_bias, const void* w_up, const void* w_gate, const void* w_down,
                const moe_shared_w* w_shared, int32_t top_k, void* out, void* stream) {
  if (!h) return MOE_ERR_INVALID_ARG;
  return forward_impl(h, x, T, w_router, router_bias, w_up, w_gate, w_down, w_shared, top_k, out,
                      static_cast<cudaStream_t>(stream));
}

int moe_forward_host(moe_handle* h, const void* x_host, int32_t T, const void* w_router,
                     const float* router_bias, const void* w_up, const void* w_gate,
                     const void* w_down, const moe_shared_w* w_shared, int32_t top_k,
                     void* out_host, void* stream) {
  if (!h) return MOE_ERR_INVALID_ARG;
  if (!h->x_stage || !h->out_stage) return MOE_ERR_NOT_READY;
  int rc;
  if ((rc = check_tokens(h, T, top_k))) return rc;
  if (!x_host || !out_host) return MOE_ERR_INVALID_ARG;
  if ((rc = select_device(h))) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // staging slot 0 may still be in use by queued asynchronous calls
  if (h->async_pending && (rc = moe_forward_host_join(h, stream, 1))) return rc;
  const size_t xb = (size_t)T * h->cfg.hidden * 2;
  const size_t ob = (size_t)T * h->cfg.hidden * ((h->cfg.flags & MOE_FLAG_OUT_BF16) ? 2 : 4);
  if (T > 0 && cudaMemcpyAsync(h->x_stage, x_host, xb, cudaMemcpyHostToDevice, st) != cudaSuccess)
    return MOE_ERR_CUDA;
  if ((rc = forward_impl(h, h->x_stage, T, w_router, router_bias, w_up, w_gate, w_down, w_shared,
                         top_k, h->out_stage, st)))
    return rc;
  if (T > 0 && cudaMemcpyAsync(out_host, h->out_stage, ob, cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return MOE_ERR_CUDA;
  return check_cuda(cudaStreamSynchronize(st));
}

int moe_forward_host_async(moe_handle* h, const void* x_host, int32_t T, const void* w_router,
                           const float* router_bias, const void* w_up, const void* w_gate,
                           const void* w_down, const moe_shared_w* w_shared, int32_t top_k,
                           void* out_host, void* stream) {
  if (!h) return MOE_ERR_INVALID_ARG;
  if (!h->x_stage || !h->out_stage || !h->copy_in) return MOE_ERR_NOT_READY;
  int rc;
  if ((rc = check_tokens(h, T, top_k))) return rc;
  if (!x_host || !out_host) return MOE_ERR_INVALID_ARG;
  if ((rc = select_device(h))) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int s = h->async_slot;
  h->async_slot ^= 1;
  void* xs = static_cast<char*>(h->x_stage) + (size_t)s * h->x_slot_bytes;
  void* os = reinterpret_cast<char*>(h->out_stage) + (size_t)s * h->out_slot_bytes;
  const size_t xb = (size_t)T * h->cfg.hidden * 2;
  const size_t ob = (size_t)T * h->cfg.hidden * ((h->cfg.flags & MOE_FLAG_OUT_BF16) ? 2 : 4);
  // copy in: this slot's x buffer is free once the forward that read it two calls ago is done
  if (h->slot_used[s] && cudaStreamWaitEvent(h->copy_in, h->ev_done[s], 0) != cudaSuccess) return MOE_ERR_CUDA;
  if (T > 0 && cudaMemcpyAsync(xs, x_host, xb, cudaMemcpyHostToDevice, h->copy_in) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (cudaEventRecord(h->ev_in[s], h->copy_in) != cudaSuccess) return MOE_ERR_CUDA;
  // forward on the caller's stream, once x is in and this slot's previous result is copied out
  if (cudaStreamWaitEvent(st, h->ev_in[s], 0) != cudaSuccess) return MOE_ERR_CUDA;
  if (h->slot_used[s] && cudaStreamWaitEvent(st, h->ev_out[s], 0) != cudaSuccess) return MOE_ERR_CUDA;
  if ((rc = forward_impl(h, xs, T, w_router, router_bias, w_up, w_gate, w_down, w_shared, top_k, os, st)))
    return rc;
  if (cudaEventRecord(h->ev_done[s], st) != cudaSuccess) return MOE_ERR_CUDA;
  // copy back
  if (cudaStreamWaitEvent(h->copy_out, h->ev_done[s], 0) != cudaSuccess) return MOE_ERR_CUDA;
  if (T > 0 && cudaMemcpyAsync(out_host, os, ob, cudaMemcpyDeviceToHost, h->copy_out) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (cudaEventRecord(h->ev_out[s], h->copy_out) != cudaSuccess) return MOE_ERR_CUDA;
  h->slot_used[s] = true;
  h->async_pending = true;
  return MOE_OK;
}

int moe_forward_host_join(moe_handle* h, void* stream, int32_t block) {
  if (!h) return MOE_ERR_INVALID_ARG;
  int rc;
  if ((rc = select_device(h))) return rc;
  if (!h->async_pending) return MOE_OK;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  for (int s = 0; s < 2; ++s)
    if (h->slot_used[s] && cudaStreamWaitEvent(st, h->ev_out[s], 0) != cudaSuccess) return MOE_ERR_CUDA;
  if (block) {
    if (cudaStreamSynchronize(h->copy_out) != cudaSuccess) return MOE_ERR_CUDA;
    h->async_pending = false;
  }
  return MOE_OK;
}

int moe_get_status(moe_handle* h, int32_t* device_status) {
  if (!h) return MOE_ERR_INVALID_ARG;
  int rc;
  if ((rc = select_device(h))) return rc;
  if (cudaStreamSynchronize(h->last_stream) != cudaSuccess) {
    if (device_status) *device_status = 0;
    return MOE_ERR_CUDA;
  }
  int32_t st = 0;
  if (cudaMemcpy(&st, &h->ws.meta->status, sizeof st, cudaMemcpyDeviceToHost) != cudaSuccess)
    return MOE_ERR_CUDA;
  const int32_t zero = 0;
  if (cudaMemcpy(&h->ws.meta->status, &zero, sizeof zero, cudaMemcpyHostToDevice) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (device_status) *device_status = st;
  if (st & kStatusTimeout) return MOE_ERR_DEVICE_TIMEOUT;
  return MOE_OK;
}

int moe_router_logits(moe_handle* h, const void* x, int32_t T, const void* w_router,
                      const float* router_bias, float* logits, void* stream) {
  if (!h) return MOE_ERR_INVALID_ARG;
  if (T < 0 || T > h->cfg.max_tokens || !x || !w_router || !logits) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(w_router) || !aligned16(logits)) return MOE_ERR_MISALIGNED;
  int rc;
  if ((rc = select_device(h))) return rc;
  if (T == 0) return MOE_OK;
  const int E = h->cfg.num_experts, H = h->cfg.hidden, bn = router_bn(E, T, h->num_sms);
  CUtensorMap xm, wm;
  if ((rc = encode_map(h, &xm, x, H, T, (uint64_t)H * 2, kBK, kBM))) return rc;
  if ((rc = cached_map(h, &wm, w_router, H, E, (uint64_t)H * 2, kBK, bn))) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  h->last_stream = st;
  return check_cuda(launch_router(xm, wm, router_bias, logits, T, E, H, bn, 1, h->ws.meta, h->timeout_ns, st));
}

int moe_gate_topk(moe_handle* h, const float* logits, int32_t T, int32_t top_k, int32_t* topk_ids,
                  float* topk_w, void* stream) {
  if (!h) return MOE_ERR_INVALID_ARG;
  int rc;
  if ((rc = check_tokens(h, T, top_k))) return rc;
  if (!logits || !topk_ids || !topk_w) return MOE_ERR_INVALID_ARG;
  if ((rc = select_device(h))) return rc;
  if (T == 0) return MOE_OK;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  h->last_stream = st;
  const Shape sh = make_shape(h, T, top_k);
  return check_cuda(launch_gate(logits, 1, nullptr, topk_ids, topk_w, h->ws, sh, false, false, 0, st));
}

int moe_align_block_size(moe_handle* h, const int32_t* topk_ids, int32_t T, int32_t top_k,
                         int32_t* sorted_ids, int32_t* expert_ids, int32_t* num_post_padded,
                         void* stream) {
  if (!h) return MOE_ERR_INVALID_ARG;
  int rc;
  if ((rc = check_tokens(h, T, top_k))) return rc;
  if ((T > 0 && !topk_ids) || !sorted_ids || !expert_ids || !num_post_padded) return MOE_ERR_INVALID_ARG;
  if ((rc = select_device(h))) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  h->last_stream = st;
  const Shape sh = make_shape(h, T, top_k);
  if ((rc = check_cuda(launch_hist(topk_ids, h->ws, sh, h->gate_smem, st)))) return rc;
  return check_cuda(launch_scatter(topk_ids, sorted_ids, expert_ids, num_post_padded, nullptr, h->ws, sh,
                                   2 * h->num_sms, st));
}

int moe_debug_outputs(moe_handle* h, float* logits, int32_t* topk_ids, float* topk_w,
                      int32_t* sorted_ids, int32_t* expert_ids, int32_t* num_post_padded,
                      void* stream) {
  if (!h) return MOE_ERR_INVALID_ARG;
  if (!h->have_forward) return MOE_ERR_NOT_READY;
  int rc;
  if ((rc = select_device(h))) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t T = h->last_T, k = h->last_k, E = h->cfg.num_experts;
  const Workspace& w = h->ws;
  auto cp = [&](void* dst, const void* src, size_t bytes) {
    if (!dst || bytes == 0) return MOE_OK;
    return check_cuda(cudaMemcpyAsync(dst, src, bytes, cudaMemcpyDeviceToDevice, st));
  };
  if ((rc = cp(logits, w.logits, T * E * 4))) return rc;
  if ((rc = cp(topk_ids, w.topk_ids, T * k * 4))) return rc;
  if ((rc = cp(topk_w, w.topk_w, T * k * 4))) return rc;
  if ((rc = cp(sorted_ids, w.sorted_ids, (size_t)moe_sorted_len(h, (int)T, (int)k) * 4))) return rc;
  if ((rc = cp(expert_ids, w.expert_ids, (size_t)moe_blocks_len(h, (int)T, (int)k) * 4))) return rc;
  if ((rc = cp(num_post_padded, &w.meta->P, 4))) return rc;
  return MOE_OK;
}

int moe_debug_expert_rows(moe_handle* h, void* h_rows, void* y_rows, int32_t* row_of_slot,
                          int32_t* num_routed_tiles, void* stream) {
  if (!h) return MOE_ERR_INVALID_ARG;
  if (!h->have_forward) return MOE_ERR_NOT_READY;
  if (h_rows && h->last_shape == 4) return MOE_ERR_NOT_READY;  // MXFP8 keeps h quantised
  int rc;
  if ((rc = select_device(h))) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const Workspace& w = h->ws;
  auto cp = [&](void* dst, const void* src, size_t bytes) {
    if (!dst || bytes == 0) return MOE_OK;
    return check_cuda(cudaMemcpyAsync(dst, src, bytes, cudaMemcpyDeviceToDevice, st));
  };
  const size_t rows = (size_t)h->tile_rows;
  if ((rc = cp(h_rows, w.h, rows * w.ldh * 2))) return rc;
  if ((rc = cp(y_rows, w.y, rows * h->cfg.hidden * 2))) return rc;
  if ((rc = cp(row_of_slot, w.row_of_slot, (size_t)h->last_T * h->last_k * 4))) return rc;
  if ((rc = cp(num_routed_tiles, &w.meta->num_routed_tiles, 4))) return rc;
  return MOE_OK;
}

int moe_stage_times(moe_handle* h, float* ms, int32_t n) {
  if (!h || !ms || n < 1) return MOE_ERR_INVALID_ARG;
  if (!h->timing || h->timed == 0) return MOE_ERR_NOT_READY;
  const int m = h->timed;
  const size_t K = kNumStages + 1;
  h->timed = 0;
  for (int i = 0; i < std::min(n, kNumStages); ++i) ms[i] = 0.f;
  if (cudaEventSynchronize(h->ev[(size_t)(m - 1) * K + kNumStages]) != cudaSuccess) return MOE_ERR_CUDA;
  for (int f = 0; f < m; ++f)
    for (int i = 0; i < std::min(n, kNumStages); ++i) {
      float t = 0.f;
      if (cudaEventElapsedTime(&t, h->ev[(size_t)f * K + i], h->ev[(size_t)f * K + i + 1]) != cudaSuccess)
        return MOE_ERR_CUDA;
      ms[i] += t / m;
    }
  return MOE_OK;
}

int moe_query(const moe_handle* h, int32_t which, int64_t* value) {
  if (!h || !value) return MOE_ERR_INVALID_ARG;
  switch (which) {
    case 0: *value = h->num_sms; return MOE_OK;
    case 1: *value = h->last_workers; return MOE_OK;
    case 2: *value = (int64_t)h->ws_bytes; return MOE_OK;
    case 3:
    case 4: {
      if (!h->have_forward) return MOE_ERR_NOT_READY;
      if (cudaSetDevice(h->device) != cudaSuccess) return MOE_ERR_CUDA;
      if (cudaStreamSynchronize(h->last_stream) != cudaSuccess) return MOE_ERR_CUDA;
      DeviceMeta m{};
      if (cudaMemcpy(&m, h->ws.meta, sizeof m, cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
      *value = (which == 3) ? m.total_tasks : m.num_tiles;
      return MOE_OK;
    }
    case 5: *value = h->last_lag; return MOE_OK;
    case 6: *value = h->last_tile_m; return MOE_OK;
    case 7: *value = h->max_pairs; return MOE_OK;
    case 8: *value = h->last_shape; return MOE_OK;
    case 9: *value = h->tile_rows; return MOE_OK;
    case 10: *value = h->ws.ldh; return MOE_OK;
    case 11: *value = h->last_kernels; return MOE_OK;
    case 12: *value = ((h->cfg.flags & MOE_FLAG_MXFP8) ? h->mx_fused_ok : h->fused_ok) ? 1 : 0; return MOE_OK;
    default: return MOE_ERR_INVALID_ARG;
  }
}

int moe_trace_read(moe_handle* h, int64_t* records, int64_t cap, int64_t* n) {
  if (!h || !records || !n || cap < 0) return MOE_ERR_INVALID_ARG;
  if (h->ws.trace_cap == 0) return MOE_ERR_NOT_READY;
  int64_t total = 0;
  int rc;
  if ((rc = moe_query(h, 3, &total))) return rc;
  const int64_t m = std::min<int64_t>(std::min<int64_t>(total, h->ws.trace_cap), cap);
  if (m > 0 && cudaMemcpy(records, h->ws.trace, (size_t)m * 4 * 8, cudaMemcpyDeviceToHost) != cudaSuccess)
    return MOE_ERR_CUDA;
  *n = m;
  return MOE_OK;
}

int moe_trace_waits(moe_handle* h, int64_t* waits, int32_t rows, int32_t* n_rows) {
  if (!h || !waits || !n_rows || rows < 0) return MOE_ERR_INVALID_ARG;
  if (!h->ws.waits || !h->have_forward) return MOE_ERR_NOT_READY;
  int rc;
  if ((rc = select_device(h))) return rc;
  if (cudaStreamSynchronize(h->last_stream) != cudaSuccess) return MOE_ERR_CUDA;
  const int m = std::min(rows, h->num_sms);
  if (m > 0 && cudaMemcpy(waits, h->ws.waits, (size_t)m * kNumWaits * 8, cudaMemcpyDeviceToHost) != cudaSuccess)
    return MOE_ERR_CUDA;
  *n_rows = m;
  return MOE_OK;
}

int moe_debug_inject_stall(moe_handle* h, int32_t extra) {
  if (!h || extra < 0) return MOE_ERR_INVALID_ARG;
  h->dep_extra_next = extra;
  return MOE_OK;
}

}  // extern "C"
