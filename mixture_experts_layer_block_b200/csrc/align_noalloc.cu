// align_noalloc.cu -- moe_align_block_size without a handle and without any allocation.
//
// Some callers cannot allocate device memory on our behalf: a serving runtime that reserves
// all of HBM for its own allocator up front (so that its memory budget stays exact and no
// other component may call cudaMalloc), or a latency-critical path where a cudaMalloc, which
// may synchronise the device, is not acceptable. The handle API allocates its workspace in
// moe_init, so such callers cannot use it. This entry point runs the same histogram, scan and
// scatter kernels as moe_align_block_size, but their scratch memory (chunk histograms, chunk
// prefixes, segment offsets, kept counts and the completion ticket) lives in a fixed array
// compiled into this library, so nothing is allocated at any time. The caller passes the
// inputs and outputs as before.
//
// Limits: num_experts <= 256 and T * top_k <= 131072 (the array holds 32 chunk histograms of
// 256 experts); larger sizes are rejected with MOE_ERR_UNSUPPORTED.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <mutex>

#include "launch.h"
#include "moe_b200.h"

namespace moe {
namespace {

constexpr int kNaMaxExperts = 256;
constexpr int64_t kNaMaxSlots = 131072;
// layout (ints): DeviceMeta (16) | chunk_hist [32][256] | chunk_base [32][256] |
//                expert_off [257] | expert_kept [256]
constexpr int kNaMetaInts = 16;
constexpr int kNaHistInts = kMaxChunks * kNaMaxExperts;
constexpr int kNaScratchInts = kNaMetaInts + 2 * kNaHistInts + (kNaMaxExperts + 1) + kNaMaxExperts;
static_assert(sizeof(DeviceMeta) == kNaMetaInts * sizeof(int), "DeviceMeta layout");

// Every GPU that loads this library holds one copy of this array until the process exits.
static __device__ __align__(256) int32_t g_align_scratch[kNaScratchInts];

constexpr int kNaMaxDevices = 64;
struct DeviceSetup {
  bool ready = false;
  unsigned long long ctx_id = 0;  // the device context the address below belongs to
  int32_t* scratch = nullptr;     // device address of g_align_scratch in that context
  int num_sms = 0;
};
DeviceSetup g_setup[kNaMaxDevices];
std::mutex g_setup_mu;

// Driver entry points (through the runtime, so no link-time dependency on libcuda) that name
// the calling thread's current context. A cudaDeviceReset destroys the context whose address
// was cached; the next context of the same device gets a new id, which triggers a new set-up.
typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);
CtxGetCurrentFn g_ctx_get_current = nullptr;
CtxGetIdFn g_ctx_get_id = nullptr;

// Id of the current context, 0 when the runtime has not made one current yet.
int current_ctx_id(unsigned long long* id) {
  *id = 0;
  if (!g_ctx_get_current || !g_ctx_get_id) {
    void* f1 = nullptr;
    void* f2 = nullptr;
    cudaDriverEntryPointQueryResult q1{}, q2{};
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f1, cudaEnableDefault, &q1) != cudaSuccess ||
        q1 != cudaDriverEntryPointSuccess || !f1 ||
        cudaGetDriverEntryPoint("cuCtxGetId", &f2, cudaEnableDefault, &q2) != cudaSuccess ||
        q2 != cudaDriverEntryPointSuccess || !f2)
      return MOE_ERR_CUDA;
    g_ctx_get_current = reinterpret_cast<CtxGetCurrentFn>(f1);
    g_ctx_get_id = reinterpret_cast<CtxGetIdFn>(f2);
  }
  CUcontext ctx = nullptr;
  if (g_ctx_get_current(&ctx) != CUDA_SUCCESS) return MOE_ERR_CUDA;
  if (ctx && g_ctx_get_id(ctx, id) != CUDA_SUCCESS) return MOE_ERR_CUDA;
  return MOE_OK;
}

// Once per device context, with that device current: the array's device address (the name of
// the array in host code is only a host-side stand-in, never a device pointer) and the SM
// count. Done again when the device's context has changed since (after a cudaDeviceReset).
int device_setup(int dev, DeviceSetup** out) {
  if (dev < 0 || dev >= kNaMaxDevices) return MOE_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_setup_mu);
  DeviceSetup& s = g_setup[dev];
  unsigned long long id = 0;
  int rc = current_ctx_id(&id);
  if (rc != MOE_OK) return rc;
  if (!s.ready || id == 0 || id != s.ctx_id) {
    s.ready = false;
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_align_scratch) != cudaSuccess || p == nullptr) return MOE_ERR_CUDA;
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
      return MOE_ERR_CUDA;
    // the symbol lookup made the device's context current if it was not yet
    if ((rc = current_ctx_id(&id)) != MOE_OK) return rc;
    s.scratch = static_cast<int32_t*>(p);
    s.num_sms = sms;
    s.ctx_id = id;
    s.ready = true;
  }
  *out = &s;
  return MOE_OK;
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" MOE_API int moe_align_block_size_noalloc(const int32_t* topk_ids, int32_t T, int32_t top_k,
                                                    int32_t num_experts, int32_t block_m,
                                                    float capacity_factor, int32_t* sorted_ids,
                                                    int32_t* expert_ids, int32_t* num_post_padded,
                                                    void* stream) {
  if (T < 0 || top_k < 1 || top_k > 32 || num_experts < 1 || top_k > num_experts || block_m < 1 ||
      block_m > 4096 || !(capacity_factor >= 0.f) || std::isinf(capacity_factor))
    return MOE_ERR_INVALID_ARG;
  if ((T > 0 && !topk_ids) || !sorted_ids || !expert_ids || !num_post_padded) return MOE_ERR_INVALID_ARG;
  if (num_experts > kNaMaxExperts || (int64_t)T * top_k > kNaMaxSlots) return MOE_ERR_UNSUPPORTED;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
  DeviceSetup* ds = nullptr;
  int rc = device_setup(dev, &ds);
  if (rc != MOE_OK) return rc;

  const int E = num_experts;
  Shape sh{};
  sh.T = T;
  sh.E = E;
  sh.k = top_k;
  sh.block_m = block_m;
  sh.capacity = 0;
  if (capacity_factor > 0.f) {
    const double c = std::ceil((double)capacity_factor * (double)T * (double)top_k / (double)E);
    sh.capacity = (int)std::min<double>(c, (double)T * top_k);
  }
  sh.chunk_tokens = ceil_div(std::max(kMinChunkTokens, ceil_div(std::max(T, 1), kMaxChunks)),
                             kGateTokensPerCta) * kGateTokensPerCta;
  sh.num_chunks = std::max(1, ceil_div(T, sh.chunk_tokens));
  sh.sorted_len = T * top_k + E * (block_m - 1);
  sh.blocks_len = ceil_div(sh.sorted_len, block_m);

  // every launch fits in 48 KB of dynamic shared memory (the default limit); the limits are
  // only ever raised, under the same lock moe_init takes, so a concurrent moe_init cannot
  // lower them between this check and the launches
  const size_t hist_smem = gate_smem_bytes(sh, 0);
  const size_t scatter_smem = scatter_smem_bytes(E, sh.chunk_tokens * top_k);
  if (hist_smem > 48 * 1024 || scatter_smem > 48 * 1024) return MOE_ERR_UNSUPPORTED;
  if (raise_align_smem(0, hist_smem, scatter_smem) != cudaSuccess) return MOE_ERR_CUDA;

  Workspace ws{};
  int32_t* base = ds->scratch;
  ws.meta = reinterpret_cast<DeviceMeta*>(base);
  ws.chunk_hist = base + kNaMetaInts;
  ws.chunk_base = ws.chunk_hist + kNaHistInts;
  ws.expert_off = ws.chunk_base + kNaHistInts;
  ws.expert_kept = ws.expert_off + (kNaMaxExperts + 1);

  // The array keeps whatever the previous call left in it: clear the counters and the
  // histograms this call accumulates into (the kernels expect them to start at zero).
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(ws.meta, 0, sizeof(DeviceMeta), st) != cudaSuccess) return MOE_ERR_CUDA;
  if (cudaMemsetAsync(ws.chunk_hist, 0, (size_t)sh.num_chunks * E * sizeof(int32_t), st) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (launch_hist(topk_ids, ws, sh, hist_smem, st) != cudaSuccess) return MOE_ERR_CUDA;
  if (launch_scatter(topk_ids, sorted_ids, expert_ids, num_post_padded, nullptr, ws, sh, 2 * ds->num_sms, st) !=
      cudaSuccess)
    return MOE_ERR_CUDA;
  return MOE_OK;
}
