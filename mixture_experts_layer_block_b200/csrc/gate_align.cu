// gate_align.cu -- gating (top-k softmax, renormalised) and align (moe_align_block_size).
//
// Gating (Weave blog section 1.1; vLLM execution analysis, topk_softmax): one warp per
// token, 64 tokens per CTA; each lane holds E/32 logits (adding the router's K-split
// partials in split order); k rounds of a warp arg-max (ties to
// the lower expert index) select the experts in descending order; the weights are the
// selected softmax probabilities renormalised over the selection, i.e.
// exp(v_j - v_0) / sum_i exp(v_i - v_0). Each warp loads its next token while it selects
// the current one.
//
// Align (vLLM PR #53280 summary: per-expert counts, exclusive cumsum, cooperative writes of
// token ids and block ids; the reviewer's variant that uses every block of the grid):
//   1. each CTA of the gating (or histogram) kernel counts its slots per expert and adds the
//      counts into its token chunk's histogram (integer atomics; at most 32 chunks);
//   2. the last CTA to finish scans: per expert, the counts of earlier chunks (loaded in
//      parallel into shared memory), the capacity cut, the padded segment offsets, and for
//      the forward also the m-tile list and the task schedule of the expert-GEMM kernel;
//   3. a grid-wide kernel writes sorted_ids: one CTA per chunk, one warp per sub-chunk,
//      ranks from __match_any_sync, warp offsets from a per-chunk prefix over warps; and
//      every CTA writes its share of the padding sentinels and expert_ids (one thread per
//      entry).
#include <algorithm>
#include <climits>
#include <cmath>
#include <mutex>

#include "launch.h"
#include "route.cuh"

namespace moe {

// ------------------------------------------------------------------------------------------
// one token's logits (the sum of the router's S K-split partials, in split order) into the
// registers of a warp: lane l holds experts l, l + 32, ...
// ------------------------------------------------------------------------------------------
template <int VPL, int S>
__device__ __forceinline__ void load_token(const float* __restrict__ row, size_t part_stride, int E,
                                           int lane, float (&v)[VPL]) {
  float p[S][VPL];
#pragma unroll
  for (int s = 0; s < S; ++s)
#pragma unroll
    for (int j = 0; j < VPL; ++j) {
      const int e = lane + 32 * j;
      p[s][j] = (e < E) ? __ldcg(row + s * part_stride + e) : 0.f;
    }
#pragma unroll
  for (int j = 0; j < VPL; ++j) {
    float a = p[0][j];
#pragma unroll
    for (int s = 1; s < S; ++s) a += p[s][j];
    v[j] = (lane + 32 * j < E) ? a : -INFINITY;
  }
}

// Add this CTA's counts into its chunk's histogram; the last CTA runs the scans.
__device__ void finish_histogram(const Workspace& ws, const Shape& sh, bool tiles, const int* hist,
                                 int chunk, int* sm) {
  __shared__ int s_last;
  for (int e = threadIdx.x; e < sh.E; e += blockDim.x)
    if (hist[e]) atomicAdd(ws.chunk_hist + (size_t)chunk * sh.E + e, hist[e]);
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) s_last = (atomicAdd(&ws.meta->hist_done, 1) == (int)gridDim.x - 1);
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  align_scans(ws, sh, tiles, sm);
  if (threadIdx.x == 0) ws.meta->hist_done = 0;
}

// ------------------------------------------------------------------------------------------
// kernels
// ------------------------------------------------------------------------------------------
// smem: hist[E] | scan area. One CTA per kGateTokensPerCta tokens (a chunk holds a whole
// number of CTAs). `parts` holds S partial logits [S][T][E]; with logits_out non-null the
// sums are written there.
template <int VPL, int S>
__global__ void __launch_bounds__(kGateThreads)
    gate_kernel(const float* __restrict__ parts, float* __restrict__ logits_out,
                int32_t* __restrict__ topk_ids, float* __restrict__ topk_w, Workspace ws, Shape sh,
                int hist_on, int tiles) {
  griddep_wait();
  griddep_launch_dependents();
  extern __shared__ int smem_i[];
  int* hist = smem_i;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int kWarps = kGateThreads / 32;
  const int t0 = blockIdx.x * kGateTokensPerCta;
  const int t1 = min(sh.T, t0 + kGateTokensPerCta);
  const size_t pstride = (size_t)sh.T * sh.E;
  if (hist_on) {
    for (int e = threadIdx.x; e < sh.E; e += blockDim.x) hist[e] = 0;
    __syncthreads();
  }
  float vnext[VPL];
  int t = t0 + warp;
  if (t < t1) load_token<VPL, S>(parts + (size_t)t * sh.E, pstride, sh.E, lane, vnext);
  for (; t < t1; t += kWarps) {
    float v[VPL];
#pragma unroll
    for (int j = 0; j < VPL; ++j) v[j] = vnext[j];
    if (t + kWarps < t1) load_token<VPL, S>(parts + (size_t)(t + kWarps) * sh.E, pstride, sh.E, lane, vnext);
    if (logits_out) {
#pragma unroll
      for (int j = 0; j < VPL; ++j)
        if (lane + 32 * j < sh.E) logits_out[(size_t)t * sh.E + lane + 32 * j] = v[j];
    }
    int id;
    float w;
    warp_topk_softmax<VPL>(v, sh.E, sh.k, lane, id, w);
    if (lane < sh.k) {
      topk_ids[(size_t)t * sh.k + lane] = id;
      topk_w[(size_t)t * sh.k + lane] = w;
      if (hist_on) atomicAdd(&hist[id], 1);
    }
  }
  if (!hist_on) return;
  __syncthreads();
  finish_histogram(ws, sh, tiles != 0, hist, t0 / sh.chunk_tokens, smem_i + sh.E);
}

__global__ void __launch_bounds__(kGateThreads)
    hist_kernel(const int32_t* __restrict__ topk_ids, Workspace ws, Shape sh) {
  griddep_wait();
  griddep_launch_dependents();
  extern __shared__ int smem_i[];
  int* hist = smem_i;
  for (int e = threadIdx.x; e < sh.E; e += blockDim.x) hist[e] = 0;
  __syncthreads();
  const int t0 = blockIdx.x * kGateTokensPerCta;
  const int64_t s0 = (int64_t)t0 * sh.k;
  const int64_t s1 = (int64_t)min(sh.T, t0 + kGateTokensPerCta) * sh.k;
  for (int64_t s = s0 + threadIdx.x; s < s1; s += blockDim.x) {
    const int e = topk_ids[s];
    if (e >= 0 && e < sh.E) atomicAdd(&hist[e], 1);  // ids outside [0, E) are skipped
  }
  __syncthreads();
  finish_histogram(ws, sh, false, hist, t0 / sh.chunk_tokens, smem_i + sh.E);
}

// smem: off[E+1] | kept[E] | tile0[E] | wcnt[16][E] | ids[chunk slots]
// CTA c < num_chunks sorts the slots of token chunk c: warp w owns a contiguous run of the
// chunk's slots; pass 1 counts them per expert, a per-expert prefix over the warps (seeded
// with the chunk prefix of the scan) gives every warp its first rank, pass 2 writes. With
// `row_of_slot` non-null, also records for every slot its row in the tile-ordered buffers
// (first tile of its expert * 128 + its rank), or -1 when the slot was dropped. Every CTA
// then writes its share of the padding sentinels and of expert_ids.
__global__ void __launch_bounds__(kGateThreads)
    scatter_kernel(const int32_t* __restrict__ topk_ids, int32_t* __restrict__ sorted_ids,
                   int32_t* __restrict__ expert_ids, int32_t* __restrict__ num_post_padded,
                   int32_t* __restrict__ row_of_slot, Workspace ws, Shape sh) {
  griddep_wait();
  griddep_launch_dependents();
  extern __shared__ int smem_i[];
  constexpr int kWarps = kGateThreads / 32;
  const int E = sh.E;
  int* off = smem_i;
  int* kept = off + E + 1;
  int* tile0 = kept + E;
  int* wcnt = tile0 + E;
  int* ids = wcnt + kWarps * E;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int e = threadIdx.x; e <= E; e += blockDim.x) off[e] = __ldcg(ws.expert_off + e);
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    kept[e] = __ldcg(ws.expert_kept + e);
    if (row_of_slot) tile0[e] = __ldcg(ws.expert_tile0 + e);
  }
  const int P = __ldcg(ws.expert_off + E);
  const int S = sh.T * sh.k;

  const int c = blockIdx.x;
  if (c < sh.num_chunks) {
    const int s0 = c * sh.chunk_tokens * sh.k;
    const int n = min(sh.T, (c + 1) * sh.chunk_tokens) * sh.k - s0;
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
      const int e = topk_ids[s0 + i];
      ids[i] = (e >= 0 && e < E) ? e : -1;
    }
    for (int i = threadIdx.x; i < kWarps * E; i += blockDim.x) wcnt[i] = 0;
    __syncthreads();
    const int per = ceil_div(ceil_div(n, kWarps), 32) * 32;
    const int w0 = min(n, warp * per), w1 = min(n, w0 + per);
    int* cnt = wcnt + warp * E;
    // pass 1: per-warp counts
    for (int base = w0; base < w1; base += 32) {
      const int e = (base + lane < w1) ? ids[base + lane] : -1;
      const unsigned mask = __match_any_sync(0xffffffffu, e);
      if (e >= 0 && lane == __ffs(mask) - 1) cnt[e] += __popc(mask);
    }
    __syncthreads();
    // per expert: first rank of every warp = chunk prefix + counts of the earlier warps
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
      int run = __ldcg(ws.chunk_base + (size_t)c * E + e);
      for (int w = 0; w < kWarps; ++w) {
        const int x = wcnt[w * E + e];
        wcnt[w * E + e] = run;
        run += x;
      }
    }
    __syncthreads();
    // pass 2: stable writes
    for (int base = w0; base < w1; base += 32) {
      const bool in = base + lane < w1;
      const int e = in ? ids[base + lane] : -1;
      const unsigned mask = __match_any_sync(0xffffffffu, e);
      const int rank = __popc(mask & ((1u << lane) - 1u));
      const int c0 = (e >= 0) ? cnt[e] : 0;
      __syncwarp();
      const int s = s0 + base + lane;
      if (e >= 0) {
        const int r = c0 + rank;
        const bool keep = sh.capacity == 0 || r < sh.capacity;
        if (keep) sorted_ids[off[e] + r] = s;
        if (row_of_slot) row_of_slot[s] = keep ? tile0[e] * sh.tile_m + r : -1;
        if (rank == 0) cnt[e] = c0 + __popc(mask);
      } else if (in && row_of_slot) {
        row_of_slot[s] = -1;  // an expert id outside [0, E)
      }
      __syncwarp();
    }
  } else {
    __syncthreads();
  }

  // padding sentinels and block -> expert ids, one thread per entry, grid-wide
  const int gt = blockIdx.x * blockDim.x + threadIdx.x;
  const int nt = gridDim.x * blockDim.x;
  for (int i = gt; i < sh.sorted_len; i += nt) {
    bool pad = true;
    if (i < P) {
      const int e = segment_of(off, E, i);
      pad = (i - off[e]) >= kept[e];
    }
    if (pad) sorted_ids[i] = S;
  }
  for (int b = gt; b < sh.blocks_len; b += nt) {
    const int i = b * sh.block_m;
    expert_ids[b] = (i < P) ? segment_of(off, E, i) : -1;
  }
  if (gt == 0 && num_post_padded) *num_post_padded = P;
  // a forward's task table: one thread per scheduling unit, starting with the CTAs that sort no
  // chunk (the schedule's scans ran in the gating kernel)
  if (row_of_slot && ws.task_tab) {
    const int U = __ldcg(&ws.meta->num_units), Mg = __ldcg(&ws.meta->num_groups);
    const int Mgr = __ldcg(&ws.meta->num_routed_groups);
    const int first = (int)((blockIdx.x + gridDim.x - min(sh.num_chunks, (int)gridDim.x)) % gridDim.x);
    for (int u = first * blockDim.x + threadIdx.x; u < U; u += nt)
      write_unit_tasks(ws, sh, u, __ldcg(&ws.unit_start[u]), Mg, Mgr);
  }
}

// ------------------------------------------------------------------------------------------
// launchers
// ------------------------------------------------------------------------------------------
size_t gate_smem_bytes(const Shape& sh, int max_units) {
  const int buf = std::max(sh.E + 1, max_units + 1);
  return sizeof(int) * (size_t)(sh.E /*hist*/ + 64 + 3 * sh.E + kMaxChunks * kScanGroup + buf);
}

size_t scatter_smem_bytes(int E, int chunk_slots) {
  return sizeof(int) * (size_t)(E + 1 + 2 * E + (kGateThreads / 32) * E + chunk_slots);
}

static int gate_grid(const Shape& sh) { return std::max(1, ceil_div(sh.T, kGateTokensPerCta)); }

template <int VPL, int S>
static cudaError_t launch_gate_vs(const float* parts, float* logits_out, int32_t* ids, float* w,
                                  const Workspace& ws, const Shape& sh, bool hist, bool tiles,
                                  size_t smem, cudaStream_t st) {
  return launch_k(gate_kernel<VPL, S>, dim3(gate_grid(sh)), dim3(kGateThreads), hist ? smem : 0, st, parts,
                  logits_out, ids, w, ws, sh, hist ? 1 : 0, tiles ? 1 : 0);
}

template <int VPL>
static cudaError_t launch_gate_v(const float* parts, int splits, float* logits_out, int32_t* ids,
                                 float* w, const Workspace& ws, const Shape& sh, bool hist,
                                 bool tiles, size_t smem, cudaStream_t st) {
  if (splits == 4) return launch_gate_vs<VPL, 4>(parts, logits_out, ids, w, ws, sh, hist, tiles, smem, st);
  if (splits == 2) return launch_gate_vs<VPL, 2>(parts, logits_out, ids, w, ws, sh, hist, tiles, smem, st);
  return launch_gate_vs<VPL, 1>(parts, logits_out, ids, w, ws, sh, hist, tiles, smem, st);
}

cudaError_t launch_gate(const float* parts, int splits, float* logits_out, int32_t* topk_ids,
                        float* topk_w, const Workspace& ws, const Shape& sh, bool hist, bool tiles,
                        size_t smem, cudaStream_t st) {
#define MOE_GATE(V) \
  launch_gate_v<V>(parts, splits, logits_out, topk_ids, topk_w, ws, sh, hist, tiles, smem, st)
  if (sh.E <= 32) return MOE_GATE(1);
  if (sh.E <= 64) return MOE_GATE(2);
  if (sh.E <= 128) return MOE_GATE(4);
  if (sh.E <= 256) return MOE_GATE(8);
  if (sh.E <= 512) return MOE_GATE(16);
  return MOE_GATE(32);
#undef MOE_GATE
}

cudaError_t launch_hist(const int32_t* topk_ids, const Workspace& ws, const Shape& sh, size_t smem,
                        cudaStream_t st) {
  return launch_k(hist_kernel, dim3(gate_grid(sh)), dim3(kGateThreads), smem, st, topk_ids, ws, sh);
}

cudaError_t launch_scatter(const int32_t* topk_ids, int32_t* sorted_ids, int32_t* expert_ids,
                           int32_t* num_post_padded, int32_t* row_of_slot, const Workspace& ws,
                           const Shape& sh, int grid, cudaStream_t st) {
  const size_t smem = scatter_smem_bytes(sh.E, sh.chunk_tokens * sh.k);
  return launch_k(scatter_kernel, dim3(std::max(grid, sh.num_chunks)), dim3(kGateThreads), smem, st, topk_ids,
                  sorted_ids, expert_ids, num_post_padded, row_of_slot, ws, sh);
}

namespace {

// One lock for every change of these kernels' shared memory limits: moe_init (any thread, any
// device) and the allocation-free align both go through raise_align_smem.
std::mutex g_align_smem_mu;

// Raise (never lower) one kernel's dynamic shared memory limit on the current device. The
// limit is kept per kernel and per device context, so a handle on another device, or an
// earlier call with a larger need, never leaves a launch with less than it asked for.
template <typename K>
cudaError_t raise_one(K* kernel, size_t bytes) {
  if (bytes == 0) return cudaSuccess;
  cudaFuncAttributes a{};
  cudaError_t err = cudaFuncGetAttributes(&a, kernel);
  if (err != cudaSuccess) return err;
  if ((size_t)a.maxDynamicSharedSizeBytes >= bytes) return cudaSuccess;
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

template <int VPL>
cudaError_t raise_gate(size_t s) {
  cudaError_t err;
  if ((err = raise_one(gate_kernel<VPL, 1>, s))) return err;
  if ((err = raise_one(gate_kernel<VPL, 2>, s))) return err;
  return raise_one(gate_kernel<VPL, 4>, s);
}

}  // namespace

cudaError_t raise_align_smem(size_t gate_bytes, size_t hist_bytes, size_t scatter_bytes) {
  std::lock_guard<std::mutex> lock(g_align_smem_mu);
  cudaError_t err = cudaSuccess;
  if ((err = raise_gate<1>(gate_bytes)) || (err = raise_gate<2>(gate_bytes)) || (err = raise_gate<4>(gate_bytes)) ||
      (err = raise_gate<8>(gate_bytes)) || (err = raise_gate<16>(gate_bytes)) || (err = raise_gate<32>(gate_bytes)))
    return err;
  if ((err = raise_one(hist_kernel, hist_bytes))) return err;
  return raise_one(scatter_kernel, scatter_bytes);
}

}  // namespace moe
