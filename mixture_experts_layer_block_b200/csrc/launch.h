// launch.h -- host-side launchers of the kernels (implemented next to each kernel).
#pragma once

#include <cuda_runtime.h>

#include <utility>

#include "common.cuh"

namespace moe {

// Launch with programmatic stream serialisation: the kernel may be scheduled while the previous
// kernel of the stream finishes, runs its prologue, and waits (griddep_wait) before it touches
// global memory; the previous kernel lets it in with griddep_launch_dependents.
template <typename... KArgs, typename... Args>
cudaError_t launch_k(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                     Args&&... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Tensor maps of the persistent expert-GEMM kernel.
struct alignas(64) GemmMaps {
  CUtensorMap x_tile;    // x [T][H], box {64, 128} (shared-expert tiles)
  CUtensorMap xs;        // gathered rows [routed_rows][H], box {64, 128}
  CUtensorMap y;         // y [rows][H] bf16, box {64, 128} (store)
  CUtensorMap w_up;      // [E*D][H], box {64, 128}
  CUtensorMap w_gate;    // [E*D][H], box {64, 128}
  CUtensorMap w_down;    // [E*H][D], box {64, 256}
  CUtensorMap h_routed;  // h [rows][D], row stride ldh, box {64, 128}
  CUtensorMap ws_up;     // [Ds][H]
  CUtensorMap ws_gate;   // [Ds][H]
  CUtensorMap ws_down;   // [H][Ds]
  CUtensorMap h_shared;  // h [rows][Ds], row stride ldh
  // the same four A operands with 32-row boxes: the one-SM kernel loads a tile of at most 96
  // rows as whole 32-row boxes instead of one 128-row box
  CUtensorMap x_tile32, xs32, h_routed32, h_shared32;
};

// Router projection: logits[T][E] = x W^T (+ bias). x_map box {64,128}, w_map box {64,BN}.
// With splits > 1 (1, 2 or 4) the K loop is split over blockIdx.z and `logits` receives the
// partials [splits][T][E] (bias in partial 0).
size_t router_smem_bytes(int BN);
int router_splits(int T, int E, int H, int BN, int num_sms);
cudaError_t launch_router(const CUtensorMap& x_map, const CUtensorMap& w_map, const float* bias,
                          float* logits, int T, int E, int H, int BN, int splits, DeviceMeta* meta,
                          int64_t timeout_ns, cudaStream_t stream);

// Gating of logits given as `splits` partials [splits][T][E] (1, 2 or 4; summed in split
// order, and the sums written to logits_out when it is non-null). With `hist`, also the
// per-chunk expert histogram and, in the last CTA, the scans (and the tile/task tables when
// `tiles`).
size_t gate_smem_bytes(const Shape& sh, int max_units);
cudaError_t launch_gate(const float* parts, int splits, float* logits_out, int32_t* topk_ids,
                        float* topk_w, const Workspace& ws, const Shape& sh, bool hist, bool tiles,
                        size_t smem, cudaStream_t stream);

// Histogram of given topk_ids (standalone align), with the same last-CTA scans (no tiles).
cudaError_t launch_hist(const int32_t* topk_ids, const Workspace& ws, const Shape& sh, size_t smem,
                        cudaStream_t stream);

// Grid-wide align writes (and the tile row of every slot when row_of_slot is non-null).
size_t scatter_smem_bytes(int E, int chunk_slots);
cudaError_t launch_scatter(const int32_t* topk_ids, int32_t* sorted_ids, int32_t* expert_ids,
                           int32_t* num_post_padded, int32_t* row_of_slot, const Workspace& ws,
                           const Shape& sh, int grid, cudaStream_t stream);

// Raise (never lower) the dynamic shared memory limits of the gating, histogram and scatter
// kernels on the current device to at least these (0 = leave as is), under one process-wide
// lock, so that concurrent callers on any thread or device only ever raise them.
cudaError_t raise_align_smem(size_t gate_bytes, size_t hist_bytes, size_t scatter_bytes);

// Copy each kept slot's x row into the tile-ordered buffer ws.xs.
cudaError_t launch_gather_rows(const uint16_t* x, const Workspace& ws, const Shape& sh, int grid,
                               cudaStream_t stream);

// out[t] = (shared row of t) + sum_j y[row_of_slot[t*k+j]], in that order, summed in fp32 and
// stored as fp32 (or rounded to bf16 when bf16_out).
cudaError_t launch_combine(void* out, bool bf16_out, const Workspace& ws, const Shape& sh, cudaStream_t stream);

// Persistent expert GEMMs in one of three shapes: general (128-row tiles), tail (the same with
// tails of at most 32 rows merged into the previous tile's tasks; needs sh.merge_tail = 1) and
// small (batches of at most 16 tokens; its maps use 16-row boxes for x_tile, xs, h_routed and
// h_shared).
// kShapeTwo: every group of two m-tiles of one expert runs as one task set whose tasks compute
// both tiles from the same weight stages (needs sh.merge_tail = 2).
enum GemmShape : int { kShapeGeneral = 0, kShapeSmall = 1, kShapeTail = 2, kShapeSmallFused = 3, kShapeTwo = 4 };
size_t gemm_smem_bytes(int shape);
cudaError_t launch_moe_gemm(const GemmMaps& maps, const Workspace& ws, const Shape& sh, int grid, int shape,
                            cudaStream_t stream);

// The whole forward of a batch of at most 16 tokens (and at most 256 experts) as one persistent
// launch of `grid` CTAs, all resident at once (cooperative launch): every CTA computes the router
// logits of a slice of the experts; the last to finish takes the gating, the align scans and
// writes and publishes the schedule; every CTA gathers its share of the x rows, then claims
// expert-GEMM tasks (small-tile shape) as the standalone kernel does; the CTA that finishes the
// last down task of a 256-column block combines that block for every token.
cudaError_t launch_moe_small_fused(const GemmMaps& maps, const Workspace& ws, const Shape& sh,
                                   const FrontArgs& fa, int grid, cudaStream_t stream);

// The same GEMMs with 256-row m-tiles on `pairs` 2-CTA clusters (sh.tile_m = 256; its maps use
// 32-row boxes for x_tile, xs, h_routed, h_shared and y, and 128-row boxes for w_down, ws_down).
size_t gemm_pair_smem_bytes();
cudaError_t launch_moe_gemm_pair(const GemmMaps& maps, const Workspace& ws, const Shape& sh, int pairs,
                                 cudaStream_t stream);

// One-time kernel attribute setup (dynamic shared memory limits).
cudaError_t configure_kernels(size_t gate_smem);

}  // namespace moe
