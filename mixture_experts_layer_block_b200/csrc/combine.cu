// combine.cu -- the two memory-bound steps around the expert GEMMs.
//
// gather_rows_kernel: copies every kept slot's token row x[t] into the tile-ordered buffer
//   xs (row = first tile of its expert * tile height + its rank in the expert), so that the
//   up/gate GEMM reads its A operand as plain TMA boxes. One warp per slot, 16-byte vectors.
//
// combine_kernel: the sum over experts of the Mixture-of-Kittens layer equation
//   x' = W_shared(x) + sum_{e in top-k} w_e (W_down^e SwiGLU(...)).
//   The down-GEMM epilogue already wrote w_s * (W_down^e h_s) for every kept slot s into its
//   tile row of y (bf16, like the per-slot intermediate cache of the vLLM execution
//   analysis); this kernel adds, per token, the shared-expert row first and then the slots
//   j = 0..k-1 in order (dropped slots skipped), in fp32. The order is fixed, so the result
//   does not depend on the schedule. The sum is stored as fp32, or rounded once to bf16.
//   One warp per (token, 512 columns).
#include <algorithm>

#include "launch.h"

namespace moe {

__global__ void __launch_bounds__(256)
    gather_rows_kernel(const uint16_t* __restrict__ x, Workspace ws, Shape sh) {
  griddep_wait();
  griddep_launch_dependents();
  const int lane = threadIdx.x & 31;
  const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int nw = (gridDim.x * blockDim.x) >> 5;
  const int S = sh.T * sh.k;
  const int nvec = sh.H / 8;  // 16-byte vectors per row (H is a multiple of 8)
  for (int s = gw; s < S; s += nw) {
    const int row = __ldcg(ws.row_of_slot + s);
    if (row < 0) continue;
    const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)(s / sh.k) * sh.H);
    uint4* dst = reinterpret_cast<uint4*>(ws.xs + (size_t)row * sh.H);
    int i = lane;
    for (; i + 96 < nvec; i += 128) {
      const uint4 a = __ldg(src + i), b = __ldg(src + i + 32), c = __ldg(src + i + 64),
                  d = __ldg(src + i + 96);
      dst[i] = a;
      dst[i + 32] = b;
      dst[i + 64] = c;
      dst[i + 96] = d;
    }
    for (; i < nvec; i += 32) dst[i] = __ldg(src + i);
  }
}

// One warp per (token, 512 columns); each lane sums 8 columns in each 256-column half.
template <bool kBf16>
__global__ void __launch_bounds__(256)
    combine_kernel(void* __restrict__ out, Workspace ws, Shape sh) {
  griddep_wait();
  griddep_launch_dependents();
  const int lane = threadIdx.x & 31;
  const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int nw = (gridDim.x * blockDim.x) >> 5;
  const int Mr = __ldcg(&ws.meta->num_routed_tiles);
  const int nblk = ceil_div(sh.H, 512);
  const int64_t items = (int64_t)sh.T * nblk;
  for (int64_t it = gw; it < items; it += nw) {
    const int t = (int)(it / nblk);
    const int c0 = (int)(it % nblk) * 512 + lane * 8, c1 = c0 + 256;
    // this token's rows in y: the shared-expert row first, then its slots in order
    const int myrow = (lane < sh.k) ? __ldcg(ws.row_of_slot + (size_t)t * sh.k + lane) : -1;
    // every lane stays for the shuffles below; lanes past the row's end only skip memory
    const bool has0 = c0 < sh.H, has1 = c1 < sh.H;
    float a0[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    float a1[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    if (sh.Ds > 0) {
      const uint16_t* srow = ws.y + ((size_t)Mr * sh.tile_m + t) * sh.H;
      if (has0) add_bf16x8(a0, __ldcg(reinterpret_cast<const uint4*>(srow + c0)));
      if (has1) add_bf16x8(a1, __ldcg(reinterpret_cast<const uint4*>(srow + c1)));
    }
    for (int j = 0; j < sh.k; ++j) {
      const int row = __shfl_sync(0xffffffffu, myrow, j);
      if (row < 0) continue;  // the same for every lane
      const uint16_t* yr = ws.y + (size_t)row * sh.H;
      if (has0) add_bf16x8(a0, __ldcg(reinterpret_cast<const uint4*>(yr + c0)));
      if (has1) add_bf16x8(a1, __ldcg(reinterpret_cast<const uint4*>(yr + c1)));
    }
    const size_t orow = (size_t)t * sh.H;
    if (has0) store8<kBf16>(out, orow + c0, a0);
    if (has1) store8<kBf16>(out, orow + c1, a1);
  }
}

cudaError_t launch_gather_rows(const uint16_t* x, const Workspace& ws, const Shape& sh, int grid,
                               cudaStream_t stream) {
  return launch_k(gather_rows_kernel, dim3(grid), dim3(256), 0, stream, x, ws, sh);
}

cudaError_t launch_combine(void* out, bool bf16_out, const Workspace& ws, const Shape& sh, cudaStream_t stream) {
  const int64_t warps = (int64_t)sh.T * ceil_div(sh.H, 512);
  const int grid = (int)std::min<int64_t>((warps + 7) / 8, 148 * 16);
  if (bf16_out) return launch_k(combine_kernel<true>, dim3(grid), dim3(256), 0, stream, out, ws, sh);
  return launch_k(combine_kernel<false>, dim3(grid), dim3(256), 0, stream, out, ws, sh);
}

}  // namespace moe
