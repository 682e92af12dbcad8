// mx_quant.cu -- MXFP8 quantisation of bf16 rows: expert weights (once, through the C ABI) and
// each forward's x rows, written straight into the tile-ordered operand buffer of the MXFP8
// expert GEMMs (and, for a shared expert, into a token-ordered copy).
//
// One warp per row; lane l takes the 32-element blocks l, l + 32, ... of the row: it reads the
// block's 64 bytes, finds its largest magnitude, and writes 32 E4M3 codes and one scale code
// (mx.cuh gives the format and the scale layout).
#include "launch.h"
#include "mx.cuh"

namespace moe {

namespace {

constexpr int kMxQuantThreads = 256;

__global__ void __launch_bounds__(kMxQuantThreads)
    mx_quantize_kernel(const uint16_t* __restrict__ src, int64_t R, int K, uint8_t* __restrict__ q,
                       uint8_t* __restrict__ sf) {
  griddep_wait();
  griddep_launch_dependents();
  const int lane = threadIdx.x & 31;
  constexpr int kWarps = kMxQuantThreads / 32;
  const int nb = K / kMxBlock;
  for (int64_t r = (int64_t)blockIdx.x * kWarps + threadIdx.x / 32; r < R; r += (int64_t)gridDim.x * kWarps) {
    for (int b = lane; b < nb; b += 32) {
      float v[32];
      load_bf16x32(src + r * K + b * kMxBlock, v);
      uint32_t w[8];
      const uint32_t code = mx_quantize_block(v, w);
      store_codes32(q + r * K + b * kMxBlock, w);
      sf[mx_sf_offset(r, b, K)] = (uint8_t)code;
    }
  }
}

// One warp per token: its x row is quantised once and written to the token-ordered copy (when
// `token_order`) and to the tile row of each kept slot of the token.
__global__ void __launch_bounds__(kMxQuantThreads)
    mx_gather_kernel(const uint16_t* __restrict__ x, Workspace ws, MxBuffers mx, Shape sh, int token_order) {
  griddep_wait();
  griddep_launch_dependents();
  const int lane = threadIdx.x & 31;
  constexpr int kWarps = kMxQuantThreads / 32;
  const int H = sh.H, nb = H / kMxBlock, k = sh.k;
  for (int t = blockIdx.x * kWarps + threadIdx.x / 32; t < sh.T; t += gridDim.x * kWarps) {
    for (int b = lane; b < nb; b += 32) {
      float v[32];
      load_bf16x32(x + (size_t)t * H + b * kMxBlock, v);
      uint32_t w[8];
      const uint8_t code = (uint8_t)mx_quantize_block(v, w);
      if (token_order) {
        store_codes32(mx.xq + (size_t)t * H + b * kMxBlock, w);
        mx.sf_xq[mx_sf_offset(t, b, H)] = code;
      }
      for (int j = 0; j < k; ++j) {
        const int row = __ldg(ws.row_of_slot + (size_t)t * k + j);
        if (row < 0) continue;  // dropped by the capacity limit
        store_codes32(mx.xs + (size_t)row * H + b * kMxBlock, w);
        mx.sf_xs[mx_sf_offset(row, b, H)] = code;
      }
    }
  }
}

}  // namespace

cudaError_t launch_mx_quantize(const uint16_t* src, int64_t R, int K, uint8_t* q, uint8_t* sf, int grid,
                               cudaStream_t stream) {
  return launch_k(mx_quantize_kernel, dim3(grid), dim3(kMxQuantThreads), 0, stream, src, R, K, q, sf);
}

cudaError_t launch_mx_gather(const uint16_t* x, const Workspace& ws, const MxBuffers& mx, const Shape& sh,
                             bool token_order, int grid, cudaStream_t stream) {
  return launch_k(mx_gather_kernel, dim3(grid), dim3(kMxQuantThreads), 0, stream, x, ws, mx, sh,
                  token_order ? 1 : 0);
}

}  // namespace moe
