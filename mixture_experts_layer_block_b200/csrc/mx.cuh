// mx.cuh -- MXFP8 experts: the data layout of quantised operands, E4M3 conversion, and the
// block-scaled tcgen05 wrappers.
//
// Format (the pages name MXFP8 experts -- Mixture-of-Kittens blog, introduction; FlashMoE
// review, "future directions" -- without defining it; read as the OCP Microscaling format):
// E4M3 elements in blocks of 32 consecutive elements along the contraction dimension, each
// block with one E8M0 scale 2^(floor(log2 amax) - 8) (code = exponent + 127, 0 for a zero
// block); elements are v / scale rounded to nearest even with saturation at 448.
//
// Layout in HBM. An operand [R][K] (R and K multiples of 128) is held as its E4M3 codes [R][K]
// (row-major, one byte each) and its scale codes in 512-byte atoms: atom (R/128 row blocks x
// K/128 column blocks, column blocks fastest) holds the scales of 128 rows x 4 blocks of 32,
// with the scale of row r (0..127 in the atom) and block b (0..3) at byte
// (r % 32) * 16 + (r / 32) * 4 + b. That is the order in which one tcgen05.cp of shape
// 32x128b.warpx4 moves an atom into four TMEM columns (lane r % 32, column r / 32, byte b,
// copied to all four lane quarters), where the block-scaled MMA reads the scales of block b
// of a 128-row operand tile through the scale-factor id b of its instruction descriptor.
#pragma once

#include <cuda.h>

#include "common.cuh"

namespace moe {

constexpr int kMxBlock = 32;          // elements per E8M0 scale
constexpr int kMxBK = 128;            // K elements (= bytes) per pipeline stage: one swizzle row
constexpr int kMxUK = 32;             // K per block-scaled tcgen05.mma
constexpr int kSfAtomBytes = 512;     // scales of 128 rows x 4 blocks

// Byte offset of the scale of (row r, block b) in the scale array of an [R][K] operand.
__host__ __device__ inline size_t mx_sf_offset(int64_t r, int b, int64_t K) {
  return ((size_t)(r >> 7) * (size_t)(K >> 7) + (size_t)(b >> 2)) * kSfAtomBytes + (size_t)(r & 31) * 16 +
         (size_t)((r >> 5) & 3) * 4 + (size_t)(b & 3);
}

// Byte offset of the scale atom of (row block rb, column block kq) of an [R][K] operand.
__host__ __device__ inline size_t mx_atom_offset(int64_t rb, int64_t kq, int64_t K) {
  return ((size_t)rb * (size_t)(K >> 7) + (size_t)kq) * kSfAtomBytes;
}

// 32 bf16 values at p (64 bytes, 16-byte aligned) widened to fp32.
__device__ __forceinline__ void load_bf16x32(const uint16_t* p, float (&v)[32]) {
  const uint4* p4 = reinterpret_cast<const uint4*>(p);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint4 w = __ldcg(p4 + i);
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      v[8 * i + 2 * j] = __uint_as_float(ws[j] << 16);
      v[8 * i + 2 * j + 1] = __uint_as_float(ws[j] & 0xffff0000u);
    }
  }
}

__device__ __forceinline__ void store_codes32(uint8_t* p, const uint32_t (&q)[8]) {
  uint4* p4 = reinterpret_cast<uint4*>(p);
  p4[0] = make_uint4(q[0], q[1], q[2], q[3]);
  p4[1] = make_uint4(q[4], q[5], q[6], q[7]);
}

// Tensor maps of the MXFP8 expert GEMMs (E4M3 operands as 8-bit elements, 128-byte swizzle).
struct alignas(64) MxMaps {
  CUtensorMap x_tile;  // xq [T][H], box {128, 128} (shared-expert tiles read tokens in order)
  CUtensorMap xs;      // xs [routed rows][H], box {128, 128}
  CUtensorMap h;       // h [rows][ldh], box {128, 128}: stored by up tasks, loaded by down tasks
  CUtensorMap y;       // y [rows][H] bf16, box {64, 128} (store)
  CUtensorMap w_up, w_gate;    // [E*D][H], box {128, 128}
  CUtensorMap w_down;          // [E*H][D], box {128, 256}
  CUtensorMap ws_up, ws_gate;  // [Ds][H]
  CUtensorMap ws_down;         // [H][Ds]
  // the A operands with 32-row boxes: a tile of at most 96 rows is loaded as whole 32-row boxes
  CUtensorMap x_tile32, xs32, h32;
};

// Quantised activations (workspace) and the weights' scale arrays.
struct MxBuffers {
  uint8_t* xq;           // [T][H] x in token order (read by shared-expert tiles)
  uint8_t* sf_xq;
  uint8_t* xs;           // [routed rows][H] kept slots' x rows in tile order
  uint8_t* sf_xs;
  uint8_t* h;            // [rows][ldh] SwiGLU activations in tile order
  uint8_t* sf_h;
  const uint8_t* sf_up;    // scales of W_up [E*D][H]
  const uint8_t* sf_gate;  // W_gate [E*D][H]
  const uint8_t* sf_down;  // W_down [E*H][D]
  const uint8_t* sfs_up;   // shared expert: [Ds][H], [Ds][H], [H][Ds]
  const uint8_t* sfs_gate;
  const uint8_t* sfs_down;
};

// ---- device helpers --------------------------------------------------------------------------

// E8M0 code of a block whose largest magnitude is amax: floor(log2 amax) - 8 + 127, clamped at
// 0 (an fp32 exponent field of at most 8, a zero or a subnormal maximum included).
__device__ __forceinline__ uint32_t mx_scale_code(float amax) {
  const int ebits = (int)((__float_as_uint(amax) >> 23) & 0xFFu);
  return ebits > 8 ? (uint32_t)(ebits - 8) : 0u;
}

// 1 / scale = 2^(127 - code) as an fp32 (code <= 246, so the exponent stays normal).
__device__ __forceinline__ float mx_inv_scale(uint32_t code) { return __uint_as_float((254u - code) << 23); }

// Two fp32 values to E4M3 (round to nearest even, saturating at +-448): lo in bits 0-7.
__device__ __forceinline__ uint32_t cvt_e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// 32 values (one block) -> 8 words of E4M3 codes (element i in byte i % 4 of word i / 4) and
// the block's scale code.
__device__ __forceinline__ uint32_t mx_quantize_block(const float (&v)[32], uint32_t (&q)[8]) {
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[i]));
  const uint32_t code = mx_scale_code(amax);
  const float inv = mx_inv_scale(code);
#pragma unroll
  for (int i = 0; i < 8; ++i)
    q[i] = cvt_e4m3x2(v[4 * i] * inv, v[4 * i + 1] * inv) | (cvt_e4m3x2(v[4 * i + 2] * inv, v[4 * i + 3] * inv) << 16);
  return code;
}

// Untiled bulk copy global -> shared, completing `bytes` on the mbarrier (16-byte aligned
// addresses, size a multiple of 16).
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Shared-memory descriptor of one scale atom for tcgen05.cp: 32 rows of 16 bytes, no swizzle
// (8-row core matrices 128 bytes apart).
__device__ __forceinline__ uint64_t sdesc_sf_atom(uint32_t saddr) {
  return static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4) | (static_cast<uint64_t>(1) << 16) |
         (static_cast<uint64_t>(128 >> 4) << 32) | (static_cast<uint64_t>(1) << 46);
}

// Copy one scale atom from shared memory into TMEM columns taddr .. taddr + 3 of all 128 lanes.
__device__ __forceinline__ void tmem_copy_sf_atom(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

// Instruction descriptor of kind::mxf8f6f4 with E4M3 A and B (format 0), both K-major, E8M0
// scales (bit 23), N >> 3 (17-22), M >> 4 (24-28), and the byte of each scale column that
// holds this MMA's block: bits 4-5 (B) and 29-30 (A).
__host__ __device__ constexpr uint32_t idesc_mxf8_e4m3(int M, int N, int sf_id) {
  return (static_cast<uint32_t>(sf_id) << 4) | (static_cast<uint32_t>(N >> 3) << 17) | (1u << 23) |
         (static_cast<uint32_t>(M >> 4) << 24) | (static_cast<uint32_t>(sf_id) << 29);
}

// D (+)= (A * scales_A) (B * scales_B)^T over K = 32, with the scales in TMEM.
__device__ __forceinline__ void umma_mxf8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}

// ---- host launchers (mx_quant.cu, moe_gemm_mx.cu) ---------------------------------------------

// Quantise the rows of a bf16 matrix [R][K] (R, K multiples of 128): codes q [R][K] and scales.
cudaError_t launch_mx_quantize(const uint16_t* src, int64_t R, int K, uint8_t* q, uint8_t* sf, int grid,
                               cudaStream_t stream);

// Quantise each token's x row once: to xq (token order, when the layer has a shared expert) and
// to the tile row of every kept slot of the token in xs.
cudaError_t launch_mx_gather(const uint16_t* x, const Workspace& ws, const MxBuffers& mx, const Shape& sh,
                             bool token_order, int grid, cudaStream_t stream);

size_t gemm_mx_smem_bytes();
cudaError_t configure_gemm_mx_kernel();
cudaError_t launch_moe_gemm_mx(const MxMaps& maps, const Workspace& ws, const MxBuffers& mx, const Shape& sh,
                               int grid, cudaStream_t stream);

// The whole MXFP8 forward of at most 16 tokens (and at most 256 experts) as one cooperative
// launch of `grid` CTAs, as launch_moe_small_fused does for bf16 experts; the front's row gather
// quantises the x rows.
cudaError_t launch_moe_mx_small_fused(const MxMaps& maps, const Workspace& ws, const MxBuffers& mx, const Shape& sh,
                                      const FrontArgs& fa, int grid, cudaStream_t stream);
int mx_small_fused_blocks_per_sm();

}  // namespace moe
