// router.cu -- router projection logits[T][E] = x[T][H] . W_router[E][H]^T (+ bias[E]).
//
// Router projection of the Mixture-of-Kittens layer ("Overlapping compute and communication
// in MoE": the router projection picks the top-k routed experts of each token). A dense
// contraction, so it runs on the tensor cores: one CTA per 128 x BN output tile and K split
// (blockIdx.z), TMA-fed smem ring (x tile 128 x 64, W tile BN x 64, both 128-byte swizzled;
// BN = 16..256, one N tile for up to 256 experts),
// tcgen05.mma with the fp32 accumulator in TMEM, and an epilogue warpgroup that stores fp32
// rows. With K split S ways (S = 1, 2 or 4, so that few tokens still fill the GPU) CTA z
// writes partial z of [S][T][E] (the bias goes into partial 0); the gating kernel adds the
// partials in split order, so the sum does not depend on which CTA finished first.
//
// Warp roles: warp 0 TMA producer, warp 1 TMEM allocator + MMA issuer, warps 2-5 epilogue.
#include <algorithm>

#include "launch.h"

namespace moe {

namespace {

constexpr int kRThreads = 192;
constexpr int kRABytes = kBM * kBK * 2;

__device__ __forceinline__ uint32_t tmem_cols_for(int bn) {
  return bn <= 32 ? 32u : (bn <= 64 ? 64u : (bn <= 128 ? 128u : 256u));
}

// Ring depth for an N tile of BN rows: kRouterStages, or fewer so that the ring stays within
// 192 KB of shared memory (4 stages of 48 KB at BN = 256).
__host__ __device__ inline int router_stages(int BN) {
  const int stage_bytes = kRABytes + ((BN * kBK * 2 + 1023) & ~1023);
  const int fit = (192 * 1024) / stage_bytes;
  return fit < kRouterStages ? fit : kRouterStages;
}

// 32 lanes x 16 columns
__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

}  // namespace

__global__ void __launch_bounds__(kRThreads, 1)
    router_kernel(const __grid_constant__ CUtensorMap x_map, const __grid_constant__ CUtensorMap w_map,
                  const float* __restrict__ bias, float* __restrict__ logits, int T, int E, int H,
                  int BN, int kb_per_split, DeviceMeta* meta, int64_t timeout_ns) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // aligned by pointer arithmetic on the shared array (not through an integer), so that the
  // compiler keeps every access through `smem` in the shared address space
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const int b_bytes = BN * kBK * 2;
  const int stage_bytes = kRABytes + ((b_bytes + 1023) & ~1023);
  const int nst = router_stages(BN);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + nst * stage_bytes);
  uint64_t* empty = full + kRouterStages;  // barrier arrays sized for the deepest ring
  uint64_t* acc_full = empty + kRouterStages;
  uint64_t* drain = acc_full + 1;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * kBM, n0 = blockIdx.y * BN;
  const int kb0 = blockIdx.z * kb_per_split;
  const int nk = min(ceil_div(H, kBK) - kb0, kb_per_split);  // >= 1 by construction of the grid
  logits += (size_t)blockIdx.z * T * E;
  if (blockIdx.z != 0) bias = nullptr;
  const uint32_t ncols = tmem_cols_for(BN);

  if (threadIdx.x == 0) {
    for (int i = 0; i < nst; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(drain, 1);
    *s_abort = 0;
    fence_mbar_init();
    tma_prefetch_desc(&x_map);
    tma_prefetch_desc(&w_map);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(s_tmem), ncols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;
  uint32_t nfill = 0;  // TMA fills issued (producer lane)
  griddep_wait();  // inputs of earlier kernels are complete from here on
  griddep_launch_dependents();

  if (warp == 0) {
    if (lane == 0) {
      uint32_t stage = 0, phase = 0;
      for (int kb = 0; kb < nk; ++kb, ++nfill) {
        if (!wait_bar(&empty[stage], phase ^ 1, meta, s_abort, timeout_ns, kSiteRouter)) break;
        const uint32_t a = smem_u32(smem + stage * stage_bytes);
        mbar_arrive_expect_tx(&full[stage], kRABytes + b_bytes);
        tma_load_2d(a, &x_map, &full[stage], (kb0 + kb) * kBK, m0);
        tma_load_2d(a + kRABytes, &w_map, &full[stage], (kb0 + kb) * kBK, n0);
        if (++stage == (uint32_t)nst) { stage = 0; phase ^= 1; }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(kBM, BN);
      uint32_t stage = 0, phase = 0;
      bool ok = true;
      for (int kb = 0; kb < nk; ++kb) {
        if (!wait_bar(&full[stage], phase, meta, s_abort, timeout_ns, kSiteRouter)) { ok = false; break; }
        tc_fence_after();
        const uint32_t a = smem_u32(smem + stage * stage_bytes);
        const uint32_t b = a + kRABytes;
#pragma unroll
        for (int kk = 0; kk < kBK / kUK; ++kk)
          umma_bf16(tmem, sdesc_kmajor_sw128(a + kk * 32), sdesc_kmajor_sw128(b + kk * 32), idesc,
                    (kb | kk) != 0);
        umma_commit(&empty[stage]);
        if (++stage == (uint32_t)nst) { stage = 0; phase ^= 1; }
      }
      if (ok) umma_commit(acc_full);
    }
    __syncwarp();
  } else {
    // epilogue: thread owns one output row
    const int q = warp & 3;
    const int row = q * 32 + lane;
    const int t = m0 + row;
    const bool ok = wait_bar(acc_full, 0, meta, s_abort, timeout_ns, kSiteRouter);
    tc_fence_after();
    if (ok) {
      for (int c = 0; c < BN; c += 16) {
        uint32_t v[16];
        tmem_ld_32x32b_x16(tmem + (static_cast<uint32_t>(q * 32) << 16) + c, v);
        tmem_ld_wait();
        if (t < T) {
          float* dst = logits + (size_t)t * E + n0 + c;
          if ((E & 3) == 0) {  // rows are 16-byte aligned: vector stores of 4 logits
#pragma unroll
            for (int j = 0; j < 16; j += 4) {
              if (n0 + c + j >= E) break;
              float4 o = make_float4(__uint_as_float(v[j]), __uint_as_float(v[j + 1]), __uint_as_float(v[j + 2]),
                                     __uint_as_float(v[j + 3]));
              if (bias) {
                o.x += bias[n0 + c + j];
                o.y += bias[n0 + c + j + 1];
                o.z += bias[n0 + c + j + 2];
                o.w += bias[n0 + c + j + 3];
              }
              *reinterpret_cast<float4*>(dst + j) = o;
            }
          } else {
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const int e = n0 + c + j;
              if (e < E) dst[j] = __uint_as_float(v[j]) + (bias ? bias[e] : 0.f);
            }
          }
        }
      }
    }
  }

  // teardown: every TMA fill and every MMA this CTA issued must have landed before the
  // shared memory and TMEM are released (only waits after an abort)
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) drain_fills(full, nst, nfill, meta, timeout_ns);
  if (threadIdx.x == 32) {
    umma_commit(drain);
    wait_bar_drain(drain, 0, meta, timeout_ns);
  }
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, ncols);
}

size_t router_smem_bytes(int BN) {
  const int b_bytes = BN * kBK * 2;
  const int stage_bytes = kRABytes + ((b_bytes + 1023) & ~1023);
  return (size_t)router_stages(BN) * stage_bytes + 1024 /*align*/ + 256 /*barriers*/;
}

int router_splits(int T, int E, int H, int BN, int num_sms) {
  const int tiles = ceil_div(T, kBM) * ceil_div(E, BN);
  const int nk = ceil_div(H, kBK);
  // S in {1, 2, 4}: about one wave of CTAs, and at least kRouterStages K steps per CTA
  int S = 1;
  while (S < kMaxRouterSplits && 2 * S * tiles <= num_sms && nk / (2 * S) >= router_stages(BN)) S *= 2;
  return S;
}

cudaError_t launch_router(const CUtensorMap& x_map, const CUtensorMap& w_map, const float* bias,
                          float* logits, int T, int E, int H, int BN, int splits, DeviceMeta* meta,
                          int64_t timeout_ns, cudaStream_t stream) {
  const int nk = ceil_div(H, kBK);
  const int kps = ceil_div(nk, splits);  // splits divides the K steps evenly or leaves a short tail
  dim3 grid(ceil_div(T, kBM), ceil_div(E, BN), ceil_div(nk, kps));
  if ((int)grid.z != splits) return cudaErrorInvalidValue;  // the gating sums exactly `splits` partials
  return launch_k(router_kernel, grid, dim3(kRThreads), router_smem_bytes(BN), stream, x_map, w_map, bias,
                  logits, T, E, H, BN, kps, meta, timeout_ns);
}

cudaError_t configure_router_kernel() {
  size_t most = 0;
  for (int bn = 16; bn <= kRouterMaxN; bn *= 2) most = std::max(most, router_smem_bytes(bn));
  return cudaFuncSetAttribute(router_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)most);
}

}  // namespace moe
