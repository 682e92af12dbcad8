// moe_gemm_pair.cu -- the persistent grouped expert GEMM on pairs of SMs.
//
// Same computation, task decomposition and scheduler as moe_gemm.cu (the Mixture-of-Kittens
// layer equation; tiles, an atomic task counter and a lagged unit-major task order as in the
// Weave blog, sections 2.1-2.2 and 5.1), with the m-tile grown to 256 rows and each tile
// computed by a cluster of two CTAs on two SMs:
//  - one tcgen05.mma.cta_group::2 (M = 256, N = 256, K = 16) is issued by CTA 0 and computes
//    the tile's first part in CTA 0's tensor memory and the second part in CTA 1's;
//  - each CTA stages its own A rows and HALF of B (128 of the 256 N rows) per K step, so a
//    K step moves 32 KB through each SM instead of 48 KB for a one-SM 128 x 256 tile doing
//    the same work per SM. The operand rings of these GEMMs are refilled from L2 and HBM at
//    a rate bounded by the bytes in flight per SM, so fewer bytes per MMA means more MMAs;
//  - up tasks: CTA 0 holds 128 rows of W_up, CTA 1 the matching 128 rows of W_gate, so both
//    accumulators hold U | G side by side, exactly as in the one-SM kernel;
//  - the tile's n rows are split between the CTAs in whole 32-row boxes (CTA 0 about half,
//    at most 128), so that a tile of up to 128 rows still moves only half of its A and B
//    bytes through each SM. Rows a CTA does not own stay stale in shared memory; their
//    results land in tensor-memory lanes that are never stored.
//
// Pipeline (per CTA: warp 0 TMA producer, warp 1 MMA issuer (CTA 0 only), warps 2-5 epilogue):
//  - CTA 0's producer claims tasks and writes each into both CTAs' task rings (remote
//    shared-memory stores, published by a release.cluster arrival on CTA 1's task barrier);
//  - both producers wait on their own `empty` barrier and fill their own stage, counting the
//    bytes on CTA 0's `full` barrier (two arrivals per fill, one per producer);
//  - the MMA issuer's commits arrive on both CTAs' `empty` and `acc_full` barriers at once;
//  - both CTAs' epilogue warps release an accumulator and a task slot on CTA 0's barriers.
// Teardown: CTA 1 passes its fill count to CTA 0, which completes any fill only one producer
// issued (after an abort) and waits for every fill and MMA before either CTA leaves.
#include "launch.h"

namespace moe {

namespace {

constexpr int kPStages = 6;
constexpr int kPABytes = kBM * kBK * 2;      // 16 KB: up to 128 rows of A
constexpr int kPBBytes = 128 * kBK * 2;      // 16 KB: this CTA's half of B
constexpr int kPStageBytes = kPABytes + kPBBytes;
constexpr int kPBox = 32;                    // rows per A load box and per result store box
constexpr int kPBoxBytes = kPBox * kBK * 2;  // 4 KB
constexpr int kPStagingOff = kPStages * kPStageBytes;
constexpr int kPBarOff = kPStagingOff + kNumStaging * kStagingBytes;
// full[S], empty[S], acc_full[2], acc_empty[2], task_full[R], task_empty[R], drain
constexpr int kPNumBars = 2 * kPStages + 4 + 2 * kTaskSlots + 1;
constexpr int kPRingOff = kPBarOff + ((kPNumBars * 8 + 63) & ~63);
constexpr int kPMiscOff = kPRingOff + kTaskSlots * (int)sizeof(Task);
constexpr int kPBytes = kPMiscOff + 64;
static_assert(kPStageBytes % 1024 == 0 && kPABytes % 1024 == 0, "1024-byte aligned operand tiles");
static_assert(kPBytes + 1024 <= 227 * 1024, "shared memory budget");
static_assert(sizeof(Task) % 4 == 0, "task ring entries are copied as words");
constexpr int kTaskWords = (int)sizeof(Task) / 4;

__device__ __forceinline__ int n1_of(int expert, const Shape& sh) {
  return ceil_div(expert == sh.E ? sh.Ds : sh.D, kBN1);
}

// The rows [r0, r0 + m) of an n-row tile (n <= 256) that CTA `rank` computes.
__device__ __forceinline__ void pair_rows(int n, uint32_t rank, int& r0, int& m) {
  const int a = min(n, min(kBM, ceil_div(ceil_div(n, 2), kPBox) * kPBox));
  r0 = rank == 0 ? 0 : a;
  m = rank == 0 ? a : n - a;
}

// wait_bar for barriers whose arrivals publish data written into this CTA's shared memory by
// the other CTA.
__device__ __noinline__ bool wait_bar_cluster(uint64_t* bar, uint32_t parity, DeviceMeta* meta,
                                              volatile int* s_abort, int64_t limit_ns, int site) {
  if (mbar_try_wait_cluster(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  uint32_t n = 0;
  while (true) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    if ((++n & 7u) == 0) {
      if (aborted(meta, s_abort)) return false;
      if (static_cast<int64_t>(globaltimer_ns() - t0) > limit_ns) {
        raise_error(meta, s_abort, kStatusTimeout | site);
        return false;
      }
    }
  }
}

__device__ __forceinline__ Task shfl_task(const Task& t) {
  Task r;
  const int32_t* a = reinterpret_cast<const int32_t*>(&t);
  int32_t* b = reinterpret_cast<int32_t*>(&r);
#pragma unroll
  for (int i = 0; i < kTaskWords; ++i) b[i] = __shfl_sync(0xffffffffu, a[i], 0);
  return r;
}

}  // namespace

__global__ void __launch_bounds__(kGemmThreads, 1)
    moe_gemm_pair_kernel(const __grid_constant__ GemmMaps maps, Workspace ws, Shape sh) {
  constexpr int kStages = kPStages;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // both CTAs get the same layout: the MMA addresses the two CTAs' operands at equal offsets
  // aligned by pointer arithmetic on the shared array (not through an integer), so that the
  // compiler keeps every access through `smem` in the shared address space
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kPBarOff);
  uint64_t* full = bars;
  uint64_t* empty = full + kStages;
  uint64_t* acc_full = empty + kStages;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* task_full = acc_empty + 2;
  uint64_t* task_empty = task_full + kTaskSlots;
  uint64_t* drain = task_empty + kTaskSlots;
  Task* ring = reinterpret_cast<Task*>(smem + kPRingOff);
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + kPMiscOff);
  volatile int* s_abort = reinterpret_cast<volatile int*>(smem + kPMiscOff + 4);
  volatile uint32_t* s_peer_nfill = reinterpret_cast<volatile uint32_t*>(smem + kPMiscOff + 8);
  volatile int* s_epi_go = reinterpret_cast<volatile int*>(smem + kPMiscOff + 12);  // [2]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  DeviceMeta* meta = ws.meta;
  const int64_t limit = sh.timeout_ns;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&full[i], 2);  // one arrival per producer (CTA 0's barrier is the one used)
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 8);  // 4 epilogue warps x 2 CTAs
    }
    for (int i = 0; i < kTaskSlots; ++i) {
      mbar_init(&task_full[i], 1);
      mbar_init(&task_empty[i], 10);  // MMA lane + 4 + 4 epilogue warps + CTA 1's producer
    }
    mbar_init(drain, 1);
    *s_abort = 0;
    *s_peer_nfill = 0;
    fence_mbar_init();
    tma_prefetch_desc(&maps.xs);
    tma_prefetch_desc(&maps.y);
    tma_prefetch_desc(&maps.w_up);
    tma_prefetch_desc(&maps.w_gate);
    tma_prefetch_desc(&maps.w_down);
    tma_prefetch_desc(&maps.h_routed);
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(s_tmem), 2 * kAccCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();  // barriers of both CTAs initialised before any remote arrival
  tc_fence_after();
  const uint32_t tmem_base = *s_tmem;
  griddep_wait();
  // CTA 0's barriers, addressed from either CTA
  const uint32_t full_c0 = mapa_shared(smem_u32(full), 0);
  const uint32_t acc_empty_c0 = mapa_shared(smem_u32(acc_empty), 0);
  const uint32_t task_empty_c0 = mapa_shared(smem_u32(task_empty), 0);
  uint32_t nfill = 0;
  bool mma_issued = false;

  if (warp == 0) {
    // ===================================== producers ====================================
    const int nk1 = ceil_div(sh.H, kBK);
    const uint32_t ring_c1 = mapa_shared(smem_u32(ring), 1);
    const uint32_t task_full_c1 = mapa_shared(smem_u32(task_full), 1);
    const int total = __ldcg(&meta->total_tasks);
    const int Mg = __ldcg(&meta->num_groups), Mgr = __ldcg(&meta->num_routed_groups);
    const int U = __ldcg(&meta->num_units);
    int u_cur = 0;
    uint32_t stage = 0, phase = 0, slot = 0, slot_phase = 0;
    int next_tau = 0, batch_end = 0;  // a claim takes sh.claim_batch consecutive ids
    while (true) {
      Task t;
      bool ok = true;
      if (rank == 0) {
        int tau = 0;
        if (lane == 0) {
          if (next_tau >= batch_end) {
            next_tau = atomicAdd(&meta->task_counter, sh.claim_batch);
            batch_end = next_tau + sh.claim_batch;
          }
          tau = aborted(meta, s_abort) ? total : next_tau++;
        }
        tau = __shfl_sync(0xffffffffu, tau, 0);
        t.id = tau;
        t.kind = kTaskStop;
        t.tile = t.expert = t.row0 = t.nrows = t.n0 = t.nk = t.nrows2 = 0;
        t.ntiles = 1;
        if (tau < total) {
          u_cur = find_unit(ws.unit_start, U, tau, u_cur);
          const TaskPos pos = decode_task(ws, sh, u_cur, tau, Mg, Mgr);
          t.kind = pos.kind;
          t.tile = pos.tile;
          const int nt = pos.nt;
          t.expert = __ldcg(&ws.tile_expert[t.tile]);
          t.row0 = __ldcg(&ws.tile_row0[t.tile]);
          t.nrows = __ldcg(&ws.tile_nrows[t.tile]);
          const int Dt = (t.expert == sh.E) ? sh.Ds : sh.D;
          if (t.kind == kTaskUp) {
            t.n0 = nt * kBN1;
            t.nk = nk1;
          } else {
            t.n0 = nt * kBN2;
            t.nk = ceil_div(Dt, kBK);
          }
        }
        // publish to both CTAs' rings
        if (lane == 0) {
          ok = wait_bar(&task_empty[slot], slot_phase ^ 1, meta, s_abort, limit, kSiteProducerTask);
          if (ok) {
            ring[slot] = t;
            const uint32_t* w = reinterpret_cast<const uint32_t*>(&t);
#pragma unroll
            for (int i = 0; i < kTaskWords; ++i)
              st_cluster_u32(ring_c1 + slot * (uint32_t)sizeof(Task) + 4u * i, w[i]);
            mbar_arrive(&task_full[slot]);
            mbar_arrive_release_cluster(task_full_c1 + 8u * slot);
          }
        }
      } else {
        if (lane == 0) {
          ok = wait_bar_cluster(&task_full[slot], slot_phase, meta, s_abort, limit, kSiteProducerTask);
          if (ok) {
            t = ring[slot];
            mbar_arrive_cluster(task_empty_c0 + 8u * slot);
          } else {
            t.kind = kTaskStop;
          }
        }
        t = shfl_task(t);
      }
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      if (!ok || t.kind == kTaskStop) break;
      if (++slot == kTaskSlots) { slot = 0; slot_phase ^= 1; }
      if (rank == 0 && ws.trace_cap > 0 && lane == 0 && t.id < ws.trace_cap) {
        ws.trace[(size_t)t.id * 4 + 0] = blockIdx.x >> 1;
        ws.trace[(size_t)t.id * 4 + 1] = t.id;
        ws.trace[(size_t)t.id * 4 + 2] = (int64_t)globaltimer_ns();
      }
      const bool shared = (t.expert == sh.E);
      // a down task needs both CTAs' results of every up task of its tile
      if (t.kind == kTaskDown) {
        if (lane == 0) {
          ok = wait_count(&ws.done1[t.tile], 2 * n1_of(t.expert, sh) + sh.dep_extra, meta, s_abort, limit);
          if (ok) fence_proxy_async_global();
        }
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        if (!ok) break;
      }
      int r0, m;
      pair_rows(t.nrows, rank, r0, m);
      const int nbox = ceil_div(m, kPBox);
      const uint32_t bytes = (uint32_t)nbox * kPBoxBytes + kPBBytes;
      const bool up = (t.kind == kTaskUp);
      const CUtensorMap* amap = up ? (shared ? &maps.x_tile : &maps.xs) : (shared ? &maps.h_shared : &maps.h_routed);
      const int arow = (up && shared) ? t.row0 + r0 : t.tile * sh.tile_m + r0;
      const CUtensorMap* bmap = up ? (rank == 0 ? (shared ? &maps.ws_up : &maps.w_up) : (shared ? &maps.ws_gate : &maps.w_gate))
                                   : (shared ? &maps.ws_down : &maps.w_down);
      const int brow = up ? (shared ? t.n0 : t.expert * sh.D + t.n0)
                          : (shared ? t.n0 : t.expert * sh.H + t.n0) + (int)rank * 128;
      for (int kb = 0; kb < t.nk; ++kb) {
        if (lane == 0) ok = wait_bar(&empty[stage], phase ^ 1, meta, s_abort, limit, kSiteProducerEmpty);
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        if (!ok) break;
        if (lane == 0) {
          const uint32_t a = smem_u32(smem + stage * kPStageBytes);
          const uint32_t b = a + kPABytes;
          const uint32_t fb = full_c0 + 8u * stage;
          if (rank == 0) mbar_arrive_expect_tx(&full[stage], bytes);
          else mbar_arrive_expect_tx_cluster(fb, bytes);
          for (int j = 0; j < nbox; ++j) tma_load_2d_pair(a + j * kPBoxBytes, amap, fb, kb * kBK, arow + j * kPBox);
          tma_load_2d_pair(b, bmap, fb, kb * kBK, brow);
        }
        __syncwarp();
        ++nfill;
        if (++stage == kStages) { stage = 0; phase ^= 1; }
      }
      if (!ok) break;
    }
  } else if (warp == 1) {
    // ================================= MMA issuer (CTA 0) ===============================
    if (rank == 0 && lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(2 * kBM, kUmmaN);
      uint32_t stage = 0, phase = 0, slot = 0, slot_phase = 0, acc = 0, acc_phase = 0;
      while (true) {
        if (!wait_bar(&task_full[slot], slot_phase, meta, s_abort, limit, kSiteMmaTask)) break;
        const Task t = ring[slot];
        if (t.kind == kTaskStop) break;
        if (!wait_bar(&acc_empty[acc], acc_phase ^ 1, meta, s_abort, limit, kSiteMmaAcc)) break;
        tc_fence_after();
        const uint32_t d = tmem_base + acc * kAccCols;
        bool ok = true;
        for (int kb = 0; kb < t.nk; ++kb) {
          if (!wait_bar(&full[stage], phase, meta, s_abort, limit, kSiteMmaFull)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a = smem_u32(smem + stage * kPStageBytes);
          const uint32_t b = a + kPABytes;
#pragma unroll
          for (int kk = 0; kk < kBK / kUK; ++kk)
            umma_bf16_pair(d, sdesc_kmajor_sw128(a + kk * 32), sdesc_kmajor_sw128(b + kk * 32), idesc,
                           (kb | kk) != 0);
          mma_issued = true;
          umma_commit_pair_mc(&empty[stage], 3);
          if (++stage == kStages) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        umma_commit_pair_mc(&acc_full[acc], 3);
        mbar_arrive(&task_empty[slot]);
        if (++acc == 2) { acc = 0; acc_phase ^= 1; }
        if (++slot == kTaskSlots) { slot = 0; slot_phase ^= 1; }
      }
    }
    __syncwarp();
  } else {
    // ===================================== epilogue =====================================
    // Each thread owns one TMEM lane = row (r0 + row) of the tile part of this CTA. Results go
    // through two 128-byte-swizzled staging buffers and TMA stores of 32-row boxes (only the
    // boxes of this CTA's rows, so the two CTAs never write the same rows).
    const int q = warp & 3;
    const int row = q * 32 + lane;
    const bool leader = (warp == 2 && lane == 0);
    uint8_t* staging = smem + kPStagingOff;
    uint32_t slot = 0, slot_phase = 0, acc = 0, acc_phase = 0, sb = 0;
    auto put_row = [&](uint8_t* buf, const uint32_t (&w)[32]) {
#pragma unroll
      for (int j = 0; j < 8; ++j)
        *reinterpret_cast<uint4*>(buf + row * 128 + ((j ^ (row & 7)) << 4)) =
            make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
    };
    for (uint32_t it = 0;; ++it) {
      // one thread waits for the task and its accumulator and tells the other 127 through the
      // named barrier, so that the four warps always take the same branch (a warp that left
      // the loop alone would strand the others at the next named barrier); the decision word
      // is double-buffered, rewritten only after every thread passed the next loop barrier
      if (leader) {
        int go = 0;
        const bool got = rank == 0 ? wait_bar(&task_full[slot], slot_phase, meta, s_abort, limit, kSiteEpiTask)
                                   : wait_bar_cluster(&task_full[slot], slot_phase, meta, s_abort, limit, kSiteEpiTask);
        if (got && ring[slot].kind != kTaskStop)
          go = wait_bar(&acc_full[acc], acc_phase, meta, s_abort, limit, kSiteEpiAcc) ? 1 : 0;
        s_epi_go[it & 1] = go;
      }
      named_bar_sync(1, 128);
      if (s_epi_go[it & 1] == 0) break;
      const Task t = ring[slot];
      tc_fence_after();
      const uint32_t tacc = tmem_base + acc * kAccCols + (static_cast<uint32_t>(q * 32) << 16);
      const bool shared = (t.expert == sh.E);
      int r0, m;
      pair_rows(t.nrows, rank, r0, m);
      const bool active = q * 32 < m;  // warp-uniform: this warp holds rows of the part
      const int nbox = ceil_div(m, kPBox);
      const int trow = t.tile * sh.tile_m + r0;  // first h / y row of this CTA's part
      if (t.kind == kTaskUp) {
        const CUtensorMap* hmap = shared ? &maps.h_shared : &maps.h_routed;
#pragma unroll 1
        for (int cc = 0; cc < kBN1 / 64; ++cc) {
          uint8_t* buf = staging + sb * kStagingBytes;
          uint32_t pk[32];
          if (active) {
#pragma unroll
            for (int half = 0; half < 2; ++half) {
              uint32_t u[32], g[32];
              tmem_ld_32x32b_x32(tacc + cc * 64 + half * 32, u);
              tmem_ld_32x32b_x32(tacc + kBN1 + cc * 64 + half * 32, g);
              tmem_ld_wait();
#pragma unroll
              for (int j = 0; j < 16; ++j) {
                const float u0 = __uint_as_float(u[2 * j]), u1 = __uint_as_float(u[2 * j + 1]);
                const float g0 = __uint_as_float(g[2 * j]), g1 = __uint_as_float(g[2 * j + 1]);
                pk[half * 16 + j] = pack_bf16x2(__fdividef(u0, 1.0f + __expf(-u0)) * g0,
                                                __fdividef(u1, 1.0f + __expf(-u1)) * g1);
              }
            }
          }
          if (cc == kBN1 / 64 - 1) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(acc_empty_c0 + 8u * acc);
          }
          if (leader) bulk_wait_group_read<kNumStaging - 1>();
          named_bar_sync(1, 128);
          if (active) put_row(buf, pk);
          fence_proxy_async_shared();
          named_bar_sync(1, 128);
          if (leader) {
            for (int j = 0; j < nbox; ++j)
              tma_store_2d(hmap, smem_u32(buf) + j * kPBox * 128, t.n0 + cc * 64, trow + j * kPBox);
            bulk_commit_group();
          }
          sb ^= 1;
        }
        // publish this CTA's part of h before the tile's counter moves
        if (leader) {
          bulk_wait_group<0>();
          fence_proxy_async_global();
          __threadfence();
          red_release_add_gpu(&ws.done1[t.tile], 1);
        }
      } else {
        float w = 0.f;
        if (row < m) {
          if (shared) {
            w = 1.f;
          } else {
            const int s = __ldcg(&ws.sorted_ids[t.row0 + r0 + row]);
            w = __ldcg(&ws.topk_w[s]);
          }
        }
#pragma unroll 1
        for (int cc = 0; cc < kBN2 / 64; ++cc) {
          uint8_t* buf = staging + sb * kStagingBytes;
          uint32_t pk[32];
          if (active) {
#pragma unroll
            for (int half = 0; half < 2; ++half) {
              uint32_t v[32];
              tmem_ld_32x32b_x32(tacc + cc * 64 + half * 32, v);
              tmem_ld_wait();
#pragma unroll
              for (int j = 0; j < 16; ++j)
                pk[half * 16 + j] = pack_bf16x2(w * __uint_as_float(v[2 * j]), w * __uint_as_float(v[2 * j + 1]));
            }
          }
          if (cc == kBN2 / 64 - 1) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(acc_empty_c0 + 8u * acc);
          }
          if (leader) bulk_wait_group_read<kNumStaging - 1>();
          named_bar_sync(1, 128);
          if (active) put_row(buf, pk);
          fence_proxy_async_shared();
          named_bar_sync(1, 128);
          if (leader) {
            for (int j = 0; j < nbox; ++j)
              tma_store_2d(&maps.y, smem_u32(buf) + j * kPBox * 128, t.n0 + cc * 64, trow + j * kPBox);
            bulk_commit_group();
          }
          sb ^= 1;
        }
      }
      if (lane == 0) mbar_arrive_cluster(task_empty_c0 + 8u * slot);
      if (rank == 0 && ws.trace_cap > 0 && leader && t.id < ws.trace_cap)
        ws.trace[(size_t)t.id * 4 + 3] = (int64_t)globaltimer_ns();
      if (++acc == 2) { acc = 0; acc_phase ^= 1; }
      if (++slot == kTaskSlots) { slot = 0; slot_phase ^= 1; }
    }
    if (leader) bulk_wait_group<0>();
  }

  griddep_launch_dependents();
  // teardown: every fill of either CTA completes on CTA 0's `full` barriers, and every MMA
  // writes both CTAs' tensor memory, so CTA 0 drains both before either CTA moves on
  tc_fence_before();
  if (rank == 1 && threadIdx.x == 0) st_cluster_u32(mapa_shared(smem_u32((const void*)s_peer_nfill), 0), nfill);
  cluster_sync_all();
  if (rank == 0 && threadIdx.x == 0) {
    // after an abort one producer may have issued up to a ring's worth of fills the other did
    // not: arrive for the missing producer so that those phases complete when the bytes land
    const uint32_t np = *s_peer_nfill;
    const uint32_t lo = min(nfill, np), hi = max(nfill, np);
    for (uint32_t i = lo; i < hi && i < lo + kStages; ++i) mbar_arrive(&full[i % kStages]);
    drain_fills(full, kStages, hi, meta, limit);
  }
  if (rank == 0 && threadIdx.x == 32 && mma_issued) {
    umma_commit_pair(drain);
    wait_bar_drain(drain, 0, meta, limit);
  }
  cluster_sync_all();
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem_base, 2 * kAccCols);
}

size_t gemm_pair_smem_bytes() { return (size_t)kPBytes + 1024; }

cudaError_t launch_moe_gemm_pair(const GemmMaps& maps, const Workspace& ws, const Shape& sh, int pairs,
                                 cudaStream_t stream) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(2 * pairs);
  cfg.blockDim = dim3(kGemmThreads);
  cfg.dynamicSmemBytes = gemm_pair_smem_bytes();
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, moe_gemm_pair_kernel, maps, ws, sh);
}

// Sets the kernel's shared-memory limit and returns how many 2-CTA clusters fit on the device
// at once (0 if none).
cudaError_t configure_gemm_pair_kernel(int* max_pairs) {
  *max_pairs = 0;
  cudaError_t e = cudaFuncSetAttribute(moe_gemm_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)gemm_pair_smem_bytes());
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(2);
  cfg.blockDim = dim3(kGemmThreads);
  cfg.dynamicSmemBytes = gemm_pair_smem_bytes();
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaOccupancyMaxActiveClusters(max_pairs, (void*)moe_gemm_pair_kernel, &cfg);
}

}  // namespace moe
