// moe_gemm.cu -- the persistent grouped expert GEMM with the atomic tile scheduler.
//
// What it computes (Mixture-of-Kittens blog, "Overlapping compute and communication in
// MoE"): for every kept slot s = (t, j) routed to expert e,
//     h_s  = SiLU(W_up^e x_t) (.) (W_gate^e x_t)                   (bf16, kept in HBM/L2)
//     y_s   = w_s * W_down^e h_s                                   (bf16, per slot row)
// plus the shared expert over every token with weight 1.
//
// How (Weave blog, sections 2.1-2.2 and 5.1: tile decomposition, an atomic task counter,
// one persistent CTA per SM that claims tasks until the queue is empty):
//  - m-tile: up to 128 sorted rows of one expert (align output), or 128 tokens of the
//    shared expert.
//  - up task   (tile, n): A = the tile's 128 x rows (pre-gathered in tile order into xs by
//    the gather kernel; shared-expert tiles read x directly); B = 128 rows of W_up^e stacked
//    on 128 rows of W_gate^e; one tcgen05.mma of N = 256 per K step, so TMEM holds U | G; the
//    epilogue writes h = SiLU(U) * G (bf16) for columns n*128 .. n*128+127 and counts the
//    tile's done1.
//  - down task (tile, n): waits until done1[tile] covers every up task of the tile (bounded
//    spin), then A = the tile's h rows, B = 256 rows of W_down^e; the epilogue scales each
//    row by its router weight and writes it (bf16) to the tile's rows of y. The combine
//    kernel sums each token's rows in slot order in fp32.
//  - epilogue results go through 16 KB shared-memory staging buffers (128-byte swizzled)
//    and asynchronous TMA tensor stores, so the epilogue warps release TMEM and move on
//    while the stores drain.
//  - consecutive tiles of one expert are scheduled as groups of two whose tasks are numbered
//    n-major (the two tasks that read the same weight rows are claimed back to back); in the
//    tail shape a group of a full tile and a tail of at most 32 rows runs as one task set that
//    computes both tiles from the same B stages into the two TMEM accumulators.
//  - task ids are numbered in units: unit u = up tasks of group u, then down tasks of group
//    u - lag. A down task's dependencies always have smaller ids, and claims are monotone,
//    so the earliest unfinished task can always make progress (no deadlock). A claim finds
//    its unit with one warp-wide round of loads.
//  - ablation (MOE_FLAG_STATIC_QUOTA): CTAs walk a fixed share of the experts' tasks instead
//    of claiming from the counter.
//
// Warp roles (192 threads, one CTA per SM): warp 0 claims tasks and issues TMA into the
// operand ring (general shape 4 x 48 KB, tail shape 4 x 52 KB, small-tile shape 6 x 34 KB);
// warp 1 allocates 512 TMEM columns (two 256-column fp32 accumulators) and issues tcgen05.mma
// from one lane; warps 2-5 drain TMEM (tcgen05.ld) in the epilogue. Producer -> consumers: a
// 4-entry task ring guarded by mbarriers. Every wait is bounded (globaltimer); a wait that
// runs out records a status code, sets the abort flag, and every CTA drains its in-flight
// copies and MMAs and exits.
#include "launch.h"
#include "front.cuh"
#include "route.cuh"

namespace moe {

namespace {

// Three shapes of the kernel (GemmShape). The general one moves 128-row A tiles through a
// 4 x 48 KB ring and writes its epilogue results with TMA stores from two staging buffers.
// The tail shape adds a 4 KB slot per stage for the 32 rows of a tail tile that rides along in
// the tasks of its expert's previous tile (4 x 52 KB ring), which leaves room for one staging
// buffer only. The small-tile one serves batches of at most 16 tokens (every m-tile then holds
// at most 16 rows): it moves 16-row A boxes (2 KB), so the same shared memory holds a
// 6 x 34 KB ring and 50% more weight bytes in flight per SM, and its epilogue stores the valid
// rows directly. Its MMAs stay M=128: rows 16..127 read the stage's B bytes (finite values)
// and their results are never stored.
template <int kShape>
struct Cfg {
  static constexpr bool kSmall = (kShape == kShapeSmall || kShape == kShapeSmallFused);
  static constexpr bool kTwo = (kShape == kShapeTwo);
  static constexpr bool kTail = (kShape == kShapeTail) || kTwo;  // a task may carry a second tile
  static constexpr int kStagesN = kSmall ? 6 : (kTwo ? 3 : kStages);
  static constexpr int kARows = kSmall ? 16 : kBM;
  static constexpr int kABytesN = kARows * kBK * 2;
  static constexpr int kTailBytesN = kTwo ? kBM * kBK * 2 : (kTail ? kTailRows * kBK * 2 : 0);
  static constexpr int kStageBytesN = kABytesN + kTailBytesN + kBBytes;
  static constexpr int kNumStagingN = kSmall ? 0 : ((kTail && !kTwo) ? 1 : kNumStaging);
  static constexpr int kStagingOff = kStagesN * kStageBytesN;
  static constexpr int kBarOff = kStagingOff + kNumStagingN * kStagingBytes;
  // barriers: full[S], empty[S], acc_full[2], acc_empty[2], task_full[R], task_empty[R], drain
  static constexpr int kNumBars = 2 * kStagesN + 4 + 2 * kTaskSlots + 1;
  static constexpr int kRingOff = kBarOff + ((kNumBars * 8 + 63) & ~63);
  static constexpr int kMiscOff = kRingOff + kTaskSlots * (int)sizeof(Task);
  // the fused small-batch forward keeps every slot's tile row (row_of_slot) in shared memory
  // the fused small-batch forward keeps its schedule (FusedSched) in shared memory
  static constexpr int kFusedOff = kMiscOff + 64;
  static constexpr int kBytes = kFusedOff + (kShape == kShapeSmallFused ? (int)((sizeof(FusedSched) + 15) & ~15) : 0);
  static_assert(kStageBytesN % 1024 == 0 && kABytesN % 1024 == 0 && kTailBytesN % 1024 == 0,
                "1024-byte aligned operand tiles");
  static_assert(kBytes + 1024 <= 227 * 1024, "shared memory budget");
};

__device__ __forceinline__ int n1_of(int expert, const Shape& sh) {
  return ceil_div(expert == sh.E ? sh.Ds : sh.D, kBN1);
}

}  // namespace

template <int kShape>
__global__ void __launch_bounds__(kGemmThreads, 1)
    moe_gemm_kernel(const __grid_constant__ GemmMaps maps, Workspace ws, Shape sh, FrontArgs fa) {
  using C = Cfg<kShape>;
  constexpr bool kSmall = C::kSmall;
  constexpr bool kFused = (kShape == kShapeSmallFused);
  constexpr bool kTail = C::kTail;
  constexpr int kStages = C::kStagesN;
  constexpr int kStageBytes = C::kStageBytesN;
  constexpr int kABytes = C::kABytesN;
  constexpr int kBOff = C::kABytesN + C::kTailBytesN;  // B's offset in a stage
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // aligned by pointer arithmetic on the shared array (not through an integer), so that the
  // compiler keeps every access through `smem` in the shared address space
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  uint64_t* full = bars;
  uint64_t* empty = full + kStages;
  uint64_t* acc_full = empty + kStages;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* task_full = acc_empty + 2;
  uint64_t* task_empty = task_full + kTaskSlots;
  uint64_t* drain = task_empty + kTaskSlots;
  Task* ring = reinterpret_cast<Task*>(smem + C::kRingOff);
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + C::kMiscOff);
  volatile int* s_abort = reinterpret_cast<volatile int*>(smem + C::kMiscOff + 4);
  volatile int* s_epi_go = reinterpret_cast<volatile int*>(smem + C::kMiscOff + 8);  // [2]
  volatile int* s_front = reinterpret_cast<volatile int*>(smem + C::kMiscOff + 16);  // fused: ok
  FusedSched* fs = reinterpret_cast<FusedSched*>(smem + C::kFusedOff);  // fused: the schedule

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  DeviceMeta* meta = ws.meta;
  const int64_t limit = sh.timeout_ns;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 4);  // one arrival per epilogue warp
    }
    for (int i = 0; i < kTaskSlots; ++i) {
      mbar_init(&task_full[i], 1);
      mbar_init(&task_empty[i], 5);  // MMA lane + 4 epilogue warps
    }
    mbar_init(drain, 1);
    *s_abort = 0;
    fence_mbar_init();
    tma_prefetch_desc(&maps.xs);
    tma_prefetch_desc(&maps.y);
    tma_prefetch_desc(&maps.w_up);
    tma_prefetch_desc(&maps.w_gate);
    tma_prefetch_desc(&maps.w_down);
    tma_prefetch_desc(&maps.h_routed);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(s_tmem), 2 * kAccCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *s_tmem;
  griddep_wait();  // inputs of earlier kernels are complete from here on
  uint32_t nfill = 0;  // TMA stage fills issued by this CTA (producer warp)
  bool mma_issued = false;

  // wait accounting while tracing (globaltimer ns, per role thread; see kWait* in common.cuh)
  const bool tracing = ws.trace_cap > 0;
  int64_t wacc[kNumWaits];
#pragma unroll
  for (int i = 0; i < kNumWaits; ++i) wacc[i] = 0;
  auto now = [&]() -> int64_t { return tracing ? (int64_t)globaltimer_ns() : 0; };

  bool run_tasks = true;
  const int64_t t_front = now();
  if constexpr (kFused) {
    // the front, by all 192 threads; the operand ring is free until the first TMA fill. CTA 0
    // resets the forward's counters, every CTA computes its router slice, then, once every
    // slice is in, the whole schedule for itself (no CTA waits for another's tables)
    int* fsm = reinterpret_cast<int*>(smem);
    if (blockIdx.x == 0) front_reset(ws, sh);
    front_router(fa, ws, sh, reinterpret_cast<float*>(fsm));
    __syncthreads();
    const int64_t t_r = now();
    if (threadIdx.x == 0) s_front[0] = front_arrive(ws, fa, meta, limit) ? 1 : 0;
    __syncthreads();
    int64_t ts[4] = {0, 0, 0, 0};
    const int64_t t_arrived = now();
    run_tasks = s_front[0] != 0;
    if (run_tasks) {
      front_schedule(fa, ws, sh, fsm, fs, blockIdx.x == 0, ts);
      __syncthreads();
    }
    const int64_t t_s = now();
    if (run_tasks) front_gather(fa, ws, sh, fs->slot_row);
    // the ring's generic-proxy writes come before the TMA fills that reuse it
    fence_proxy_async_shared();
    __syncthreads();
    if (threadIdx.x == 0) {
      wacc[kFrontRouter] = t_r - t_front;
      wacc[kFrontSchedule] = t_s - t_r;
      wacc[kFrontGather] = now() - t_s;
      wacc[kFrontLast] = tracing && blockIdx.x == 0 ? 1 : 0;
      if (tracing) {
        wacc[kSchedArrive] = t_arrived - t_r;
        wacc[kSchedLogits] = ts[0] - t_arrived;
        wacc[kSchedGating] = ts[1] - ts[0];
        wacc[kSchedTables] = ts[2] - ts[1];
        wacc[kSchedWrites] = ts[3] - ts[2];
        wacc[kSchedPublish] = t_s - ts[3];
      }
    }
  }

  if (!run_tasks) {
    // the schedule never came (bounded wait ran out): nothing was issued, go to the teardown
  } else if (warp == 0) {
    // ===================================== producer =====================================
    const int total = kFused ? fs->n_tasks : __ldcg(&meta->total_tasks);
    const int Mg = __ldcg(&meta->num_groups), Mgr = __ldcg(&meta->num_routed_groups);
    const int U = __ldcg(&meta->num_units);
    const int nk1 = ceil_div(sh.H, kBK);
    int u_cur = 0;
    uint32_t stage = 0, phase = 0, slot = 0, slot_phase = 0;
    // Static per-expert quota (ablation): X slots (experts, plus the shared expert) over G CTAs.
    // With G >= X each slot gets floor(G/X) CTAs, which take its tasks in turn, and the CTAs
    // left over stay idle; with G < X, CTA c takes slots c, c+G, ... one after the other.
    const int X = sh.E + (sh.Ds > 0 ? 1 : 0), G = (int)gridDim.x;
    const int q = (G >= X) ? G / X : 1;
    int sq_slot = (G >= X) ? (int)blockIdx.x / q : (int)blockIdx.x;
    const int sq_r = (G >= X) ? (int)blockIdx.x % q : 0;
    const int sq_stride = (G >= X) ? X : G;
    SlotIter sq_it;
    int sq_j = 0;
    if (sh.static_quota && lane == 0 && sq_slot < X) sq_it.start(ws, sq_slot);
    // Claims run ahead by less than a ring: the id of the next task is fetched from the counter
    // while the current task's last kStages stages are issued, so the atomic's round trip
    // overlaps them, but a claimed task is never held for longer than one ring drains (a held
    // task is one no idle CTA can take at the end of the queue). The held id is always the next
    // task this producer starts, and every task it waits for has a smaller id, so the smallest
    // unfinished task still always makes progress.
    // A claim takes sh.claim_batch consecutive ids; batch_end is one past the held batch.
    const uint64_t w_policy = kSmall ? policy_evict_first() : 0;
    int next_tau = 0, batch_end = 0;
    if (!sh.static_quota && lane == 0) {
      next_tau = atomicAdd(&meta->task_counter, sh.claim_batch);
      batch_end = next_tau + sh.claim_batch;
    }
    // with the task table, the claimed task's entry is loaded one stage after the claim
    const bool use_tab = ws.task_tab != nullptr && !sh.static_quota && !kFused;
    int4 next_ent = make_int4(0, 0, 0, 0);
    int ent_tau = -1;  // the claim whose entry next_ent holds
    const int64_t t_loop = now();
    while (true) {
      const int64_t t_top = now();
      int tau = 0, unit = 0;
      if (sh.static_quota) {
        if (lane == 0) {
          tau = total;  // stop unless a task of this CTA's slots remains
          while (!aborted(meta, s_abort) && sq_slot < X) {
            int u = 0;
            const int cand = sq_it.next(ws, sh, Mg, Mgr, u);
            if (cand < 0) {
              sq_slot += sq_stride;
              sq_j = 0;
              if (sq_slot < X) sq_it.start(ws, sq_slot);
              continue;
            }
            if (sq_j++ % q == sq_r) {
              tau = cand;
              unit = u;
              break;
            }
          }
        }
        unit = __shfl_sync(0xffffffffu, unit, 0);
      } else if (lane == 0) {
        tau = aborted(meta, s_abort) ? total : next_tau;
      }
      tau = __shfl_sync(0xffffffffu, tau, 0);
      Task t;
      t.id = tau;
      t.ntiles = 1;
      t.nrows2 = 0;
      if (tau >= total) {
        t.kind = kTaskStop;
      } else if (kFused) {
        if (lane == 0) fused_task(*fs, sh, tau, t);
        t.kind = __shfl_sync(0xffffffffu, t.kind, 0);
        t.tile = __shfl_sync(0xffffffffu, t.tile, 0);
        t.expert = __shfl_sync(0xffffffffu, t.expert, 0);
        t.row0 = __shfl_sync(0xffffffffu, t.row0, 0);
        t.nrows = __shfl_sync(0xffffffffu, t.nrows, 0);
        t.n0 = __shfl_sync(0xffffffffu, t.n0, 0);
        t.ntiles = 1;
        t.nrows2 = 0;
        t.nk = t.kind == kTaskUp ? nk1 : ceil_div(t.expert == sh.E ? sh.Ds : sh.D, kBK);
      } else if (use_tab) {
        int4 ent = next_ent;
        if (lane == 0 && ent_tau != tau) ent = __ldcg(ws.task_tab + tau);
        ent.x = __shfl_sync(0xffffffffu, ent.x, 0);
        ent.y = __shfl_sync(0xffffffffu, ent.y, 0);
        ent.z = __shfl_sync(0xffffffffu, ent.z, 0);
        ent.w = __shfl_sync(0xffffffffu, ent.w, 0);
        t.tile = ent.x;
        t.expert = ent.y;
        t.row0 = ent.z;
        t.nrows = ent.w & 511;
        t.kind = (ent.w >> 19) & 1;
        t.ntiles = kTail ? (((ent.w >> 18) & 1) ? 2 : 1) : 1;
        t.nrows2 = t.ntiles == 2 ? (ent.w >> 9) & 511 : 0;
        const int nt = ent.w >> 20;
        if (t.kind == kTaskUp) {
          t.n0 = nt * kBN1;
          t.nk = nk1;
        } else {
          t.n0 = nt * kBN2;
          t.nk = ceil_div(t.expert == sh.E ? sh.Ds : sh.D, kBK);
        }
      } else {
        u_cur = sh.static_quota ? unit : find_unit(ws.unit_start, U, tau, u_cur);
        const TaskPos pos = decode_task(ws, sh, u_cur, tau, Mg, Mgr);
        t.kind = pos.kind;
        t.tile = pos.tile;
        const int nt = pos.nt;
        t.expert = __ldcg(&ws.tile_expert[t.tile]);
        t.row0 = __ldcg(&ws.tile_row0[t.tile]);
        t.nrows = __ldcg(&ws.tile_nrows[t.tile]);
        t.ntiles = kTail ? pos.ntiles : 1;
        t.nrows2 = (t.ntiles == 2) ? __ldcg(&ws.tile_nrows[t.tile + 1]) : 0;
        const int Dt = (t.expert == sh.E) ? sh.Ds : sh.D;
        if (t.kind == kTaskUp) {
          t.n0 = nt * kBN1;
          t.nk = nk1;
        } else {
          t.n0 = nt * kBN2;
          t.nk = ceil_div(Dt, kBK);
        }
      }
      // publish the task to the MMA and epilogue warps
      bool ok = true;
      if (lane == 0) {
        const int64_t t0 = now();
        ok = wait_bar(&task_empty[slot], slot_phase ^ 1, meta, s_abort, limit, kSiteProducerTask);
        const int64_t t1 = now();
        wacc[kWaitProdRing] += t1 - t0;
        wacc[kWaitProdClaim] += t0 - t_top;
        if (ok) {
          ring[slot] = t;
          mbar_arrive(&task_full[slot]);
        }
      }
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      if (!ok || t.kind == kTaskStop) break;
      if (++slot == kTaskSlots) { slot = 0; slot_phase ^= 1; }
      const int claim_kb = t.nk > kStages ? t.nk - kStages : 0;  // stage at which the next id is claimed
      if (ws.trace_cap > 0 && lane == 0) {
        // claim time goes to the trace slot of this task id (written again at completion)
        if (tau < ws.trace_cap) {
          ws.trace[(size_t)tau * 4 + 0] = blockIdx.x;
          ws.trace[(size_t)tau * 4 + 1] = tau;
          ws.trace[(size_t)tau * 4 + 2] = (int64_t)globaltimer_ns();
        }
      }
      const bool shared = (t.expert == sh.E);
      // fused small-batch forward: an up task of a routed tile needs the tile's gathered x rows
      if (kFused && t.kind == kTaskUp && !shared) {
        if (lane == 0) {
          const int64_t t0 = now();
          ok = wait_count(&ws.gather_done[t.tile], t.nrows, meta, s_abort, limit);
          wacc[kWaitProdDep] += now() - t0;
          if (ok) fence_proxy_async_global();
        }
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        if (!ok) break;
      }
      // a down task needs every up task of its tile(s)
      if (t.kind == kTaskDown) {
        if (lane == 0) {
          const int need = n1_of(t.expert, sh) + sh.dep_extra;
          const int64_t t0 = now();
          ok = wait_count(&ws.done1[t.tile], need, meta, s_abort, limit);
          if (ok && t.ntiles == 2) ok = wait_count(&ws.done1[t.tile + 1], need, meta, s_abort, limit);
          wacc[kWaitProdDep] += now() - t0;
          if (ok) fence_proxy_async_global();
        }
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        if (!ok) break;
      }
      const int wrow_up = shared ? t.n0 : t.expert * sh.D + t.n0;
      const int wrow_dn = shared ? t.n0 : t.expert * sh.H + t.n0;
      // A operand: one box of kARows rows, or (general shape, tiles of at most 96 rows) only
      // the 32-row boxes that hold the tile's rows; the rest of the A slot keeps stale rows,
      // whose results land in output rows past the tile's end
      const bool up = (t.kind == kTaskUp);
      const int nbox = (!kSmall && t.nrows <= 3 * kPairBoxRows) ? ceil_div(t.nrows, kPairBoxRows) : 0;
      // the second tile of a two-tile task: one 32-row box (tail shape), or (two-tile shape) its
      // 32-row boxes when it has at most 96 rows, else one 128-row box
      const int nbox2 = t.ntiles != 2 ? 0
                        : (!C::kTwo || t.nrows2 <= 3 * kPairBoxRows ? ceil_div(t.nrows2, kPairBoxRows) : -1);
      const uint32_t stage_tx = (nbox ? (uint32_t)nbox * kPairBoxRows * kBK * 2 : (uint32_t)kABytes) + kBBytes +
                                (nbox2 < 0 ? (uint32_t)kABytes : (uint32_t)nbox2 * kPairBoxRows * kBK * 2);
      const CUtensorMap* amap = up ? (shared ? &maps.x_tile : &maps.xs) : (shared ? &maps.h_shared : &maps.h_routed);
      const CUtensorMap* amap32 =
          up ? (shared ? &maps.x_tile32 : &maps.xs32) : (shared ? &maps.h_shared32 : &maps.h_routed32);
      const int arow = (up && shared) ? t.row0 : t.tile * kBM;
      const int arow2 = (up && shared) ? t.row0 + kBM : (t.tile + 1) * kBM;  // a merged tail's rows
      for (int kb = 0; kb < t.nk; ++kb) {
        if (lane == 0) {
          const int64_t t0 = now();
          ok = wait_bar(&empty[stage], phase ^ 1, meta, s_abort, limit, kSiteProducerEmpty);
          wacc[kWaitProdEmpty] += now() - t0;
        }
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        if (!ok) break;
        if (lane == 0) {
          const uint32_t a = smem_u32(smem + stage * kStageBytes);
          const uint32_t b = a + kBOff;
          mbar_arrive_expect_tx(&full[stage], stage_tx);
          // A: the tile's rows of x in tile order (routed: gathered copy; shared: the tokens),
          // or of h for down tasks
          if (nbox == 0) {
            tma_load_2d(a, amap, &full[stage], kb * kBK, arow);
          } else {
            for (int j = 0; j < nbox; ++j)
              tma_load_2d(a + j * kPairBoxRows * 128, amap32, &full[stage], kb * kBK, arow + j * kPairBoxRows);
          }
          if (kTail && nbox2 < 0) {
            tma_load_2d(a + kABytes, amap, &full[stage], kb * kBK, arow2);
          } else if (kTail) {
            for (int j = 0; j < nbox2; ++j)
              tma_load_2d(a + kABytes + j * kPairBoxRows * 128, amap32, &full[stage], kb * kBK,
                          arow2 + j * kPairBoxRows);
          }
          // B: weight rows. At most 16 tokens, every expert has one tile and its weights are read
          // exactly once: they are loaded with an evict-first L2 hint, so that streaming them does
          // not push out of L2 what the forward reads again (x, h, y, the schedule, its code)
          auto load_w = [&](uint32_t dst, const CUtensorMap* map, int c1) {
            if constexpr (kSmall)
              tma_load_2d_hint(dst, map, &full[stage], kb * kBK, c1, w_policy);
            else
              tma_load_2d(dst, map, &full[stage], kb * kBK, c1);
          };
          if (up) {
            load_w(b, shared ? &maps.ws_up : &maps.w_up, wrow_up);
            load_w(b + kBN1 * 128, shared ? &maps.ws_gate : &maps.w_gate, wrow_up);
          } else {
            load_w(b, shared ? &maps.ws_down : &maps.w_down, wrow_dn);
          }
        }
        if (kb == claim_kb && !sh.static_quota && lane == 0) {
          if (tau + 1 < batch_end) {
            next_tau = tau + 1;
          } else {
            next_tau = atomicAdd(&meta->task_counter, sh.claim_batch);
            batch_end = next_tau + sh.claim_batch;
          }
        }
        if (kb == claim_kb + 1 && use_tab && lane == 0 && next_tau < total) {
          next_ent = __ldcg(ws.task_tab + next_tau);
          ent_tau = next_tau;
        }
        __syncwarp();
        ++nfill;
        if (++stage == kStages) { stage = 0; phase ^= 1; }
      }
      if (!ok) break;
    }
    wacc[kWaitProdLoop] = now() - t_loop;
  } else if (warp == 1) {
    // ===================================== MMA issuer ===================================
    // A task uses the next accumulator, or both when it also computes a merged tail tile; each
    // accumulator's barriers are phased by its own use count.
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(kBM, kUmmaN);
      uint32_t stage = 0, phase = 0, slot = 0, slot_phase = 0, next = 0, use0 = 0, use1 = 0;
      const int64_t t_loop = now();
      while (true) {
        int64_t t0 = now();
        const bool got = wait_bar(&task_full[slot], slot_phase, meta, s_abort, limit, kSiteMmaTask);
        wacc[kWaitMmaTask] += now() - t0;
        if (!got) break;
        const Task t = ring[slot];
        if (t.kind == kTaskStop) break;
        const uint32_t a0 = next, a1 = next ^ 1u;
        const bool two = kTail && (t.ntiles == 2);
        t0 = now();
        if (!wait_bar(&acc_empty[a0], ((a0 ? use1 : use0) & 1u) ^ 1u, meta, s_abort, limit, kSiteMmaAcc)) break;
        if (two && !wait_bar(&acc_empty[a1], ((a1 ? use1 : use0) & 1u) ^ 1u, meta, s_abort, limit, kSiteMmaAcc))
          break;
        wacc[kWaitMmaAcc] += now() - t0;
        tc_fence_after();
        const uint32_t d0 = tmem_base + a0 * kAccCols, d1 = tmem_base + a1 * kAccCols;
        bool ok = true;
        for (int kb = 0; kb < t.nk; ++kb) {
          t0 = now();
          if (!wait_bar(&full[stage], phase, meta, s_abort, limit, kSiteMmaFull)) { ok = false; break; }
          wacc[kWaitMmaFull] += now() - t0;
          tc_fence_after();
          const uint32_t a = smem_u32(smem + stage * kStageBytes);
          const uint32_t b = a + kBOff;
#pragma unroll
          for (int kk = 0; kk < kBK / kUK; ++kk)
            umma_bf16(d0, sdesc_kmajor_sw128(a + kk * 32), sdesc_kmajor_sw128(b + kk * 32), idesc,
                      (kb | kk) != 0);
          if (two) {
            // the tail's 32 rows sit in the slot after A; its other 96 MMA rows read the start of
            // B and land in accumulator rows that are never stored
#pragma unroll
            for (int kk = 0; kk < kBK / kUK; ++kk)
              umma_bf16(d1, sdesc_kmajor_sw128(a + kABytes + kk * 32), sdesc_kmajor_sw128(b + kk * 32), idesc,
                        (kb | kk) != 0);
          }
          mma_issued = true;
          umma_commit(&empty[stage]);
          if (++stage == kStages) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        umma_commit(&acc_full[a0]);
        if (a0) ++use1; else ++use0;
        if (two) {
          umma_commit(&acc_full[a1]);
          if (a1) ++use1; else ++use0;
        } else {
          next ^= 1u;
        }
        mbar_arrive(&task_empty[slot]);
        if (++slot == kTaskSlots) { slot = 0; slot_phase ^= 1; }
      }
      wacc[kWaitMmaLoop] = now() - t_loop;
    }
    __syncwarp();
  } else {
    // ===================================== epilogue =====================================
    // Each thread owns one tile row (its TMEM lane). Per chunk of 128 bytes per row: drain
    // TMEM to registers, convert, write the row into a 128-byte-swizzled staging buffer, and
    // let one thread issue the TMA store of the 128-row box.
    const int q = warp & 3;          // TMEM lane quarter this warp may read
    const int row = q * 32 + lane;   // tile row owned by this thread
    const bool leader = (warp == 2 && lane == 0);
    uint8_t* staging = smem + C::kStagingOff;
    // accumulator bookkeeping mirrors the MMA issuer: a task uses `next`, or both
    // accumulators when it carries a merged tail tile; barriers are phased per accumulator
    uint32_t slot = 0, slot_phase = 0, next = 0, use0 = 0, use1 = 0;
    // One thread waits for the next task and its accumulator and tells the other 127 through
    // the named barrier, so the four warps always take the same branch (a warp that left the
    // loop alone would strand the others at the next named barrier). The decision word is
    // double-buffered: it is rewritten only after every thread passed the next loop barrier.
    auto epilogue_next = [&](uint32_t it) -> bool {
      if (leader) {
        int go = 0;
        const int64_t t0 = now();
        const bool got = wait_bar(&task_full[slot], slot_phase, meta, s_abort, limit, kSiteEpiTask);
        const int64_t t1 = now();
        wacc[kWaitEpiTask] += t1 - t0;
        if (got && ring[slot].kind != kTaskStop) {
          const uint32_t a1 = next ^ 1u;
          go = wait_bar(&acc_full[next], (next ? use1 : use0) & 1u, meta, s_abort, limit, kSiteEpiAcc) ? 1 : 0;
          if (go && ring[slot].ntiles == 2)
            go = wait_bar(&acc_full[a1], (a1 ? use1 : use0) & 1u, meta, s_abort, limit, kSiteEpiAcc) ? 1 : 0;
          wacc[kWaitEpiAcc] += now() - t1;
        }
        s_epi_go[it & 1] = go;
      }
      named_bar_sync(1, 128);
      if (s_epi_go[it & 1] == 0) return false;
      tc_fence_after();
      return true;
    };
    // after a task: count the accumulators it used and move `next` past a single one
    auto accs_done = [&](int ntiles) {
      if (next) ++use1; else ++use0;
      if (ntiles == 2) {
        if (next) ++use0; else ++use1;
      } else {
        next ^= 1u;
      }
    };
    const int64_t t_loop = now();
    if constexpr (kSmall) {
      // at most 16 valid rows per tile: only the warp of TMEM lanes 0-31 has work, and the
      // valid rows are stored straight from registers (no staging, no TMA stores)
      for (uint32_t it = 0;; ++it) {
        if (!epilogue_next(it)) break;
        const Task t = ring[slot];
        const uint32_t tacc = tmem_base + next * kAccCols + (static_cast<uint32_t>(q * 32) << 16);
        const bool shared = (t.expert == sh.E);
        const bool has_rows = q * 32 < t.nrows;  // warp-uniform
        const bool valid = row < t.nrows;
        if (t.kind == kTaskUp) {
          const int Dt = shared ? sh.Ds : sh.D;
          uint16_t* hrow = ws.h + (size_t)(t.tile * kBM + row) * ws.ldh;
          if (has_rows) {
#pragma unroll 1
            for (int cc = 0; cc < kBN1 / 64; ++cc) {
              uint32_t pk[32];
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
              const int col = t.n0 + cc * 64;
              if (valid) {
#pragma unroll
                for (int v = 0; v < 8; ++v)
                  if (col + 8 * v + 8 <= Dt)
                    *reinterpret_cast<uint4*>(hrow + col + 8 * v) =
                        make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
              }
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&acc_empty[next]);
          // publish h: this tile's down tasks read it with TMA (async proxy) on other SMs
          fence_proxy_async_global();
          __threadfence();
          named_bar_sync(1, 128);
          if (leader) red_release_add_gpu(&ws.done1[t.tile], 1);
        } else {
          float w = 0.f;
          if (valid) {
            if (shared) {
              w = 1.f;
            } else if constexpr (kFused) {
              w = fs->slot_w[fs->row_slot[t.tile * kSmallRows + row]];
            } else {
              const int s = __ldcg(&ws.sorted_ids[t.row0 + row]);
              w = __ldcg(&ws.topk_w[s]);
            }
          }
          uint16_t* yrow = ws.y + (size_t)(t.tile * kBM + row) * sh.H;
          if (has_rows) {
#pragma unroll 1
            for (int cc = 0; cc < kBN2 / 64; ++cc) {
              uint32_t pk[32];
#pragma unroll
              for (int half = 0; half < 2; ++half) {
                uint32_t v[32];
                tmem_ld_32x32b_x32(tacc + cc * 64 + half * 32, v);
                tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < 16; ++j)
                  pk[half * 16 + j] = pack_bf16x2(w * __uint_as_float(v[2 * j]), w * __uint_as_float(v[2 * j + 1]));
              }
              const int col = t.n0 + cc * 64;
              if (valid) {
#pragma unroll
                for (int v = 0; v < 8; ++v)
                  if (col + 8 * v + 8 <= sh.H)
                    *reinterpret_cast<uint4*>(yrow + col + 8 * v) =
                        make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
              }
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&acc_empty[next]);
          if constexpr (kFused) {
            // count this task's rows per token; the row that completes a token's column block
            // has that token's block combined by one epilogue warp
            const int64_t tc0 = now();
            const int n = fused_down_done(fa, ws, sh, *fs, t, row, fs->comb_list, leader);
            const int64_t dt = now() - tc0;
            wacc[kCombineCount] += dt;
            if (n > 0) wacc[kCombineRun] += dt;
          }
        }
        if (lane == 0) mbar_arrive(&task_empty[slot]);
        if (ws.trace_cap > 0 && leader && t.id < ws.trace_cap)
          ws.trace[(size_t)t.id * 4 + 3] = (int64_t)globaltimer_ns();
        accs_done(1);
        if (++slot == kTaskSlots) { slot = 0; slot_phase ^= 1; }
      }
    } else {
    // write 8 x 16 bytes (one 128-byte row) into staging buffer `buf` with the 128B swizzle
    auto put_row = [&](uint8_t* buf, const uint32_t (&w)[32]) {
#pragma unroll
      for (int j = 0; j < 8; ++j)
        *reinterpret_cast<uint4*>(buf + row * 128 + ((j ^ (row & 7)) << 4)) =
            make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
    };
    uint32_t sb = 0;  // staging buffer in use (the tail shape has one, the general shape two)
    // One tile of the task: accumulator `a` holds its rows (lane = row); results go to rows
    // tile*128 .. of h (up) or y (down).
    auto process_tile = [&](const Task& t, int tile, int row0, int nrows, uint32_t a) {
      const uint32_t tacc = tmem_base + a * kAccCols + (static_cast<uint32_t>(q * 32) << 16);
      const bool shared = (t.expert == sh.E);
      if (t.kind == kTaskUp) {
        // h = SiLU(U) * G, two chunks of 64 bf16 columns
#pragma unroll 1
        for (int cc = 0; cc < kBN1 / 64; ++cc) {
          uint32_t pk[32];
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
              // SiLU(u) * g with a fast reciprocal (the result is rounded to bf16)
              pk[half * 16 + j] = pack_bf16x2(__fdividef(u0, 1.0f + __expf(-u0)) * g0,
                                              __fdividef(u1, 1.0f + __expf(-u1)) * g1);
            }
          }
          if (cc == kBN1 / 64 - 1) {  // every TMEM read of this accumulator is done: release it
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[a]);
          }
          uint8_t* buf = staging + sb * kStagingBytes;
          if (leader) bulk_wait_group_read<C::kNumStagingN - 1>();  // buffer sb is no longer read
          named_bar_sync(1, 128);
          put_row(buf, pk);
          fence_proxy_async_shared();
          named_bar_sync(1, 128);
          if (leader) {
            tma_store_2d(shared ? &maps.h_shared : &maps.h_routed, smem_u32(buf), t.n0 + cc * 64, tile * kBM);
            bulk_commit_group();
          }
          if constexpr (C::kNumStagingN > 1) sb ^= 1;
        }
        // publish h: the stores must be complete and visible to other SMs' TMA loads before
        // the tile's counter moves
        if (leader) {
          bulk_wait_group<0>();
          fence_proxy_async_global();
          __threadfence();
          red_release_add_gpu(&ws.done1[tile], 1);
        }
      } else {
        // y = w * (h W_down^T) rounded to bf16, four chunks of 64 columns
        float w = 0.f;
        if (row < nrows) {
          if (shared) {
            w = 1.f;
          } else {
            const int s = __ldcg(&ws.sorted_ids[row0 + row]);
            w = __ldcg(&ws.topk_w[s]);
          }
        }
#pragma unroll 1
        for (int cc = 0; cc < kBN2 / 64; ++cc) {
          uint32_t pk[32];
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            uint32_t v[32];
            tmem_ld_32x32b_x32(tacc + cc * 64 + half * 32, v);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 16; ++j)
              pk[half * 16 + j] = pack_bf16x2(w * __uint_as_float(v[2 * j]), w * __uint_as_float(v[2 * j + 1]));
          }
          if (cc == kBN2 / 64 - 1) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[a]);
          }
          uint8_t* buf = staging + sb * kStagingBytes;
          if (leader) bulk_wait_group_read<C::kNumStagingN - 1>();
          named_bar_sync(1, 128);
          put_row(buf, pk);
          fence_proxy_async_shared();
          named_bar_sync(1, 128);
          if (leader) {
            tma_store_2d(&maps.y, smem_u32(buf), t.n0 + cc * 64, tile * kBM);
            bulk_commit_group();
          }
          if constexpr (C::kNumStagingN > 1) sb ^= 1;
        }
      }
    };
    for (uint32_t it = 0;; ++it) {
      if (!epilogue_next(it)) break;
      const Task t = ring[slot];
      process_tile(t, t.tile, t.row0, t.nrows, next);
      if (kTail && t.ntiles == 2) process_tile(t, t.tile + 1, t.row0 + kBM, t.nrows2, next ^ 1u);
      if (lane == 0) mbar_arrive(&task_empty[slot]);
      if (ws.trace_cap > 0 && leader && t.id < ws.trace_cap)
        ws.trace[(size_t)t.id * 4 + 3] = (int64_t)globaltimer_ns();
      accs_done(kTail ? t.ntiles : 1);
      if (++slot == kTaskSlots) { slot = 0; slot_phase ^= 1; }
    }
    // the staging buffer must not be released while a store still reads it
    if (leader) bulk_wait_group<0>();
    }
    wacc[kWaitEpiLoop] = now() - t_loop;
    wacc[kFrontToEnd] = now() - t_front;
  }
  // wait accounting of this CTA: each role's recording thread adds its entries
  if (tracing && ws.waits != nullptr && ((warp == 0 && lane == 0) || threadIdx.x == 32 || (warp == 2 && lane == 0))) {
#pragma unroll
    for (int i = 0; i < kNumWaits; ++i)
      if (wacc[i]) atomicAdd(reinterpret_cast<unsigned long long*>(ws.waits + (size_t)blockIdx.x * kNumWaits + i),
                             (unsigned long long)wacc[i]);
  }

  // the next kernel may start its prologue once every CTA has finished its tasks (not earlier:
  // its waiting CTAs would share the SMs with the tensor-core pipeline)
  griddep_launch_dependents();
  // teardown: every TMA fill and tcgen05 op issued by this CTA must be complete before the
  // CTA releases TMEM and exits (this only waits after an abort)
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) drain_fills(full, kStages, nfill, meta, limit);
  if (threadIdx.x == 32) {
    if (mma_issued) {
      umma_commit(drain);
      wait_bar_drain(drain, 0, meta, limit);
    }
  }
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, 2 * kAccCols);
}

size_t gemm_smem_bytes(int shape) {
  // (the fused shape's layout is the small shape's plus its schedule)
  const int bytes = shape == kShapeSmallFused ? Cfg<kShapeSmallFused>::kBytes
                    : shape == kShapeSmall    ? Cfg<kShapeSmall>::kBytes
                    : shape == kShapeTail     ? Cfg<kShapeTail>::kBytes
                    : shape == kShapeTwo      ? Cfg<kShapeTwo>::kBytes
                                              : Cfg<kShapeGeneral>::kBytes;
  return (size_t)bytes + 1024;
}

cudaError_t launch_moe_gemm(const GemmMaps& maps, const Workspace& ws, const Shape& sh, int grid, int shape,
                            cudaStream_t stream) {
  const size_t smem = gemm_smem_bytes(shape);
  const FrontArgs fa{};
  if (shape == kShapeSmall)
    return launch_k(moe_gemm_kernel<kShapeSmall>, dim3(grid), dim3(kGemmThreads), smem, stream, maps, ws, sh, fa);
  if (shape == kShapeTail)
    return launch_k(moe_gemm_kernel<kShapeTail>, dim3(grid), dim3(kGemmThreads), smem, stream, maps, ws, sh, fa);
  if (shape == kShapeTwo)
    return launch_k(moe_gemm_kernel<kShapeTwo>, dim3(grid), dim3(kGemmThreads), smem, stream, maps, ws, sh, fa);
  return launch_k(moe_gemm_kernel<kShapeGeneral>, dim3(grid), dim3(kGemmThreads), smem, stream, maps, ws, sh, fa);
}

cudaError_t launch_moe_small_fused(const GemmMaps& maps, const Workspace& ws, const Shape& sh,
                                   const FrontArgs& fa, int grid, cudaStream_t stream) {
  // every CTA waits at the front's arrival for all the others: all must be resident at once
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kGemmThreads);
  cfg.dynamicSmemBytes = gemm_smem_bytes(kShapeSmallFused);
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, moe_gemm_kernel<kShapeSmallFused>, maps, ws, sh, fa);
}

int small_fused_blocks_per_sm() {
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, moe_gemm_kernel<kShapeSmallFused>, kGemmThreads,
                                                    gemm_smem_bytes(kShapeSmallFused)) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return n;
}

cudaError_t configure_gemm_kernel() {
  cudaError_t e = cudaFuncSetAttribute(moe_gemm_kernel<kShapeSmall>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)gemm_smem_bytes(kShapeSmall));
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(moe_gemm_kernel<kShapeSmallFused>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)gemm_smem_bytes(kShapeSmallFused));
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(moe_gemm_kernel<kShapeTail>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)gemm_smem_bytes(kShapeTail));
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(moe_gemm_kernel<kShapeTwo>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)gemm_smem_bytes(kShapeTwo));
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(moe_gemm_kernel<kShapeGeneral>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)gemm_smem_bytes(kShapeGeneral));
}

}  // namespace moe
