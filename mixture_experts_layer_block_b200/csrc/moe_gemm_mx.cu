// moe_gemm_mx.cu -- the persistent grouped expert GEMMs with MXFP8 experts.
//
// Same tasks and scheduler as the bf16 kernel (Weave blog, sections 2.1-2.2 and 5.1: one
// persistent CTA per SM claiming (tile, n) tasks from an atomic counter; units of a group's up
// tasks followed, `lag` units later, by its down tasks), on operands quantised to MXFP8
// (mx.cuh): x rows (gather kernel), every expert weight (once, by the caller) and h, which the
// up tasks' epilogue quantises as they write it.
//
//  - up task (tile, n): A = the tile's 128 x rows, B = 128 rows of W_up^e on 128 rows of
//    W_gate^e; per 128-K stage four block-scaled MMAs (kind::mxf8f6f4, M=128, N=256, K=32)
//    with their scales copied from shared memory into TMEM (tcgen05.cp) just before them. The
//    epilogue computes h = SiLU(U) * G in fp32, quantises it per 32 columns and writes 128
//    bytes of codes per row (TMA store) and 4 scale codes per row (one 32-bit store).
//  - down task (tile, n): after the tile's up tasks, A = its quantised h rows, B = 256 rows of
//    W_down^e; the epilogue writes y = w * (h W_down^T) in bf16, as in the bf16 kernel, and the
//    same combine kernel sums each token's rows.
//
// TMEM: one 256-column fp32 accumulator (columns 0-255) and, per stage, 16 columns of scales
// (A's atom in 4 columns, B's two atoms in 8). The scales leave no room for a second
// accumulator, so the MMAs of a task wait for the epilogue of the task before it; the producer
// keeps filling the 4-stage ring meanwhile.
//
// Warp roles and bounded waits as in the bf16 kernel: warp 0 producer, warp 1 MMA issuer (one
// lane), warps 2-5 epilogue.
#include "front.cuh"
#include "launch.h"
#include "mx.cuh"

namespace moe {

namespace {

// kSmall (batches of at most 16 tokens: every tile holds at most 16 rows): the A slot holds one
// 32-row box, so the same shared memory holds a fifth stage (more weight bytes in flight per SM).
template <bool kSmall>
struct MxCfg {
  static constexpr int kStages = kSmall ? 5 : 4;
  static constexpr int kABytes = (kSmall ? kPairBoxRows : kBM) * kMxBK;  // 4 KB or 16 KB
  static constexpr int kBBytes = kUmmaN * kMxBK;       // 32 KB
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kSfStageBytes = 2048;           // SFA atom at 0, SFB atoms at 512 and 1024
  static constexpr int kSfOff = kStages * kStageBytes;
  static constexpr int kStagingOff = kSfOff + kStages * kSfStageBytes;
  static constexpr int kBarOff = kStagingOff + kStagingBytes;
  // barriers: full[S], empty[S], acc_full, acc_empty, task_full[R], task_empty[R], drain
  static constexpr int kNumBars = 2 * kStages + 2 + 2 * kTaskSlots + 1;
  static constexpr int kRingOff = kBarOff + ((kNumBars * 8 + 63) & ~63);
  static constexpr int kMiscOff = kRingOff + kTaskSlots * (int)sizeof(Task);
  // the fused small-batch forward keeps every slot's tile row (row_of_slot) in shared memory
  // the fused small-batch forward keeps its schedule (FusedSched) in shared memory
  static constexpr int kFusedOff = kMiscOff + 64;
  static constexpr int kBytes = kFusedOff + (kSmall ? (int)((sizeof(FusedSched) + 15) & ~15) : 0);
  static constexpr uint32_t kSfCol0 = kAccCols;        // first TMEM column of the scale slots
  static constexpr uint32_t kSfColsPerStage = 16;
  static_assert(kStageBytes % 1024 == 0 && kSfOff % 1024 == 0, "1024-byte aligned operand tiles");
  static_assert(kBytes + 1024 <= 227 * 1024, "shared memory budget");
  static_assert(kMiscOff % 8 == 0, "8-byte words in the misc area");
  static_assert(kSfCol0 + kStages * kSfColsPerStage <= 2 * kAccCols, "TMEM budget");
};

__device__ __forceinline__ int n1_of(int expert, const Shape& sh) {
  return ceil_div(expert == sh.E ? sh.Ds : sh.D, kBN1);
}

// kFused: the whole forward of at most 16 tokens in one launch (front.cuh): router slices, each
// CTA's own schedule once every slice is in, the MXFP8 row gather, then the tasks; the down task
// that brings in a token's last row of a 256-column block combines that token's block.
template <bool kFused, bool kSmall>
__global__ void __launch_bounds__(kGemmThreads, 1)
    moe_gemm_mx_kernel(const __grid_constant__ MxMaps maps, Workspace ws, MxBuffers mx, Shape sh, FrontArgs fa) {
  static_assert(!kFused || kSmall, "the fused forward is for batches of at most 16 tokens");
  using C = MxCfg<kSmall>;
  constexpr int kStages = C::kStages;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // aligned by pointer arithmetic on the shared array (not through an integer), so that the
  // compiler keeps every access through `smem` in the shared address space
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  uint64_t* full = bars;
  uint64_t* empty = full + kStages;
  uint64_t* acc_full = empty + kStages;
  uint64_t* acc_empty = acc_full + 1;
  uint64_t* task_full = acc_empty + 1;
  uint64_t* task_empty = task_full + kTaskSlots;
  uint64_t* drain = task_empty + kTaskSlots;
  Task* ring = reinterpret_cast<Task*>(smem + C::kRingOff);
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + C::kMiscOff);
  volatile int* s_abort = reinterpret_cast<volatile int*>(smem + C::kMiscOff + 4);
  volatile int* s_epi_go = reinterpret_cast<volatile int*>(smem + C::kMiscOff + 8);  // [2]
  // (misc + 16 .. + 39: the epilogue leader's wait sums)
  volatile int* s_front = reinterpret_cast<volatile int*>(smem + C::kMiscOff + 40);  // fused: ok
  FusedSched* fs = reinterpret_cast<FusedSched*>(smem + C::kFusedOff);  // fused: the schedule

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  DeviceMeta* meta = ws.meta;
  const int64_t limit = sh.timeout_ns;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 4);  // one arrival per epilogue warp
    for (int i = 0; i < kTaskSlots; ++i) {
      mbar_init(&task_full[i], 1);
      mbar_init(&task_empty[i], 5);  // MMA lane + 4 epilogue warps
    }
    mbar_init(drain, 1);
    *s_abort = 0;
    fence_mbar_init();
    tma_prefetch_desc(&maps.xs);
    tma_prefetch_desc(&maps.h);
    tma_prefetch_desc(&maps.y);
    tma_prefetch_desc(&maps.w_up);
    tma_prefetch_desc(&maps.w_gate);
    tma_prefetch_desc(&maps.w_down);
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
  uint32_t nfill = 0;
  bool mma_issued = false;

  // wait accounting while tracing, as in the bf16 kernel (globaltimer ns; each role's recording
  // thread keeps its own sums and adds them to its CTA's row at the end of its loop)
  const bool tracing = ws.trace_cap > 0;
  auto now = [&]() -> int64_t { return tracing ? (int64_t)globaltimer_ns() : 0; };
  auto add_wait = [&](int kind, int64_t v) {
    if (tracing && ws.waits != nullptr && v != 0)
      atomicAdd(reinterpret_cast<unsigned long long*>(ws.waits + (size_t)blockIdx.x * kNumWaits + kind),
                (unsigned long long)v);
  };

  bool run_tasks = true;
  if constexpr (kFused) {
    // the front, by all 192 threads, as in the bf16 kernel; the operand ring is free until the
    // first TMA fill
    const int64_t t_front = now();
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
    if (run_tasks) front_gather_mx(fa, ws, mx, sh, fs->slot_row, fs->n_routed);
    // the ring's generic-proxy writes come before the TMA fills that reuse it
    fence_proxy_async_shared();
    __syncthreads();
    if (threadIdx.x == 0) {
      add_wait(kFrontRouter, t_r - t_front);
      add_wait(kFrontSchedule, t_s - t_r);
      add_wait(kFrontGather, now() - t_s);
      add_wait(kFrontLast, tracing && blockIdx.x == 0 ? 1 : 0);
      if (tracing) {
        add_wait(kSchedArrive, t_arrived - t_r);
        add_wait(kSchedLogits, ts[0] - t_arrived);
        add_wait(kSchedGating, ts[1] - ts[0]);
        add_wait(kSchedTables, ts[2] - ts[1]);
        add_wait(kSchedWrites, ts[3] - ts[2]);
        add_wait(kSchedPublish, t_s - ts[3]);
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
    const int H = sh.H;
    int u_cur = 0;
    uint32_t stage = 0, phase = 0, slot = 0, slot_phase = 0;
    // claims as in the bf16 kernel: the next id while the current task's last ring-depth of
    // stages is issued, its task-table entry one stage later
    const bool weights_once = sh.T <= kSmallRows;
    const uint64_t w_policy = weights_once ? policy_evict_first() : 0;
    int next_tau = 0, batch_end = 0;
    if (lane == 0) {
      next_tau = atomicAdd(&meta->task_counter, sh.claim_batch);
      batch_end = next_tau + sh.claim_batch;
    }
    const bool use_tab = ws.task_tab != nullptr && !kFused;
    int4 next_ent = make_int4(0, 0, 0, 0);
    int ent_tau = -1;
    const int64_t t_loop = now();
    int64_t w_empty = 0, w_dep = 0, w_ring = 0, w_claim = 0;
    while (true) {
      const int64_t t_top = now();
      int tau = 0;
      if (lane == 0) tau = aborted(meta, s_abort) ? total : next_tau;
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
        t.nk = t.kind == kTaskUp ? H / kMxBK : (t.expert == sh.E ? sh.Ds : sh.D) / kMxBK;
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
        const int nt = ent.w >> 20;
        const int Dt = (t.expert == sh.E) ? sh.Ds : sh.D;
        if (t.kind == kTaskUp) {
          t.n0 = nt * kBN1;
          t.nk = H / kMxBK;
        } else {
          t.n0 = nt * kBN2;
          t.nk = Dt / kMxBK;
        }
      } else {
        u_cur = find_unit(ws.unit_start, U, tau, u_cur);
        const TaskPos pos = decode_task(ws, sh, u_cur, tau, Mg, Mgr);
        t.kind = pos.kind;
        t.tile = pos.tile;
        t.expert = __ldcg(&ws.tile_expert[t.tile]);
        t.row0 = __ldcg(&ws.tile_row0[t.tile]);
        t.nrows = __ldcg(&ws.tile_nrows[t.tile]);
        const int Dt = (t.expert == sh.E) ? sh.Ds : sh.D;
        if (t.kind == kTaskUp) {
          t.n0 = pos.nt * kBN1;
          t.nk = H / kMxBK;
        } else {
          t.n0 = pos.nt * kBN2;
          t.nk = Dt / kMxBK;
        }
      }
      bool ok = true;
      if (lane == 0) {
        const int64_t t0 = now();
        ok = wait_bar(&task_empty[slot], slot_phase ^ 1, meta, s_abort, limit, kSiteProducerTask);
        if (ok) {
          ring[slot] = t;
          mbar_arrive(&task_full[slot]);
        }
        w_ring += now() - t0;
        w_claim += t0 - t_top;
      }
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      if (!ok || t.kind == kTaskStop) break;
      if (++slot == kTaskSlots) { slot = 0; slot_phase ^= 1; }
      const int claim_kb = t.nk > kStages ? t.nk - kStages : 0;
      if (ws.trace_cap > 0 && lane == 0 && tau < ws.trace_cap) {
        ws.trace[(size_t)tau * 4 + 0] = blockIdx.x;
        ws.trace[(size_t)tau * 4 + 1] = tau;
        ws.trace[(size_t)tau * 4 + 2] = (int64_t)globaltimer_ns();
      }
      const bool shared = (t.expert == sh.E);
      const bool up = (t.kind == kTaskUp);
      if (kFused && up) {
        // the tile's quantised x rows (or, for the shared tile, every token's) are gathered
        if (lane == 0) {
          const int64_t t0 = now();
          ok = wait_count(&ws.gather_done[t.tile], t.nrows, meta, s_abort, limit);
          if (ok) fence_proxy_async_global();
          w_dep += now() - t0;
        }
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        if (!ok) break;
      }
      if (!up) {
        if (lane == 0) {
          const int64_t t0 = now();
          ok = wait_count(&ws.done1[t.tile], n1_of(t.expert, sh) + sh.dep_extra, meta, s_abort, limit);
          if (ok) fence_proxy_async_global();  // h (codes and scales) is read by the async proxy
          w_dep += now() - t0;
        }
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        if (!ok) break;
      }
      const int Dt = shared ? sh.Ds : sh.D;
      const int wrow_up = shared ? t.n0 : t.expert * sh.D + t.n0;
      const int wrow_dn = shared ? t.n0 : t.expert * H + t.n0;
      const CUtensorMap* amap = up ? (shared ? &maps.x_tile : &maps.xs) : &maps.h;
      const CUtensorMap* amap32 = up ? (shared ? &maps.x_tile32 : &maps.xs32) : &maps.h32;
      const int arow = (up && shared) ? t.row0 : t.tile * kBM;
      // A: one 128-row box, or (tiles of at most 96 rows) only the 32-row boxes that hold the
      // tile's rows; the rest of the A slot keeps stale rows, whose results land in accumulator
      // rows that are never stored
      // (small: every tile has at most 16 rows, one 32-row box in the 4 KB A slot; the MMA's other
      // 96 rows read the start of B, and their results are never stored either)
      const int nbox = kSmall ? 1 : ((t.nrows <= 3 * kPairBoxRows) ? ceil_div(t.nrows, kPairBoxRows) : 0);
      const uint32_t a_bytes = nbox ? (uint32_t)(nbox * kPairBoxRows * kMxBK) : (uint32_t)C::kABytes;
      // scale atoms: A's row block (128-aligned rows), B's row blocks
      const uint8_t* sfa = up ? (shared ? mx.sf_xq + mx_atom_offset(t.row0 >> 7, 0, H)
                                        : mx.sf_xs + mx_atom_offset(t.tile, 0, H))
                              : mx.sf_h + mx_atom_offset(t.tile, 0, ws.ldh);
      const uint8_t* sfb0;
      const uint8_t* sfb1;
      uint32_t sfb_bytes = 2 * kSfAtomBytes;
      if (up) {
        sfb0 = (shared ? mx.sfs_up : mx.sf_up) + mx_atom_offset(wrow_up >> 7, 0, H);
        sfb1 = (shared ? mx.sfs_gate : mx.sf_gate) + mx_atom_offset(wrow_up >> 7, 0, H);
      } else {
        const int rows_dn = shared ? H : sh.E * H;  // W_down's rows (multiples of 128)
        sfb0 = (shared ? mx.sfs_down : mx.sf_down) + mx_atom_offset(wrow_dn >> 7, 0, Dt);
        sfb1 = sfb0 + (size_t)(Dt / kMxBK) * kSfAtomBytes;
        // the last 128 rows of a 256-row box past the end of W_down: TMA fills zeros, and the
        // scales of those rows (results in columns that are never stored) are not fetched
        if (wrow_dn + kBM >= rows_dn) sfb_bytes = kSfAtomBytes;
      }
      const uint32_t stage_tx = a_bytes + (uint32_t)C::kBBytes + kSfAtomBytes + sfb_bytes;
      for (int kb = 0; kb < t.nk; ++kb) {
        if (lane == 0) {
          const int64_t t0 = now();
          ok = wait_bar(&empty[stage], phase ^ 1, meta, s_abort, limit, kSiteProducerEmpty);
          w_empty += now() - t0;
        }
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        if (!ok) break;
        if (lane == 0) {
          const uint32_t a = smem_u32(smem + stage * C::kStageBytes);
          const uint32_t b = a + C::kABytes;
          const uint32_t sf = smem_u32(smem + C::kSfOff + stage * C::kSfStageBytes);
          mbar_arrive_expect_tx(&full[stage], stage_tx);
          if (nbox == 0) {
            tma_load_2d(a, amap, &full[stage], kb * kMxBK, arow);
          } else {
            for (int j = 0; j < nbox; ++j)
              tma_load_2d(a + j * kPairBoxRows * kMxBK, amap32, &full[stage], kb * kMxBK, arow + j * kPairBoxRows);
          }
          // weights read exactly once (at most 16 tokens: one tile per expert) carry an
          // evict-first L2 hint, as in the bf16 kernel
          auto load_w = [&](uint32_t dst, const CUtensorMap* map, int c1) {
            if (weights_once)
              tma_load_2d_hint(dst, map, &full[stage], kb * kMxBK, c1, w_policy);
            else
              tma_load_2d(dst, map, &full[stage], kb * kMxBK, c1);
          };
          if (up) {
            load_w(b, shared ? &maps.ws_up : &maps.w_up, wrow_up);
            load_w(b + kBN1 * kMxBK, shared ? &maps.ws_gate : &maps.w_gate, wrow_up);
          } else {
            load_w(b, shared ? &maps.ws_down : &maps.w_down, wrow_dn);
          }
          bulk_load(sf, sfa + (size_t)kb * kSfAtomBytes, kSfAtomBytes, &full[stage]);
          bulk_load(sf + kSfAtomBytes, sfb0 + (size_t)kb * kSfAtomBytes, kSfAtomBytes, &full[stage]);
          if (sfb_bytes > kSfAtomBytes)
            bulk_load(sf + 2 * kSfAtomBytes, sfb1 + (size_t)kb * kSfAtomBytes, kSfAtomBytes, &full[stage]);
        }
        if (kb == claim_kb && lane == 0) {
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
    if (lane == 0) {
      add_wait(kWaitProdLoop, now() - t_loop);
      add_wait(kWaitProdEmpty, w_empty);
      add_wait(kWaitProdDep, w_dep);
      add_wait(kWaitProdRing, w_ring);
      add_wait(kWaitProdClaim, w_claim);
    }
  } else if (warp == 1) {
    // ===================================== MMA issuer ===================================
    if (lane == 0) {
      uint32_t stage = 0, phase = 0, slot = 0, slot_phase = 0, use = 0;
      const int64_t t_loop = now();
      int64_t w_task = 0, w_acc = 0, w_full = 0;
      while (true) {
        int64_t t0 = now();
        if (!wait_bar(&task_full[slot], slot_phase, meta, s_abort, limit, kSiteMmaTask)) break;
        w_task += now() - t0;
        const Task t = ring[slot];
        if (t.kind == kTaskStop) break;
        t0 = now();
        if (!wait_bar(acc_empty, (use & 1u) ^ 1u, meta, s_abort, limit, kSiteMmaAcc)) break;
        w_acc += now() - t0;
        tc_fence_after();
        bool ok = true;
        for (int kb = 0; kb < t.nk; ++kb) {
          t0 = now();
          if (!wait_bar(&full[stage], phase, meta, s_abort, limit, kSiteMmaFull)) { ok = false; break; }
          w_full += now() - t0;
          tc_fence_after();
          const uint32_t a = smem_u32(smem + stage * C::kStageBytes);
          const uint32_t b = a + C::kABytes;
          const uint32_t sf = smem_u32(smem + C::kSfOff + stage * C::kSfStageBytes);
          const uint32_t tsf = tmem_base + C::kSfCol0 + stage * C::kSfColsPerStage;
          // scales into TMEM: A's atom in columns 0-3, B's rows 0-127 in 4-7 and 128-255 in 8-11
          // (tcgen05 operations of one thread run in issue order: the MMAs below see them)
          tmem_copy_sf_atom(tsf, sdesc_sf_atom(sf));
          tmem_copy_sf_atom(tsf + 4, sdesc_sf_atom(sf + kSfAtomBytes));
          tmem_copy_sf_atom(tsf + 8, sdesc_sf_atom(sf + 2 * kSfAtomBytes));
#pragma unroll
          for (int kk = 0; kk < kMxBK / kMxUK; ++kk)
            umma_mxf8(tmem_base, sdesc_kmajor_sw128(a + kk * 32), sdesc_kmajor_sw128(b + kk * 32),
                      idesc_mxf8_e4m3(kBM, kUmmaN, kk), tsf, tsf + 4, (kb | kk) != 0);
          mma_issued = true;
          umma_commit(&empty[stage]);
          if (++stage == kStages) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        umma_commit(acc_full);
        ++use;
        mbar_arrive(&task_empty[slot]);
        if (++slot == kTaskSlots) { slot = 0; slot_phase ^= 1; }
      }
      add_wait(kWaitMmaLoop, now() - t_loop);
      add_wait(kWaitMmaTask, w_task);
      add_wait(kWaitMmaAcc, w_acc);
      add_wait(kWaitMmaFull, w_full);
    }
    __syncwarp();
  } else {
    // ===================================== epilogue =====================================
    const int q = warp & 3;          // TMEM lane quarter this warp may read
    const int row = q * 32 + lane;   // tile row owned by this thread
    const bool leader = (warp == 2 && lane == 0);
    uint8_t* staging = smem + C::kStagingOff;
    uint32_t slot = 0, slot_phase = 0, use = 0;
    // the leader's wait sums live in shared memory (no registers held across the loop)
    int64_t* s_ewait = reinterpret_cast<int64_t*>(smem + C::kMiscOff + 16);  // [3]
    if (leader) s_ewait[0] = s_ewait[1] = 0, s_ewait[2] = now();
    const uint32_t tacc = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    // the leader waits for the next task and the accumulator and tells the others (the four
    // warps always take the same branch); the decision word is double-buffered
    auto epilogue_next = [&](uint32_t it) -> bool {
      if (leader) {
        int go = 0;
        const int64_t t0 = now();
        if (wait_bar(&task_full[slot], slot_phase, meta, s_abort, limit, kSiteEpiTask) && ring[slot].kind != kTaskStop) {
          const int64_t t1 = now();
          s_ewait[0] += t1 - t0;
          go = wait_bar(acc_full, use & 1u, meta, s_abort, limit, kSiteEpiAcc) ? 1 : 0;
          s_ewait[1] += now() - t1;
        }
        s_epi_go[it & 1] = go;
      }
      named_bar_sync(1, 128);
      if (s_epi_go[it & 1] == 0) return false;
      tc_fence_after();
      return true;
    };
    // one 128-byte row per thread into the staging buffer, 128-byte swizzled
    auto put_row = [&](const uint32_t (&w)[32]) {
#pragma unroll
      for (int j = 0; j < 8; ++j)
        *reinterpret_cast<uint4*>(staging + row * 128 + ((j ^ (row & 7)) << 4)) =
            make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
    };
    auto release_acc = [&]() {
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty);
    };
    // stage one 128-row x 128-byte box and store it with TMA (one staging buffer: wait until
    // the previous store has read it)
    auto store_box = [&](const CUtensorMap* map, const uint32_t (&w)[32], int c0, int r0) {
      if (leader) bulk_wait_group_read<0>();
      named_bar_sync(1, 128);
      put_row(w);
      fence_proxy_async_shared();
      named_bar_sync(1, 128);
      if (leader) {
        tma_store_2d(map, smem_u32(staging), c0, r0);
        bulk_commit_group();
      }
    };
    for (uint32_t it = 0;; ++it) {
      if (!epilogue_next(it)) break;
      const Task t = ring[slot];
      const bool shared = (t.expert == sh.E);
      // a partial tile (decode batches, tails): warps without valid rows skip the accumulator,
      // and the valid rows go straight from registers to global memory (no staging, no TMA
      // store of 128 rows)
      const bool direct = t.nrows < kBM;
      const bool has_rows = q * 32 < t.nrows;  // warp-uniform
      const bool valid = row < t.nrows;
      if (t.kind == kTaskUp) {
        // h = SiLU(U) * G for 128 columns, quantised per 32 columns
        uint32_t codes[32];
        uint32_t scales = 0;
        if (has_rows || !direct) {
#pragma unroll
          for (int j = 0; j < kBN1 / kMxBlock; ++j) {
            uint32_t u[32], g[32];
            tmem_ld_32x32b_x32(tacc + j * 32, u);
            tmem_ld_32x32b_x32(tacc + kBN1 + j * 32, g);
            tmem_ld_wait();
            if (j == kBN1 / kMxBlock - 1) release_acc();
            float hv[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const float uu = __uint_as_float(u[i]);
              hv[i] = __fdividef(uu, 1.0f + __expf(-uu)) * __uint_as_float(g[i]);
            }
            uint32_t w8[8];
            scales |= mx_quantize_block(hv, w8) << (8 * j);
#pragma unroll
            for (int i = 0; i < 8; ++i) codes[8 * j + i] = w8[i];
          }
          // this row's four scales: one 32-bit word of the tile's atom for these 128 columns
          *reinterpret_cast<uint32_t*>(mx.sf_h + mx_atom_offset(t.tile, t.n0 / kMxBK, ws.ldh) + lane * 16 + q * 4) =
              scales;
        } else {
          release_acc();
        }
        if (!direct) {
          store_box(&maps.h, codes, t.n0, t.tile * kBM);
        } else if (valid) {
          uint4* hrow = reinterpret_cast<uint4*>(mx.h + (size_t)(t.tile * kBM + row) * ws.ldh + t.n0);
#pragma unroll
          for (int v = 0; v < 8; ++v) hrow[v] = make_uint4(codes[4 * v], codes[4 * v + 1], codes[4 * v + 2], codes[4 * v + 3]);
        }
        // publish h: codes (TMA store or plain stores) and scales (plain stores) must be visible
        // to the async proxy of other SMs before the tile's counter moves
        fence_proxy_async_global();
        __threadfence();
        named_bar_sync(1, 128);
        if (leader) {
          bulk_wait_group<0>();
          fence_proxy_async_global();
          __threadfence();
          red_release_add_gpu(&ws.done1[t.tile], 1);
        }
      } else {
        float w = 0.f;
        if (row < t.nrows) {
          if (shared) {
            w = 1.f;
          } else if constexpr (kFused) {
            w = fs->slot_w[fs->row_slot[t.tile * kSmallRows + row]];
          } else {
            const int s = __ldcg(&ws.sorted_ids[t.row0 + row]);
            w = __ldcg(&ws.topk_w[s]);
          }
        }
        if (has_rows || !direct) {
          uint16_t* yrow = ws.y + (size_t)(t.tile * kBM + row) * sh.H;
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
            if (cc == kBN2 / 64 - 1) release_acc();
            const int col = t.n0 + cc * 64;
            if (!direct) {
              store_box(&maps.y, pk, col, t.tile * kBM);
            } else if (valid && col + 64 <= sh.H) {  // H is a multiple of 128: whole chunks
#pragma unroll
              for (int v = 0; v < 8; ++v)
                *reinterpret_cast<uint4*>(yrow + col + 8 * v) =
                    make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
            }
          }
        } else {
          release_acc();
        }
        if constexpr (kFused) {
          // count this task's rows per token (every fused tile is partial: each thread stored its
          // own row straight from registers); the row that completes a token's column block has
          // that token's block combined by one epilogue warp
          const int64_t tc0 = now();
          const int n = fused_down_done(fa, ws, sh, *fs, t, row, fs->comb_list, leader);
          const int64_t dt = now() - tc0;
          if (leader) {
            add_wait(kCombineCount, dt);
            if (n > 0) add_wait(kCombineRun, dt);
          }
        }
      }
      if (lane == 0) mbar_arrive(&task_empty[slot]);
      if (ws.trace_cap > 0 && leader && t.id < ws.trace_cap)
        ws.trace[(size_t)t.id * 4 + 3] = (int64_t)globaltimer_ns();
      ++use;
      if (++slot == kTaskSlots) { slot = 0; slot_phase ^= 1; }
    }
    if (leader) {
      bulk_wait_group<0>();
      add_wait(kWaitEpiLoop, now() - s_ewait[2]);
      add_wait(kWaitEpiTask, s_ewait[0]);
      add_wait(kWaitEpiAcc, s_ewait[1]);
    }
  }

  griddep_launch_dependents();
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

}  // namespace

// dynamic shared memory of the general and of the small-batch configuration
static size_t mx_smem_bytes(bool small) { return (size_t)(small ? MxCfg<true>::kBytes : MxCfg<false>::kBytes) + 1024; }

size_t gemm_mx_smem_bytes() { return mx_smem_bytes(false); }

cudaError_t configure_gemm_mx_kernel() {
  cudaError_t e = cudaFuncSetAttribute(moe_gemm_mx_kernel<false, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)mx_smem_bytes(false));
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(moe_gemm_mx_kernel<false, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)mx_smem_bytes(true));
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(moe_gemm_mx_kernel<true, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)mx_smem_bytes(true));
}

cudaError_t launch_moe_gemm_mx(const MxMaps& maps, const Workspace& ws, const MxBuffers& mx, const Shape& sh,
                               int grid, cudaStream_t stream) {
  if (sh.T <= kSmallRows)
    return launch_k(moe_gemm_mx_kernel<false, true>, dim3(grid), dim3(kGemmThreads), mx_smem_bytes(true),
                    stream, maps, ws, mx, sh, FrontArgs{});
  return launch_k(moe_gemm_mx_kernel<false, false>, dim3(grid), dim3(kGemmThreads), mx_smem_bytes(false),
                  stream, maps, ws, mx, sh, FrontArgs{});
}

cudaError_t launch_moe_mx_small_fused(const MxMaps& maps, const Workspace& ws, const MxBuffers& mx, const Shape& sh,
                                      const FrontArgs& fa, int grid, cudaStream_t stream) {
  // every CTA waits at the front's arrival for all the others: all must be resident at once
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kGemmThreads);
  cfg.dynamicSmemBytes = mx_smem_bytes(true);
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, moe_gemm_mx_kernel<true, true>, maps, ws, mx, sh, fa);
}

int mx_small_fused_blocks_per_sm() {
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, moe_gemm_mx_kernel<true, true>, kGemmThreads,
                                                    mx_smem_bytes(true)) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return n;
}

}  // namespace moe
