// common.cuh -- definitions shared by the kernels and the host API: tile sizes, workspace
// layout, device status codes, task encoding and bounded waits.
#pragma once

#include <cstdint>

#include "ptx.cuh"

namespace moe {

// ---- tile geometry of the expert GEMMs ---------------------------------------------------
constexpr int kBM = 128;        // rows (token slots) per m-tile = UMMA M
constexpr int kBK = 64;         // K elements per pipeline stage = one 128-byte swizzle row
constexpr int kUK = 16;         // K per tcgen05.mma (bf16)
constexpr int kBN1 = 128;       // D columns per up/gate task; MMA N = 2*kBN1 (up | gate)
constexpr int kBN2 = 256;       // H columns per down task; MMA N = kBN2
constexpr int kUmmaN = 256;     // N of every expert-GEMM MMA
constexpr int kStages = 4;      // smem pipeline depth
constexpr int kABytes = kBM * kBK * 2;       // 16 KB
constexpr int kBBytes = kUmmaN * kBK * 2;    // 32 KB
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kTaskSlots = 4;   // depth of the producer -> MMA/epilogue task ring
#ifndef MOE_GROUP_TILES
#define MOE_GROUP_TILES 2
#endif
// Consecutive m-tiles of one expert are scheduled as a group of up to this many: the group's
// up (and down) tasks are numbered n-major across its tiles, so the tasks that read the same
// weight rows are claimed back to back and stream those rows together through L2.
constexpr int kGroupTiles = MOE_GROUP_TILES;
constexpr int kStagingBytes = 128 * 128;  // one epilogue staging buffer: 128 rows x 128 B
constexpr int kNumStaging = 2;            // double-buffered epilogue -> TMA store staging
constexpr int kAccCols = 256;   // TMEM columns per accumulator buffer (2 buffers)
constexpr int kGemmThreads = 192;  // warp 0 producer, warp 1 MMA, warps 2-5 epilogue
constexpr int kMaxTopK = 32;       // largest top_k
constexpr int kSmallRows = 16;     // A-tile rows of the expert GEMMs' small-tile shape (T <= 16)
constexpr int kPairBoxRows = 32;   // rows per A load / result store box of the SM-pair shape

// ---- router GEMM -------------------------------------------------------------------------
constexpr int kRouterStages = 6;
constexpr int kRouterMaxN = 256;  // one N tile covers up to 256 experts: x is read once per split
constexpr int kMaxRouterSplits = 4;

// ---- gating / align ------------------------------------------------------------------------
constexpr int kGateThreads = 512;
constexpr int kMaxChunks = 32;     // token chunks of the histogram (chunk = ceil(T/32) >= 64)
constexpr int kMinChunkTokens = 64;
constexpr int kGateTokensPerCta = 16;  // gating CTAs: 16 warps x 1 token
constexpr int kMaxExperts = 1024;
constexpr int kFusedMaxExperts = 256;  // the fused small-batch forward's gating holds 8 logits per lane

// ---- device status word --------------------------------------------------------------------
constexpr int kStatusTimeout = 1 << 30;     // | where-code
enum WaitSite : int {
  kSiteProducerEmpty = 1,
  kSiteProducerTask = 2,
  kSiteDependency = 3,
  kSiteMmaTask = 4,
  kSiteMmaAcc = 5,
  kSiteMmaFull = 6,
  kSiteEpiTask = 7,
  kSiteEpiAcc = 8,
  kSiteDrain = 9,
  kSiteRouter = 10,
  kSiteFront = 11,  // fused small-batch forward: not every CTA arrived in time
};

// Counters and scalars that live in device memory (one int each).
struct DeviceMeta {
  int task_counter;   // atomic work queue head
  int abort;          // set by any wait that gave up; every CTA then drains and exits
  int status;         // first device error code (0 = ok)
  int hist_done;      // CTAs of the histogram kernel that finished (last one scans)
  int num_tiles;      // m-tiles of this forward (routed + shared)
  int total_tasks;    // tasks of this forward
  int num_units;      // scheduling units (tiles + lag)
  int P;              // num_post_padded
  int trace_count;    // trace records written
  int num_routed_tiles;  // m-tiles of routed experts (shared-expert tiles follow them)
  int num_groups;     // scheduling groups of up to kGroupTiles tiles of one expert
  int num_routed_groups;  // groups of routed experts (shared-expert groups follow them)
  int pad[4];
};

// The fused small-batch forward's arrival counter, on a 128-byte line of its own: each CTA adds
// 1 once its router slice is in, so forward n is complete when it reaches n times the grid size
// (it is never reset).
struct FrontSync {
  int front_done;
  int pad0[31];
};

// Per-CTA wait accounting of the expert-GEMM kernel while tracing (ns of %globaltimer, summed
// over the CTA's tasks): what each role's issuing thread waited for, and how long its loop ran.
enum WaitKind : int {
  kWaitProdEmpty = 0,  // producer: a free operand stage
  kWaitProdDep = 1,    // producer: a down task's up tasks (or, fused, a tile's gathered rows)
  kWaitProdRing = 2,   // producer: a free task-ring entry
  kWaitProdClaim = 3,  // producer: claiming and decoding the next task
  kWaitMmaFull = 4,    // MMA lane: a filled operand stage
  kWaitMmaAcc = 5,     // MMA lane: a free accumulator (the epilogue of the task before)
  kWaitMmaTask = 6,    // MMA lane: the next task
  kWaitEpiTask = 7,    // epilogue: the next task
  kWaitEpiAcc = 8,     // epilogue: a finished accumulator
  kWaitProdLoop = 9,   // producer loop duration
  kWaitMmaLoop = 10,   // MMA loop duration
  kWaitEpiLoop = 11,   // epilogue loop duration
  // the fused small-batch forward's front, per CTA (0 for the other kernels)
  kFrontRouter = 12,   // this CTA's router slice
  kFrontSchedule = 13, // the arrival and this CTA's schedule
  kFrontGather = 14,   // this CTA's share of the row gather
  kFrontLast = 15,     // 1 for CTA 0 (which also writes the align outputs)
  kFrontToEnd = 16,    // from the front's start to the end of the epilogue loop
  // the steps of this CTA's schedule
  kSchedArrive = 17,   // waiting for every CTA's router slice
  kSchedLogits = 18,   // loading every token's logits
  kSchedGating = 19,   // top-k and softmax of every token
  kSchedTables = 20,   // counts, offsets, tiles and units (one warp)
  kSchedWrites = 21,   // the CTA's schedule in shared memory (slot rows and weights, tiles)
  kSchedPublish = 22,  // CTA 0: the align and tile outputs for the host (0 elsewhere)
  // the fused forward's combine (epilogue leader, summed over this CTA's down tasks)
  kCombineCount = 23,  // the per-token counters and combines after each down task
  kCombineRun = 24,    // the same, for the down tasks that combined at least one token
  kNumWaits = 25,
};

// Task kinds in the ring.
constexpr int kTaskUp = 0;     // up/gate GEMM + SwiGLU -> h
constexpr int kTaskDown = 1;   // down GEMM + weighted combine -> out
constexpr int kTaskStop = -1;

struct Task {
  int32_t kind;
  int32_t tile;    // m-tile index
  int32_t expert;  // routed expert, or E for the shared expert
  int32_t row0;    // first sorted row (routed) or first token (shared)
  int32_t nrows;   // valid rows in the tile (1..128)
  int32_t n0;      // first output column (D for up tasks, H for down tasks)
  int32_t nk;      // K stages
  int32_t id;      // global task id
  int32_t ntiles;  // 1, or 2: the task also computes the next tile (rows row0 + 128 ...), a
                   // tail of nrows2 <= kTailRows rows, from the same B stages
  int32_t nrows2;  // valid rows of that second tile
};
constexpr int kTailRows = 32;  // a tile this short rides along with its expert's previous tile

// Pointers into the workspace handed to the kernels.
struct Workspace {
  DeviceMeta* meta;
  float* logits;         // [T][E]
  float* logit_parts;    // [splits*T][E]    K-split partial router logits
  int32_t* topk_ids;     // [T][k]
  float* topk_w;         // [T][k]
  int32_t* chunk_hist;   // [kMaxChunks][E]
  int32_t* chunk_base;   // [kMaxChunks][E]  exclusive prefix over chunks, per expert
  int32_t* expert_off;   // [E+1]            padded segment offsets
  int32_t* expert_kept;  // [E]              kept slots per expert
  int32_t* sorted_ids;   // [sorted_len]
  int32_t* expert_ids;   // [blocks_len]
  int32_t* tile_expert;  // [max_tiles]
  int32_t* tile_row0;    // [max_tiles]
  int32_t* tile_nrows;   // [max_tiles]
  int32_t* group_tile0;  // [max_tiles]      first m-tile of each scheduling group
  int32_t* group_ntiles; // [max_tiles]      m-tiles in each group (1..kGroupTiles)
  int32_t* group_tasks;  // [max_tiles]      task sets per n-tile: group_ntiles, or 1 when the
                         //                  group's last tile is a tail merged into the tasks
                         //                  of the tile before it
  int32_t* expert_group0;  // [E + 2]        first scheduling group of each expert; [E] the
                           //                shared expert's first group, [E + 1] all groups
  int32_t* unit_start;   // [max_groups + max_lag + 1]
  int32_t* done1;        // [max_tiles]      finished up/gate tasks per tile
  int32_t* expert_tile0; // [E]              first m-tile of each expert
  int32_t* row_of_slot;  // [S]              tile row (tile*tile_m + r) of each kept slot, -1 if dropped
  uint16_t* xs;          // [routed rows][H] bf16 x rows gathered in tile order
  uint16_t* h;           // [rows][ldh] bf16 SwiGLU activations, tile order
  uint16_t* y;           // [rows][H] bf16 router-weighted expert outputs per tile row
  int64_t* trace;        // [trace_cap][4]
  int32_t trace_cap;
  int32_t ldh;           // row stride of h in elements (max(D, D_shared))
  FrontSync* front;      // fused small-batch forward's counters
  int4* task_tab;        // [task_cap] every task of the forward, decoded (task_entry), or null
  int32_t task_cap;
  int64_t* waits;        // [grid][kNumWaits] per-CTA wait accounting while tracing, or null
  int32_t* tok_done;     // [16][ceil(H / kBN2)] fused small-batch forward: a token's rows finished
                         //   per 256-column block (the down task that finishes the last one
                         //   combines that token's block)
  int32_t* gather_done;  // [max_tiles]       fused small-batch forward: x rows gathered per tile
};

// What the fused small-batch forward (router, gating, align, gather, expert GEMMs and combine
// in one launch) reads and writes besides the workspace.
struct FrontArgs {
  const uint16_t* x;         // [T][H] bf16
  const uint16_t* w_router;  // [E][H] bf16
  const float* bias;         // [E] fp32, or null
  void* out;                 // [T][H] fp32, or bf16 when out_bf16
  int32_t out_bf16;
  int32_t epoch;             // this forward's number (the arrival counter's target / grid size)
};

// Shapes and knobs of one forward, passed by value.
constexpr int kMaxClaimBatch = 64;  // largest moe_config.claim_batch

struct Shape {
  int32_t T, H, D, Ds, E, k, block_m;
  int32_t capacity;      // C, 0 = dropless
  int32_t chunk_tokens;  // tokens per histogram chunk
  int32_t num_chunks;
  int32_t sorted_len, blocks_len;
  int32_t lag;           // scheduling lag in units between a tile's up and down tasks
  int32_t dep_extra;     // testing hook: extra up completions a down task waits for
  int32_t tile_m;        // rows per m-tile of the expert GEMMs: 128, or 256 on SM pairs
  int32_t merge_tail;    // 1: a group of a full tile and a tail of <= kTailRows rows runs as one
                         //    task set (the one-SM tail shape); 2: every group of two tiles does
                         //    (the two-tile shape); 0: never
  int32_t static_quota;  // 1: each CTA works through a fixed share of the experts (ablation)
  int32_t claim_batch;   // consecutive task ids one claim on the counter takes (>= 1)
  int64_t timeout_ns;
};

__host__ __device__ inline int ceil_div(int a, int b) { return (a + b - 1) / b; }

// ---- error raising and bounded waits -------------------------------------------------------
__device__ __forceinline__ void raise_error(DeviceMeta* meta, volatile int* s_abort, int code) {
  atomicCAS(&meta->status, 0, code);
  atomicExch(&meta->abort, 1);
  if (s_abort) *s_abort = 1;
}

__device__ __forceinline__ bool aborted(const DeviceMeta* meta, const volatile int* s_abort) {
  return (s_abort && *s_abort) || *reinterpret_cast<const volatile int*>(&meta->abort);
}

// Wait until the phase of parity `parity` of `bar` completed. Gives up (returns false) when
// the kernel is aborting or after `limit_ns`, in which case it raises a timeout error.
static __device__ __noinline__ bool wait_bar(uint64_t* bar, uint32_t parity, DeviceMeta* meta,
                                      volatile int* s_abort, int64_t limit_ns, int site) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  uint32_t n = 0;
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((++n & 7u) == 0) {
      if (aborted(meta, s_abort)) return false;
      if (static_cast<int64_t>(globaltimer_ns() - t0) > limit_ns) {
        raise_error(meta, s_abort, kStatusTimeout | site);
        return false;
      }
    }
  }
}

// Teardown wait: ignores the abort flag (the work it waits for is already in flight and will
// finish), bounded by `limit_ns`.
static __device__ __noinline__ bool wait_bar_drain(uint64_t* bar, uint32_t parity, DeviceMeta* meta,
                                            int64_t limit_ns) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (static_cast<int64_t>(globaltimer_ns() - t0) > limit_ns) {
      atomicCAS(&meta->status, 0, kStatusTimeout | kSiteDrain);
      atomicExch(&meta->abort, 1);
      return false;
    }
  }
  return true;
}

// Bounded wait until *p >= need (acquire). Raises a timeout error on expiry.
static __device__ __noinline__ bool wait_count(const int* p, int need, DeviceMeta* meta,
                                        volatile int* s_abort, int64_t limit_ns) {
  if (ld_acquire_gpu(p) >= need) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    __nanosleep(128);
    if (ld_acquire_gpu(p) >= need) return true;
    if (aborted(meta, s_abort)) return false;
    if (static_cast<int64_t>(globaltimer_ns() - t0) > limit_ns) {
      raise_error(meta, s_abort, kStatusTimeout | kSiteDependency);
      return false;
    }
  }
}

// The scheduling unit u of task `tau` (unit_start[u] <= tau < unit_start[u + 1]), searched
// forward from unit `u` (each CTA claims ever larger task ids). Executed by a whole warp: each
// round compares the next 32 unit starts at once, so a claim costs one dependent load round
// however many units it skips.
__device__ __forceinline__ int find_unit(const int32_t* unit_start, int num_units, int tau, int u) {
  const int lane = threadIdx.x & 31;
  while (true) {
    const int idx = u + 1 + lane;
    const int v = idx <= num_units ? __ldcg(unit_start + idx) : 0x7fffffff;
    const int adv = __popc(__ballot_sync(0xffffffffu, v <= tau));  // unit starts never decrease
    u += adv;
    if (adv < 32) return u;
  }
}

// A task, decoded once by the schedule so that a claim costs one load: {tile, expert, first
// row, bits}, bits = nrows | nrows2 << 9 | (ntiles == 2) << 18 | kind << 19 | n-tile << 20.
__host__ __device__ inline int4 task_entry(int kind, int tile, int nt, int ntiles, int expert, int row0, int nrows,
                                           int nrows2) {
  return make_int4(tile, expert, row0,
                   nrows | (nrows2 << 9) | ((ntiles == 2 ? 1 : 0) << 18) | (kind << 19) | (nt << 20));
}

// Write the entries of unit u's tasks (ids unit_start[u] ...): the up tasks of group u, then the
// down tasks of group u - lag, in the order decode_task gives them.
__device__ inline void write_unit_tasks(const Workspace& ws, const Shape& sh, int u, int us, int Mg, int Mgr) {
  const int gl = u - sh.lag;
  int tau = us;
  for (int part = 0; part < 2; ++part) {
    const int g = part == 0 ? u : gl;
    if (g < 0 || g >= Mg) continue;
    const int gt = __ldcg(&ws.group_tasks[g]), t0 = __ldcg(&ws.group_tile0[g]), nt_ = __ldcg(&ws.group_ntiles[g]);
    const int ntiles = gt == 1 ? nt_ : 1;
    int ex[2], r0[2], nr[2];
    for (int i = 0; i < gt; ++i) {
      ex[i] = __ldcg(&ws.tile_expert[t0 + i]);
      r0[i] = __ldcg(&ws.tile_row0[t0 + i]);
      nr[i] = __ldcg(&ws.tile_nrows[t0 + i]);
    }
    const int nr2 = ntiles == 2 ? __ldcg(&ws.tile_nrows[t0 + 1]) : 0;
    const int n = part == 0 ? ceil_div(g < Mgr ? sh.D : sh.Ds, kBN1) : ceil_div(sh.H, kBN2);
    for (int o = 0; o < n * gt; ++o) {
      const int i = o % gt;
      ws.task_tab[tau++] = task_entry(part == 0 ? kTaskUp : kTaskDown, t0 + i, o / gt, ntiles, ex[i], r0[i], nr[i],
                                      ntiles == 2 ? nr2 : 0);
    }
  }
}

// Position of task `tau` of unit `u`: unit u holds the up tasks of group u, then the down tasks
// of group u - lag; inside a group the tasks run n-major over its tiles.
struct TaskPos {
  int kind, tile, nt, ntiles;
};
__device__ __forceinline__ TaskPos decode_task(const Workspace& ws, const Shape& sh, int u, int tau, int Mg,
                                               int Mgr) {
  // every load depends only on u: they go out together (one round trip per claim)
  const int gl = u - sh.lag;
  const bool has_up = u < Mg, has_dn = gl >= 0 && gl < Mg;
  const int us = __ldcg(&ws.unit_start[u]);
  const int gu = has_up ? __ldcg(&ws.group_tasks[u]) : 1;
  const int tu = has_up ? __ldcg(&ws.group_tile0[u]) : 0;
  const int nu = has_up ? __ldcg(&ws.group_ntiles[u]) : 1;
  const int gd = has_dn ? __ldcg(&ws.group_tasks[gl]) : 1;
  const int td = has_dn ? __ldcg(&ws.group_tile0[gl]) : 0;
  const int nd = has_dn ? __ldcg(&ws.group_ntiles[gl]) : 1;
  const int off = tau - us;
  const int n1u = has_up ? ceil_div(u < Mgr ? sh.D : sh.Ds, kBN1) * gu : 0;
  // a merged group (one task set for two tiles) computes both tiles in each task
  if (off < n1u) return TaskPos{kTaskUp, tu + off % gu, off / gu, gu == 1 ? nu : 1};
  const int o = off - n1u;
  return TaskPos{kTaskDown, td + o % gd, o / gd, gd == 1 ? nd : 1};
}

// The tasks of one "slot" (a routed expert, or E for the shared expert) in task-id order, for
// the static per-expert quota (ablation). The slot's groups are [g0, g1); unit u holds the up
// tasks of group u, then the down tasks of group u - lag.
struct SlotIter {
  int g0, g1, u, part, k;
  __device__ void start(const Workspace& ws, int slot) {
    g0 = __ldcg(&ws.expert_group0[slot]);
    g1 = __ldcg(&ws.expert_group0[slot + 1]);
    u = g0;
    part = 0;
    k = 0;
  }
  // The slot's next task id (and its unit in `unit`), or -1 when the slot has no more.
  __device__ int next(const Workspace& ws, const Shape& sh, int Mg, int Mgr, int& unit) {
    while (u < g1 + sh.lag) {
      const int us = __ldcg(&ws.unit_start[u]);
      const int n1u = (u < Mg) ? ceil_div(u < Mgr ? sh.D : sh.Ds, kBN1) * __ldcg(&ws.group_tasks[u]) : 0;
      if (part == 0) {
        if (u >= g0 && u < g1 && k < n1u) {
          unit = u;
          return us + k++;
        }
        part = 1;
        k = 0;
      }
      const int gl = u - sh.lag;
      if (gl >= g0 && gl < g1) {
        const int nd = __ldcg(&ws.unit_start[u + 1]) - us - n1u;
        if (k < nd) {
          unit = u;
          return us + n1u + k++;
        }
      }
      ++u;
      part = 0;
      k = 0;
    }
    return -1;
  }
};

// Wait for the last TMA fill of every stage of a ring that was filled `nfill` times in
// round-robin order (fill f of stage s completes phase f of its `full` barrier).
__device__ __forceinline__ void drain_fills(uint64_t* full, int nstages, uint32_t nfill,
                                            DeviceMeta* meta, int64_t limit_ns) {
  for (int s = 0; s < nstages; ++s) {
    if (nfill <= static_cast<uint32_t>(s)) break;
    const uint32_t fills = (nfill - 1u - s) / nstages + 1u;
    wait_bar_drain(&full[s], (fills - 1u) & 1u, meta, limit_ns);
  }
}

// ---- rows of bf16 values summed in fp32 (the combine) -----------------------------------------
// acc[i] += the i-th of 8 bf16 values packed in v (widened exactly).
__device__ __forceinline__ void add_bf16x8(float (&acc)[8], const uint4 v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    acc[2 * i] += __uint_as_float(w[i] << 16);
    acc[2 * i + 1] += __uint_as_float(w[i] & 0xffff0000u);
  }
}

// Stores 8 consecutive sums at element `off` of `out`: fp32, or bf16 rounded to nearest even.
template <bool kBf16>
__device__ __forceinline__ void store8(void* out, size_t off, const float (&a)[8]) {
  if constexpr (kBf16) {
    *reinterpret_cast<uint4*>(static_cast<uint16_t*>(out) + off) =
        make_uint4(pack_bf16x2(a[0], a[1]), pack_bf16x2(a[2], a[3]), pack_bf16x2(a[4], a[5]),
                   pack_bf16x2(a[6], a[7]));
  } else {
    float4* o = reinterpret_cast<float4*>(static_cast<float*>(out) + off);
    o[0] = make_float4(a[0], a[1], a[2], a[3]);
    o[1] = make_float4(a[4], a[5], a[6], a[7]);
  }
}

}  // namespace moe
