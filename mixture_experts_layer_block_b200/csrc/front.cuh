// front.cuh -- device code of the fused small-batch forward (at most 16 tokens, one launch):
// the front (router slices, the grid-wide arrival, every CTA's own gating, align and task
// schedule, the row gather) and the combine that the task completing a column block runs. Used
// by the bf16 and the MXFP8 expert-GEMM kernels.
#pragma once

#include "common.cuh"
#include "mx.cuh"
#include "ptx.cuh"
#include "route.cuh"

namespace moe {

namespace {

__device__ __forceinline__ void bf16x8_to_f32(const uint4 v, float (&f)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}

// Router projection (Mixture-of-Kittens blog, "Overlapping compute and communication in MoE")
// for this CTA's experts e = blockIdx.x + j * gridDim.x, two at a time: logits[t][e] =
// sum_h x[t][h] W_router[e][h] (+ bias[e]) in fp32. Each thread takes 8-wide chunks of H for
// all T <= 16 tokens; the partial sums are added over the warp, then over the warps in warp
// order. red: shared scratch of [warps][2][16] floats.
__device__ void front_router(const FrontArgs& fa, const Workspace& ws, const Shape& sh, float* red) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
  const int H = sh.H, E = sh.E, T = sh.T, nchunk = H / 8;
  for (int e0 = blockIdx.x; e0 < E; e0 += 2 * gridDim.x) {
    const int e1 = e0 + gridDim.x;
    const bool two = e1 < E;
    float a0[kSmallRows], a1[kSmallRows];
#pragma unroll
    for (int t = 0; t < kSmallRows; ++t) a0[t] = a1[t] = 0.f;
    const uint4* w0p = reinterpret_cast<const uint4*>(fa.w_router + (size_t)e0 * H);
    const uint4* w1p = reinterpret_cast<const uint4*>(fa.w_router + (size_t)(two ? e1 : e0) * H);
    for (int c = tid; c < nchunk; c += blockDim.x) {
      // every load of the chunk first (rows past T re-read row T-1; their sums are never used),
      // so that they are all in flight together
      uint4 xr[kSmallRows];
#pragma unroll
      for (int t = 0; t < kSmallRows; ++t)
        xr[t] = __ldg(reinterpret_cast<const uint4*>(fa.x + (size_t)min(t, T - 1) * H) + c);
      const uint4 wr0 = __ldg(w0p + c), wr1 = __ldg(w1p + c);
      float w0[8], w1[8];
      bf16x8_to_f32(wr0, w0);
      bf16x8_to_f32(wr1, w1);
#pragma unroll
      for (int t = 0; t < kSmallRows; ++t) {
        float xv[8];
        bf16x8_to_f32(xr[t], xv);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          a0[t] = fmaf(w0[i], xv[i], a0[t]);
          a1[t] = fmaf(w1[i], xv[i], a1[t]);
        }
      }
    }
    // transpose-reduce the 32 partial sums over the warp (31 shuffles): at each level a lane keeps
    // the half of its values selected by its lane bit and adds its partner's copy of that half;
    // lane l ends with the warp's total of value l (values 0-15: expert e0, 16-31: expert e1)
    float v[2 * kSmallRows];
#pragma unroll
    for (int t = 0; t < kSmallRows; ++t) {
      v[t] = a0[t];
      v[kSmallRows + t] = a1[t];
    }
#pragma unroll
    for (int sft = 16; sft >= 1; sft >>= 1) {
      const bool upper = (lane & sft) != 0;
#pragma unroll
      for (int i = 0; i < sft; ++i) {
        const float send = upper ? v[i] : v[i + sft];
        const float keep = upper ? v[i + sft] : v[i];
        v[i] = keep + __shfl_xor_sync(0xffffffffu, send, sft);
      }
    }
    red[warp * 2 * kSmallRows + lane] = v[0];
    __syncthreads();
    if (tid < 2 * T) {
      const int which = tid >= T ? 1 : 0, t = tid - which * T;
      if (!which || two) {
        const int e = which ? e1 : e0;
        float v = 0.f;
        for (int w = 0; w < nw; ++w) v += red[(w * 2 + which) * kSmallRows + t];
        if (fa.bias) v += fa.bias[e];
        ws.logits[(size_t)t * E + e] = v;
      }
    }
    __syncthreads();
  }
}

// Exclusive prefix of v over the lanes of warp 0 (lane order); *total = the sum of all lanes.
__device__ __forceinline__ int warp_exclusive(int v, int lane, int& total) {
  int incl = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += y;
  }
  total = __shfl_sync(0xffffffffu, incl, 31);
  return incl - v;
}

// First task id of unit u when every group is one m-tile (Mg groups, the first Mr routed): the up
// tasks of the groups before u (ceil(D/128) each for a routed group, ceil(Ds/128) for the
// shared one) plus the down tasks (ceil(H/256) each) of the groups before u - lag -- the
// exclusive scan of the unit sizes, in closed form.
__device__ __forceinline__ int unit_start_of(int u, int Mr, int Mg, const Shape& sh) {
  const int n1r = ceil_div(sh.D, kBN1), n1s = ceil_div(sh.Ds, kBN1), n2 = ceil_div(sh.H, kBN2);
  const int ups = min(u, Mg);
  const int downs = max(0, min(u - sh.lag, Mg));
  return n1r * min(ups, Mr) + n1s * max(0, ups - Mr) + n2 * downs;
}

// The schedule of a fused forward, kept by every CTA in shared memory beside the operand ring:
// the tiles (one per hit expert, in expert order, then the shared expert's), each slot's tile row
// and router weight, and each routed tile row's slot.
struct FusedSched {
  int n_tiles, n_routed, n_units, n_tasks;
  int slot_row[kSmallRows * kMaxTopK];  // tile row of slot s = t*k + j, -1 if dropped
  float slot_w[kSmallRows * kMaxTopK];  // its router weight
  int tile_exp[kFusedMaxExperts + 1];   // expert of tile g (E: the shared expert)
  int tile_row0[kFusedMaxExperts + 1];  // its first sorted row (0 for the shared tile)
  int tile_nrows[kFusedMaxExperts + 1];
  int16_t row_slot[kFusedMaxExperts * kSmallRows];  // slot of row r of routed tile g, at g*16 + r
  int tok_need[kSmallRows];             // rows of token t in y: its kept slots (+1 shared)
  int comb_list[1 + kSmallRows];        // a down task's completed tokens (count, tokens)
};

// CTA 0, before it arrives: this forward's counters start from zero. No CTA reads them before
// every CTA has arrived, and the launch before this one has completed (griddepcontrol.wait).
__device__ void front_reset(const Workspace& ws, const Shape& sh) {
  const int mt_max = min(sh.E, sh.T * sh.k) + 1;
  for (int i = threadIdx.x; i < mt_max; i += blockDim.x) {
    ws.gather_done[i] = 0;
    ws.done1[i] = 0;
  }
  for (int i = threadIdx.x; i < sh.T * ceil_div(sh.H, kBN2); i += blockDim.x) ws.tok_done[i] = 0;
  if (threadIdx.x == 0) {
    ws.meta->task_counter = 0;
    ws.meta->abort = 0;
    ws.meta->trace_count = 0;
  }
}

// Thread 0: this CTA's router slice (and CTA 0's resets) are in; wait (bounded) until every CTA's
// are. The counter only grows: forward `epoch` is complete when it reaches gridDim.x * epoch.
__device__ bool front_arrive(const Workspace& ws, const FrontArgs& fa, DeviceMeta* meta, int64_t limit_ns) {
  __threadfence();
  int* cnt = &ws.front->front_done;
  atomicAdd(cnt, 1);
  const unsigned target = (unsigned)gridDim.x * (unsigned)fa.epoch;
  auto done = [&](int v) { return (int)((unsigned)v - target) >= 0; };
  if (done(ld_acquire_gpu(cnt))) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    __nanosleep(64);
    if (done(ld_relaxed_gpu(cnt)) && done(ld_acquire_gpu(cnt))) return true;
    if (static_cast<int64_t>(globaltimer_ns() - t0) > limit_ns) {
      raise_error(meta, nullptr, kStatusTimeout | kSiteFront);
      return false;
    }
  }
}

// Run by every CTA once every router slice is in (all threads). For a batch of at most 16 tokens
// every expert receives at most 16 slots, so each hit expert has one m-tile and one scheduling
// group, and the whole schedule fits one warp's scans:
//  - gating (Weave blog section 1.1: top-k, ties to the lower expert index, softmax
//    renormalised over the selection);
//  - the align (vLLM PR #53280 summary, implementation breakdown): per-expert counts, the
//    capacity cut, padded segment offsets, each kept slot's rank (stable: ascending slot order);
//  - the tile and task schedule of the expert GEMMs: one tile per hit expert, units with the
//    dependency lag, as the align scans lay them out for a larger batch.
// The result goes to `fs`. With `write_outputs` (CTA 0) the CTA also writes the layer's outputs
// that nothing in this launch reads: top-k ids and weights, sorted_ids with its padding,
// expert_ids, row_of_slot, the tile and group tables, the unit starts and the counts (the tests
// compare them with the oracle). sm: shared scratch (ints) in the operand ring.
__device__ void front_schedule(const FrontArgs& fa, const Workspace& ws, const Shape& sh, int* sm,
                               FusedSched* fs, bool write_outputs, int64_t* ts) {
  // ts (thread 0, tracing): the end times of the steps, for the wait accounting
  const bool tracing = ws.trace_cap > 0;
  auto stamp = [&](int i) {
    if (tracing && threadIdx.x == 0) ts[i] = (int64_t)globaltimer_ns();
  };
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5, nthr = blockDim.x;
  const int E = sh.E, T = sh.T, k = sh.k, S = T * k;
  int* ids_s = sm;           // [S]
  int* cnt = ids_s + S;      // [E]
  unsigned* tmask = reinterpret_cast<unsigned*>(cnt + E);  // [E] tokens (bits) that chose e
  int* off = reinterpret_cast<int*>(tmask + E);            // [E + 1]
  int* kept = off + E + 1;   // [E]
  int* tile0 = kept + E;     // [E]
  int* s_mt = tile0 + E;     // [2]  m-tiles, and routed m-tiles, of this forward
  for (int e = tid; e < E; e += nthr) {
    cnt[e] = 0;
    tmask[e] = 0;
  }
  // gating: warp w takes tokens w, w + nw, w + 2 nw (T <= 16 <= 3 * 6); the logits of all its
  // tokens are loaded at once (one round trip), then their top-k interleaved
  constexpr int kTokPerWarp = 3;
  float v[kTokPerWarp][8];
#pragma unroll
  for (int i = 0; i < kTokPerWarp; ++i) {
    const int t = min(warp + i * nw, T - 1);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int e = lane + 32 * j;
      const float x = __ldcg(ws.logits + (size_t)t * E + min(e, E - 1));
      v[i][j] = e < E ? x : -INFINITY;
    }
  }
  __syncthreads();
  stamp(0);
  {
    int id[kTokPerWarp];
    float wt[kTokPerWarp];
    warp_topk_softmax_n<8, kTokPerWarp>(v, E, k, lane, id, wt);
#pragma unroll
    for (int i = 0; i < kTokPerWarp; ++i) {
      const int t = warp + i * nw;
      if (t < T && lane < k) {
        if (write_outputs) {
          ws.topk_ids[t * k + lane] = id[i];
          ws.topk_w[t * k + lane] = wt[i];
        }
        ids_s[t * k + lane] = id[i];
        fs->slot_w[t * k + lane] = wt[i];
        atomicAdd(&cnt[id[i]], 1);
        atomicOr(&tmask[id[i]], 1u << t);
      }
    }
  }
  __syncthreads();
  stamp(1);
  if (warp == 0) {
    // the two scans over the experts; lane l owns experts [8l, 8l + 8) (E <= 256), so lane
    // order is expert order
    const int e0 = lane * 8;
    const int bm = sh.block_m;
    const bool pow2 = (bm & (bm - 1)) == 0;
    auto padded = [&](int n) { return pow2 ? (n + bm - 1) & ~(bm - 1) : ceil_div(n, bm) * bm; };
    int kp[8], pad = 0, hit = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int e = e0 + j;
      const int n = e < E ? cnt[e] : 0;
      kp[j] = (sh.capacity > 0) ? min(n, sh.capacity) : n;
      pad += padded(kp[j]);
      hit += kp[j] > 0 ? 1 : 0;
    }
    int P, Mr;
    int o = warp_exclusive(pad, lane, P);
    int ti = warp_exclusive(hit, lane, Mr);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int e = e0 + j;
      if (e < E) {
        off[e] = o;
        kept[e] = kp[j];
        tile0[e] = ti;
        o += padded(kp[j]);
        ti += kp[j] > 0 ? 1 : 0;
      }
    }
    if (lane == 0) {
      off[E] = P;
      s_mt[0] = Mr + (sh.Ds > 0 ? 1 : 0);  // the shared expert: one tile of all T tokens
      s_mt[1] = Mr;
    }
  }
  __syncthreads();
  stamp(2);
  // the schedule of this CTA: tiles, slot rows and weights, tile rows' slots
  const int P = off[E], Mt = s_mt[0], Mr = s_mt[1], Mg = Mt, U = Mt > 0 ? Mt + sh.lag : 0;
  for (int e = tid; e < E; e += nthr) {
    const int kp = kept[e];
    if (kp > 0) {
      const int t0 = tile0[e];
      fs->tile_exp[t0] = e;
      fs->tile_row0[t0] = off[e];
      fs->tile_nrows[t0] = kp;
    }
  }
  // slot s = t*k + j: its rank in its expert is the number of earlier tokens that chose it
  for (int s = tid; s < S; s += nthr) {
    const int t = s / k, e = ids_s[s];
    const int r = __popc(tmask[e] & ((1u << t) - 1u));
    const bool keep = sh.capacity == 0 || r < sh.capacity;
    fs->slot_row[s] = keep ? tile0[e] * sh.tile_m + r : -1;
    if (keep) fs->row_slot[tile0[e] * kSmallRows + r] = (int16_t)s;
  }
  if (tid == 0) {
    if (sh.Ds > 0) {
      fs->tile_exp[Mr] = E;
      fs->tile_row0[Mr] = 0;
      fs->tile_nrows[Mr] = T;
    }
    fs->n_tiles = Mt;
    fs->n_routed = Mr;
    fs->n_units = U;
    fs->n_tasks = unit_start_of(U, Mr, Mg, sh);
    fs->comb_list[0] = 0;
  }
  // token t's rows in y: its kept slots, and its shared-expert row
  for (int t = tid; t < T; t += nthr) {
    int need = sh.Ds > 0 ? 1 : 0;
    for (int j = 0; j < k; ++j) {
      const int e = ids_s[t * k + j];
      need += (sh.capacity == 0 || __popc(tmask[e] & ((1u << t) - 1u)) < sh.capacity) ? 1 : 0;
    }
    fs->tok_need[t] = need;
    // a token without a row in y (every slot dropped, no shared expert): its output is zero,
    // written here, since no down task completes it
    if (need == 0 && write_outputs) {
      for (int c = 0; c < sh.H; c += 8) {
        const float z[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        if (fa.out_bf16) store8<true>(fa.out, (size_t)t * sh.H + c, z);
        else store8<false>(fa.out, (size_t)t * sh.H + c, z);
      }
    }
  }
  stamp(3);
  if (!write_outputs) return;
  // CTA 0: the outputs that the tests and the debug calls read after the launch
  const int bm = sh.block_m;
  for (int e = tid; e < E; e += nthr) {
    const int o = off[e], kp = kept[e], t0 = tile0[e], end = off[e + 1];
    ws.expert_off[e] = o;
    ws.expert_kept[e] = kp;
    ws.expert_tile0[e] = t0;
    ws.expert_group0[e] = t0;  // one tile per group
    if (kp > 0) {
      ws.tile_expert[t0] = e;
      ws.tile_row0[t0] = o;
      ws.tile_nrows[t0] = kp;
      ws.group_tile0[t0] = t0;
      ws.group_ntiles[t0] = 1;
      ws.group_tasks[t0] = 1;
    }
    for (int i = o + kp; i < end; ++i) ws.sorted_ids[i] = S;  // the segment's padding
    for (int b = o / bm; b < end / bm; ++b) ws.expert_ids[b] = e;
  }
  for (int s = tid; s < S; s += nthr) {
    const int t = s / k, e = ids_s[s];
    const int r = __popc(tmask[e] & ((1u << t) - 1u));
    const bool keep = sh.capacity == 0 || r < sh.capacity;
    if (keep) ws.sorted_ids[off[e] + r] = s;
    ws.row_of_slot[s] = keep ? tile0[e] * sh.tile_m + r : -1;
  }
  for (int i = P + tid; i < sh.sorted_len; i += nthr) ws.sorted_ids[i] = S;
  for (int b = P / bm + tid; b < sh.blocks_len; b += nthr) ws.expert_ids[b] = -1;
  for (int u = tid; u <= U; u += nthr) ws.unit_start[u] = unit_start_of(u, Mr, Mg, sh);
  if (tid == 0) {
    ws.expert_off[E] = P;
    if (sh.Ds > 0) {
      ws.tile_expert[Mr] = E;
      ws.tile_row0[Mr] = 0;
      ws.tile_nrows[Mr] = T;
      ws.group_tile0[Mr] = Mr;
      ws.group_ntiles[Mr] = 1;
      ws.group_tasks[Mr] = 1;
    }
    ws.expert_group0[E] = Mr;
    ws.expert_group0[E + 1] = Mg;
    DeviceMeta* m = ws.meta;
    m->P = P;
    m->num_tiles = Mt;
    m->num_routed_tiles = Mr;
    m->num_groups = Mg;
    m->num_routed_groups = Mr;
    m->num_units = U;
    m->total_tasks = unit_start_of(U, Mr, Mg, sh);
  }
}

// Task `tau` of a fused forward, from the CTA's schedule: unit u (the last unit whose first id
// is at most tau; empty units share their successor's first id) holds the up tasks of tile u,
// then the down tasks of tile u - lag, as the align scans number them for a larger batch.
__device__ __forceinline__ void fused_task(const FusedSched& fs, const Shape& sh, int tau, Task& t) {
  const int Mt = fs.n_tiles, Mr = fs.n_routed;
  int lo = 0, hi = fs.n_units - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (unit_start_of(mid, Mr, Mt, sh) <= tau) lo = mid;
    else hi = mid - 1;
  }
  const int off = tau - unit_start_of(lo, Mr, Mt, sh);
  const int nup = lo < Mt ? ceil_div(lo < Mr ? sh.D : sh.Ds, kBN1) : 0;
  const bool up = off < nup;
  const int g = up ? lo : lo - sh.lag;
  const int nt = up ? off : off - nup;
  t.kind = up ? kTaskUp : kTaskDown;
  t.tile = g;
  t.expert = fs.tile_exp[g];
  t.row0 = fs.tile_row0[g];
  t.nrows = fs.tile_nrows[g];
  t.ntiles = 1;
  t.nrows2 = 0;
  t.n0 = nt * (up ? kBN1 : kBN2);
}

// This CTA's share of the row gather: the x row of every kept slot s = blockIdx.x + j * gridDim.x
// into its tile row of xs; each row bumps its tile's gather count (release), which the tile's
// up tasks wait for before their TMA loads.
__device__ void front_gather(const FrontArgs& fa, const Workspace& ws, const Shape& sh, const int* slot_rows) {
  const int S = sh.T * sh.k, nvec = sh.H / 8;
  for (int s = blockIdx.x; s < S; s += gridDim.x) {
    const int row = slot_rows[s];
    if (row < 0) continue;
    const uint4* src = reinterpret_cast<const uint4*>(fa.x + (size_t)(s / sh.k) * sh.H);
    uint4* dst = reinterpret_cast<uint4*>(ws.xs + (size_t)row * sh.H);
    for (int i = threadIdx.x; i < nvec; i += 2 * blockDim.x) {  // two loads in flight per thread
      const int i2 = i + blockDim.x;
      const uint4 a = __ldg(src + i), b = __ldg(src + min(i2, nvec - 1));
      dst[i] = a;
      if (i2 < nvec) dst[i2] = b;
    }
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) red_release_add_gpu(ws.gather_done + row / sh.tile_m, 1);
  }
}

// The row gather of the MXFP8 experts: the x row of every kept slot s = blockIdx.x + j * gridDim.x,
// quantised to MXFP8 as the x quantiser does (one 32-element block per thread), into its tile row
// of xs and the scale atoms of sf_xs; with a shared expert, CTA b < T also quantises token b into
// the token-ordered xq / sf_xq that the shared tile (tile Mr) reads. Each written row bumps its
// tile's gather count (release) after a proxy fence, since the tile's up tasks read the codes and
// scales with TMA and bulk copies (async proxy).
__device__ void front_gather_mx(const FrontArgs& fa, const Workspace& ws, const MxBuffers& mx, const Shape& sh,
                                const int* slot_rows, int Mr) {
  const int S = sh.T * sh.k, H = sh.H, nb = H / kMxBlock;
  auto quantise_row = [&](int t, uint8_t* codes, uint8_t* sf, int64_t row) {
    for (int b = threadIdx.x; b < nb; b += blockDim.x) {
      float v[32];
      load_bf16x32(fa.x + (size_t)t * H + b * kMxBlock, v);
      uint32_t w[8];
      const uint32_t code = mx_quantize_block(v, w);
      store_codes32(codes + (size_t)row * H + b * kMxBlock, w);
      sf[mx_sf_offset(row, b, H)] = (uint8_t)code;
    }
    fence_proxy_async_global();
    __threadfence();
    __syncthreads();
  };
  for (int s = blockIdx.x; s < S; s += gridDim.x) {
    const int row = slot_rows[s];
    if (row < 0) continue;
    quantise_row(s / sh.k, mx.xs, mx.sf_xs, row);
    if (threadIdx.x == 0) red_release_add_gpu(ws.gather_done + row / sh.tile_m, 1);
  }
  if (sh.Ds > 0) {
    for (int t = blockIdx.x; t < sh.T; t += gridDim.x) {
      quantise_row(t, mx.xq, mx.sf_xq, t);
      if (threadIdx.x == 0) red_release_add_gpu(ws.gather_done + Mr, 1);
    }
  }
}

// One token's combine of columns [c*kBN2, (c+1)*kBN2) by one warp, once all of that token's rows
// of the block are in y: out[t] = y[shared row of t] + sum_j y[row of slot t*k + j], in this
// order, in fp32 (the standalone combine kernel's order, so the result is the same bit for bit).
// Lane l takes the 8 columns c*kBN2 + 8 l (the warp reads 512 contiguous bytes of a row per
// load); the rows' loads go out 8 at a time.
__device__ void combine_token_block(const FrontArgs& fa, const Workspace& ws, const Shape& sh, const FusedSched& fs,
                                    int tok, int c, int lane) {
  const int col = c * kBN2 + lane * 8;
  if (col + 8 > sh.H) return;
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  const int nr = (sh.Ds > 0 ? 1 : 0) + sh.k;
  auto row_of = [&](int j) {
    const int jj = sh.Ds > 0 ? j - 1 : j;
    return jj < 0 ? (fs.n_routed + tok / sh.tile_m) * sh.tile_m + tok % sh.tile_m : fs.slot_row[tok * sh.k + jj];
  };
  constexpr int kRound = 8;
  for (int j0 = 0; j0 < nr; j0 += kRound) {
    uint4 d[kRound];
    int rows[kRound];
#pragma unroll
    for (int q = 0; q < kRound; ++q) {
      rows[q] = j0 + q < nr ? row_of(j0 + q) : -1;
      d[q] = rows[q] >= 0 ? __ldcg(reinterpret_cast<const uint4*>(ws.y + (size_t)rows[q] * sh.H + col))
                          : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int q = 0; q < kRound; ++q)
      if (rows[q] >= 0) add_bf16x8(acc, d[q]);
  }
  if (fa.out_bf16) store8<true>(fa.out, (size_t)tok * sh.H + col, acc);
  else store8<false>(fa.out, (size_t)tok * sh.H + col, acc);
}

// After a fused down task's y stores (the 128 epilogue threads, warps 2-5; `row` is the thread's
// tile row): each valid row adds 1 to its token's counter for the task's column block with one
// acquire-release atomic (its release covers the thread's own row of y), and the row that
// completes a token's block lists the token; then one warp per listed token combines it. A
// token's block is combined as soon as its last row is in, not after the block's last task.
// s_list: shared [1 + 16] (count, tokens), zero on entry. Returns the number of tokens combined.
__device__ int fused_down_done(const FrontArgs& fa, const Workspace& ws, const Shape& sh, const FusedSched& fs,
                                const Task& t, int row, volatile int* s_list, bool leader) {
  const int nblk = ceil_div(sh.H, kBN2), c = t.n0 / kBN2;
  named_bar_sync(1, 128);  // the previous task's list is cleared
  if (row < t.nrows) {
    const int tok = (t.expert == sh.E) ? t.row0 + row : fs.row_slot[t.tile * kSmallRows + row] / sh.k;
    if (atom_add_acq_rel_gpu(&ws.tok_done[tok * nblk + c], 1) == fs.tok_need[tok] - 1) {
      __threadfence();
      s_list[1 + atomicAdd(const_cast<int*>(&s_list[0]), 1)] = tok;
    }
  }
  named_bar_sync(1, 128);
  const int n = s_list[0];
  for (int i = ((int)threadIdx.x >> 5) - 2; i < n; i += 4)
    combine_token_block(fa, ws, sh, fs, s_list[1 + i], c, (int)threadIdx.x & 31);
  named_bar_sync(1, 128);
  if (leader) s_list[0] = 0;
  return n;
}

}  // namespace

}  // namespace moe
