// route.cuh -- device code shared by the gating/align kernels and the fused small-batch
// forward: the warp top-k with renormalised softmax, a block-wide scan, the align scans
// (offsets, capacity, m-tiles, scheduling groups and task units) and the segment search.
#pragma once

#include <climits>
#include <cmath>

#include "common.cuh"

namespace moe {

// ------------------------------------------------------------------------------------------
// warp top-k + renormalised softmax of one token held in registers; lane j < k returns
// choice j
// ------------------------------------------------------------------------------------------
// A float's order as an unsigned key (larger value, larger key; -0 and +0 the same key).
__device__ __forceinline__ uint32_t order_key(float f) {
  const uint32_t u = __float_as_uint(f + 0.0f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Top-k with renormalised softmax for NT tokens at once (their dependency chains interleave):
// v[n][j] holds expert lane + 32 j of token n. Each lane first sorts its VPL candidates of every
// token (largest first, ties to the lower expert index; an odd-even merge network). Each of the
// k rounds then takes, per token, the largest remaining logit, ties to the lower expert index:
// the warp's largest head key (one redux), then the lowest expert index among the lanes whose
// head holds it (another); the winning lane drops its head. Lane r < k returns round r's expert
// in ids[n] and its weight exp(v_r - v_0) / sum_i exp(v_i - v_0) over the k chosen in w[n].
// Experts >= E and NaN logits are never chosen while another candidate is left.
template <int VPL>
__device__ __forceinline__ void lane_sort_desc(uint32_t (&key)[VPL], int (&idx)[VPL], float (&val)[VPL]) {
  // compare-exchange (a, b): a keeps the larger key, the lower index on equal keys
  auto cx = [&](int a, int b) {
    const bool sw = key[a] < key[b] || (key[a] == key[b] && idx[a] > idx[b]);
    const uint32_t ka = key[a], kb = key[b];
    const int ia = idx[a], ib = idx[b];
    const float va = val[a], vb = val[b];
    key[a] = sw ? kb : ka;
    key[b] = sw ? ka : kb;
    idx[a] = sw ? ib : ia;
    idx[b] = sw ? ia : ib;
    val[a] = sw ? vb : va;
    val[b] = sw ? va : vb;
  };
  // Batcher's odd-even merge sort, for VPL a power of two
#pragma unroll
  for (int p = 1; p < VPL; p <<= 1)
#pragma unroll
    for (int q = p; q >= 1; q >>= 1)
#pragma unroll
      for (int j = q % p; j + q < VPL; j += 2 * q)
#pragma unroll
        for (int i = 0; i < q; ++i)
          if (i + j + q < VPL && (i + j) / (2 * p) == (i + j + q) / (2 * p)) cx(i + j, i + j + q);
}

// More than 8 candidates per lane (E > 256): no sort; each round scans the lane's remaining
// candidates for its best, with the same order.
template <int VPL, int NT>
__device__ __forceinline__ void warp_topk_scan_n(const float (&v)[NT][VPL], int E, int k, int lane,
                                                 float (&my_v)[NT], float (&top_v)[NT], int (&ids)[NT]) {
  uint32_t taken[NT];
#pragma unroll
  for (int n = 0; n < NT; ++n) {
    taken[n] = 0;
#pragma unroll
    for (int j = 0; j < VPL; ++j)
      if (lane + 32 * j >= E || v[n][j] != v[n][j]) taken[n] |= 1u << j;
  }
  for (int r = 0; r < k; ++r) {
    float bv[NT];
    int bi[NT];
    uint32_t key[NT], best[NT];
    int win[NT];
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      bv[n] = -INFINITY;
      bi[n] = INT_MAX;
#pragma unroll
      for (int j = 0; j < VPL; ++j) {
        const int e = lane + 32 * j;
        if (!((taken[n] >> j) & 1u) && (v[n][j] > bv[n] || (v[n][j] == bv[n] && e < bi[n]))) {
          bv[n] = v[n][j];
          bi[n] = e;
        }
      }
      key[n] = bi[n] == INT_MAX ? 0u : order_key(bv[n]);
    }
#pragma unroll
    for (int n = 0; n < NT; ++n) best[n] = __reduce_max_sync(0xffffffffu, key[n]);
#pragma unroll
    for (int n = 0; n < NT; ++n)
      win[n] = (int)__reduce_min_sync(0xffffffffu, (uint32_t)(key[n] == best[n] ? bi[n] : INT_MAX));
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      if (win[n] != INT_MAX && (win[n] & 31) == lane) taken[n] |= 1u << (win[n] >> 5);
      const float wv = __shfl_sync(0xffffffffu, bv[n], win[n] & 31);
      if (lane == r) {
        my_v[n] = wv;
        ids[n] = win[n];
      }
      if (r == 0) top_v[n] = wv;
    }
  }
}

template <int VPL, int NT>
__device__ __forceinline__ void warp_topk_softmax_n(const float (&v)[NT][VPL], int E, int k, int lane,
                                                    int (&ids)[NT], float (&w)[NT]) {
  static_assert((VPL & (VPL - 1)) == 0, "candidates per lane: a power of two");
  float my_v[NT], top_v[NT];
  if constexpr (VPL > 8) {
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      my_v[n] = 0.f;
      top_v[n] = 0.f;
      ids[n] = -1;
    }
    warp_topk_scan_n<VPL, NT>(v, E, k, lane, my_v, top_v, ids);
  } else {
  uint32_t key[NT][VPL];
  int idx[NT][VPL];
  float val[NT][VPL];
#pragma unroll
  for (int n = 0; n < NT; ++n) {
#pragma unroll
    for (int j = 0; j < VPL; ++j) {
      const int e = lane + 32 * j;
      const bool ok = e < E && !(v[n][j] != v[n][j]);
      key[n][j] = ok ? order_key(v[n][j]) : 0u;
      idx[n][j] = ok ? e : INT_MAX;
      val[n][j] = v[n][j];
    }
    lane_sort_desc<VPL>(key[n], idx[n], val[n]);
    my_v[n] = 0.f;
    top_v[n] = 0.f;
    ids[n] = -1;
  }
  for (int r = 0; r < k; ++r) {
    uint32_t best[NT];
    int win[NT];
    // each step runs for all NT tokens before the next: the warp-wide reductions are not moved
    // across one another, so token-major code would run the NT chains one after the other
#pragma unroll
    for (int n = 0; n < NT; ++n) best[n] = __reduce_max_sync(0xffffffffu, key[n][0]);
#pragma unroll
    for (int n = 0; n < NT; ++n)
      win[n] = (int)__reduce_min_sync(0xffffffffu, (uint32_t)(key[n][0] == best[n] ? idx[n][0] : INT_MAX));
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      const bool mine = win[n] != INT_MAX && idx[n][0] == win[n];
      const float wv = __shfl_sync(0xffffffffu, val[n][0], win[n] & 31);  // the winner's value
      if (lane == r) {
        my_v[n] = wv;
        ids[n] = win[n];
      }
      if (r == 0) top_v[n] = wv;
      // the winning lane drops its head
#pragma unroll
      for (int j = 0; j + 1 < VPL; ++j) {
        key[n][j] = mine ? key[n][j + 1] : key[n][j];
        idx[n][j] = mine ? idx[n][j + 1] : idx[n][j];
        val[n][j] = mine ? val[n][j + 1] : val[n][j];
      }
      key[n][VPL - 1] = mine ? 0u : key[n][VPL - 1];
      idx[n][VPL - 1] = mine ? INT_MAX : idx[n][VPL - 1];
    }
  }
  }
#pragma unroll
  for (int n = 0; n < NT; ++n) {
    const float ex = (lane < k) ? expf(my_v[n] - top_v[n]) : 0.f;
    float s = ex;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    w[n] = ex / s;
  }
}

// One token: lane j < k returns choice j.
template <int VPL>
__device__ __forceinline__ void warp_topk_softmax(const float (&v)[VPL], int E, int k, int lane,
                                                  int& out_id, float& out_w) {
  const float (&vv)[1][VPL] = *reinterpret_cast<const float (*)[1][VPL]>(&v);
  int ids[1];
  float w[1];
  warp_topk_softmax_n<VPL, 1>(vv, E, k, lane, ids, w);
  out_id = ids[0];
  out_w = w[0];
}

// ------------------------------------------------------------------------------------------
// block-wide exclusive scan of a[0..n) in shared memory (any n), returns the total.
// Uses `tmp` (>= blockDim/32 + 1 ints). All threads must call it.
// ------------------------------------------------------------------------------------------
__device__ inline int block_exclusive_scan(int* a, int n, int* tmp) {
  const int tid = threadIdx.x, nthr = blockDim.x, lane = tid & 31, warp = tid >> 5;
  const int nwarps = nthr >> 5;
  int carry = 0;
  for (int base = 0; base < n; base += nthr * 4) {
    int loc[4];
    int sum = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int idx = base + tid * 4 + i;
      loc[i] = (idx < n) ? a[idx] : 0;
      sum += loc[i];
    }
    int incl = sum;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += y;
    }
    if (lane == 31) tmp[warp] = incl;
    __syncthreads();
    if (tid == 0) {
      int run = 0;
      for (int w = 0; w < nwarps; ++w) {
        const int x = tmp[w];
        tmp[w] = run;
        run += x;
      }
      tmp[nwarps] = run;
    }
    __syncthreads();
    int run = carry + tmp[warp] + incl - sum;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int idx = base + tid * 4 + i;
      if (idx < n) a[idx] = run;
      run += loc[i];
    }
    carry += tmp[nwarps];
    __syncthreads();
  }
  return carry;
}

// ------------------------------------------------------------------------------------------
// The scans, run by the last CTA of the histogram pass. Shared memory layout (ints):
//   tmp[64] | cnt[E] | kept[E] | offs[E] | tile[kMaxChunks * kScanGroup] | buf[max(E+1, units+1)]
// Everything the later steps need stays in shared memory (no reads of just-written globals).
// ------------------------------------------------------------------------------------------
constexpr int kScanGroup = 256;  // experts scanned per pass (tile of [chunks][256] counts)

__device__ inline void align_scans(const Workspace& ws, const Shape& sh, bool tiles, int* sm) {
  const int tid = threadIdx.x, nthr = blockDim.x;
  const int E = sh.E;
  int* tmp = sm;
  int* cnt = tmp + 64;
  int* kept = cnt + E;
  int* offs = kept + E;
  int* tile = offs + E;
  int* buf = tile + kMaxChunks * kScanGroup;
  const int nch = sh.num_chunks;

  // 1. per expert: exclusive prefix of the chunk counts (chunk_base) and the total n_e.
  //    The [chunks][group] block of counts is loaded with independent loads, then each
  //    thread scans one expert's column in shared memory.
  for (int g0 = 0; g0 < E; g0 += kScanGroup) {
    const int G = min(kScanGroup, E - g0);
    const int n = nch * G;
#pragma unroll 4
    for (int i = tid; i < n; i += nthr) {
      const int c = i / G, e = i - c * G;
      int* p = ws.chunk_hist + (size_t)c * E + g0 + e;
      tile[i] = __ldcg(p);
      *p = 0;  // the histograms start from zero at the next call
    }
    __syncthreads();
    for (int e = tid; e < G; e += nthr) {  // any block size: one expert per thread and pass
      int run = 0;
      for (int c = 0; c < nch; ++c) {
        const int v = tile[c * G + e];
        ws.chunk_base[(size_t)c * E + g0 + e] = run;
        run += v;
      }
      cnt[g0 + e] = run;
    }
    __syncthreads();
  }

  // 2. capacity cut and padded segment lengths
  for (int e = tid; e < E; e += nthr) {
    const int n = cnt[e];
    const int kp = (sh.capacity > 0) ? min(n, sh.capacity) : n;
    kept[e] = kp;
    ws.expert_kept[e] = kp;
    buf[e] = ceil_div(kp, sh.block_m) * sh.block_m;
  }
  __syncthreads();
  const int P = block_exclusive_scan(buf, E, tmp);
  for (int e = tid; e < E; e += nthr) {
    ws.expert_off[e] = buf[e];
    offs[e] = buf[e];
  }
  if (tid == 0) {
    ws.expert_off[E] = P;
    ws.meta->P = P;
  }
  __syncthreads();
  if (!tiles) return;

  // 3. m-tiles of tile_m rows: routed experts (ceil(kept/tile_m) each), then the shared expert
  //    over all tokens
  const int tm = sh.tile_m;
  for (int e = tid; e < E; e += nthr) buf[e] = ceil_div(kept[e], tm);
  __syncthreads();
  const int Mr = block_exclusive_scan(buf, E, tmp);
  for (int e = tid; e < E; e += nthr) {
    const int first = buf[e], nt = ceil_div(kept[e], tm);
    const int off = offs[e];
    ws.expert_tile0[e] = first;
    for (int i = 0; i < nt; ++i) {
      ws.tile_expert[first + i] = e;
      ws.tile_row0[first + i] = off + i * tm;
      ws.tile_nrows[first + i] = min(tm, kept[e] - i * tm);
    }
    offs[e] = first;  // the segment offsets are no longer needed: keep the first tile instead
  }
  const int Ms = (sh.Ds > 0) ? ceil_div(sh.T, tm) : 0;
  for (int j = tid; j < Ms; j += nthr) {
    ws.tile_expert[Mr + j] = E;
    ws.tile_row0[Mr + j] = j * tm;
    ws.tile_nrows[Mr + j] = min(tm, sh.T - j * tm);
  }
  const int Mt = Mr + Ms;
  __syncthreads();

  // 3b. scheduling groups: up to kGroupTiles consecutive tiles of one expert (the shared
  //     expert's tiles are grouped the same way)
  for (int e = tid; e < E; e += nthr) buf[e] = ceil_div(ceil_div(kept[e], tm), kGroupTiles);
  __syncthreads();
  const int Mgr = block_exclusive_scan(buf, E, tmp);
  // A group of two tiles whose second is a tail of at most kTailRows rows runs as one task set
  // when sh.merge_tail: each task computes both tiles from the same weight stages. With pairs of
  // tiles, a run of an odd number of tiles that ends in a tail starts with a single-tile group,
  // so that the tail closes a pair.
  auto put_group = [&](int gi, int t0, int g, int last_rows) {
    ws.group_tile0[gi] = t0;
    ws.group_ntiles[gi] = g;
    ws.group_tasks[gi] = (g == 2 && (sh.merge_tail == 2 || (sh.merge_tail == 1 && last_rows <= kTailRows))) ? 1 : g;
  };
  // tiles [start, start + g) of group j of a run of nt tiles whose last tile has last_rows rows
  auto group_span = [&](int j, int nt, int last_rows, int& start, int& g) {
    const int f = (kGroupTiles == 2 && sh.merge_tail == 1 && nt > 1 && (nt & 1) && last_rows <= kTailRows) ? 1 : 0;
    start = (f && j > 0) ? kGroupTiles * j - 1 : kGroupTiles * j;
    g = (f && j == 0) ? 1 : min(kGroupTiles, nt - start);
  };
  for (int e = tid; e < E; e += nthr) {
    const int nt = ceil_div(kept[e], tm), first = offs[e], g0 = buf[e];
    const int last_rows = kept[e] - (nt - 1) * tm;
    ws.expert_group0[e] = g0;
    for (int i = 0; i * kGroupTiles < nt; ++i) {
      int st, g;
      group_span(i, nt, last_rows, st, g);
      put_group(g0 + i, first + st, g, min(tm, kept[e] - (st + g - 1) * tm));
    }
  }
  const int Mgs = ceil_div(Ms, kGroupTiles);
  for (int j = tid; j < Mgs; j += nthr) {
    int st, g;
    group_span(j, Ms, sh.T - (Ms - 1) * tm, st, g);
    put_group(Mgr + j, Mr + st, g, min(tm, sh.T - (st + g - 1) * tm));
  }
  const int Mg = Mgr + Mgs;
  if (tid == 0) {
    ws.expert_group0[E] = Mgr;
    ws.expert_group0[E + 1] = Mg;
  }
  __syncthreads();

  // 4. schedule units: unit u holds the up/gate tasks of group u, then the down tasks of group
  //    u - lag. Task ids are unit-major, so every down task's dependencies have lower ids.
  const int U = (Mg > 0) ? Mg + sh.lag : 0;
  const int n2 = ceil_div(sh.H, kBN2);
  const int n1r = ceil_div(sh.D, kBN1), n1s = ceil_div(sh.Ds, kBN1);
  for (int u = tid; u < U; u += nthr) {
    int c = 0;
    if (u < Mg) c += ((u < Mgr) ? n1r : n1s) * ws.group_tasks[u];  // routed groups first
    if (u >= sh.lag && u - sh.lag < Mg) c += n2 * ws.group_tasks[u - sh.lag];
    buf[u] = c;
  }
  __syncthreads();
  const int total = block_exclusive_scan(buf, U, tmp);
  for (int u = tid; u < U; u += nthr) ws.unit_start[u] = buf[u];
  for (int i = tid; i < Mt; i += nthr) ws.done1[i] = 0;
  if (tid == 0) {
    ws.unit_start[U] = total;
    ws.meta->num_tiles = Mt;
    ws.meta->num_routed_tiles = Mr;
    ws.meta->num_groups = Mg;
    ws.meta->num_routed_groups = Mgr;
    ws.meta->num_units = U;
    ws.meta->total_tasks = total;
    ws.meta->task_counter = 0;
    ws.meta->abort = 0;
    ws.meta->trace_count = 0;
  }
}

__device__ __forceinline__ int segment_of(const int* off, int E, int i) {
  // largest e with off[e] <= i (off non-decreasing, off[E] = P > i)
  int lo = 0, hi = E;  // answer in [lo, hi)
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (off[mid] <= i) lo = mid;
    else hi = mid;
  }
  return lo;
}


}  // namespace moe
