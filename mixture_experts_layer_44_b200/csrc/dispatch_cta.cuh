// One CTA dispatching a small batch: per-warp counts, exclusive scan over the
// experts, stable scatter, and (when given x) the gather of the rows.
//
// DWDP-Triton-MoE-Inference-Engine README, "Dispatcher Module" and "Executor
// Module" (gather token activations).  Inside an expert the assignments keep
// ascending f = t*k + j, the flat order of metrale's ep_dispatch.rs
// (build_ep_routing_table).  Warp w owns a contiguous slice of the N
// assignments; inside a 32-lane round a lane's rank among equal experts is the
// popcount of the lower lanes in its match mask, so positions grow with f
// inside an expert and the result does not depend on the warp count.
#pragma once

#include "common.cuh"

namespace moe {

// NW warps; up to NW * 32 * ROUNDS assignments.  wc: shared [NW][E], zeroed
// by the caller before a __syncthreads; s_scan: shared [kMaxExperts].  Every
// thread of the CTA calls this (it synchronises the CTA).  Ids outside [0,E)
// are reported (MOE_ERR_BAD_INDEX), given inv_perm -1 and left out.
//
// With stage (shared, 3 * NW * 32 * ROUNDS ints) the scatter writes perm,
// packed_tok and packed_w into shared memory, and the CTA then copies the
// three arrays out in position order: a scattered 4-byte store from one SM
// costs a separate L2 write per distinct sector, a copied-out row of 32
// positions costs four.
template <int NW, int ROUNDS>
__device__ __forceinline__ void dispatch_cta(
    const int32_t* ids, const float* w, int N, int E, int k, int32_t* counts, int32_t* offsets,
    int32_t* perm, int32_t* inv_perm, int32_t* packed_tok, float* packed_w, const uint4* x,
    int row_vecs, uint4* xp, int32_t* status, int* wc, int* s_scan, int* stage = nullptr) {
  constexpr int NMAX = NW * 32 * ROUNDS;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const unsigned lt = (1u << lane) - 1u;
  const int per = (N + NW - 1) / NW;
  const int w0 = warp * per, w1 = min(N, w0 + per);
  // The warp's slice of ids and weights, read once (all loads in flight
  // together) and kept in registers for both passes; -1 marks no assignment
  // or a bad id.
  const int nr = w1 > w0 ? (w1 - w0 + 31) / 32 : 0;   // rounds this warp needs
  int eid[ROUNDS];
  float wv[ROUNDS];
#pragma unroll
  for (int i = 0; i < ROUNDS; ++i) {
    const int f = w0 + 32 * i + lane;
    eid[i] = f < w1 ? ld_prod(ids + f) : -1;
    wv[i] = packed_w != nullptr && f < w1 ? ld_prod(w + f) : 0.f;
  }
  // 1. per-warp counts over this warp's contiguous slice
#pragma unroll
  for (int i = 0; i < ROUNDS; ++i) {
    if (i >= nr) break;
    const int f = w0 + 32 * i + lane;
    if (f < w1 && (eid[i] < 0 || eid[i] >= E)) {
      report(status, MOE_ERR_BAD_INDEX);
      inv_perm[f] = -1;
      eid[i] = -1;
    }
    const int e = eid[i];
    const int key = e >= 0 ? e : -1 - lane;
    const unsigned peers = __match_any_sync(0xffffffffu, key);
    if (e >= 0 && lane == __ffs(peers) - 1) wc[warp * E + e] += __popc(peers);
  }
  __syncthreads();
  // 2. counts, inclusive scan over experts into s_scan (a shuffle scan in
  //    each warp of 32 experts, then the warp totals), per-warp bases
  //    (blockDim >= 256)
  const int e = threadIdx.x;
  int total = 0;
  if (e < E)
    for (int ww = 0; ww < NW; ++ww) total += wc[ww * E + e];
  __shared__ int s_wsum[kMaxExperts / 32];
  int incl = total;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (e < kMaxExperts && lane == 31) s_wsum[warp] = incl;
  __syncthreads();
  if (e < kMaxExperts) {
    for (int ww = 0; ww < warp; ++ww) incl += s_wsum[ww];
    s_scan[e] = incl;
  }
  __syncthreads();
  if (e < E) {
    const int excl = s_scan[e] - total;
    counts[e] = total;
    offsets[e] = excl;
    int run = excl;
    for (int ww = 0; ww < NW; ++ww) {
      const int c = wc[ww * E + e];
      wc[ww * E + e] = run;
      run += c;
    }
  }
  if (e == 0) offsets[E] = s_scan[kMaxExperts - 1];
  __syncthreads();
  // 3. stable scatter: slices in warp order, rounds in order, lanes in order
#pragma unroll
  for (int i = 0; i < ROUNDS; ++i) {
    if (i >= nr) break;
    const int f = w0 + 32 * i + lane;
    const int ex = eid[i];
    const int key = ex >= 0 ? ex : -1 - lane;
    const unsigned peers = __match_any_sync(0xffffffffu, key);
    if (ex >= 0) {
      const int p = wc[warp * E + ex] + __popc(peers & lt);
      inv_perm[f] = p;
      if (stage != nullptr) {
        stage[p] = f;
        stage[NMAX + p] = f / k;
        stage[2 * NMAX + p] = __float_as_int(wv[i]);
      } else {
        perm[p] = f;
        packed_tok[p] = f / k;
        if (packed_w) packed_w[p] = wv[i];
      }
    }
    __syncwarp();
    if (ex >= 0 && lane == __ffs(peers) - 1) wc[warp * E + ex] += __popc(peers);
    __syncwarp();
  }
  const int nrows = s_scan[kMaxExperts - 1];
  if (stage != nullptr) {
    __syncthreads();
    for (int p = threadIdx.x; p < nrows; p += NW * 32) {
      perm[p] = stage[p];
      packed_tok[p] = stage[NMAX + p];
      if (packed_w) packed_w[p] = __int_as_float(stage[2 * NMAX + p]);
    }
  }
  grid_dep_launch();
  if (x == nullptr) return;
  __syncthreads();
  // 4. gather (small total): one warp per row, 16-byte vectors, 8 loads in
  //    flight per lane before the stores
  for (int p = warp; p < nrows; p += NW) {
    const int tok = stage != nullptr ? stage[NMAX + p] : ld_prod(packed_tok + p);
    const uint4* src = x + static_cast<size_t>(tok) * row_vecs;
    uint4* dst = xp + static_cast<size_t>(p) * row_vecs;
    for (int v0 = lane; v0 < row_vecs; v0 += 32 * 8) {
      uint4 q[8];
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (v0 + 32 * j < row_vecs) q[j] = ld_prod(src + v0 + 32 * j);
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (v0 + 32 * j < row_vecs) dst[v0 + 32 * j] = q[j];
    }
  }
}

}  // namespace moe
