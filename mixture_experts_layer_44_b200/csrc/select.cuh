// Per-token softmax and top-k selection shared by the router kernels.
#pragma once

#include <float.h>

#include "common.cuh"

namespace moe {

// Order of the top-k key: larger logit first, equal logits -> lower expert id.
__device__ __forceinline__ bool better(float v1, int i1, float v2, int i2) {
  return v1 > v2 || (v1 == v2 && i1 < i2);
}

// Order-preserving 32-bit key of a float: a larger float has a larger
// unsigned key, and -0.0 and +0.0 share one key (they compare equal).  Every
// finite float has a key above 0, so 0 marks an expert out of the running.
__device__ __forceinline__ uint32_t order_key(float f) {
  const uint32_t b = __float_as_uint(f + 0.f);   // -0.0 + 0.0 = +0.0
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

__device__ __forceinline__ float key_value(uint32_t key) {
  return __uint_as_float((key & 0x80000000u) ? (key & 0x7fffffffu) : ~key);
}

// Group-limited selection (diffulex.moe.topk, GroupLimitedTopKRouter): the
// experts form `count` groups of `gsize` consecutive ids, a group scores as
// its best expert, and only the `keep` best groups (equal scores: lower group
// id first) stay in the running.  count <= 1: no limit.
struct GroupLimit {
  int gsize;
  int count;
  int keep;
};

// Bit g of the result is set when group g is kept.  key[j] is the order key
// of expert lane + 32 j (0 = no expert); gidx[j] its group.  Every lane
// returns the same mask.
template <int PER>
__device__ __forceinline__ uint32_t kept_groups(const uint32_t (&key)[PER], const int (&gidx)[PER],
                                                GroupLimit gl) {
  const int lane = threadIdx.x & 31;
  uint32_t mine = 0;                                   // score key of group `lane`
  for (int g = 0; g < gl.count; ++g) {
    uint32_t m = 0;
#pragma unroll
    for (int j = 0; j < PER; ++j)
      if (gidx[j] == g) m = key[j] > m ? key[j] : m;
    m = __reduce_max_sync(0xffffffffu, m);
    if (lane == g) mine = m;
  }
  uint32_t mask = 0;
  for (int r = 0; r < gl.keep; ++r) {
    const uint32_t best = __reduce_max_sync(0xffffffffu, mine);
    const uint32_t who = __reduce_min_sync(
        0xffffffffu, (lane < gl.count && mine == best) ? static_cast<uint32_t>(lane) : 32u);
    mask |= 1u << who;
    if (lane == static_cast<int>(who)) mine = 0;
  }
  return mask;
}

// Top-k selection and softmax weights for NTOK tokens at once, each held by
// the whole warp (lane l holds the logits of experts l, l+32, ... of every
// token; k >= 1).  Each lane first sorts its PER experts of a token by
// (logit descending, expert id ascending).  Round r then compares only the
// lanes' heads: one warp max-reduction finds the largest key, one warp
// min-reduction the lowest expert id among the heads holding it, and that
// lane pops its head.  This is the order (logit descending, expert id
// ascending) over all E.  The NTOK tokens are independent chains, so their
// reductions overlap.  The first round's logit is the row maximum m; the
// weight of a selection is exp(l - m) divided by the sum over the k
// selections (renormalize) or over all E experts.  Lane r < k writes
// selection r of token n when ids_t[n] is not null.  With a group limit the
// experts of the groups left out are out of the running before the sort (the
// softmax still spans all E; the group holding the row maximum is always
// kept, so the first selection is still the row maximum m).
template <int PER, int NTOK>
__device__ __forceinline__ void select_topk_n(const float (&v)[NTOK][PER], const bool (&live)[PER],
                                              int k, int renorm, int32_t* const (&ids_t)[NTOK],
                                              float* const (&w_t)[NTOK],
                                              GroupLimit gl = GroupLimit{1, 1, 1}) {
  const int lane = threadIdx.x & 31;
  uint32_t key[NTOK][PER], eid[NTOK][PER];
  int gidx[PER];
#pragma unroll
  for (int j = 0; j < PER; ++j)
    gidx[j] = (gl.count > 1 && live[j]) ? (lane + 32 * j) / gl.gsize : -1;
#pragma unroll
  for (int n = 0; n < NTOK; ++n) {
#pragma unroll
    for (int j = 0; j < PER; ++j) {
      key[n][j] = live[j] ? order_key(v[n][j]) : 0u;
      eid[n][j] = static_cast<uint32_t>(lane + 32 * j);
    }
    if (gl.count > 1) {
      const uint32_t kept = kept_groups<PER>(key[n], gidx, gl);
#pragma unroll
      for (int j = 0; j < PER; ++j)
        if (gidx[j] >= 0 && !((kept >> gidx[j]) & 1u)) key[n][j] = 0u;
    }
    // odd-even transposition sort, PER passes: (key descending, id ascending)
#pragma unroll
    for (int p = 0; p < PER; ++p) {
#pragma unroll
      for (int j = p & 1; j + 1 < PER; j += 2) {
        const bool sw = key[n][j + 1] > key[n][j] ||
                        (key[n][j + 1] == key[n][j] && eid[n][j + 1] < eid[n][j]);
        const uint32_t k0 = key[n][j], e0 = eid[n][j];
        key[n][j] = sw ? key[n][j + 1] : k0;
        eid[n][j] = sw ? eid[n][j + 1] : e0;
        key[n][j + 1] = sw ? k0 : key[n][j + 1];
        eid[n][j + 1] = sw ? e0 : eid[n][j + 1];
      }
    }
  }
  float m[NTOK], ssel[NTOK], my_v[NTOK];
  int my_id[NTOK];
#pragma unroll
  for (int n = 0; n < NTOK; ++n) {
    m[n] = 0.f;
    ssel[n] = 0.f;
    my_v[n] = 0.f;
    my_id[n] = 0;
  }
#pragma unroll
  for (int r = 0; r < moe::kMaxTopK; ++r) {
    if (r >= k) break;
    uint32_t kmax[NTOK], cand[NTOK], id[NTOK];
#pragma unroll
    for (int n = 0; n < NTOK; ++n) kmax[n] = __reduce_max_sync(0xffffffffu, key[n][0]);
#pragma unroll
    for (int n = 0; n < NTOK; ++n) {
      cand[n] = key[n][0] == kmax[n] ? eid[n][0] : 0xffffffffu;
      id[n] = __reduce_min_sync(0xffffffffu, cand[n]);
    }
#pragma unroll
    for (int n = 0; n < NTOK; ++n) {
      const bool pop = cand[n] == id[n];
#pragma unroll
      for (int j = 0; j + 1 < PER; ++j) {
        key[n][j] = pop ? key[n][j + 1] : key[n][j];
        eid[n][j] = pop ? eid[n][j + 1] : eid[n][j];
      }
      key[n][PER - 1] = pop ? 0u : key[n][PER - 1];
      const float bv = key_value(kmax[n]);
      if (r == 0) m[n] = bv;
      const float ex = expf(bv - m[n]);
      ssel[n] += ex;
      if (lane == r) {
        my_v[n] = ex;
        my_id[n] = static_cast<int>(id[n]);
      }
    }
  }
#pragma unroll
  for (int n = 0; n < NTOK; ++n) {
    float denom = ssel[n];
    if (!renorm) {
      float sum = 0.f;
#pragma unroll
      for (int j = 0; j < PER; ++j)
        if (live[j]) sum += expf(v[n][j] - m[n]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      denom = sum;
    }
    if (lane < k && ids_t[n] != nullptr) {
      ids_t[n][lane] = my_id[n];
      w_t[n][lane] = my_v[n] / denom;
    }
  }
}

// One token per warp (see select_topk_n).
template <int PER>
__device__ __forceinline__ void select_topk(const float* v, const bool* live, int k, int renorm,
                                            int32_t* ids_t, float* w_t,
                                            GroupLimit gl = GroupLimit{1, 1, 1}) {
  float vv[1][PER];
  bool lv[PER];
#pragma unroll
  for (int j = 0; j < PER; ++j) {
    vv[0][j] = v[j];
    lv[j] = live[j];
  }
  int32_t* const it[1] = {ids_t};
  float* const wt[1] = {w_t};
  select_topk_n<PER, 1>(vv, lv, k, renorm, it, wt, gl);
}

}  // namespace moe
