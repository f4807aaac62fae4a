// Router: gating GEMM on the CUDA cores (fp32 FMA), fused with softmax,
// warp-shuffle top-k and renormalisation.
//
// DWDP-Triton-MoE-Inference-Engine README, "Router Module": router logits,
// routing probabilities, top-k expert indices, normalized routing weights.
// diffulex.moe API reference, "diffulex.moe.topk": NaiveTopKRouter.
//
// Batches of more than 64 tokens (or more than 64 experts): a thread-block
// cluster of S CTAs (S <= 8) owns BT = 64 tokens and all E
// experts; CTA s of the cluster contracts its own slice of H.  Each CTA
// stages chunks of KC = 32 columns of x and W_gate (converted to fp32,
// transposed) in shared memory, prefetching the next chunk into registers
// while it computes the current one, and accumulates a 4-token x
// (EPAD/16)-expert register tile per thread (EPAD = 64, 128 or 256: E rounded
// up).  The S partial logit tiles are then summed through distributed shared
// memory in a fixed rank order (deterministic, no global scratch): CTA s
// finalises tokens [s*BT/S, (s+1)*BT/S) of the tile, one warp per token, which
// adds the bias, writes the logits and selects the top k by k rounds of a warp
// arg-max on the key (logit descending, expert id ascending).
#include <cooperative_groups.h>
#include <float.h>

#include <algorithm>

#include "common.cuh"

namespace cg = cooperative_groups;

namespace {

constexpr int BT = 64;    // tokens per cluster
constexpr int KC = 32;    // H chunk
constexpr int TT = 4;     // tokens per thread
constexpr int NT = 256;   // threads per CTA
constexpr int MAX_S = 8;  // CTAs per cluster

__device__ __forceinline__ bool better(float v1, int i1, float v2, int i2) {
  return v1 > v2 || (v1 == v2 && i1 < i2);
}

template <bool BF16>
__device__ __forceinline__ void load8(const void* base, size_t off, bool ok, float* f) {
  if (!ok) {
#pragma unroll
    for (int j = 0; j < 8; ++j) f[j] = 0.f;
    return;
  }
  if (BF16) {
    const uint4 q = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(base) + off);
    moe::unpack8(q, f);
  } else {
    const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(base) + off);
    const float4 a = p[0], b = p[1];
    f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
    f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
  }
}


// Softmax over the E live logits of one token held by a warp (lane l holds
// experts l, l+32, ...), then k rounds of a warp arg-max on (logit desc, id
// asc) over the experts not yet taken; lane r < k writes selection r.
template <int PER>
__device__ __forceinline__ void select_topk(const float* v, const bool* live, int k, int renorm,
                                            int32_t* ids_t, float* w_t) {
  const int lane = threadIdx.x & 31;
  float m = -FLT_MAX;
#pragma unroll
  for (int j = 0; j < PER; ++j)
    if (live[j]) m = fmaxf(m, v[j]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  float s = 0.f;
#pragma unroll
  for (int j = 0; j < PER; ++j)
    if (live[j]) s += expf(v[j] - m);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);

  bool taken[PER];
#pragma unroll
  for (int j = 0; j < PER; ++j) taken[j] = !live[j];
  float ssel = 0.f;
  float my_v = 0.f;                           // lane r < k keeps selection r
  int my_id = 0;
#pragma unroll
  for (int r = 0; r < moe::kMaxTopK; ++r) {
    if (r >= k) break;
    float bv = -FLT_MAX;
    int bi = 0x7fffffff;
#pragma unroll
    for (int j = 0; j < PER; ++j) {
      const int e = lane + 32 * j;
      if (!taken[j] && (bi == 0x7fffffff || better(v[j], e, bv, bi))) {
        bv = v[j];
        bi = e;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (oi != 0x7fffffff && (bi == 0x7fffffff || better(ov, oi, bv, bi))) {
        bv = ov;
        bi = oi;
      }
    }
#pragma unroll
    for (int j = 0; j < PER; ++j)
      if (lane + 32 * j == bi) taken[j] = true;
    const float ex = expf(bv - m);
    ssel += ex;
    if (lane == r) {
      my_v = ex;
      my_id = bi;
    }
  }
  if (lane < k) {
    const float denom = renorm ? ssel : s;
    ids_t[lane] = my_id;
    w_t[lane] = my_v / denom;
  }
}

// Small batches (T <= 64 tokens, E <= 64 experts: decode): one CTA per token.
// The 256 threads cover H in one pass of 8-element vectors (thread i takes
// vectors i, i+256, ...) and keep one partial dot product per expert; the
// partials are reduced in a fixed order (warp shuffle tree, then warps in
// order), so the logits do not depend on timing.  Warp 0 then selects.
template <bool BF16>
__global__ void __launch_bounds__(NT) route_small_kernel(const void* __restrict__ xv,
                                                         const void* __restrict__ wv,
                                                         const float* __restrict__ bias, int H,
                                                         int E, int k, int renorm,
                                                         float* __restrict__ logits,
                                                         int32_t* __restrict__ ids,
                                                         float* __restrict__ wout) {
  constexpr int EMAX = 64;
  __shared__ float part[NT / 32][EMAX];
  const int t = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float acc[EMAX];
#pragma unroll
  for (int e = 0; e < EMAX; ++e) acc[e] = 0.f;
  const int nvec = H / 8;
  for (int v = threadIdx.x; v < nvec; v += NT) {
    float xf[8];
    load8<BF16>(xv, static_cast<size_t>(t) * H + v * 8, true, xf);
#pragma unroll
    for (int e = 0; e < EMAX; ++e) {
      if (e < E) {
        float wf[8];
        load8<BF16>(wv, static_cast<size_t>(e) * H + v * 8, true, wf);
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[e] = fmaf(xf[j], wf[j], acc[e]);
      }
    }
  }
#pragma unroll
  for (int e = 0; e < EMAX; ++e) {
    if (e < E) {
      float a = acc[e];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
      if (lane == 0) part[warp][e] = a;
    }
  }
  __syncthreads();
  if (warp != 0) return;
  constexpr int PER = EMAX / 32;
  float v[PER];
  bool live[PER];
#pragma unroll
  for (int j = 0; j < PER; ++j) {
    const int e = lane + 32 * j;
    live[j] = e < E;
    float s = 0.f;
    if (live[j]) {
#pragma unroll
      for (int w = 0; w < NT / 32; ++w) s += part[w][e];
      s += bias ? bias[e] : 0.f;
      logits[static_cast<size_t>(t) * E + e] = s;
    }
    v[j] = live[j] ? s : -FLT_MAX;
  }
  if (k == 0) return;
  select_topk<PER>(v, live, k, renorm, ids + static_cast<size_t>(t) * k,
                   wout + static_cast<size_t>(t) * k);
}

template <int EPAD, bool BF16>
__global__ void __launch_bounds__(NT) route_kernel(const void* __restrict__ xv,
                                                   const void* __restrict__ wv,
                                                   const float* __restrict__ bias, int T, int H,
                                                   int E, int k, int renorm, int kc_per_cta,
                                                   float* __restrict__ logits,
                                                   int32_t* __restrict__ ids,
                                                   float* __restrict__ wout) {
  constexpr int TE = EPAD / 16;            // experts per thread
  constexpr int LS = EPAD + 1;             // padded row of the logits tile
  constexpr int WV = EPAD * (KC / 8) / NT; // W_gate vectors per thread per chunk (1, 2 or 4)
  extern __shared__ __align__(16) float sm[];
  float* x_s = sm;                         // [KC][BT]
  float* w_s = sm + KC * BT;               // [KC][EPAD]
  float* l_s = sm + KC * BT + KC * EPAD;   // [BT][LS] partial logits of this CTA

  cg::cluster_group cluster = cg::this_cluster();
  const int S = static_cast<int>(cluster.num_blocks());
  const int rank = static_cast<int>(cluster.block_rank());
  const int tid = threadIdx.x;
  const int eg = tid & 15;
  const int tg = tid >> 4;
  const int t0 = blockIdx.y * BT;
  const int h_begin = rank * kc_per_cta * KC;
  const int h_end = min(H, h_begin + kc_per_cta * KC);

  float acc[TT][TE];
#pragma unroll
  for (int i = 0; i < TT; ++i)
#pragma unroll
    for (int j = 0; j < TE; ++j) acc[i][j] = 0.f;

  // Register staging of one chunk: x (one 8-vector per thread), W (WV 8-vectors).
  const int xt = tid >> 2, xv8 = tid & 3;
  float xr[8], wr[WV][8];
  auto fetch = [&](int h0) {
    const int hh = h0 + xv8 * 8;
    load8<BF16>(xv, static_cast<size_t>(t0 + xt) * H + hh, t0 + xt < T && hh < h_end, xr);
#pragma unroll
    for (int u = 0; u < WV; ++u) {
      const int i = tid + u * NT;
      const int e = i >> 2, hv = h0 + (i & 3) * 8;
      load8<BF16>(wv, static_cast<size_t>(e) * H + hv, e < E && hv < h_end, wr[u]);
    }
  };
  auto stash = [&]() {
#pragma unroll
    for (int j = 0; j < 8; ++j) x_s[(xv8 * 8 + j) * BT + xt] = xr[j];
#pragma unroll
    for (int u = 0; u < WV; ++u) {
      const int i = tid + u * NT;
      const int e = i >> 2, v = i & 3;
#pragma unroll
      for (int j = 0; j < 8; ++j) w_s[(v * 8 + j) * EPAD + e] = wr[u][j];
    }
  };

  if (h_begin < h_end) fetch(h_begin);
  for (int h0 = h_begin; h0 < h_end; h0 += KC) {
    stash();
    __syncthreads();
    if (h0 + KC < h_end) fetch(h0 + KC);        // next chunk in flight during the FMAs
#pragma unroll 8
    for (int kk = 0; kk < KC; ++kk) {
      const float4 xq = *reinterpret_cast<const float4*>(&x_s[kk * BT + tg * TT]);
      const float xa[TT] = {xq.x, xq.y, xq.z, xq.w};
      float wa[TE];
#pragma unroll
      for (int j = 0; j < TE; j += 4) {
        const float4 q = *reinterpret_cast<const float4*>(&w_s[kk * EPAD + eg * TE + j]);
        wa[j] = q.x; wa[j + 1] = q.y; wa[j + 2] = q.z; wa[j + 3] = q.w;
      }
#pragma unroll
      for (int i = 0; i < TT; ++i)
#pragma unroll
        for (int j = 0; j < TE; ++j) acc[i][j] = fmaf(xa[i], wa[j], acc[i][j]);
    }
    __syncthreads();
  }

  // This CTA's partial logits tile.
#pragma unroll
  for (int i = 0; i < TT; ++i)
#pragma unroll
    for (int j = 0; j < TE; ++j) l_s[(tg * TT + i) * LS + eg * TE + j] = acc[i][j];
  cluster.sync();

  // Finalise tokens [rank*BT/S, (rank+1)*BT/S): one warp per token.
  constexpr int PER = EPAD / 32;
  const int warp = tid >> 5, lane = tid & 31;
  const int per_cta = (BT + S - 1) / S;
  const int tl_end = min(BT, (rank + 1) * per_cta);
  for (int tl = rank * per_cta + warp; tl < tl_end; tl += NT / 32) {
    const int t = t0 + tl;
    if (t >= T) break;
    float v[PER];
    bool live[PER];
#pragma unroll
    for (int j = 0; j < PER; ++j) {
      const int e = lane + 32 * j;
      live[j] = e < E;
      v[j] = 0.f;
    }
    for (int r = 0; r < S; ++r) {               // fixed order: deterministic sum
      const float* rl = cluster.map_shared_rank(l_s, r);
#pragma unroll
      for (int j = 0; j < PER; ++j)
        if (live[j]) v[j] += rl[tl * LS + lane + 32 * j];
    }
#pragma unroll
    for (int j = 0; j < PER; ++j) {
      const int e = lane + 32 * j;
      if (live[j]) {
        v[j] += bias ? bias[e] : 0.f;
        logits[static_cast<size_t>(t) * E + e] = v[j];
      } else {
        v[j] = -FLT_MAX;
      }
    }
    if (k == 0) continue;
    select_topk<PER>(v, live, k, renorm, ids + static_cast<size_t>(t) * k,
                     wout + static_cast<size_t>(t) * k);
  }
  cluster.sync();   // no CTA leaves while another still reads its partial tile
}

template <int EPAD, bool BF16>
cudaError_t launch_t(const void* x, const void* W, const float* b, int T, int H, int E, int k,
                     int renorm, float* logits, int32_t* ids, float* w, cudaStream_t s) {
  const size_t smem = sizeof(float) * (KC * BT + KC * EPAD + BT * (EPAD + 1));
  auto fn = route_kernel<EPAD, BF16>;
  cudaError_t err = moe_host::ensure_smem(reinterpret_cast<const void*>(fn), (int)smem);
  if (err != cudaSuccess) return err;
  const int tiles = (T + BT - 1) / BT;
  const int chunks = (H + KC - 1) / KC;
  // Enough CTAs for ~4 per SM, never more than one chunk of H each.
  int S = (4 * moe_host::num_sms() + tiles - 1) / tiles;
  S = std::max(1, std::min({S, MAX_S, chunks}));
  const int kc_per_cta = (chunks + S - 1) / S;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(S, tiles, 1);
  cfg.blockDim = dim3(NT, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = S;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  err = cudaLaunchKernelEx(&cfg, fn, x, W, b, T, H, E, k, renorm, kc_per_cta, logits, ids, w);
  if (err != cudaSuccess) return err;
  return cudaGetLastError();
}

}  // namespace

namespace moe_host {

cudaError_t launch_route(const void* x, const void* W_gate, const float* bias, int T, int H,
                         int E, int k, int renormalize, int dtype, float* logits, int32_t* ids,
                         float* w, cudaStream_t s) {
  const bool bf = dtype == MOE_BF16;
  if (T <= 64 && E <= 64) {
    if (bf)
      route_small_kernel<true><<<T, NT, 0, s>>>(x, W_gate, bias, H, E, k, renormalize, logits,
                                                ids, w);
    else
      route_small_kernel<false><<<T, NT, 0, s>>>(x, W_gate, bias, H, E, k, renormalize, logits,
                                                 ids, w);
    return cudaGetLastError();
  }
#define MOE_ROUTE_CASE(EP)                                                                  \
  if (E <= EP)                                                                              \
    return bf ? launch_t<EP, true>(x, W_gate, bias, T, H, E, k, renormalize, logits, ids, w, \
                                   s)                                                       \
              : launch_t<EP, false>(x, W_gate, bias, T, H, E, k, renormalize, logits, ids, w, s);
  MOE_ROUTE_CASE(64)
  MOE_ROUTE_CASE(128)
  MOE_ROUTE_CASE(256)
#undef MOE_ROUTE_CASE
  return cudaErrorInvalidValue;
}

}  // namespace moe_host
