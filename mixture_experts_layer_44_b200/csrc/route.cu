// Router: gating GEMM on the CUDA cores (fp32 FMA), fused with softmax,
// warp-shuffle top-k and renormalisation.
//
// DWDP-Triton-MoE-Inference-Engine README, "Router Module": router logits,
// routing probabilities, top-k expert indices, normalized routing weights.
// diffulex.moe API reference, "diffulex.moe.topk": NaiveTopKRouter.
//
// One CTA (256 threads) owns BT = 64 tokens and all E experts.  The
// contraction over H runs in chunks of KC = 32: the chunk of x and of W_gate
// is converted to fp32 and staged transposed in shared memory, and each
// thread accumulates a 4-token x (EPAD/16)-expert register tile (EPAD =
// 64, 128 or 256: E rounded up).  The
// logits tile then goes through shared memory to one warp per token, which
// adds the bias, writes the logits, and selects the top k by k rounds of a
// warp arg-max on the key (logit descending, expert id ascending).
#include <float.h>

#include <algorithm>

#include "common.cuh"

namespace {

constexpr int BT = 64;    // tokens per CTA
constexpr int KC = 32;    // H chunk
constexpr int TT = 4;     // tokens per thread
constexpr int NT = 256;   // threads

__device__ __forceinline__ bool better(float v1, int i1, float v2, int i2) {
  return v1 > v2 || (v1 == v2 && i1 < i2);
}

template <int EPAD, bool BF16>
__global__ void __launch_bounds__(NT) route_kernel(const void* __restrict__ xv,
                                                   const void* __restrict__ wv,
                                                   const float* __restrict__ bias, int T, int H,
                                                   int E, int k, int renorm,
                                                   float* __restrict__ logits,
                                                   int32_t* __restrict__ ids,
                                                   float* __restrict__ wout) {
  constexpr int TE = EPAD / 16;            // experts per thread
  constexpr int LS = EPAD + 1;             // padded row of the logits tile
  extern __shared__ __align__(16) float sm[];
  float* x_s = sm;                         // [KC][BT]
  float* w_s = sm + KC * BT;               // [KC][EPAD]
  float* l_s = sm;                         // [BT][LS], reused after the GEMM

  const int tid = threadIdx.x;
  const int eg = tid & 15;
  const int tg = tid >> 4;
  const int t0 = blockIdx.x * BT;

  float acc[TT][TE];
#pragma unroll
  for (int i = 0; i < TT; ++i)
#pragma unroll
    for (int j = 0; j < TE; ++j) acc[i][j] = 0.f;

  for (int h0 = 0; h0 < H; h0 += KC) {
    // x chunk: BT tokens x KC columns = 256 vectors of 8 elements, one per thread.
    {
      const int t = tid >> 2, v = tid & 3;
      const int hh = h0 + v * 8;
      float f[8];
      if (t0 + t < T && hh < H) {
        if (BF16) {
          const uint4 q = *reinterpret_cast<const uint4*>(
              static_cast<const __nv_bfloat16*>(xv) + static_cast<size_t>(t0 + t) * H + hh);
          moe::unpack8(q, f);
        } else {
          const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(xv) +
                                                            static_cast<size_t>(t0 + t) * H + hh);
          const float4 a = p[0], b = p[1];
          f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
          f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
        }
      } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) f[j] = 0.f;
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) x_s[(v * 8 + j) * BT + t] = f[j];
    }
    // W_gate chunk: EPAD experts x KC columns.
    for (int i = tid; i < EPAD * (KC / 8); i += NT) {
      const int e = i >> 2, v = i & 3;
      const int hh = h0 + v * 8;
      float f[8];
      if (e < E && hh < H) {
        if (BF16) {
          const uint4 q = *reinterpret_cast<const uint4*>(
              static_cast<const __nv_bfloat16*>(wv) + static_cast<size_t>(e) * H + hh);
          moe::unpack8(q, f);
        } else {
          const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(wv) +
                                                            static_cast<size_t>(e) * H + hh);
          const float4 a = p[0], b = p[1];
          f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
          f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
        }
      } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) f[j] = 0.f;
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) w_s[(v * 8 + j) * EPAD + e] = f[j];
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < KC; ++kk) {
      const float4 xq = *reinterpret_cast<const float4*>(&x_s[kk * BT + tg * TT]);
      const float xr[TT] = {xq.x, xq.y, xq.z, xq.w};
      float wr[TE];
#pragma unroll
      for (int j = 0; j < TE; j += 4) {
        const float4 q = *reinterpret_cast<const float4*>(&w_s[kk * EPAD + eg * TE + j]);
        wr[j] = q.x; wr[j + 1] = q.y; wr[j + 2] = q.z; wr[j + 3] = q.w;
      }
#pragma unroll
      for (int i = 0; i < TT; ++i)
#pragma unroll
        for (int j = 0; j < TE; ++j) acc[i][j] = fmaf(xr[i], wr[j], acc[i][j]);
    }
    __syncthreads();
  }

  // Logits tile to shared memory.
#pragma unroll
  for (int i = 0; i < TT; ++i)
#pragma unroll
    for (int j = 0; j < TE; ++j) l_s[(tg * TT + i) * LS + eg * TE + j] = acc[i][j];
  __syncthreads();

  // One warp per token: bias, logits out, softmax, top-k, weights.
  constexpr int PER = EPAD / 32;
  const int warp = tid >> 5, lane = tid & 31;
  for (int tl = warp; tl < BT; tl += NT / 32) {
    const int t = t0 + tl;
    if (t >= T) break;
    float v[PER];
    bool live[PER];
#pragma unroll
    for (int j = 0; j < PER; ++j) {
      const int e = lane + 32 * j;
      live[j] = e < E;
      v[j] = live[j] ? l_s[tl * LS + e] + (bias ? bias[e] : 0.f) : -FLT_MAX;
      if (live[j]) logits[static_cast<size_t>(t) * E + e] = v[j];
    }
    if (k == 0) continue;
    // Max over all experts and sum of exp(l - max).
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

    // k rounds of warp arg-max on (value desc, id asc) over experts not yet taken.
    bool taken[PER];
#pragma unroll
    for (int j = 0; j < PER; ++j) taken[j] = !live[j];
    int sel_id[moe::kMaxTopK];
    float sel_v[moe::kMaxTopK];
    for (int r = 0; r < k; ++r) {
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
      sel_id[r] = bi;
      sel_v[r] = bv;
#pragma unroll
      for (int j = 0; j < PER; ++j)
        if (lane + 32 * j == bi) taken[j] = true;
    }
    if (lane == 0) {
      float ex[moe::kMaxTopK];
      float ssel = 0.f;
      for (int r = 0; r < k; ++r) {
        ex[r] = expf(sel_v[r] - m);
        ssel += ex[r];
      }
      const float denom = renorm ? ssel : s;
      for (int r = 0; r < k; ++r) {
        ids[static_cast<size_t>(t) * k + r] = sel_id[r];
        wout[static_cast<size_t>(t) * k + r] = ex[r] / denom;
      }
    }
  }
}

template <int EPAD, bool BF16>
cudaError_t launch_t(const void* x, const void* W, const float* b, int T, int H, int E, int k,
                     int renorm, float* logits, int32_t* ids, float* w, cudaStream_t s) {
  const size_t smem = sizeof(float) * std::max(KC * BT + KC * EPAD, BT * (EPAD + 1));
  auto fn = route_kernel<EPAD, BF16>;
  cudaError_t err =
      cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  const int grid = (T + BT - 1) / BT;
  fn<<<grid, NT, smem, s>>>(x, W, b, T, H, E, k, renorm, logits, ids, w);
  return cudaGetLastError();
}

}  // namespace

namespace moe_host {

cudaError_t launch_route(const void* x, const void* W_gate, const float* bias, int T, int H,
                         int E, int k, int renormalize, int dtype, float* logits, int32_t* ids,
                         float* w, cudaStream_t s) {
  const bool bf = dtype == MOE_BF16;
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
