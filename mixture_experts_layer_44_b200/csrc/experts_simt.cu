// Executor, fp32: grouped SwiGLU experts in true fp32 on the CUDA cores.
//
// Same contract as the tensor-core path (DWDP README, "Executor Module";
// fused w13 [E, 2I, H] with gate w1 in rows [0,I) and up w3 in rows [I,2I)),
// for workloads whose activations and weights are fp32: TF32 tensor cores
// would not keep the 1e-5 relative bound, so these two passes use fp32 FMA.
//
// Tile = 64 packed rows of one expert x 64 output columns, K in chunks of 16
// staged in shared memory; each thread owns a 4 x 4 register tile (pass 1:
// 4 x 4 gate and 4 x 4 up accumulators).  The tile list (per-expert row
// tiles, exclusive scan) is rebuilt from `offsets` by every CTA; CTAs past
// the last tile exit.
#include <algorithm>

#include "common.cuh"

namespace {

constexpr int SBM = 64, SBN = 64, SBK = 16;
constexpr int SNT = 256;

enum { EPI_SWIGLU = 0, EPI_SCALE = 1 };

// Fill tstart[0..E] (token tiles per expert, exclusive scan) and offs[0..E].
__device__ void build_tiles(const int32_t* offsets, int E, int* offs, int* tstart) {
  if (threadIdx.x == 0) {
    int run = 0;
    for (int e = 0; e < E; ++e) {
      const int o0 = moe::ld_prod(offsets + e), o1 = moe::ld_prod(offsets + e + 1);
      offs[e] = o0;
      tstart[e] = run;
      run += (o1 - o0 + SBM - 1) / SBM;
    }
    offs[E] = moe::ld_prod(offsets + E);
    tstart[E] = run;
  }
  __syncthreads();
}

template <int EPI>
__global__ void __launch_bounds__(SNT) simt_gemm_kernel(const float* A, int K,
                                                        const int32_t* offsets,
                                                        int E, const float* __restrict__ B,
                                                        int rows_per_expert, int I,
                                                        const float* pw,
                                                        float* __restrict__ out, int ldo) {
  __shared__ int offs[moe::kMaxExperts + 1];
  __shared__ int tstart[moe::kMaxExperts + 1];
  constexpr int NB = EPI == EPI_SWIGLU ? 2 * SBN : SBN;   // weight rows staged per chunk
  __shared__ __align__(16) float As[SBK][SBM + 4];
  __shared__ __align__(16) float Bs[SBK][NB + 4];

  moe::grid_dep_wait();
  build_tiles(offsets, E, offs, tstart);
  const int t = blockIdx.x;
  if (t >= tstart[E]) return;
  int e = 0;
  while (e + 1 < E && tstart[e + 1] <= t) ++e;
  const int r0 = offs[e] + (t - tstart[e]) * SBM;      // first packed row
  const int rend = offs[e + 1];
  const int c0 = blockIdx.y * SBN;                      // first output column
  const float* Be = B + static_cast<size_t>(e) * rows_per_expert * K;

  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4] = {};
  float acu[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += SBK) {
    for (int i = threadIdx.x; i < SBM * SBK; i += SNT) {
      const int r = i / SBK, kk = i % SBK;
      const int gr = r0 + r, gk = k0 + kk;
      As[kk][r] = (gr < rend && gk < K) ? moe::ld_prod(A + static_cast<size_t>(gr) * K + gk) : 0.f;
    }
    for (int i = threadIdx.x; i < NB * SBK; i += SNT) {
      const int r = i / SBK, kk = i % SBK;
      const int gk = k0 + kk;
      int wrow;
      if (EPI == EPI_SWIGLU) wrow = r < SBN ? c0 + r : I + c0 + (r - SBN);
      else wrow = c0 + r;
      const bool ok = gk < K && (EPI == EPI_SWIGLU ? (c0 + (r % SBN)) < I : wrow < rows_per_expert);
      Bs[kk][r] = ok ? Be[static_cast<size_t>(wrow) * K + gk] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < SBK; ++kk) {
      float a[4], b[4], u[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tx * 4 + j];
      if (EPI == EPI_SWIGLU) {
#pragma unroll
        for (int j = 0; j < 4; ++j) u[j] = Bs[kk][SBN + tx * 4 + j];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
          if (EPI == EPI_SWIGLU) acu[i][j] = fmaf(a[i], u[j], acu[i][j]);
        }
    }
    __syncthreads();
  }
  const int ncols = EPI == EPI_SWIGLU ? I : rows_per_expert;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int gr = r0 + ty * 4 + i;
    if (gr >= rend) continue;
    const float sc = EPI == EPI_SCALE ? (pw ? moe::ld_prod(pw + gr) : 1.f) : 1.f;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int gc = c0 + tx * 4 + j;
      if (gc >= ncols) continue;
      float v;
      if (EPI == EPI_SWIGLU) {
        const float g = acc[i][j];
        v = g / (1.f + expf(-g)) * acu[i][j];
      } else {
        v = acc[i][j] * sc;
      }
      out[static_cast<size_t>(gr) * ldo + gc] = v;
    }
  }
  moe::grid_dep_launch();
}

}  // namespace

namespace moe_host {

cudaError_t launch_experts_simt(const void* x_packed, const int32_t* offsets,
                                const float* packed_w, const void* w13, const void* w2, int N,
                                int H, int I, int E, void* h, void* y, cudaStream_t s) {
  const int mt_bound = (N + SBM - 1) / SBM + E;
  dim3 g1(mt_bound, (I + SBN - 1) / SBN);
  const float* no_w = nullptr;
  cudaError_t err = launch_pdl(simt_gemm_kernel<EPI_SWIGLU>, g1, dim3(SNT), 0, s, 0,
                               static_cast<const float*>(x_packed), H, offsets, E,
                               static_cast<const float*>(w13), 2 * I, I, no_w,
                               static_cast<float*>(h), I);
  if (err != cudaSuccess) return err;
  dim3 g2(mt_bound, (H + SBN - 1) / SBN);
  return launch_pdl(simt_gemm_kernel<EPI_SCALE>, g2, dim3(SNT), 0, s, 0,
                    static_cast<const float*>(h), I, offsets, E, static_cast<const float*>(w2), H,
                    I, packed_w, static_cast<float*>(y), H);
}

}  // namespace moe_host
