// Merger: inverse-permutation gather-reduce back to token order.
//
// DWDP-Triton-MoE-Inference-Engine README, "Merger Module": restore
// token-major assignment order, accumulate the top-k expert outputs, reshape
// to the token layout.  out[t] = sum_{j<k} y_packed[inv_perm[t*k+j]] in j
// order with an fp32 accumulator (deterministic: no atomics), plus
// sigmoid(gate_logit[t]) * shared[t] for the always-on shared expert
// (diffulex.moe.layer, SharedExpertMLP).
//
// y_packed and the shared expert's output come in the executor's output type
// (fp16 or fp32); the k terms and the shared term are added in fp32 and
// rounded once, to the output type.
//
// One CTA per token at a time (grid-stride over tokens); each thread owns
// 16-byte vectors of the hidden dimension, so every load and store is a
// 128-bit access.  The k source rows of a token are independent loads that
// are all in flight together.
//
// Masked-local merge (expert parallelism, metrale ep_dispatch.rs: "the served
// EP MoE is masked-local plus all-reduce"): with an expert range, only rows
// of the experts [lo_e, hi_e) -- packed rows [offsets[lo_e], offsets[hi_e)) --
// are added; a rank's other assignments belong to other ranks' experts.  The
// partial sums of all ranks are then added across ranks and rounded once by
// moe_finalize.
#include <algorithm>

#include "common.cuh"

namespace {

constexpr int CNT = 256;   // threads per CTA of the finalize kernel

// Eight consecutive elements of an fp32 or fp16 row, as fp32 (read at L2:
// the rows come from the kernels just before).
template <bool BF>
struct Vec8;
template <>
struct Vec8<false> {
  float4 a, b;
  __device__ __forceinline__ void load(const void* base, size_t row, int H, int v) {
    const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(base) + row * H) + 2 * v;
    a = moe::ld_prod(p);
    b = moe::ld_prod(p + 1);
  }
  __device__ __forceinline__ void get(float* f) const {
    f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
    f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
  }
};
template <>
struct Vec8<true> {
  uint4 q;
  __device__ __forceinline__ void load(const void* base, size_t row, int H, int v) {
    q = moe::ld_prod(reinterpret_cast<const uint4*>(static_cast<const __half*>(base) + row * H) +
                     v);
  }
  __device__ __forceinline__ void get(float* f) const { moe::unpack8_f16(q, f); }
};

// NT threads per CTA (one token at a time): 256 while the tokens fit one
// wave of 8 CTAs per SM (decode: the shortest chain per token), 128 above it
// (16 tokens in flight per SM: Qwen1.5 T = 8192 merger 51 -> 44 us).
template <bool Y_F16, bool OUT_BF16, int KT, int NT>
__global__ void __launch_bounds__(NT) combine_kernel(const void* y,
                                                      const int32_t* inv_perm,
                                                      int T, int H, int k, int N,
                                                      const void* shared,
                                                      const float* sgate,
                                                      const int32_t* range_offs,
                                                      int lo_e, int hi_e,
                                                      void* __restrict__ outv, int32_t* status) {
  const int nvec = H / 8;                               // 8 outputs per thread step
  __shared__ int rows[moe::kMaxTopK];
  __shared__ float gate;
  moe::grid_dep_wait();
  int rlo = 0, rhi = N;                                 // rows that contribute
  if (range_offs != nullptr) {
    rlo = moe::ld_prod(range_offs + lo_e);
    rhi = moe::ld_prod(range_offs + hi_e);
  }
  for (int t = blockIdx.x; t < T; t += gridDim.x) {
    __syncthreads();
    if (threadIdx.x < k) {
      int p = moe::ld_prod(inv_perm + static_cast<size_t>(t) * k + threadIdx.x);
      if (p < 0 || p >= N) {
        moe::report(status, MOE_ERR_BAD_INDEX);
        p = -1;
      } else if (p < rlo || p >= rhi) {
        p = -1;                                         // another rank's expert
      }
      rows[threadIdx.x] = p;
    }
    if (threadIdx.x == 0)
      gate = shared ? (sgate ? 1.f / (1.f + expf(-moe::ld_prod(sgate + t))) : 1.f) : 0.f;
    __syncthreads();
    for (int v = threadIdx.x; v < nvec; v += NT) {
      float acc[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = 0.f;
      // all k rows' loads first (in flight together), then the sums in j order
      Vec8<Y_F16> yv[KT];
#pragma unroll
      for (int j = 0; j < KT; ++j)
        if (rows[j] >= 0) yv[j].load(y, static_cast<size_t>(rows[j]), H, v);
#pragma unroll
      for (int j = 0; j < KT; ++j) {
        if (rows[j] >= 0) {
          float f[8];
          yv[j].get(f);
#pragma unroll
          for (int i = 0; i < 8; ++i) acc[i] += f[i];
        }
      }
      if (shared) {
        const float g = gate;
        Vec8<Y_F16> sv;
        sv.load(shared, static_cast<size_t>(t), H, v);
        float f[8];
        sv.get(f);
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = fmaf(g, f[i], acc[i]);
      }
      if (OUT_BF16) {
        reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(outv) + static_cast<size_t>(t) * H)[v] =
            make_uint4(moe::pack_bf16x2(acc[0], acc[1]), moe::pack_bf16x2(acc[2], acc[3]),
                       moe::pack_bf16x2(acc[4], acc[5]), moe::pack_bf16x2(acc[6], acc[7]));
      } else {
        float4* dst = reinterpret_cast<float4*>(static_cast<float*>(outv) + static_cast<size_t>(t) * H) + 2 * v;
        dst[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
        dst[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
      }
    }
  }
  moe::grid_dep_launch();
}

// out = acc rounded once to the output type (bf16 or fp32 copy).
template <bool OUT_BF16>
__global__ void __launch_bounds__(CNT) finalize_kernel(const float4* acc,
                                                       size_t nvec8, void* __restrict__ outv) {
  moe::grid_dep_wait();
  for (size_t v = blockIdx.x * static_cast<size_t>(CNT) + threadIdx.x; v < nvec8;
       v += static_cast<size_t>(gridDim.x) * CNT) {
    const float4 a = moe::ld_prod(acc + 2 * v), b = moe::ld_prod(acc + 2 * v + 1);
    if (OUT_BF16) {
      reinterpret_cast<uint4*>(outv)[v] =
          make_uint4(moe::pack_bf16x2(a.x, a.y), moe::pack_bf16x2(a.z, a.w),
                     moe::pack_bf16x2(b.x, b.y), moe::pack_bf16x2(b.z, b.w));
    } else {
      float4* d = reinterpret_cast<float4*>(outv) + 2 * v;
      d[0] = a;
      d[1] = b;
    }
  }
  moe::grid_dep_launch();
}

}  // namespace

namespace moe_host {

cudaError_t launch_finalize(const float* acc, int T, int H, int dtype, void* out,
                            cudaStream_t s) {
  const size_t nvec8 = static_cast<size_t>(T) * H / 8;
  const int grid = static_cast<int>(std::max<size_t>(
      1, std::min<size_t>((nvec8 + CNT - 1) / CNT, static_cast<size_t>(num_sms()) * 8)));
  const float4* a = reinterpret_cast<const float4*>(acc);
  return dtype == MOE_BF16
             ? launch_pdl(finalize_kernel<true>, dim3(grid), dim3(CNT), 0, s, 0, a, nvec8, out)
             : launch_pdl(finalize_kernel<false>, dim3(grid), dim3(CNT), 0, s, 0, a, nvec8, out);
}

template <bool Y_F16, bool OUT_BF16>
cudaError_t launch_combine_t(const void* y, const int32_t* inv_perm, int T, int H, int k,
                             const void* shared, const float* shared_gate, void* out,
                             int32_t* status, cudaStream_t s, const int32_t* range_offs,
                             int lo_e, int hi_e) {
  const bool narrow = T > num_sms() * 8;
  const int grid = std::max(1, std::min(T, num_sms() * (narrow ? 16 : 8)));
  const int N = T * k;
  // k is a template parameter so that exactly k rows are loaded, all in flight.
#define MOE_COMBINE_K(KV)                                                                      \
  case KV:                                                                                     \
    return narrow ? launch_pdl(combine_kernel<Y_F16, OUT_BF16, KV, 128>, dim3(grid), dim3(128), \
                               0, s, 0, y, inv_perm, T, H, k, N, shared, shared_gate,          \
                               range_offs, lo_e, hi_e, out, status)                            \
                  : launch_pdl(combine_kernel<Y_F16, OUT_BF16, KV, 256>, dim3(grid), dim3(256), \
                               0, s, 0, y, inv_perm, T, H, k, N, shared, shared_gate,          \
                               range_offs, lo_e, hi_e, out, status);
  switch (k) {
    MOE_COMBINE_K(1)
    MOE_COMBINE_K(2)
    MOE_COMBINE_K(3)
    MOE_COMBINE_K(4)
    MOE_COMBINE_K(5)
    MOE_COMBINE_K(6)
    MOE_COMBINE_K(7)
    MOE_COMBINE_K(8)
    default:
      return cudaErrorInvalidValue;
  }
#undef MOE_COMBINE_K
}

cudaError_t launch_combine(const void* y, int y_dtype, const int32_t* inv_perm, int T, int H,
                           int k, const void* shared, const float* shared_gate, int dtype,
                           void* out, int32_t* status, cudaStream_t s,
                           const int32_t* range_offs, int lo_e, int hi_e) {
  const bool yb = y_dtype == MOE_F16, ob = dtype == MOE_BF16;
  if (yb && ob)
    return launch_combine_t<true, true>(y, inv_perm, T, H, k, shared, shared_gate, out, status,
                                        s, range_offs, lo_e, hi_e);
  if (yb)
    return launch_combine_t<true, false>(y, inv_perm, T, H, k, shared, shared_gate, out, status,
                                         s, range_offs, lo_e, hi_e);
  if (ob)
    return launch_combine_t<false, true>(y, inv_perm, T, H, k, shared, shared_gate, out, status,
                                         s, range_offs, lo_e, hi_e);
  return launch_combine_t<false, false>(y, inv_perm, T, H, k, shared, shared_gate, out, status,
                                        s, range_offs, lo_e, hi_e);
}

}  // namespace moe_host
