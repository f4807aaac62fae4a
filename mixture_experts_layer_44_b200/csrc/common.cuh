// Shared helpers of the libmoe_b200 kernels: status codes, bf16 conversion,
// vector types and the bounded-wait clock.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include <string>
#include <utility>

#include "../../include/moe_b200.h"

namespace moe {

// Largest sizes the kernels are written for (checked on the host).
constexpr int kMaxExperts = 256;
constexpr int kMaxTopK = 8;

// Budget of every bounded wait in a kernel (nanoseconds).  A correct kernel
// waits microseconds at most; the budget only bounds a wait that would
// otherwise never end, after which the kernel reports MOE_ERR_TIMEOUT.
constexpr uint64_t kWaitBudgetNs = 2000ull * 1000ull * 1000ull;

// Record the first device-side error in the caller's status word.
__device__ __forceinline__ void report(int32_t* status, int32_t code) {
  if (status != nullptr) atomicCAS(status, 0, code);
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ float bf16_to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }

// Programmatic dependent launch.  Every kernel here is launched so that it may
// start while the previous kernel on the stream finishes; it does its
// independent set-up, then grid_dep_wait() before the first read of anything
// the previous kernel wrote (the wait returns once that kernel has completed
// and its writes are visible).  grid_dep_launch() lets the next kernel begin
// launching once every CTA of this one has called it (or exited).
__device__ __forceinline__ void grid_dep_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void grid_dep_launch() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Loads of data that an earlier kernel of the stream produced.  Every kernel
// here is launched with programmatic dependent launch, so it can be resident
// while its producer still runs; the read-only data path (ld.global.nc) is
// only valid for data that stays constant for a kernel's whole lifetime.
// Such data is therefore read at L2, the point of coherence (ld.global.cg),
// after griddepcontrol.wait.  Constant weights keep the read-only path.
template <typename T>
__device__ __forceinline__ T ld_prod(const T* p) {
  return __ldcg(p);
}

// Unpack 8 bf16 (one 16-byte vector) into floats.
__device__ __forceinline__ void unpack8(const uint4& v, float* f) {
  const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 t = __bfloat1622float2(p[i]);
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}

// 16-byte read-only global load, issued where it stands: a batch of these is
// in flight together before any of the values is used.
__device__ __forceinline__ uint4 ld_nc_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 t = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&t);
}

// Two fp32 values rounded to fp16 (nearest even), lo in the low half.
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  __half2 t = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&t);
}

// Eight fp16 values (one 16-byte word) as fp32.
__device__ __forceinline__ void unpack8_f16(const uint4& v, float* f) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    __half2 h = *reinterpret_cast<const __half2*>(&w[i]);
    const float2 t = __half22float2(h);
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}

// Largest finite fp16 value: a larger fp32 value does not fit an fp16 output.
constexpr float kF16Max = 65504.f;

}  // namespace moe

// Host-side internal launchers (one translation unit each).  They assume the
// arguments were validated by the ABI layer and return a cudaError_t.
namespace moe_host {
// n_groups > 1: group-limited selection (topk_groups of n_groups groups kept).
cudaError_t launch_route(const void* x, const void* W_gate, const float* bias, int T, int H,
                         int E, int k, int renormalize, int dtype, float* logits,
                         int32_t* ids, float* w, int32_t* status, cudaStream_t s,
                         int n_groups = 1, int topk_groups = 1);
// launch_route plus the shared expert's gate logit sg[t] = x[t] . wsg: in the
// same launch where the router has room for it (small batches with E + 1 <=
// 64; the bf16 tensor-core router), else a second launch.
cudaError_t launch_route_gated(const void* x, const void* W_gate, const float* bias,
                               const void* wsg, int T, int H, int E, int k, int renormalize,
                               int dtype, float* logits, int32_t* ids, float* w, float* sg,
                               int32_t* status, cudaStream_t s, int n_groups, int topk_groups);
// Router and dispatcher in one launch (T <= 64, E <= 64, H <= 32768,
// 1 <= k <= 8; with a shared expert's gate row wsg, E + 1 <= 64, and its
// logit per token goes to sg): route_dispatch_fits says whether a shape
// qualifies.
bool route_dispatch_fits(int T, int H, int E, int k, bool gate = false);
cudaError_t launch_route_dispatch(const void* x, const void* W_gate, const float* bias, int T,
                                  int H, int E, int k, int renormalize, int dtype, float* logits,
                                  int32_t* ids, float* w, int32_t* counts, int32_t* offsets,
                                  int32_t* perm, int32_t* inv_perm, int32_t* packed_tok,
                                  float* packed_w, void* x_packed, int32_t* counter,
                                  int32_t* status, cudaStream_t s, int n_groups = 1,
                                  int topk_groups = 1, const void* wsg = nullptr,
                                  float* sg = nullptr);
// With wsg (bf16 [H]) the shared expert's gate logit x . wsg goes to sg [T] in
// the same launch; cudaErrorNotSupported when a CTA's slice of H is too long
// to stage it.
cudaError_t launch_route_tc(const void* x, const void* W_gate, const float* bias, int T, int H,
                            int E, int k, int renormalize, float* logits, int32_t* ids, float* w,
                            int32_t* status, cudaStream_t s, int n_groups, int topk_groups,
                            const void* wsg = nullptr, float* sg = nullptr);
size_t dispatch_ws_bytes(int T, int k, int E);
cudaError_t launch_dispatch(const int32_t* ids, const float* w, const void* x, int T, int H,
                            int E, int k, int dtype, int32_t* counts, int32_t* offsets,
                            int32_t* perm, int32_t* inv_perm, int32_t* packed_tok,
                            float* packed_w, void* x_packed, void* ws, int32_t* status,
                            cudaStream_t s);
size_t experts_ws_bytes();
// The optional shared expert of moe_experts_shared: every row of x [T,H]
// through w13 [2I,H] / w2 [H,I] into h [T,I] (bf16) and y [T,H] (fp32).
struct SharedGroup {
  const void* x;
  int T;
  const void* w13;
  const void* w2;
  int I;
  void* h;
  void* y;
};
cudaError_t launch_experts_tc(const void* x_packed, const int32_t* offsets,
                              const float* packed_w, const void* w13, const void* w2, int N,
                              int H, int I, int E, void* h, void* y, bool y_f16,
                              const SharedGroup* sh,
                              void* ws, size_t ws_bytes, int32_t* status, cudaStream_t s,
                              const char** why);
cudaError_t launch_experts_simt(const void* x_packed, const int32_t* offsets,
                                const float* packed_w, const void* w13, const void* w2, int N,
                                int H, int I, int E, void* h, void* y, cudaStream_t s);
// range_offs != NULL: only packed rows [range_offs[lo_e], range_offs[hi_e]) are added.
cudaError_t launch_combine(const void* y, int y_dtype, const int32_t* inv_perm, int T, int H,
                           int k, const void* shared, const float* shared_gate, int dtype,
                           void* out,
                           int32_t* status, cudaStream_t s, const int32_t* range_offs = nullptr,
                           int lo_e = 0, int hi_e = 0);
cudaError_t launch_finalize(const float* acc, int T, int H, int dtype, void* out,
                            cudaStream_t s);
// Rows [offsets[lo_e], offsets[hi_e]) of x_packed gathered from x by packed_tok.
cudaError_t launch_gather(const void* x, const int32_t* packed_tok, const int32_t* offsets,
                          int lo_e, int hi_e, int N, int H, int dtype, void* x_packed,
                          int32_t* status, cudaStream_t s);
size_t ep_partition_ws_bytes(long long n);
cudaError_t launch_ep_partition(const int32_t* ids, const float* w, int n, int top_k,
                                unsigned lo, unsigned hi, int32_t* l_tok, int32_t* l_eid,
                                float* l_w, int32_t* r_tok, int32_t* r_eid, float* r_w,
                                int32_t* bucket_counts, void* ws, cudaStream_t s);
cudaError_t launch_ep_owner(const int32_t* ids, int n, int E, int R, int32_t* owner,
                            int32_t* status, cudaStream_t s);
cudaError_t launch_ep_pack_ids(const int32_t* ids, const int32_t* perm, const int32_t* offsets,
                               int n, int E, int R, int32_t* local, cudaStream_t s);
cudaError_t launch_probe_wait_timeout(int32_t* status, int budget_us, cudaStream_t s);
int num_sms();
void set_last_error(const std::string& msg);   // the message moe_last_error() returns
// cudaFuncSetAttribute(MaxDynamicSharedMemorySize) once per (device, kernel, size).
cudaError_t ensure_smem(const void* kernel, int bytes);

// Count one kernel enqueued by this library (moe_launch_count).
void note_launch();

// Budget of the main-loop waits of the tensor-core kernels (nanoseconds):
// kWaitBudgetNs unless moe_test_set_wait_budget_ns shortened it.
uint64_t main_wait_budget_ns();

// Launch with programmatic stream serialization (and a cluster of cluster_x
// CTAs along x when cluster_x > 0).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t s, int cluster_x, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  int n = 0;
  attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[n].val.programmaticStreamSerializationAllowed = 1;
  ++n;
  if (cluster_x > 0) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = cluster_x;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e == cudaSuccess) note_launch();
  return e;
}
}  // namespace moe_host
