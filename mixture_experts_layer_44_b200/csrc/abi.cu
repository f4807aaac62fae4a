// extern "C" entry points of libmoe_b200.so (declared in include/moe_b200.h):
// host-side argument checks, then the stage launchers.  No call allocates
// device memory or synchronises the stream (except moe_read_status).
#include <stdio.h>
#include <string.h>

#include <atomic>
#include <map>
#include <mutex>
#include <string>
#include <tuple>

#include "common.cuh"
#include "sm100_ptx.cuh"

namespace {

thread_local std::string g_err;
std::atomic<unsigned long long> g_launches{0};
std::atomic<unsigned long long> g_main_wait_ns{moe::kWaitBudgetNs};

int fail(int code, const std::string& msg) {
  g_err = msg;
  return code;
}

int cuda_fail(cudaError_t e, const char* where) {
  g_err = std::string(where) + ": " + cudaGetErrorString(e);
  return MOE_ERR_CUDA;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

#define REQ(cond, code, msg)                 \
  do {                                       \
    if (!(cond)) return fail(code, msg);   \
  } while (0)

int check_dtype(int dtype) {
  if (dtype != MOE_F32 && dtype != MOE_BF16)
    return fail(MOE_ERR_INVALID_ARG, "dtype must be MOE_F32 (0) or MOE_BF16 (1)");
  return MOE_OK;
}

// The type of y_packed and of a shared expert's output.
int check_y_dtype(int y_dtype) {
  if (y_dtype != MOE_F32 && y_dtype != MOE_F16)
    return fail(MOE_ERR_INVALID_ARG, "y_dtype must be MOE_F32 (0) or MOE_F16 (2)");
  return MOE_OK;
}

// Bounded-wait self-test: one thread waits on an mbarrier nothing arrives on.
__global__ void probe_wait_kernel(int32_t* status, uint64_t budget_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x != 0) return;
  const uint32_t b = moe::smem_addr(&bar);
  moe::mbar_init(b, 1);
  moe::fence_barrier_init();
  if (!moe::mbar_wait(b, 0, budget_ns)) moe::report(status, MOE_ERR_TIMEOUT);
}

}  // namespace

namespace moe_host {
void set_last_error(const std::string& msg) { g_err = msg; }
void note_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }
uint64_t main_wait_budget_ns() { return g_main_wait_ns.load(std::memory_order_relaxed); }

cudaError_t ensure_smem(const void* kernel, int bytes) {
  static std::mutex mu;
  static std::map<std::tuple<int, const void*>, int> done;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  auto key = std::make_tuple(dev, kernel);
  auto it = done.find(key);
  if (it != done.end() && it->second >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) done[key] = bytes;
  return e;
}

cudaError_t launch_probe_wait_timeout(int32_t* status, int budget_us, cudaStream_t s) {
  probe_wait_kernel<<<1, 32, 0, s>>>(status, static_cast<uint64_t>(budget_us) * 1000ull);
  if (cudaPeekAtLastError() == cudaSuccess) moe_host::note_launch();
  return cudaGetLastError();
}
}  // namespace moe_host

extern "C" {

int moe_abi_version(void) { return 5; }

unsigned long long moe_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

const char* moe_last_error(void) { return g_err.c_str(); }

namespace {

int route_impl(const char* fn, const void* x, const void* W_gate, const float* bias, int T,
               int H, int E, int k, int renormalize, int n_groups, int topk_groups, int dtype,
               float* logits, int32_t* topk_ids, float* topk_w, int32_t* status, void* stream,
               const void* wsg = nullptr, float* sg = nullptr) {
  const std::string f = std::string(fn) + ": ";
  if (int r = check_dtype(dtype)) return r;
  REQ(x && W_gate && logits, MOE_ERR_INVALID_ARG, f + "null x, W_gate or logits");
  REQ(T >= 1 && H >= 1, MOE_ERR_INVALID_ARG, f + "T and H must be >= 1");
  REQ(E >= 1 && E <= moe::kMaxExperts, MOE_ERR_INVALID_ARG, f + "E must be in [1, 256]");
  REQ(k >= 0 && k <= E && k <= moe::kMaxTopK, MOE_ERR_INVALID_ARG,
      f + "k must be in [0, min(E, 8)]");
  REQ(k == 0 || (topk_ids && topk_w), MOE_ERR_INVALID_ARG, f + "null topk_ids or topk_w");
  REQ(H % 8 == 0, MOE_ERR_INVALID_ARG, f + "H must be a multiple of 8");
  REQ(aligned16(x) && aligned16(W_gate), MOE_ERR_INVALID_ARG,
      f + "x and W_gate must be 16-byte aligned");
  REQ(aligned4(logits) && aligned4(topk_ids) && aligned4(topk_w) && aligned4(bias) &&
          aligned4(status),
      MOE_ERR_INVALID_ARG, f + "outputs, bias and status must be 4-byte aligned");
  REQ(static_cast<long long>(T) * (H > E ? H : E) < (1ll << 31), MOE_ERR_INVALID_ARG,
      f + "T*H too large");
  if (n_groups > 1) {
    REQ(n_groups <= 32 && E % n_groups == 0, MOE_ERR_INVALID_ARG,
        f + "n_groups must divide E and be at most 32");
    REQ(topk_groups >= 1 && topk_groups <= n_groups, MOE_ERR_INVALID_ARG,
        f + "topk_groups must be in [1, n_groups]");
    REQ(k >= 1 && k <= topk_groups * (E / n_groups), MOE_ERR_INVALID_ARG,
        f + "k must be in [1, topk_groups * E / n_groups]");
  }
  cudaError_t e =
      wsg != nullptr
          ? moe_host::launch_route_gated(x, W_gate, bias, wsg, T, H, E, k, renormalize != 0,
                                         dtype, logits, topk_ids, topk_w, sg, status,
                                         static_cast<cudaStream_t>(stream), n_groups,
                                         topk_groups)
          : moe_host::launch_route(x, W_gate, bias, T, H, E, k, renormalize != 0, dtype,
                                   logits, topk_ids, topk_w, status,
                                   static_cast<cudaStream_t>(stream), n_groups, topk_groups);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, (f + "launch").c_str());
}

}  // namespace

int moe_route(const void* x, const void* W_gate, const float* bias, int T, int H, int E, int k,
              int renormalize, int dtype, float* logits, int32_t* topk_ids, float* topk_w,
              int32_t* status, void* stream) {
  g_err.clear();
  return route_impl("moe_route", x, W_gate, bias, T, H, E, k, renormalize, 1, 1, dtype, logits,
                    topk_ids, topk_w, status, stream);
}

int moe_route_grouped(const void* x, const void* W_gate, const float* bias, int T, int H, int E,
                      int k, int renormalize, int n_groups, int topk_groups, int dtype,
                      float* logits, int32_t* topk_ids, float* topk_w, int32_t* status,
                      void* stream) {
  g_err.clear();
  REQ(n_groups >= 1, MOE_ERR_INVALID_ARG, "moe_route_grouped: n_groups must be >= 1");
  return route_impl("moe_route_grouped", x, W_gate, bias, T, H, E, k, renormalize, n_groups,
                    topk_groups, dtype, logits, topk_ids, topk_w, status, stream);
}

int moe_route_gated(const void* x, const void* W_gate, const float* bias,
                    const void* w_gate_shared, int T, int H, int E, int k, int renormalize,
                    int n_groups, int topk_groups, int dtype, float* logits, int32_t* topk_ids,
                    float* topk_w, float* shared_gate_logit, int32_t* status, void* stream) {
  g_err.clear();
  REQ(n_groups >= 1, MOE_ERR_INVALID_ARG, "moe_route_gated: n_groups must be >= 1");
  REQ(w_gate_shared && shared_gate_logit, MOE_ERR_INVALID_ARG,
      "moe_route_gated: null w_gate_shared or shared_gate_logit");
  REQ(aligned16(w_gate_shared) && aligned4(shared_gate_logit), MOE_ERR_INVALID_ARG,
      "moe_route_gated: w_gate_shared must be 16-byte and shared_gate_logit 4-byte aligned");
  return route_impl("moe_route_gated", x, W_gate, bias, T, H, E, k, renormalize, n_groups,
                    topk_groups, dtype, logits, topk_ids, topk_w, status, stream, w_gate_shared,
                    shared_gate_logit);
}

size_t moe_dispatch_workspace_bytes(int T, int k, int E) {
  if (T < 1 || k < 1 || E < 1) return 0;
  return moe_host::dispatch_ws_bytes(T, k, E);
}

int moe_dispatch(const int32_t* topk_ids, const float* topk_w, const void* x, int T, int H, int E,
                 int k, int dtype, int32_t* counts, int32_t* offsets, int32_t* perm,
                 int32_t* inv_perm, int32_t* packed_tok, float* packed_w, void* x_packed,
                 void* ws, size_t ws_bytes, int32_t* status, void* stream) {
  g_err.clear();
  if (int r = check_dtype(dtype)) return r;
  REQ(topk_ids && counts && offsets && perm && inv_perm && packed_tok, MOE_ERR_INVALID_ARG,
      "moe_dispatch: null ids or output");
  REQ(!topk_w || packed_w, MOE_ERR_INVALID_ARG, "moe_dispatch: topk_w given but packed_w is null");
  REQ(T >= 1, MOE_ERR_INVALID_ARG, "moe_dispatch: T must be >= 1");
  REQ(E >= 1 && E <= moe::kMaxExperts, MOE_ERR_INVALID_ARG, "moe_dispatch: E must be in [1, 256]");
  REQ(k >= 1 && k <= moe::kMaxTopK, MOE_ERR_INVALID_ARG, "moe_dispatch: k must be in [1, 8]");
  REQ(static_cast<long long>(T) * k < (1ll << 30), MOE_ERR_INVALID_ARG, "moe_dispatch: T*k too large");
  REQ(aligned4(topk_ids) && aligned4(topk_w) && aligned4(counts) && aligned4(offsets) &&
          aligned4(perm) && aligned4(inv_perm) && aligned4(packed_tok) && aligned4(packed_w),
      MOE_ERR_INVALID_ARG, "moe_dispatch: index arrays must be 4-byte aligned");
  REQ(aligned4(status), MOE_ERR_INVALID_ARG, "moe_dispatch: status must be 4-byte aligned");
  if (x) {
    REQ(x_packed, MOE_ERR_INVALID_ARG, "moe_dispatch: x given but x_packed is null");
    REQ(H >= 1 && H % 8 == 0, MOE_ERR_INVALID_ARG, "moe_dispatch: H must be a positive multiple of 8");
    REQ(aligned16(x) && aligned16(x_packed), MOE_ERR_INVALID_ARG,
        "moe_dispatch: x and x_packed must be 16-byte aligned");
    REQ(static_cast<long long>(T) * k * H < (1ll << 40), MOE_ERR_INVALID_ARG,
        "moe_dispatch: T*k*H too large");
  }
  const size_t need = moe_host::dispatch_ws_bytes(T, k, E);
  REQ(ws && ws_bytes >= need && aligned16(ws), MOE_ERR_INVALID_ARG,
      "moe_dispatch: workspace missing, misaligned or smaller than moe_dispatch_workspace_bytes()");
  cudaError_t e = moe_host::launch_dispatch(topk_ids, topk_w, x, T, H, E, k, dtype, counts,
                                            offsets, perm, inv_perm, packed_tok, packed_w,
                                            x_packed, ws, status, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_dispatch launch");
}

int moe_route_dispatch(const void* x, const void* W_gate, const float* bias,
                       const void* w_gate_shared, int T, int H, int E, int k, int renormalize,
                       int n_groups, int topk_groups, int dtype, float* logits,
                       int32_t* topk_ids, float* topk_w, float* shared_gate_logit, int32_t* counts,
                       int32_t* offsets, int32_t* perm, int32_t* inv_perm, int32_t* packed_tok,
                       float* packed_w, void* x_packed, int32_t* counter, int32_t* status,
                       void* stream) {
  g_err.clear();
  if (int r = check_dtype(dtype)) return r;
  const std::string f = "moe_route_dispatch: ";
  REQ(x && W_gate && logits && topk_ids && topk_w, MOE_ERR_INVALID_ARG,
      f + "null x, W_gate, logits, topk_ids or topk_w");
  REQ(counts && offsets && perm && inv_perm && packed_tok && packed_w && counter,
      MOE_ERR_INVALID_ARG, f + "null dispatch output or counter");
  REQ((w_gate_shared == nullptr) == (shared_gate_logit == nullptr), MOE_ERR_INVALID_ARG,
      f + "w_gate_shared and shared_gate_logit come together");
  const int gate = w_gate_shared != nullptr ? 1 : 0;
  REQ(T >= 1 && T <= 64, MOE_ERR_INVALID_ARG, f + "T must be in [1, 64]");
  REQ(E >= 1 && E + gate <= 64, MOE_ERR_INVALID_ARG,
      f + (gate ? "E must be in [1, 63] with a shared gate" : "E must be in [1, 64]"));
  REQ(H >= 8 && H % 8 == 0 && H <= 32768, MOE_ERR_INVALID_ARG,
      f + "H must be a multiple of 8 in [8, 32768]");
  REQ(k >= 1 && k <= E && k <= moe::kMaxTopK, MOE_ERR_INVALID_ARG,
      f + "k must be in [1, min(E, 8)]");
  REQ(n_groups >= 1, MOE_ERR_INVALID_ARG, f + "n_groups must be >= 1");
  if (n_groups > 1) {
    REQ(n_groups <= 32 && E % n_groups == 0, MOE_ERR_INVALID_ARG,
        f + "n_groups must divide E and be at most 32");
    REQ(topk_groups >= 1 && topk_groups <= n_groups, MOE_ERR_INVALID_ARG,
        f + "topk_groups must be in [1, n_groups]");
    REQ(k <= topk_groups * (E / n_groups), MOE_ERR_INVALID_ARG,
        f + "k must be in [1, topk_groups * E / n_groups]");
  }
  REQ(aligned16(x) && aligned16(W_gate) && aligned16(x_packed) && aligned16(w_gate_shared),
      MOE_ERR_INVALID_ARG, f + "x, W_gate, w_gate_shared and x_packed must be 16-byte aligned");
  REQ(aligned4(logits) && aligned4(topk_ids) && aligned4(topk_w) && aligned4(bias) &&
          aligned4(shared_gate_logit) &&
          aligned4(counts) && aligned4(offsets) && aligned4(perm) && aligned4(inv_perm) &&
          aligned4(packed_tok) && aligned4(packed_w) && aligned4(counter) && aligned4(status),
      MOE_ERR_INVALID_ARG, f + "index arrays, bias, counter and status must be 4-byte aligned");
  cudaError_t e = moe_host::launch_route_dispatch(
      x, W_gate, bias, T, H, E, k, renormalize != 0, dtype, logits, topk_ids, topk_w, counts,
      offsets, perm, inv_perm, packed_tok, packed_w, x_packed, counter, status,
      static_cast<cudaStream_t>(stream), n_groups, n_groups > 1 ? topk_groups : 1, w_gate_shared,
      shared_gate_logit);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_route_dispatch launch");
}

size_t moe_experts_workspace_bytes(int N, int H, int I, int E, int dtype) {
  (void)N; (void)H; (void)I; (void)E;
  return dtype == MOE_BF16 ? moe_host::experts_ws_bytes() : 0;
}

namespace {

// Shared body of moe_experts and moe_experts_shared (sh == NULL: no shared
// expert).
int experts_impl(const char* fn, const void* x_packed, const int32_t* offsets,
                 const float* packed_w, const void* w13, const void* w2, int N, int H, int I,
                 int E, int dtype, int y_dtype, void* h, void* y_packed,
                 const moe_host::SharedGroup* sh, void* ws, size_t ws_bytes, int32_t* status,
                 void* stream) {
  const std::string f = std::string(fn) + ": ";
  if (int r = check_dtype(dtype)) return r;
  if (int r = check_y_dtype(y_dtype)) return r;
  REQ(dtype == MOE_BF16 || y_dtype == MOE_F32, MOE_ERR_UNSUPPORTED,
      f + "fp32 layers keep y_packed in fp32 (y_dtype must be MOE_F32)");
  REQ(N >= 0, MOE_ERR_INVALID_ARG, f + "N must be >= 0");
  if (N == 0 && sh == nullptr) return MOE_OK;
  REQ(x_packed && offsets && w13 && w2 && h && y_packed, MOE_ERR_INVALID_ARG,
      f + "null input or output");
  REQ(H >= 1 && I >= 1, MOE_ERR_INVALID_ARG, f + "H and I must be >= 1");
  REQ(E >= 1 && E <= moe::kMaxExperts, MOE_ERR_INVALID_ARG, f + "E must be in [1, 256]");
  REQ(H % 8 == 0 && I % 8 == 0, MOE_ERR_INVALID_ARG, f + "H and I must be multiples of 8");
  REQ(aligned16(x_packed) && aligned16(w13) && aligned16(w2) && aligned16(h) && aligned16(y_packed),
      MOE_ERR_INVALID_ARG, f + "tensors must be 16-byte aligned");
  REQ(aligned4(offsets) && aligned4(packed_w) && aligned4(status), MOE_ERR_INVALID_ARG,
      f + "offsets / packed_w / status must be 4-byte aligned");
  REQ(aligned16(ws), MOE_ERR_INVALID_ARG, f + "ws must be 16-byte aligned");
  REQ(static_cast<long long>(N) * (H > I ? H : I) < (1ll << 40) && N < (1 << 30),
      MOE_ERR_INVALID_ARG, f + "N too large");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (dtype == MOE_BF16) {
    REQ(H % 256 == 0 && I % 64 == 0, MOE_ERR_UNSUPPORTED,
        f + "the bf16 tensor-core path needs H % 256 == 0 and I % 64 == 0");
    const char* why = "";
    e = moe_host::launch_experts_tc(x_packed, offsets, packed_w, w13, w2, N, H, I, E, h, y_packed,
                                    y_dtype == MOE_F16, sh, ws, ws_bytes, status, s, &why);
    if (e != cudaSuccess && why[0]) return fail(MOE_ERR_CUDA, f + why);
  } else {
    REQ(sh == nullptr, MOE_ERR_UNSUPPORTED,
        f + "fp32: call moe_experts for the routed and for the shared expert");
    e = moe_host::launch_experts_simt(x_packed, offsets, packed_w, w13, w2, N, H, I, E, h,
                                      y_packed, s);
  }
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, (f + "launch").c_str());
}

}  // namespace

int moe_experts(const void* x_packed, const int32_t* offsets, const float* packed_w,
                const void* w13, const void* w2, int N, int H, int I, int E, int dtype,
                int y_dtype, void* h, void* y_packed, void* ws, size_t ws_bytes,
                int32_t* status, void* stream) {
  g_err.clear();
  return experts_impl("moe_experts", x_packed, offsets, packed_w, w13, w2, N, H, I, E, dtype,
                      y_dtype, h, y_packed, nullptr, ws, ws_bytes, status, stream);
}

int moe_experts_shared(const void* x_packed, const int32_t* offsets, const float* packed_w,
                       const void* w13, const void* w2, int N, int H, int I, int E,
                       const void* x, int T, const void* w13s, const void* w2s, int I_s,
                       int dtype, int y_dtype, void* h, void* y_packed, void* h_s, void* y_s,
                       void* ws, size_t ws_bytes, int32_t* status, void* stream) {
  g_err.clear();
  REQ(x && w13s && w2s && h_s && y_s, MOE_ERR_INVALID_ARG,
      "moe_experts_shared: null shared-expert input or output");
  REQ(T >= 1 && I_s >= 1, MOE_ERR_INVALID_ARG, "moe_experts_shared: T and I_s must be >= 1");
  REQ(aligned16(x) && aligned16(w13s) && aligned16(w2s) && aligned16(h_s) && aligned16(y_s),
      MOE_ERR_INVALID_ARG, "moe_experts_shared: shared-expert tensors must be 16-byte aligned");
  REQ(I_s % 64 == 0, MOE_ERR_UNSUPPORTED, "moe_experts_shared: I_s must be a multiple of 64");
  REQ(static_cast<long long>(T) * (H > I_s ? H : I_s) < (1ll << 40) && T < (1 << 30),
      MOE_ERR_INVALID_ARG, "moe_experts_shared: T too large");
  const moe_host::SharedGroup sh{x, T, w13s, w2s, I_s, h_s, y_s};
  return experts_impl("moe_experts_shared", x_packed, offsets, packed_w, w13, w2, N, H, I, E,
                      dtype, y_dtype, h, y_packed, &sh, ws, ws_bytes, status, stream);
}

int moe_combine(const void* y_packed, int y_dtype, const int32_t* inv_perm, int T, int H, int k,
                const void* shared, const float* shared_gate_logit, int dtype, void* out,
                int32_t* status, void* stream) {
  g_err.clear();
  if (int r = check_dtype(dtype)) return r;
  if (int r = check_y_dtype(y_dtype)) return r;
  REQ(y_packed && inv_perm && out, MOE_ERR_INVALID_ARG, "moe_combine: null y_packed, inv_perm or out");
  REQ(T >= 1 && H >= 1, MOE_ERR_INVALID_ARG, "moe_combine: T and H must be >= 1");
  REQ(k >= 1 && k <= moe::kMaxTopK, MOE_ERR_INVALID_ARG, "moe_combine: k must be in [1, 8]");
  REQ(H % 8 == 0, MOE_ERR_INVALID_ARG, "moe_combine: H must be a multiple of 8");
  REQ(aligned16(y_packed) && aligned16(out) && aligned16(shared), MOE_ERR_INVALID_ARG,
      "moe_combine: y_packed, shared and out must be 16-byte aligned");
  REQ(aligned4(inv_perm) && aligned4(shared_gate_logit) && aligned4(status), MOE_ERR_INVALID_ARG,
      "moe_combine: inv_perm / gate / status must be 4-byte aligned");
  REQ(static_cast<long long>(T) * k < (1ll << 30), MOE_ERR_INVALID_ARG, "moe_combine: T*k too large");
  cudaError_t e = moe_host::launch_combine(y_packed, y_dtype, inv_perm, T, H, k, shared,
                                           shared_gate_logit, dtype, out, status,
                                           static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_combine launch");
}

int moe_combine_range(const void* y_packed, int y_dtype, const int32_t* inv_perm,
                      const int32_t* offsets, int E, int expert_start, int expert_end, int T,
                      int H, int k, const void* shared, const float* shared_gate_logit,
                      int dtype, void* out, int32_t* status, void* stream) {
  g_err.clear();
  if (int r = check_dtype(dtype)) return r;
  if (int r = check_y_dtype(y_dtype)) return r;
  REQ(y_packed && inv_perm && offsets && out, MOE_ERR_INVALID_ARG,
      "moe_combine_range: null y_packed, inv_perm, offsets or out");
  REQ(T >= 1 && H >= 1, MOE_ERR_INVALID_ARG, "moe_combine_range: T and H must be >= 1");
  REQ(k >= 1 && k <= moe::kMaxTopK, MOE_ERR_INVALID_ARG, "moe_combine_range: k must be in [1, 8]");
  REQ(E >= 1 && E <= moe::kMaxExperts, MOE_ERR_INVALID_ARG, "moe_combine_range: E must be in [1, 256]");
  REQ(expert_start >= 0 && expert_start <= expert_end && expert_end <= E, MOE_ERR_INVALID_ARG,
      "moe_combine_range: need 0 <= expert_start <= expert_end <= E");
  REQ(H % 8 == 0, MOE_ERR_INVALID_ARG, "moe_combine_range: H must be a multiple of 8");
  REQ(aligned16(y_packed) && aligned16(out) && aligned16(shared), MOE_ERR_INVALID_ARG,
      "moe_combine_range: y_packed, shared and out must be 16-byte aligned");
  REQ(aligned4(inv_perm) && aligned4(offsets) && aligned4(shared_gate_logit) && aligned4(status),
      MOE_ERR_INVALID_ARG, "moe_combine_range: index / gate / status arrays must be 4-byte aligned");
  REQ(static_cast<long long>(T) * k < (1ll << 30), MOE_ERR_INVALID_ARG,
      "moe_combine_range: T*k too large");
  cudaError_t e = moe_host::launch_combine(y_packed, y_dtype, inv_perm, T, H, k, shared,
                                           shared_gate_logit, dtype, out, status,
                                           static_cast<cudaStream_t>(stream), offsets,
                                           expert_start, expert_end);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_combine_range launch");
}

int moe_finalize(const float* acc, int T, int H, int dtype, void* out, void* stream) {
  g_err.clear();
  if (int r = check_dtype(dtype)) return r;
  REQ(acc && out, MOE_ERR_INVALID_ARG, "moe_finalize: null acc or out");
  REQ(T >= 1 && H >= 1 && H % 8 == 0, MOE_ERR_INVALID_ARG,
      "moe_finalize: need T >= 1 and H a positive multiple of 8");
  REQ(aligned16(acc) && aligned16(out), MOE_ERR_INVALID_ARG,
      "moe_finalize: acc and out must be 16-byte aligned");
  cudaError_t e = moe_host::launch_finalize(acc, T, H, dtype, out, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_finalize launch");
}

int moe_gather(const void* x, const int32_t* packed_tok, const int32_t* offsets, int E,
               int expert_start, int expert_end, int N, int H, int dtype, void* x_packed,
               int32_t* status, void* stream) {
  g_err.clear();
  if (int r = check_dtype(dtype)) return r;
  REQ(x && packed_tok && offsets && x_packed, MOE_ERR_INVALID_ARG,
      "moe_gather: null x, packed_tok, offsets or x_packed");
  REQ(N >= 1 && H >= 1 && H % 8 == 0, MOE_ERR_INVALID_ARG,
      "moe_gather: need N >= 1 and H a positive multiple of 8");
  REQ(E >= 1 && E <= moe::kMaxExperts, MOE_ERR_INVALID_ARG, "moe_gather: E must be in [1, 256]");
  REQ(expert_start >= 0 && expert_start <= expert_end && expert_end <= E, MOE_ERR_INVALID_ARG,
      "moe_gather: need 0 <= expert_start <= expert_end <= E");
  REQ(aligned16(x) && aligned16(x_packed), MOE_ERR_INVALID_ARG,
      "moe_gather: x and x_packed must be 16-byte aligned");
  REQ(aligned4(packed_tok) && aligned4(offsets) && aligned4(status), MOE_ERR_INVALID_ARG,
      "moe_gather: index and status arrays must be 4-byte aligned");
  REQ(N < (1 << 30) && static_cast<long long>(N) * H < (1ll << 40), MOE_ERR_INVALID_ARG,
      "moe_gather: N too large");
  cudaError_t e = moe_host::launch_gather(x, packed_tok, offsets, expert_start, expert_end, N, H,
                                          dtype, x_packed, status, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_gather launch");
}

size_t moe_ep_partition_workspace_bytes(int num_tokens, int top_k) {
  if (num_tokens < 0 || top_k < 1) return 0;
  return moe_host::ep_partition_ws_bytes(static_cast<long long>(num_tokens) * top_k);
}

int moe_ep_partition(const int32_t* gate_indices, size_t n_indices, const float* gate_weights,
                     size_t n_weights, int num_tokens, int top_k, int local_expert_start,
                     int local_expert_end, int32_t* local_token_indices,
                     int32_t* local_expert_ids, float* local_weights,
                     int32_t* remote_token_indices, int32_t* remote_expert_ids,
                     float* remote_weights, int32_t* bucket_counts, void* ws, size_t ws_bytes,
                     void* stream) {
  g_err.clear();
  REQ(num_tokens >= 0 && top_k >= 1, MOE_ERR_INVALID_ARG,
      "moe_ep_partition: need num_tokens >= 0 and top_k >= 1");
  const long long total = static_cast<long long>(num_tokens) * top_k;
  REQ(total < (1ll << 31), MOE_ERR_INVALID_ARG, "moe_ep_partition: num_tokens*top_k too large");
  // The page's build_ep_routing_table panics on these two; here they are errors.
  REQ(static_cast<long long>(n_indices) == total, MOE_ERR_INVALID_ARG,
      "gate_indices length mismatch");
  REQ(static_cast<long long>(n_weights) == total, MOE_ERR_INVALID_ARG,
      "gate_weights length mismatch");
  REQ(local_expert_start >= 0 && local_expert_start <= local_expert_end, MOE_ERR_INVALID_ARG,
      "moe_ep_partition: need 0 <= local_expert_start <= local_expert_end");
  REQ(bucket_counts != nullptr, MOE_ERR_INVALID_ARG, "moe_ep_partition: null bucket_counts");
  REQ(total == 0 || (gate_indices && gate_weights && local_token_indices && local_expert_ids &&
                     local_weights && remote_token_indices && remote_expert_ids && remote_weights),
      MOE_ERR_INVALID_ARG, "moe_ep_partition: null input or bucket array");
  REQ(aligned4(gate_indices) && aligned4(gate_weights) && aligned4(local_token_indices) &&
          aligned4(local_expert_ids) && aligned4(local_weights) &&
          aligned4(remote_token_indices) && aligned4(remote_expert_ids) &&
          aligned4(remote_weights) && aligned4(bucket_counts),
      MOE_ERR_INVALID_ARG, "moe_ep_partition: arrays must be 4-byte aligned");
  const size_t need = moe_host::ep_partition_ws_bytes(total);
  REQ(total <= 2048 || (ws && ws_bytes >= need && aligned4(ws)), MOE_ERR_INVALID_ARG,
      "moe_ep_partition: workspace missing or smaller than moe_ep_partition_workspace_bytes()");
  cudaError_t e = moe_host::launch_ep_partition(
      gate_indices, gate_weights, static_cast<int>(total), top_k,
      static_cast<unsigned>(local_expert_start), static_cast<unsigned>(local_expert_end),
      local_token_indices, local_expert_ids, local_weights, remote_token_indices,
      remote_expert_ids, remote_weights, bucket_counts, ws, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_ep_partition launch");
}

int moe_ep_owner(const int32_t* ids, int n, int E, int world, int32_t* owner, int32_t* status,
                 void* stream) {
  g_err.clear();
  REQ(ids && owner, MOE_ERR_INVALID_ARG, "moe_ep_owner: null ids or owner");
  REQ(n >= 1 && E >= 1 && world >= 1 && world <= E, MOE_ERR_INVALID_ARG,
      "moe_ep_owner: need n >= 1 and 1 <= world <= E");
  REQ(aligned4(ids) && aligned4(owner) && aligned4(status), MOE_ERR_INVALID_ARG,
      "moe_ep_owner: arrays must be 4-byte aligned");
  cudaError_t e = moe_host::launch_ep_owner(ids, n, E, world, owner, status,
                                            static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_ep_owner launch");
}

int moe_ep_pack_ids(const int32_t* ids, const int32_t* perm, const int32_t* offsets, int n,
                    int E, int world, int32_t* local_ids, void* stream) {
  g_err.clear();
  REQ(ids && perm && offsets && local_ids, MOE_ERR_INVALID_ARG,
      "moe_ep_pack_ids: null ids, perm, offsets or local_ids");
  REQ(n >= 1 && E >= 1 && world >= 1 && world <= E, MOE_ERR_INVALID_ARG,
      "moe_ep_pack_ids: need n >= 1 and 1 <= world <= E");
  REQ(aligned4(ids) && aligned4(perm) && aligned4(offsets) && aligned4(local_ids),
      MOE_ERR_INVALID_ARG, "moe_ep_pack_ids: arrays must be 4-byte aligned");
  cudaError_t e = moe_host::launch_ep_pack_ids(ids, perm, offsets, n, E, world, local_ids,
                                               static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_ep_pack_ids launch");
}

int moe_read_status(const int32_t* status, void* stream, int32_t* host_status) {
  g_err.clear();
  REQ(status && host_status, MOE_ERR_INVALID_ARG, "moe_read_status: null pointer");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemcpyAsync(host_status, status, sizeof(int32_t), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_read_status");
}

int moe_test_set_wait_budget_ns(unsigned long long ns) {
  g_err.clear();
  if (ns == 0) ns = moe::kWaitBudgetNs;
  REQ(ns >= 1000 && ns <= moe::kWaitBudgetNs, MOE_ERR_INVALID_ARG,
      "moe_test_set_wait_budget_ns: budget must be 0 (default) or in [1000, 2e9] ns");
  g_main_wait_ns.store(ns, std::memory_order_relaxed);
  return MOE_OK;
}

int moe_probe_wait_timeout(int32_t* status, int budget_us, void* stream) {
  g_err.clear();
  REQ(status && aligned4(status), MOE_ERR_INVALID_ARG, "moe_probe_wait_timeout: bad status pointer");
  REQ(budget_us >= 1 && budget_us <= 2000000, MOE_ERR_INVALID_ARG,
      "moe_probe_wait_timeout: budget_us must be in [1, 2000000]");
  cudaError_t e = moe_host::launch_probe_wait_timeout(status, budget_us,
                                                      static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_probe_wait_timeout launch");
}

}  // extern "C"
