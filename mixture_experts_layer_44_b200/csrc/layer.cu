// The whole layer behind one handle: DWDP-Triton-MoE-Inference-Engine README,
// "Runtime Integration Layer" (router -> dispatcher -> executor -> merger,
// each stage consuming the previous one's output), as a C object.
//
// moe_layer_create checks the shapes once and carves every buffer the four
// stages need out of ONE device block the caller allocated (the library still
// allocates no device memory).  moe_layer_forward runs the stages on device
// activations.  moe_layer_forward_host takes pinned host activations: it
// keeps two device copies of x and of out and runs the upload, the layer and
// the download on three streams ordered by events, so that while step i
// computes, step i+1 uploads and step i-1 downloads.  Every copy is one plain
// cudaMemcpyAsync.
#include <stdio.h>
#include <string.h>

#include <new>
#include <string>

#include "common.cuh"

struct moe_layer {
  moe_layer_desc d;
  int N;
  int es;                        // activation bytes
  int y_dtype;                   // y_packed and the shared expert's output
  int ys;                        // their element bytes
  bool fuse_shared;
  // device buffers (carved from the caller's block)
  void* x[2];
  void* out[2];
  float* logits;
  int32_t* ids;
  float* w;
  int32_t* counts;
  int32_t* offsets;
  int32_t* perm;
  int32_t* inv_perm;
  int32_t* packed_tok;
  float* packed_w;
  void* x_packed;
  void* h;
  void* y_packed;
  void* dws;
  size_t dws_bytes;
  void* ews;
  size_t ews_bytes;
  int32_t* status;
  int32_t* counter;              // ticket of the fused small-batch route+dispatch
  float* sg_logit;
  void* sh_h;
  void* sh_y;
  int32_t* sh_offsets;
  // host-buffer pipeline
  cudaStream_t s_in, s_comp, s_out;
  cudaEvent_t ev_entry, x_ready[2], x_free[2], out_ready[2], out_free[2];
  int parity;
};

namespace {

size_t up256(size_t b) { return (b + 255) / 256 * 256; }

// Byte layout of the block: offsets of every buffer (a null `base` only sizes).
struct Carve {
  uint8_t* base;
  size_t used = 0;
  void* take(size_t bytes) {
    void* p = base ? base + used : nullptr;
    used += up256(bytes);
    return p;
  }
};

size_t layout(moe_layer* L, uint8_t* base) {
  const moe_layer_desc& d = L->d;
  Carve c{base};
  const size_t T = d.T, H = d.H, E = d.E, k = d.k, I = d.I, N = T * k, es = L->es;
  L->x[0] = c.take(T * H * es);
  L->x[1] = c.take(T * H * es);
  L->out[0] = c.take(T * H * es);
  L->out[1] = c.take(T * H * es);
  L->logits = static_cast<float*>(c.take(T * E * 4));
  L->ids = static_cast<int32_t*>(c.take(N * 4));
  L->w = static_cast<float*>(c.take(N * 4));
  L->counts = static_cast<int32_t*>(c.take(E * 4));
  L->offsets = static_cast<int32_t*>(c.take((E + 1) * 4));
  L->perm = static_cast<int32_t*>(c.take(N * 4));
  L->inv_perm = static_cast<int32_t*>(c.take(N * 4));
  L->packed_tok = static_cast<int32_t*>(c.take(N * 4));
  L->packed_w = static_cast<float*>(c.take(N * 4));
  L->x_packed = c.take(N * H * es);
  L->h = c.take(N * I * es);
  L->y_packed = c.take(N * H * L->ys);
  L->dws_bytes = moe_host::dispatch_ws_bytes(d.T, d.k, d.E);
  L->dws = c.take(L->dws_bytes);
  L->ews_bytes = d.dtype == MOE_BF16 ? moe_host::experts_ws_bytes() : 0;
  L->ews = L->ews_bytes ? c.take(L->ews_bytes) : nullptr;
  L->status = static_cast<int32_t*>(c.take(8));   // status, then the route+dispatch ticket
  L->counter = L->status + 1;
  if (d.w13s != nullptr) {
    L->sg_logit = static_cast<float*>(c.take(T * 4));
    L->sh_h = c.take(T * static_cast<size_t>(d.I_s) * es);
    L->sh_y = c.take(T * H * L->ys);
    L->sh_offsets = static_cast<int32_t*>(c.take(8));
  } else {
    L->sg_logit = nullptr;
    L->sh_h = nullptr;
    L->sh_y = nullptr;
    L->sh_offsets = nullptr;
  }
  return c.used;
}

const char* check_desc(const moe_layer_desc* d) {
  if (d == nullptr) return "null descriptor";
  if (d->dtype != MOE_F32 && d->dtype != MOE_BF16) return "dtype must be MOE_F32 or MOE_BF16";
  if (d->T < 1 || d->H < 8 || d->H % 8 || d->I < 8 || d->I % 8) return "bad T, H or I";
  if (d->E < 1 || d->E > moe::kMaxExperts) return "E must be in [1, 256]";
  if (d->k < 1 || d->k > d->E || d->k > moe::kMaxTopK) return "k must be in [1, min(E, 8)]";
  if (!d->W_gate || !d->w13 || !d->w2) return "null W_gate, w13 or w2";
  {
    auto mis = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) != 0; };
    if (mis(d->W_gate) || mis(d->w13) || mis(d->w2) || mis(d->w13s) || mis(d->w2s) ||
        mis(d->w_sg))
      return "weights must be 16-byte aligned";
  }
  if (d->dtype == MOE_BF16 && (d->H % 256 || d->I % 64))
    return "bf16 layers need H % 256 == 0 and I % 64 == 0";
  if (d->w13s != nullptr) {
    if (!d->w2s || !d->w_sg || d->I_s < 8 || d->I_s % 8) return "incomplete shared expert";
    if (d->dtype == MOE_BF16 && d->I_s % 64) return "bf16 shared experts need I_s % 64 == 0";
  }
  if (d->n_groups > 1 && (d->n_groups > 32 || d->E % d->n_groups || d->topk_groups < 1 ||
                          d->topk_groups > d->n_groups ||
                          d->k > d->topk_groups * (d->E / d->n_groups)))
    return "bad group limit (n_groups, topk_groups)";
  if (static_cast<long long>(d->T) * d->k * d->H >= (1ll << 40)) return "T*k*H too large";
  return nullptr;
}

cudaError_t run_layer(moe_layer* L, const void* x, void* out, cudaStream_t s) {
  const moe_layer_desc& d = L->d;
  const int ng = d.n_groups > 1 ? d.n_groups : 1;
  cudaError_t e;
  const bool shared = d.w13s != nullptr;
  bool gate_done = false;       // the shared expert's gate logit is written
  if (moe_host::route_dispatch_fits(d.T, d.H, d.E, d.k, shared)) {
    // decode batches: router (and the shared expert's gate) and dispatcher in one launch
    e = moe_host::launch_route_dispatch(x, d.W_gate, d.bias, d.T, d.H, d.E, d.k,
                                        d.renormalize != 0, d.dtype, L->logits, L->ids, L->w,
                                        L->counts, L->offsets, L->perm, L->inv_perm,
                                        L->packed_tok, L->packed_w, L->x_packed, L->counter,
                                        L->status, s, ng, d.topk_groups,
                                        shared ? d.w_sg : nullptr,
                                        shared ? L->sg_logit : nullptr);
    gate_done = shared;
  } else {
    e = shared ? moe_host::launch_route_gated(x, d.W_gate, d.bias, d.w_sg, d.T, d.H, d.E, d.k,
                                              d.renormalize != 0, d.dtype, L->logits, L->ids,
                                              L->w, L->sg_logit, L->status, s, ng,
                                              d.topk_groups)
               : moe_host::launch_route(x, d.W_gate, d.bias, d.T, d.H, d.E, d.k,
                                        d.renormalize != 0, d.dtype, L->logits, L->ids, L->w,
                                        L->status, s, ng, d.topk_groups);
    gate_done = shared;
    if (e == cudaSuccess)
      e = moe_host::launch_dispatch(L->ids, L->w, x, d.T, d.H, d.E, d.k, d.dtype, L->counts,
                                    L->offsets, L->perm, L->inv_perm, L->packed_tok,
                                    L->packed_w, L->x_packed, L->dws, L->status, s);
  }
  if (e != cudaSuccess) return e;
  const char* why = "";
  if (shared && !gate_done) {
    e = moe_host::launch_route(x, d.w_sg, nullptr, d.T, d.H, 1, 0, 0, d.dtype, L->sg_logit,
                               nullptr, nullptr, L->status, s);
    if (e != cudaSuccess) return e;
  }
  if (d.dtype == MOE_BF16) {
    moe_host::SharedGroup g{x, d.T, d.w13s, d.w2s, d.I_s, L->sh_h, L->sh_y};
    e = moe_host::launch_experts_tc(L->x_packed, L->offsets, L->packed_w, d.w13, d.w2, L->N, d.H,
                                    d.I, d.E, L->h, L->y_packed, L->y_dtype == MOE_F16,
                                    shared ? &g : nullptr, L->ews,
                                    L->ews_bytes, L->status, s, &why);
  } else {
    e = moe_host::launch_experts_simt(L->x_packed, L->offsets, L->packed_w, d.w13, d.w2, L->N,
                                      d.H, d.I, d.E, L->h, L->y_packed, s);
    if (e == cudaSuccess && shared)
      e = moe_host::launch_experts_simt(x, L->sh_offsets, nullptr, d.w13s, d.w2s, d.T, d.H,
                                        d.I_s, 1, L->sh_h, L->sh_y, s);
  }
  if (e != cudaSuccess) return e;
  return moe_host::launch_combine(L->y_packed, L->y_dtype, L->inv_perm, d.T, d.H, d.k,
                                  shared ? L->sh_y : nullptr, shared ? L->sg_logit : nullptr,
                                  d.dtype, out, L->status, s);
}

int fail(int code, const std::string& msg) {
  moe_host::set_last_error(msg);
  return code;
}

int cuda_fail(cudaError_t e, const char* where) {
  moe_host::set_last_error(std::string(where) + ": " + cudaGetErrorString(e));
  return MOE_ERR_CUDA;
}

void destroy_handles(moe_layer* L) {
  if (L->s_in) cudaStreamDestroy(L->s_in);
  if (L->s_comp) cudaStreamDestroy(L->s_comp);
  if (L->s_out) cudaStreamDestroy(L->s_out);
  cudaEvent_t* evs[] = {&L->ev_entry, &L->x_ready[0], &L->x_ready[1], &L->x_free[0],
                        &L->x_free[1], &L->out_ready[0], &L->out_ready[1], &L->out_free[0],
                        &L->out_free[1]};
  for (cudaEvent_t* e : evs)
    if (*e) cudaEventDestroy(*e);
}

}  // namespace

extern "C" {

size_t moe_layer_workspace_bytes(const moe_layer_desc* d) {
  if (check_desc(d) != nullptr) return 0;
  moe_layer tmp;
  memset(&tmp, 0, sizeof(tmp));
  tmp.d = *d;
  tmp.es = d->dtype == MOE_BF16 ? 2 : 4;
  tmp.y_dtype = d->dtype == MOE_BF16 && !d->y_f32 ? MOE_F16 : MOE_F32;
  tmp.ys = tmp.y_dtype == MOE_F16 ? 2 : 4;
  return layout(&tmp, nullptr);
}

int moe_layer_create(const moe_layer_desc* d, void* workspace, size_t workspace_bytes,
                     void* stream, moe_layer** out) {
  moe_host::set_last_error("");
  if (out == nullptr) return fail(MOE_ERR_INVALID_ARG, "moe_layer_create: null out");
  *out = nullptr;
  if (const char* why = check_desc(d)) return fail(MOE_ERR_INVALID_ARG, std::string("moe_layer_create: ") + why);
  const size_t need = moe_layer_workspace_bytes(d);
  if (workspace == nullptr || workspace_bytes < need ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return fail(MOE_ERR_INVALID_ARG,
                "moe_layer_create: workspace missing, not 256-byte aligned or smaller than "
                "moe_layer_workspace_bytes() = " + std::to_string(need));
  moe_layer* L = new (std::nothrow) moe_layer;
  if (L == nullptr) return fail(MOE_ERR_INVALID_ARG, "moe_layer_create: out of host memory");
  memset(L, 0, sizeof(*L));
  L->d = *d;
  if (L->d.n_groups < 1) L->d.n_groups = 1;
  L->es = d->dtype == MOE_BF16 ? 2 : 4;
  L->y_dtype = d->dtype == MOE_BF16 && !d->y_f32 ? MOE_F16 : MOE_F32;
  L->ys = L->y_dtype == MOE_F16 ? 2 : 4;
  L->N = d->T * d->k;
  layout(L, static_cast<uint8_t*>(workspace));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaSuccess;
  // the experts' split-K counters and the status word start at zero
  if (L->ews) e = cudaMemsetAsync(L->ews, 0, L->ews_bytes, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(L->status, 0, 8, s);   // status and ticket
  if (e == cudaSuccess && L->sh_offsets) {
    static thread_local int32_t so[2];
    so[0] = 0;
    so[1] = d->T;
    e = cudaMemcpyAsync(L->sh_offsets, so, 8, cudaMemcpyHostToDevice, s);
  }
  // Set-up done before the first forward call can be enqueued (and `so` must
  // outlive its copy).
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  const unsigned fl = cudaStreamNonBlocking;
  if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&L->s_in, fl);
  if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&L->s_comp, fl);
  if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&L->s_out, fl);
  cudaEvent_t* evs[] = {&L->ev_entry, &L->x_ready[0], &L->x_ready[1], &L->x_free[0],
                        &L->x_free[1], &L->out_ready[0], &L->out_ready[1], &L->out_free[0],
                        &L->out_free[1]};
  for (cudaEvent_t* ev : evs)
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(ev, cudaEventDisableTiming);
  if (e != cudaSuccess) {
    destroy_handles(L);
    delete L;
    return cuda_fail(e, "moe_layer_create");
  }
  *out = L;
  return MOE_OK;
}

int moe_layer_destroy(moe_layer* L) {
  if (L == nullptr) return MOE_OK;
  cudaStreamSynchronize(L->s_in);
  cudaStreamSynchronize(L->s_comp);
  cudaStreamSynchronize(L->s_out);
  destroy_handles(L);
  delete L;
  return MOE_OK;
}

int moe_layer_forward(moe_layer* L, const void* x, void* out, void* stream) {
  moe_host::set_last_error("");
  if (L == nullptr || x == nullptr || out == nullptr)
    return fail(MOE_ERR_INVALID_ARG, "moe_layer_forward: null layer, x or out");
  if ((reinterpret_cast<uintptr_t>(x) & 15u) || (reinterpret_cast<uintptr_t>(out) & 15u))
    return fail(MOE_ERR_INVALID_ARG, "moe_layer_forward: x and out must be 16-byte aligned");
  cudaError_t e = run_layer(L, x, out, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_layer_forward");
}

int moe_layer_forward_host(moe_layer* L, const void* x_host, void* out_host, void* stream) {
  moe_host::set_last_error("");
  if (L == nullptr || x_host == nullptr || out_host == nullptr)
    return fail(MOE_ERR_INVALID_ARG, "moe_layer_forward_host: null layer, x_host or out_host");
  const size_t bytes = static_cast<size_t>(L->d.T) * L->d.H * L->es;
  const int b = L->parity;
  L->parity ^= 1;
  cudaError_t e = cudaEventRecord(L->ev_entry, static_cast<cudaStream_t>(stream));
  // upload: after the caller's prior work, and after the step that last read x[b]
  if (e == cudaSuccess) e = cudaStreamWaitEvent(L->s_in, L->ev_entry, 0);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(L->s_in, L->x_free[b], 0);
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(L->x[b], x_host, bytes, cudaMemcpyHostToDevice, L->s_in);
  if (e == cudaSuccess) e = cudaEventRecord(L->x_ready[b], L->s_in);
  // the layer: once x[b] is in and the download of the step that last wrote out[b] is done
  if (e == cudaSuccess) e = cudaStreamWaitEvent(L->s_comp, L->x_ready[b], 0);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(L->s_comp, L->out_free[b], 0);
  if (e == cudaSuccess) e = run_layer(L, L->x[b], L->out[b], L->s_comp);
  if (e == cudaSuccess) e = cudaEventRecord(L->x_free[b], L->s_comp);
  if (e == cudaSuccess) e = cudaEventRecord(L->out_ready[b], L->s_comp);
  // download
  if (e == cudaSuccess) e = cudaStreamWaitEvent(L->s_out, L->out_ready[b], 0);
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(out_host, L->out[b], bytes, cudaMemcpyDeviceToHost, L->s_out);
  if (e == cudaSuccess) e = cudaEventRecord(L->out_free[b], L->s_out);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_layer_forward_host");
}

int moe_layer_join(moe_layer* L, void* stream) {
  moe_host::set_last_error("");
  if (L == nullptr) return fail(MOE_ERR_INVALID_ARG, "moe_layer_join: null layer");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaSuccess;
  for (int b = 0; b < 2 && e == cudaSuccess; ++b) {
    e = cudaStreamWaitEvent(s, L->out_free[b], 0);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(s, L->x_free[b], 0);
  }
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_layer_join");
}

int moe_layer_status(moe_layer* L, void* stream, int32_t* host_status) {
  moe_host::set_last_error("");
  if (L == nullptr || host_status == nullptr)
    return fail(MOE_ERR_INVALID_ARG, "moe_layer_status: null layer or host_status");
  int r = moe_layer_join(L, stream);
  if (r != MOE_OK) return r;
  return moe_read_status(L->status, stream, host_status);
}

void* moe_layer_buffer(moe_layer* L, const char* name) {
  if (L == nullptr || name == nullptr) return nullptr;
  if (!strcmp(name, "logits")) return L->logits;
  if (!strcmp(name, "ids")) return L->ids;
  if (!strcmp(name, "w")) return L->w;
  if (!strcmp(name, "counts")) return L->counts;
  if (!strcmp(name, "offsets")) return L->offsets;
  if (!strcmp(name, "inv_perm")) return L->inv_perm;
  if (!strcmp(name, "perm")) return L->perm;
  if (!strcmp(name, "packed_tok")) return L->packed_tok;
  if (!strcmp(name, "packed_w")) return L->packed_w;
  if (!strcmp(name, "x_packed")) return L->x_packed;
  if (!strcmp(name, "h")) return L->h;
  if (!strcmp(name, "y_packed")) return L->y_packed;
  if (!strcmp(name, "status")) return L->status;
  return nullptr;
}

}  // extern "C"
