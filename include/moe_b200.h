/*
 * moe_b200.h -- C ABI of libmoe_b200.so: the forward pass of one
 * Mixture-of-Experts layer on one NVIDIA B200 (sm_100a).
 *
 * The four stage calls follow the stage contracts of the
 * DWDP-Triton-MoE-Inference-Engine README: the Router ("Router Module"),
 * the Dispatcher ("Dispatcher Module"), the Executor ("Executor Module")
 * and the Merger ("Merger Module"), chained in the order its "Runtime
 * Integration Layer" section gives.  Each stage reads only what the
 * previous one wrote.
 *
 * Conventions shared by every call
 *  - Pointers named as device pointers must point to device memory of the
 *    current CUDA device; tensors are dense and row-major; bf16 means the
 *    IEEE-like bfloat16 (1-8-7) bit pattern, fp32 means IEEE binary32.
 *  - The caller owns every buffer.  The library allocates no device memory,
 *    keeps no pointer after a call returns, and never synchronises the
 *    stream on these calls.  All work is enqueued on `stream` (a
 *    cudaStream_t; NULL = the legacy default stream) and runs asynchronously.
 *  - Return value: MOE_OK, or a moe_status_t describing a host-side
 *    argument check failure (nothing is enqueued) or a launch failure
 *    (MOE_ERR_CUDA).  moe_last_error() then gives a one-line message.
 *  - Errors found on the device (an expert id outside [0, E), an inverse
 *    permutation entry outside [0, N), a bounded wait that ran out) are
 *    written to the optional device word `status` (int32, caller-zeroed):
 *    the first error code stays, later ones do not overwrite it.  Kernels
 *    never trap: a bad entry is skipped and reported.  moe_read_status()
 *    copies the word to the host.
 *  - Sizes: 1 <= T; 1 <= E <= 256; 0 <= k <= min(E, 8) (k = 0 only in
 *    moe_route, "logits only"; moe_dispatch takes 1 <= k <= 8 and ids that
 *    may repeat within a token); H, I >= 1 with H % 8 == 0 and I % 8 == 0
 *    (whole 16-byte vectors); the bf16 tensor-core expert path also needs
 *    H % 256 == 0 and I % 64 == 0, else moe_experts returns
 *    MOE_ERR_UNSUPPORTED.  Activation and weight tensors must be 16-byte
 *    aligned; index, weight and status arrays 4-byte aligned.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,  /* bad size, null or misaligned pointer        */
  MOE_ERR_UNSUPPORTED = 2,  /* valid but not implemented for this shape    */
  MOE_ERR_CUDA = 3,         /* a CUDA launch / runtime call failed         */
  MOE_ERR_TIMEOUT = 4,      /* (device status) a bounded wait ran out      */
  MOE_ERR_BAD_INDEX = 5,    /* (device status) an index was out of range   */
  MOE_ERR_OVERFLOW = 6      /* (device status) a value beyond the fp16 range
                               was stored in an fp16 y_packed (it became inf) */
} moe_status_t;

typedef enum {
  MOE_F32 = 0,   /* activations, weights and outputs in fp32              */
  MOE_BF16 = 1,  /* activations, weights and outputs in bf16, fp32 inside  */
  MOE_F16 = 2    /* fp16: only as the type of y_packed and of the shared
                    expert's output (y_dtype) of a bf16 layer               */
} moe_dtype_t;

/* Version of this ABI (bumped on any added entry point or signature change). */
int moe_abi_version(void);

/* Number of kernels this library has enqueued in this process so far (all
 * threads, all devices).  The difference across a region of calls is the
 * number of GPU kernels those calls launched. */
unsigned long long moe_launch_count(void);

/* Message for the last non-OK return on the calling thread ("" if none).
 * The string stays valid until the next call on this thread. */
const char* moe_last_error(void);

/*
 * moe_route -- Router.  DWDP README, "Router Module": router logits, routing
 * probabilities, top-k expert indices and normalized routing weights;
 * diffulex.moe API reference, "diffulex.moe.topk" (NaiveTopKRouter, the
 * standard top-k router).
 *
 *   logits[t,e] = sum_h x[t,h] * W_gate[e,h] + bias[e]      (fp32 sums)
 *   p[t,:]      = softmax(logits[t,:]) over all E             (fp32)
 *   topk_ids[t,j], j < k: the k experts with the largest logits, in
 *               descending order; equal logits -> lower expert id first
 *   topk_w[t,j] = p[t, topk_ids[t,j]]; if renormalize, divided by the
 *               sum of the k selected probabilities
 *
 *   x        device [T,H] (dtype)          W_gate  device [E,H] (dtype)
 *   bias     device [E] fp32, or NULL (no bias)
 *   logits   device [T,E] fp32, written
 *   topk_ids device [T,k] int32, written (may be NULL when k == 0)
 *   topk_w   device [T,k] fp32, written  (may be NULL when k == 0)
 *   status   device int32, or NULL: the first device-side error
 *            (MOE_ERR_TIMEOUT) is recorded there with atomicCAS from 0
 *   k == 0 computes the logits only (e.g. a shared expert's scalar gate
 *   logit with E == 1).  Inputs are assumed finite.
 *
 *   fp32: the sums are fp32 FMA chains on the CUDA cores.  bf16 with more
 *   than 64 tokens or more than 64 experts: the contraction runs on the
 *   tensor cores (bf16 products are exact in fp32; fp32 accumulation in
 *   TMEM); smaller bf16 batches use fp32 FMA.  Results are deterministic
 *   for a given device and shape.
 */
int moe_route(const void* x, const void* W_gate, const float* bias,
              int T, int H, int E, int k, int renormalize, int dtype,
              float* logits, int32_t* topk_ids, float* topk_w, int32_t* status,
              void* stream);

/*
 * moe_route_grouped -- Router with group-limited expert selection
 * (diffulex.moe API reference, "diffulex.moe.topk": GroupLimitedTopKRouter).
 * The page gives no rule; the one implemented is the plainest reading:
 *   the E experts form n_groups groups of E / n_groups consecutive ids;
 *   a group's score is the largest logit among its experts;
 *   the topk_groups groups with the highest scores are kept (equal scores:
 *   lower group id first);
 *   topk_ids = the k largest logits among the kept groups' experts, ordered
 *   and tie-broken as in moe_route.
 * logits and topk_w are defined as in moe_route (the softmax spans all E
 * experts; renormalize divides by the k selected probabilities).
 * n_groups == 1 is moe_route.  Needs n_groups <= 32, E % n_groups == 0,
 * 1 <= topk_groups <= n_groups and 1 <= k <= topk_groups * E / n_groups;
 * otherwise MOE_ERR_INVALID_ARG.  All other arguments as moe_route.
 */
int moe_route_grouped(const void* x, const void* W_gate, const float* bias, int T, int H, int E,
                      int k, int renormalize, int n_groups, int topk_groups, int dtype,
                      float* logits, int32_t* topk_ids, float* topk_w, int32_t* status,
                      void* stream);

/*
 * moe_route_gated -- moe_route_grouped plus the always-on shared expert's
 * gate logit (diffulex.moe.layer, SharedExpertMLP: the sigmoid gate that
 * scales the shared expert's output; moe_combine applies the sigmoid):
 *   shared_gate_logit[t] = x[t] . w_gate_shared      (fp32 accumulate, no bias)
 * The gate row is contracted in the router's own launch where the router has
 * room for it -- small batches (T <= 64, E + 1 <= 64, H <= 32768) as row E,
 * the bf16 tensor-core router (T > 64) by the warps that are otherwise idle
 * during its main loop, from the x tiles already in shared memory -- else in
 * a second launch (moe_route with E = 1, k = 0 on that row).  Either way x is
 * read from HBM once per launch.  The routed outputs are those of
 * moe_route_grouped; where the gate changes the router's row block (E + 1
 * passing a power of two) their logits can differ from it in fp32 summation
 * order.
 *   w_gate_shared      device [H] (dtype), 16-byte aligned
 *   shared_gate_logit  device [T] f32
 *   All other arguments as moe_route_grouped (n_groups = 1: plain top-k).
 */
int moe_route_gated(const void* x, const void* W_gate, const float* bias,
                    const void* w_gate_shared, int T, int H, int E, int k, int renormalize,
                    int n_groups, int topk_groups, int dtype, float* logits, int32_t* topk_ids,
                    float* topk_w, float* shared_gate_logit, int32_t* status, void* stream);

/* Bytes of device scratch moe_dispatch needs for (T, k, E). */
size_t moe_dispatch_workspace_bytes(int T, int k, int E);

/*
 * moe_dispatch -- Dispatcher.  DWDP README, "Dispatcher Module": converts
 * token-major routing assignments into an expert-major layout with
 * per-expert counts, expert offsets, token permutation, inverse permutation,
 * packed token indices and packed routing weights; plus the Executor's
 * "gather token activations" step ("Executor Module") into x_packed.
 *
 * Assignment f = t*k + j is entry j of token t (row-major [T,k], the flat
 * order of metrale's ep_dispatch.rs, build_ep_routing_table).  N = T*k.
 *   counts[e]      number of f with topk_ids[f] == e               [E]
 *   offsets[e]     exclusive prefix sum of counts; offsets[E] = N  [E+1]
 *   p(f)           offsets[e] + #{f' < f : topk_ids[f'] == e}  (stable:
 *                  equal experts keep ascending f, i.e. token order)
 *   perm[p(f)] = f,  inv_perm[f] = p(f),  packed_tok[p] = perm[p] / k,
 *   packed_w[p] = topk_w[perm[p]],  x_packed[p,:] = x[packed_tok[p],:]
 *
 *   topk_ids device [T,k] int32     topk_w device [T,k] fp32 (or NULL: no
 *   packed_w output)                 x device [T,H] (dtype), or NULL to
 *   skip the gather (x_packed then unused)
 *   counts, offsets, perm, inv_perm, packed_tok  device int32, written
 *   packed_w  device [N] fp32, written (ignored if topk_w is NULL)
 *   x_packed  device [N,H] (dtype), written
 *   ws        device scratch of at least moe_dispatch_workspace_bytes()
 *   status    device int32 or NULL.  An id outside [0,E) sets
 *             MOE_ERR_BAD_INDEX; that assignment is left out of every
 *             output (inv_perm[f] = -1) and offsets[E] < N.
 */
int moe_dispatch(const int32_t* topk_ids, const float* topk_w, const void* x,
                 int T, int H, int E, int k, int dtype,
                 int32_t* counts, int32_t* offsets, int32_t* perm, int32_t* inv_perm,
                 int32_t* packed_tok, float* packed_w, void* x_packed,
                 void* ws, size_t ws_bytes, int32_t* status, void* stream);

/*
 * moe_dispatch_noalloc -- moe_dispatch for callers that cannot allocate
 * device memory at the point where they dispatch: a C host program whose GPU
 * memory is carved up by someone else, a plugin of a framework that does not
 * expose its allocator, or a serving loop that forbids allocation once it is
 * running.  The pages have no counterpart; it exists only so that such a
 * caller needs no workspace.
 *
 * Same arguments, outputs, ordering and status reporting as moe_dispatch,
 * without `ws` / `ws_bytes`: the per-block count table lives in one fixed
 * array of the library (a file-scope __device__ array of 128 KiB that every
 * GPU which loads the library holds until the process exits).  The call
 * allocates nothing.
 *   - Limit: ceil(T*k / 2048) * E <= 32768 (e.g. T*k <= 524288 at E = 128;
 *     up to T*k = 65536 the table always fits); larger problems return
 *     MOE_ERR_INVALID_ARG with a message naming the limit.  Use moe_dispatch
 *     with a workspace for them.
 *   - The first call on a device looks up the array's device address on that
 *     device (cudaGetSymbolAddress), so make that first call before any
 *     stream capture.  The address is cached per device and CUDA context and
 *     looked up again when the context changes (after cudaDeviceReset, the
 *     next call does the look-up again: make it outside a capture too).
 *   - All calls share the one array and it keeps the last call's contents
 *     (nothing in it needs to start at zero).  Two calls whose work overlaps
 *     on the GPU (different streams, or different host threads) race on it:
 *     order them on one stream.
 */
int moe_dispatch_noalloc(const int32_t* topk_ids, const float* topk_w, const void* x,
                         int T, int H, int E, int k, int dtype,
                         int32_t* counts, int32_t* offsets, int32_t* perm, int32_t* inv_perm,
                         int32_t* packed_tok, float* packed_w, void* x_packed,
                         int32_t* status, void* stream);

/*
 * moe_route_dispatch -- moe_route_grouped followed by moe_dispatch, in one
 * launch, for small batches (decode).  The Router and the Dispatcher of the
 * DWDP README ("Router Module", "Dispatcher Module", chained as its "Runtime
 * Integration Layer" gives) produce exactly the outputs of the two separate
 * calls on the same arguments (bit for bit: the same routing arithmetic and
 * the same stable order).
 *
 * One CTA per token routes it; the CTA that finishes last (found with an
 * atomic ticket on `counter`: no CTA waits for another) then counts, scans
 * and scatters all T*k assignments, and gathers x_packed when the rows total
 * at most 128 KiB (a second, multi-CTA gather kernel otherwise).
 *
 *   Arguments as moe_route_grouped (n_groups = 1: plain top-k) and
 *   moe_dispatch, with topk_ids / topk_w as the routed outputs it writes and
 *   then reads back (both required, k >= 1).
 *   x_packed  device [N,H] (dtype), or NULL to skip the gather.
 *   counter   device int32, zero before the first call; every call leaves it
 *             at zero again.  Calls that may overlap on the GPU (different
 *             streams) need different counters.
 *   w_gate_shared      device [H] (dtype): the always-on shared expert's gate
 *                      row (diffulex.moe.layer, SharedExpertMLP), or NULL;
 *   shared_gate_logit  device [T] f32: x[t] . w_gate_shared (no bias), the
 *                      logit moe_combine's sigmoid gate takes; NULL exactly
 *                      when w_gate_shared is.  The gate is contracted as one
 *                      more row beside the E experts, in the same launch, and
 *                      takes no part in the selection; it equals moe_route
 *                      with E = 1, k = 0 on that row up to fp32 summation
 *                      order.  When E + 1 passes a power of two, the routed
 *                      rows are contracted in a larger block too, and their
 *                      logits can then differ from the call without the gate
 *                      in fp32 summation order (the bit-for-bit identity with
 *                      the two separate calls holds without a gate).
 *   Needs 1 <= T <= 64, 1 <= E <= 64 (E <= 63 with a shared gate),
 *   H <= 32768 and 1 <= k <= min(E, 8): other shapes return
 *   MOE_ERR_INVALID_ARG (use the two separate calls).
 *   No workspace.
 */
int moe_route_dispatch(const void* x, const void* W_gate, const float* bias,
                       const void* w_gate_shared, int T, int H, int E, int k, int renormalize,
                       int n_groups, int topk_groups, int dtype, float* logits,
                       int32_t* topk_ids, float* topk_w, float* shared_gate_logit,
                       int32_t* counts, int32_t* offsets, int32_t* perm, int32_t* inv_perm,
                       int32_t* packed_tok, float* packed_w, void* x_packed,
                       int32_t* counter, int32_t* status, void* stream);

/* Bytes of device scratch moe_experts can use (bf16 path: per-tile counters
 * plus 128 KiB partial slots, 4 per SM; fp32 path: 0). */
size_t moe_experts_workspace_bytes(int N, int H, int I, int E, int dtype);

/*
 * moe_experts -- Executor.  DWDP README, "Executor Module": for scheduled
 * expert-major ranges, execute the expert modules, apply routing weights
 * and write packed expert outputs.  Experts are SwiGLU MLPs whose gate and
 * up projections are fused in one [E, 2I, H] buffer, gate (w1) in rows
 * [0, I) and up (w3) in rows [I, 2I) of each expert's slot (the w13_weight
 * layout of modelexpress-client's test_reshard_refit_moe_experts.py).
 *
 * For every expert e and every row p in [offsets[e], offsets[e+1]):
 *   h[p,i]        = silu(x_packed[p,:] . w13[e,i,:]) * (x_packed[p,:] . w13[e,I+i,:])
 *   y_packed[p,c] = packed_w[p] * (h[p,:] . w2[e,c,:])
 * with silu(z) = z / (1 + exp(-z)), fp32 accumulation, and (bf16) h
 * rounded to bf16 before the second product (it is the operand of a bf16
 * tensor-core product).  y_packed is stored in y_dtype: fp16 (each element
 * rounded once, to nearest, after the fp32 accumulation and the
 * routing-weight scale: a relative error of at most 2^-11, half the bytes to
 * write here and to read in the merger) or fp32 (the merger then adds the k
 * fp32 terms before the output's only rounding).  An fp16 element whose
 * magnitude exceeds 65504 becomes inf and sets MOE_ERR_OVERFLOW in status.
 * fp32 layers take y_dtype = MOE_F32 only.
 *
 *   x_packed device [N,H]       offsets device [E+1] int32 (read on the
 *   device; the host never needs the split)
 *   packed_w device [N] fp32, or NULL for all-ones (e.g. a shared expert)
 *   w13 device [E,2I,H]         w2 device [E,H,I]
 *   h        device [N,I] (dtype) scratch, written
 *   y_dtype  MOE_F16 or MOE_F32 (bf16 layers), MOE_F32 (fp32 layers);
 *            otherwise MOE_ERR_INVALID_ARG / MOE_ERR_UNSUPPORTED
 *   y_packed device [N,H] (y_dtype), written; rows outside every expert's
 *            range are left untouched
 *   ws/ws_bytes  device scratch of moe_experts_workspace_bytes() bytes,
 *            ZERO-FILLED before its first use (the kernels leave it zeroed
 *            again; re-zero it after a MOE_ERR_TIMEOUT).  With it, a pass with
 *            fewer tiles than two per SM splits K and reduces the fp32
 *            partials in a fixed order (deterministic).  NULL / 0 is allowed:
 *            no split.  Calls that share one ws must not overlap on the GPU.
 *   status   device int32 or NULL (timeouts, fp16 overflow)
 * offsets must be non-decreasing with offsets[E] <= N (as moe_dispatch
 * writes them); rows are trusted to lie in [0, N).
 */
int moe_experts(const void* x_packed, const int32_t* offsets, const float* packed_w,
                const void* w13, const void* w2, int N, int H, int I, int E, int dtype,
                int y_dtype, void* h, void* y_packed, void* ws, size_t ws_bytes,
                int32_t* status, void* stream);

/*
 * moe_experts_shared -- the Executor of moe_experts plus one shared expert
 * in the same pair of launches (diffulex.moe.layer, "SharedExpertMLP": an
 * expert every token goes through).  The routed part is exactly moe_experts.
 * The shared part computes, for every t < T,
 *   h_s[t,i] = silu(x[t,:] . w13s[i,:]) * (x[t,:] . w13s[I_s+i,:])
 *   y_s[t,c] = h_s[t,:] . w2s[c,:]                 (no routing weight)
 * Its tiles are scheduled first, beside the routed ones, so the weight
 * streams of both share every SM instead of running one after the other.
 * bf16 only (fp32 returns MOE_ERR_UNSUPPORTED: call moe_experts twice).
 *
 *   x    device [T,H] bf16          w13s device [2*I_s,H]   w2s device [H,I_s]
 *   h_s  device [T,I_s] bf16, written   y_s device [T,H] (y_dtype), written
 *   I_s % 64 == 0; all other arguments, results and rules as moe_experts.
 */
int moe_experts_shared(const void* x_packed, const int32_t* offsets, const float* packed_w,
                       const void* w13, const void* w2, int N, int H, int I, int E,
                       const void* x, int T, const void* w13s, const void* w2s, int I_s,
                       int dtype, int y_dtype, void* h, void* y_packed, void* h_s, void* y_s,
                       void* ws, size_t ws_bytes, int32_t* status, void* stream);

/*
 * moe_combine -- Merger.  DWDP README, "Merger Module": restore token-major
 * assignment order, accumulate the top-k expert outputs and reshape back to
 * the token layout.  Routing weights were already applied by moe_experts.
 *
 *   out[t,:] = sum_{j=0..k-1} y_packed[inv_perm[t*k+j],:]   (j in order,
 *              fp32 sum, one rounding to the output type)
 *            + sigmoid(shared_gate_logit[t]) * shared[t,:]   (if shared)
 *
 *   y_packed device [N,H] (y_dtype: MOE_F16 or MOE_F32), N = T*k
 *   inv_perm device [N] int32
 *   shared   device [T,H] (y_dtype) or NULL (a moe_experts output with E = 1);
 *            shared_gate_logit device [T] fp32 or NULL (gate 1 when shared
 *            is given without it): the always-on shared expert of
 *            diffulex.moe.layer (SharedExpertMLP)
 *   dtype    type of `out` (MOE_BF16 or MOE_F32)
 *   out      device [T,H] (dtype), written
 *   status   device int32 or NULL: an inv_perm entry outside [0,N) sets
 *            MOE_ERR_BAD_INDEX and contributes nothing.
 */
int moe_combine(const void* y_packed, int y_dtype, const int32_t* inv_perm, int T, int H, int k,
                const void* shared, const float* shared_gate_logit, int dtype,
                void* out, int32_t* status, void* stream);

/*
 * ---- Expert and tensor parallelism: the pieces a rank runs --------------
 *
 * metrale ep_dispatch.rs (module doc): the served expert-parallel MoE is
 * "masked-local plus all-reduce".  A rank that owns experts [s, e) of E runs
 * the full router and dispatcher on its tokens, then
 *   moe_gather(..., s, e, ...)          rows of its experts only,
 *   moe_experts(x_packed, offsets + s, packed_w, w13_local, w2_local, N, H,
 *               I, e - s, ...)          its experts (offsets hold absolute
 *                                       packed rows, so the rank's slice of
 *                                       offsets is a valid table for them),
 *   moe_combine_range(..., s, e, ..., MOE_F32, partial)
 *                                       its share of every token's sum,
 * the caller adds the ranks' fp32 partials (an all-reduce), and
 * moe_finalize rounds the sum once.  Tensor parallelism (diffulex.moe.layer,
 * TPFusedMoE; the modelexpress refit test's INTER_PER_TP slices, "w1 low, w3
 * high") is the same with every expert present on every rank but its I
 * split: rank r holds rows [r*I/tp, (r+1)*I/tp) of each half of w13 as one
 * [E, 2*I/tp, H] buffer and the same columns of w2 as [E, H, I/tp]; its
 * moe_experts (with I/tp) and moe_combine (fp32 out) give a partial that the
 * all-reduce and moe_finalize complete.
 */

/*
 * moe_gather -- the Executor's "gather token activations for scheduled
 * expert ranges" (DWDP README, "Executor Module") for the experts
 * [expert_start, expert_end) alone:
 *   x_packed[p,:] = x[packed_tok[p],:]  for p in [offsets[expert_start],
 *                                              offsets[expert_end])
 * Other rows of x_packed are left untouched.  moe_dispatch with x == NULL
 * followed by moe_gather over [0, E) is moe_dispatch with x.
 *
 *   x          device [T,H] (dtype)        packed_tok device [N] int32 and
 *   offsets    device [E+1] int32, as moe_dispatch writes them (trusted:
 *              rows and tokens in range)
 *   0 <= expert_start <= expert_end <= E;  N = rows of x_packed (T*k)
 *   x_packed   device [N,H] (dtype), written in the range only
 */
int moe_gather(const void* x, const int32_t* packed_tok, const int32_t* offsets, int E,
               int expert_start, int expert_end, int N, int H, int dtype, void* x_packed,
               int32_t* status, void* stream);

/*
 * moe_combine_range -- masked-local Merger: moe_combine restricted to the
 * rows of experts [expert_start, expert_end) (packed rows [offsets[s],
 * offsets[e])); a token's other assignments contribute nothing:
 *   out[t,:] = sum_{j<k, s <= id(t,j) < e} y_packed[inv_perm[t*k+j],:]
 *              (j in order, fp32)  + sigmoid(gate[t]) * shared[t,:] if given
 * Written as `dtype` (MOE_F32 for a partial that an all-reduce will add).
 * Arguments and errors as moe_combine, plus offsets (device [E+1] int32)
 * and 0 <= expert_start <= expert_end <= E.
 */
int moe_combine_range(const void* y_packed, int y_dtype, const int32_t* inv_perm,
                      const int32_t* offsets, int E, int expert_start, int expert_end, int T,
                      int H, int k, const void* shared, const float* shared_gate_logit,
                      int dtype, void* out, int32_t* status, void* stream);

/*
 * moe_finalize -- the one rounding after the ranks' partial outputs were
 * added: out[t,h] = acc[t,h] rounded to `dtype` (bf16: round to nearest
 * even; fp32: a copy).  acc device [T,H] fp32, out device [T,H] (dtype);
 * both 16-byte aligned, H % 8 == 0.
 */
int moe_finalize(const float* acc, int T, int H, int dtype, void* out, void* stream);

/* Bytes of device scratch moe_ep_partition needs (0 for num_tokens * top_k
 * <= 2048, when one block does all the work). */
size_t moe_ep_partition_workspace_bytes(int num_tokens, int top_k);

/*
 * moe_ep_partition -- metrale ep_dispatch.rs, "EpRoutingTable" /
 * "build_ep_routing_table", on the device: the row-major [num_tokens, top_k]
 * assignments split into a local bucket (expert id in [local_expert_start,
 * local_expert_end)) and a remote bucket (every other id).  Entry i of a
 * bucket is the triple (*_token_indices[i], *_expert_ids[i], *_weights[i])
 * of one assignment; both buckets keep the order the assignments were given
 * (flat index token * top_k + j ascending).  Expert ids are global (not
 * rank-relative) and compared as unsigned 32-bit values, like the page's
 * u32 ids.
 *
 *   gate_indices device [n_indices] int32, gate_weights device [n_weights] f32
 *   n_indices / n_weights must both equal num_tokens * top_k: otherwise
 *       MOE_ERR_INVALID_ARG with the message "gate_indices length mismatch" /
 *       "gate_weights length mismatch" (where the page's function panics)
 *   local_* and remote_* device arrays of num_tokens * top_k entries each
 *       (the caller cannot know the split in advance); bucket i is written
 *       in entries [0, bucket_counts[i])
 *   bucket_counts device int32[2]: local count, remote count (they add up
 *       to num_tokens * top_k, the table's total_count)
 *   ws / ws_bytes: device scratch of moe_ep_partition_workspace_bytes()
 *   num_tokens >= 0, top_k >= 1, 0 <= local_expert_start <= local_expert_end
 */
int moe_ep_partition(const int32_t* gate_indices, size_t n_indices, const float* gate_weights,
                     size_t n_weights, int num_tokens, int top_k, int local_expert_start,
                     int local_expert_end, int32_t* local_token_indices,
                     int32_t* local_expert_ids, float* local_weights,
                     int32_t* remote_token_indices, int32_t* remote_expert_ids,
                     float* remote_weights, int32_t* bucket_counts, void* ws, size_t ws_bytes,
                     void* stream);

/*
 * All-to-all dispatcher (diffulex.moe API reference, "diffulex.moe.dispatcher":
 * NaiveA2ADispatcher / TokenDispatcher move tokens between ranks for expert
 * execution).  With the E experts split over `world` ranks in contiguous
 * ranges (rank q owns [floor(E*q/world), floor(E*(q+1)/world))):
 *
 * moe_ep_owner -- owner[f] = the rank owning expert ids[f], f < n.  An id
 * outside [0, E) gives owner -1 and sets MOE_ERR_BAD_INDEX in `status`
 * (device int32 or NULL).  ids, owner: device int32 [n].
 * Dispatching the [T,k] owner table with moe_dispatch (E = world) groups a
 * rank's assignments by destination, in assignment order inside each group.
 *
 * moe_ep_pack_ids -- for the rows p < offsets[world] of that dispatch:
 *   local_ids[p] = ids[perm[p]] - (first expert of its owner),
 * the expert id the receiving rank uses for its own [0, E_local) experts.
 * ids device [n] int32 (the routed expert ids), perm / offsets the owner
 * dispatch's outputs (device [n] / [world+1] int32), local_ids device [n].
 */
int moe_ep_owner(const int32_t* ids, int n, int E, int world, int32_t* owner, int32_t* status,
                 void* stream);
int moe_ep_pack_ids(const int32_t* ids, const int32_t* perm, const int32_t* offsets, int n,
                    int E, int world, int32_t* local_ids, void* stream);

/*
 * ---- The whole layer behind one handle -----------------------------------
 *
 * DWDP README, "Runtime Integration Layer": router -> dispatcher ->
 * executor -> merger, each stage consuming the previous stage's output.  A
 * moe_layer holds a layer's shapes and weights (device pointers the caller
 * keeps alive) and every intermediate buffer, carved from ONE device block
 * the caller allocates (moe_layer_workspace_bytes; 256-byte aligned): the
 * library allocates no device memory here either.  It owns three CUDA
 * streams and a few events (host objects) for moe_layer_forward_host.
 */
typedef struct moe_layer_desc {
  int T, H, E, k, I;          /* tokens per call, hidden, experts, top-k, expert width */
  int dtype;                  /* MOE_F32 or MOE_BF16 */
  int renormalize;            /* divide the k weights by their sum */
  int n_groups, topk_groups;  /* group-limited routing when n_groups > 1 */
  const void* W_gate;         /* device [E,H] */
  const float* bias;          /* device [E] fp32 or NULL */
  const void* w13;            /* device [E,2I,H] */
  const void* w2;             /* device [E,H,I] */
  int I_s;                    /* shared expert width (when w13s != NULL) */
  const void* w13s;           /* device [2I_s,H] or NULL: no shared expert */
  const void* w2s;            /* device [H,I_s] */
  const void* w_sg;           /* device [H]: the shared expert's gate vector */
  int y_f32;                  /* bf16 layers: keep y_packed and the shared expert's
                                 output in fp32 (0: in fp16, see moe_experts) */
} moe_layer_desc;

typedef struct moe_layer moe_layer;   /* opaque */

/* Device bytes moe_layer_create needs for `d` (0 if d is invalid). */
size_t moe_layer_workspace_bytes(const moe_layer_desc* d);

/* Check `d` once (the rules of the stage calls), carve the buffers out of
 * `workspace` and zero what must start at zero (enqueued on `stream`, which
 * is then synchronised once).  *out receives the handle. */
int moe_layer_create(const moe_layer_desc* d, void* workspace, size_t workspace_bytes,
                     void* stream, moe_layer** out);

/* Wait for the handle's streams and free its host objects (not the workspace). */
int moe_layer_destroy(moe_layer* L);

/* The layer on device activations: x device [T,H] (dtype) -> out device
 * [T,H] (dtype), enqueued on `stream`, as moe_route, moe_dispatch,
 * moe_experts(_shared) and moe_combine chained. */
int moe_layer_forward(moe_layer* L, const void* x, void* out, void* stream);

/*
 * The layer on HOST activations: x_host [T,H] -> out_host [T,H], both host
 * memory of the activation type (pinned, so that the copies run
 * asynchronously).  Enqueues, without waiting for completion:
 *   upload x_host into one of two device copies of x (one cudaMemcpyAsync,
 *   after the work already on `stream` and after the step that last used
 *   that copy), the layer, and the download into out_host (one
 *   cudaMemcpyAsync), on three internal streams.  Consecutive calls
 *   therefore overlap: one step uploads while the previous one computes and
 *   the one before it downloads.
 * x_host must stay unchanged and out_host unread until the step is done:
 * moe_layer_join(L, s) makes stream s wait for every step enqueued so far.
 */
int moe_layer_forward_host(moe_layer* L, const void* x_host, void* out_host, void* stream);

/* Make `stream` wait for all work enqueued on L so far. */
int moe_layer_join(moe_layer* L, void* stream);

/* moe_layer_join, then copy L's device status word to *host_status
 * (synchronises `stream`). */
int moe_layer_status(moe_layer* L, void* stream, int32_t* host_status);

/* Device address of one of L's intermediate buffers, for inspection:
 * "logits", "ids", "w", "counts", "offsets", "perm", "inv_perm",
 * "packed_tok", "packed_w", "x_packed", "h", "y_packed" (fp16, or fp32 with
 * y_f32), "status"; NULL for any other name. */
void* moe_layer_buffer(moe_layer* L, const char* name);

/* Copy the device status word to *host_status after the stream's prior work
 * (synchronises `stream`).  Returns MOE_OK or MOE_ERR_CUDA. */
int moe_read_status(const int32_t* status, void* stream, int32_t* host_status);

/*
 * moe_probe_wait_timeout -- self-test of the bounded-wait machinery every
 * persistent kernel here uses.  Launches one CTA that waits on an mbarrier
 * nothing ever arrives on, with a budget of `budget_us` microseconds
 * (1..2,000,000); the wait gives up, writes MOE_ERR_TIMEOUT to `status`
 * (device int32) and the kernel returns normally.  Used by the tests to
 * check that a wait which runs out is reported, not hung.
 */
int moe_probe_wait_timeout(int32_t* status, int budget_us, void* stream);

/*
 * moe_test_set_wait_budget_ns -- testing hook for failure detection.  Sets the
 * budget of the main-loop waits of the tensor-core kernels (the grouped GEMM
 * and the tensor-core router) for launches made after the call, process
 * wide: 0 restores the default (2 s); otherwise 1000 <= ns <= 2e9.  With a
 * budget of a few microseconds ordinary waits for copies and MMAs run out,
 * so the kernels report MOE_ERR_TIMEOUT and take their abort path (their
 * drain waits keep the full budget: every issued copy and MMA completes
 * before a CTA leaves, and TMEM is freed).  Results of such launches are
 * undefined; re-zero a moe_experts workspace used by one.  Not for
 * production use.
 */
int moe_test_set_wait_budget_ns(unsigned long long ns);

#ifdef __cplusplus
}
#endif
#endif /* MOE_B200_H */
